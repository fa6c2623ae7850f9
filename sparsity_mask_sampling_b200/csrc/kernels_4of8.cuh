// kernels_4of8.cuh -- the 4:8 sampler kernels (C = 70 candidates per block of 8 weights).
//
// MaskLLM (paper-graph-ui summary of arXiv 2409.17481) s.3.2 / s.3.4, generalised from 2:4
// to 4:8 as the method states (N:M with C(M,N) candidates); the candidate order is the
// lexicographic order of the ascending position 4-tuples.
//
// Work mapping: one thread owns one block and walks all 70 candidates fully unrolled, so
// every candidate's keep mask is a compile-time constant (no divergence, no table lookups).
// A block's logits are 280 B, so a thread reading its own row would make each warp access
// stride 280 B; instead a CTA stages its tile of kBlocksPerCta logit rows through shared
// memory with coalesced copies, and AdamW runs as a flat, coalesced pass over the tile.
#pragma once

#include <type_traits>

#include "device_common.cuh"

namespace mllm {
namespace k48 {

constexpr int C = 70;
constexpr int kCtaThreads = 128;
constexpr int kBlocksPerCta = kCtaThreads;  // one block per thread
constexpr int kTileFloats = kBlocksPerCta * C;
// The forward's CTA is two independent 128-thread halves that share one logarithm table:
// each half stages and computes its own tiles and meets only on its own named barrier, so an
// SM holds 16 warps (two such CTAs) where 128-thread CTAs, each with its own table, fit 12.
constexpr int kFwdHalves = 2;
constexpr int kFwdThreads = kFwdHalves * kCtaThreads;
constexpr int kFwdDynSmem = kFwdHalves * kTileFloats * (int)sizeof(float);
constexpr int kBwdDynSmem = 2 * kTileFloats * (int)sizeof(float);
constexpr int kStepDynSmem = kTileFloats * (int)sizeof(float);  // the one-launch step: one tile buffer

// Keep mask (bit j = position j) of candidate i: the i-th 4-subset of {0..7} in
// lexicographic order of ascending index tuples. Only ever evaluated at compile time.
__host__ __device__ constexpr uint32_t cand_mask(int i) {
    int r = 0;
    for (int a = 0; a < 8; ++a)
        for (int b = a + 1; b < 8; ++b)
            for (int c = b + 1; c < 8; ++c)
                for (int d = c + 1; d < 8; ++d)
                    if (r++ == i) return (1u << a) | (1u << b) | (1u << c) | (1u << d);
    return 0u;
}

// The 70 keep masks as a device table, for lookups by a runtime index (the prior given as a
// candidate index); built at compile time from cand_mask.
struct Cand48Table {
    uint8_t m[C];
    constexpr Cand48Table() : m{} {
        for (int i = 0; i < C; ++i) m[i] = (uint8_t)cand_mask(i);
    }
};
__device__ const Cand48Table g_cand48{};

// Compile-time loop: f(std::integral_constant<int, I>) for I in [B, E).
template <int B, int E, class F>
__device__ __forceinline__ void static_for(F &&f) {
    if constexpr (B < E) {
        f(std::integral_constant<int, B>{});
        static_for<B + 1, E>(f);
    }
}

// --------------------------------------------------------------------------- tile staging

// Tile staging. A tile of nb blocks is nb*280 bytes, 16-byte aligned at its start (tiles
// begin at multiples of kBlocksPerCta blocks). stage_in issues asynchronous 16-byte copies
// (cp.async, no registers involved) for every whole 16-byte chunk, plus one 8-byte tail when
// nb is odd, then waits for them; the caller synchronises the CTA afterwards.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// lt: the thread's index among the kCtaThreads threads that share the tile.
__device__ __forceinline__ void stage_in(float *dst, const float *src, int n, int lt = threadIdx.x) {
    const int n4 = n >> 2;  // whole 16-byte chunks
    for (int i = lt; i < n4; i += kCtaThreads) cp_async16(dst + 4 * i, src + 4 * i);
    if ((n & 3) && lt == 0) {  // n = nb*70 is even: at most one 8-byte tail
        *reinterpret_cast<float2 *>(dst + 4 * n4) = __ldcs(reinterpret_cast<const float2 *>(src + 4 * n4));
    }
    cp_async_wait_all();
}

__device__ __forceinline__ void stage_out(float *dst, const float *src, int n) {
    const int n4 = n >> 2;
    for (int i = threadIdx.x; i < n4; i += kCtaThreads)
        __stcs(reinterpret_cast<float4 *>(dst) + i, reinterpret_cast<const float4 *>(src)[i]);
    if ((n & 3) && threadIdx.x == 0)
        __stcs(reinterpret_cast<float2 *>(dst + 4 * n4), *reinterpret_cast<const float2 *>(src + 4 * n4));
}

// Ask L2 to fetch [p, p + bytes) now (a bulk prefetch; no data returns to the SM).
__device__ __forceinline__ void prefetch_l2(const void *p, int bytes) {
    bytes &= ~15;
    if (bytes > 0) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

template <bool kF32>
__device__ __forceinline__ void load8(const void *base, int64_t b, float w[8]) {
    if (kF32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + b * 8);
        const float4 a = ld_stream(p), c = ld_stream(p + 1);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
    } else {
        const uint4 a = ld_stream(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(base) + b * 8));
        w[0] = bf16lo(a.x); w[1] = bf16hi(a.x); w[2] = bf16lo(a.y); w[3] = bf16hi(a.y);
        w[4] = bf16lo(a.z); w[5] = bf16hi(a.z); w[6] = bf16lo(a.w); w[7] = bf16hi(a.w);
    }
}

template <bool kF32>
__device__ __forceinline__ void store8(void *base, int64_t b, const float x[8]) {
    if (kF32) {
        float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(base) + b * 8);
        st_stream(p, make_float4(x[0], x[1], x[2], x[3]));
        st_stream(p + 1, make_float4(x[4], x[5], x[6], x[7]));
    } else {
        st_stream(reinterpret_cast<uint4 *>(static_cast<uint16_t *>(base) + b * 8),
                  make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                             pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7])));
    }
}

// --------------------------------------------------------------------------- per-block math

// The per-block math below runs on the paired fp32 instructions of sm_100 (__ffma2_rn,
// __fmul2_rn, __fadd2_rn), two candidates or two positions per instruction; each component
// rounds exactly as the scalar form and every sum keeps its order, so the results are
// bit-identical to one-at-a-time evaluation. w2[k] holds candidates 2k and 2k+1.
constexpr int C2 = C / 2;

// max(a, b, c) in one instruction (the three-input form of max.f32, sm_100); NaN operands
// are passed over as by fmaxf.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Perturbed logits w_c = fma(kappa, pi_c, g_c) for all 70 candidates, and their maximum.
__device__ __forceinline__ float perturbed(const float *pi_row, uint64_t gid, const StepScalars &sc,
                                           const NlogCtx &L, float2 w2[C2]) {
    float mx = -INFINITY;
    const float2 *pi2 = reinterpret_cast<const float2 *>(pi_row);  // rows are 280 B: 8-byte aligned
#pragma unroll
    for (int gr = 0; gr < 12; ++gr) {
        uint32_t u[6];
        if (sc.noise_on) fields21_unit(block_words(sc, gid, (uint32_t)gr), u);
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int c = 6 * gr + 2 * k;
            if (c < C) {
                const float2 g = sc.noise_on ? gumbel_unit2(u[2 * k], u[2 * k + 1], L) : make_float2(0.f, 0.f);
                const float2 wc = __ffma2_rn(f2(sc.kappa), pi2[c / 2], g);
                w2[c / 2] = wc;
                mx = fmax3(mx, wc.x, wc.y);
            }
        }
    }
    return mx;
}

// Sums over candidates, formed per half of the block. A candidate's four kept positions are
// a subset of positions 0-3 (its low half) and a subset of positions 4-7 (its high half);
// each of the 16 subsets of a half occurs among the 70 candidates. In the forward each e_c
// goes into one of 16 buckets by its low half and one of 16 by its high half; the sum over
// the candidates that keep position j (or prune it) is the sum of the 8 buckets of j's half
// whose subset holds j (or lacks it). In the backward a candidate's
// sum_{j kept} P_j - sum_{j pruned} Q_j is D_lo[low half] + D_hi[high half], where
// D[s] = sum_{j in s} P_j - sum_{j in the half, not in s} Q_j is formed once per subset. The
// terms are those of Eq.7 and its derivative; only the association of the fp32 additions
// differs from sums taken in candidate order.
__host__ __device__ constexpr uint32_t lo4(int c) { return cand_mask(c) & 0xFu; }
__host__ __device__ constexpr uint32_t hi4(int c) { return cand_mask(c) >> 4; }
__host__ __device__ constexpr bool first_lo(int c) {
    for (int k = 0; k < c; ++k)
        if (lo4(k) == lo4(c)) return false;
    return true;
}
__host__ __device__ constexpr bool first_hi(int c) {
    for (int k = 0; k < c; ++k)
        if (hi4(k) == hi4(c)) return false;
    return true;
}
__host__ __device__ constexpr int top_bit(int s) {
    int b = -1;
    for (; s; s >>= 1) ++b;
    return b;
}

// Sum of the buckets B[s] whose subset s holds bit kBit (kHas) or lacks it, in ascending s.
template <int kBit, bool kHas>
__device__ __forceinline__ float bucket_sum(const float B[16]) {
    constexpr int s0 = kHas ? (1 << kBit) : 0;  // the smallest such subset
    float acc = B[s0];
    static_for<s0 + 1, 16>([&](auto I) {
        constexpr int s = decltype(I)::value;
        if constexpr (((s >> kBit) & 1) == (kHas ? 1 : 0)) acc = __fadd_rn(acc, B[s]);
    });
    return acc;
}

// e_c = 2^((w_c - max) c2) in place; returns sum e; ms2 = sums over c with j in S_c and, when
// kComp, mc2 = sums over c with j not in S_c (pairs of positions 2p, 2p+1).
template <bool kComp>
__device__ __forceinline__ float soft_sums(float2 w2[C2], float mx, float c2, float2 ms2[4], float2 mc2[4]) {
    float BL[16], BH[16];  // buckets by low-half and by high-half subset
    const float m2 = __fmul_rn(mx, c2);  // (w - max) c2 = w c2 - fl(max c2): a common rounding that cancels
    auto put = [&](auto I, float e) {
        constexpr int c = decltype(I)::value;
        if constexpr (first_lo(c)) BL[lo4(c)] = e;
        else BL[lo4(c)] = __fadd_rn(BL[lo4(c)], e);
        if constexpr (first_hi(c)) BH[hi4(c)] = e;
        else BH[hi4(c)] = __fadd_rn(BH[hi4(c)], e);
    };
    static_for<0, C2>([&](auto I) {
        constexpr int k = decltype(I)::value;
        const float2 a = __ffma2_rn(w2[k], f2(c2), f2(-m2));
        const float e0 = ex2_approx(a.x), e1 = ex2_approx(a.y);
        w2[k] = make_float2(e0, e1);
        put(std::integral_constant<int, 2 * k>{}, e0);
        put(std::integral_constant<int, 2 * k + 1>{}, e1);
    });
    ms2[0] = make_float2(bucket_sum<0, true>(BL), bucket_sum<1, true>(BL));
    ms2[1] = make_float2(bucket_sum<2, true>(BL), bucket_sum<3, true>(BL));
    ms2[2] = make_float2(bucket_sum<0, true>(BH), bucket_sum<1, true>(BH));
    ms2[3] = make_float2(bucket_sum<2, true>(BH), bucket_sum<3, true>(BH));
    if (kComp) {
        mc2[0] = make_float2(bucket_sum<0, false>(BL), bucket_sum<1, false>(BL));
        mc2[1] = make_float2(bucket_sum<2, false>(BL), bucket_sum<3, false>(BL));
        mc2[2] = make_float2(bucket_sum<0, false>(BH), bucket_sum<1, false>(BH));
        mc2[3] = make_float2(bucket_sum<2, false>(BH), bucket_sum<3, false>(BH));
    }
    // sum e: every candidate sits in exactly one low-half bucket (a pairwise tree over them)
    float t8[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) t8[q] = __fadd_rn(BL[2 * q], BL[2 * q + 1]);
#pragma unroll
    for (int q = 0; q < 4; ++q) t8[q] = __fadd_rn(t8[2 * q], t8[2 * q + 1]);
    return __fadd_rn(__fadd_rn(t8[0], t8[1]), __fadd_rn(t8[2], t8[3]));
}

// D[s] = sum_{j in s} P_j - sum_{j in the half, not in s} Q_j for the 16 subsets s of the
// half kBase..kBase+3 (subset sums in ascending position order).
template <int kBase>
__device__ __forceinline__ void half_diffs(const float P[8], const float Q[8], float D[16]) {
    float SP[16], SQ[16];
    static_for<1, 16>([&](auto I) {
        constexpr int s = decltype(I)::value;
        constexpr int hb = top_bit(s), rest = s & ~(1 << hb);
        if constexpr (rest == 0) {
            SP[s] = P[kBase + hb];
            SQ[s] = Q[kBase + hb];
        } else {
            SP[s] = __fadd_rn(SP[rest], P[kBase + hb]);
            SQ[s] = __fadd_rn(SQ[rest], Q[kBase + hb]);
        }
    });
    D[0] = -SQ[15];
    D[15] = SP[15];
    static_for<1, 15>([&](auto I) {
        constexpr int s = decltype(I)::value;
        D[s] = __fsub_rn(SP[s], SQ[15 ^ s]);
    });
}

// AdamW, PyTorch step order, two elements (bit-identical to adamw on each).
__device__ __forceinline__ void adamw2(float2 &p, float2 &m, float2 &v, float2 g, const StepScalars &s) {
    const float2 pd = __fmul2_rn(p, f2(s.decay));
    m = __ffma2_rn(f2(s.beta1), m, __fmul2_rn(f2(s.one_minus_beta1), g));
    v = __ffma2_rn(f2(s.beta2), v, __fmul2_rn(f2(s.one_minus_beta2), __fmul2_rn(g, g)));
    const float2 denom = __ffma2_rn(make_float2(sqrt_approx(v.x), sqrt_approx(v.y)), f2(s.inv_sqrt_bc2), f2(s.eps));
    p = __ffma2_rn(f2(-s.step_size), make_float2(__fdividef(m.x, denom.x), __fdividef(m.y, denom.y)), pd);
}
__device__ __forceinline__ void adamw4(float4 &p, float4 &m, float4 &v, float4 g, const StepScalars &s) {
    float2 pa = make_float2(p.x, p.y), pb = make_float2(p.z, p.w), ma = make_float2(m.x, m.y),
           mb = make_float2(m.z, m.w), va = make_float2(v.x, v.y), vb = make_float2(v.z, v.w);
    adamw2(pa, ma, va, make_float2(g.x, g.y), s);
    adamw2(pb, mb, vb, make_float2(g.z, g.w), s);
    p = make_float4(pa.x, pa.y, pb.x, pb.y);
    m = make_float4(ma.x, ma.y, mb.x, mb.y);
    v = make_float4(va.x, va.y, vb.x, vb.y);
}

// AdamW, PyTorch step order, one element.
__device__ __forceinline__ void adamw(float &p, float &m, float &v, float g, const StepScalars &s) {
    const float pd = __fmul_rn(p, s.decay);
    m = __fmaf_rn(s.beta1, m, __fmul_rn(s.one_minus_beta1, g));
    v = __fmaf_rn(s.beta2, v, __fmul_rn(s.one_minus_beta2, __fmul_rn(g, g)));
    const float denom = __fmaf_rn(sqrt_approx(v), s.inv_sqrt_bc2, s.eps);
    p = __fmaf_rn(-s.step_size, __fdividef(m, denom), pd);
}

// Gradient of one block's logits (Eq.6-Eq.8 backward) into grow[C] from e_c (in w2),
// r = 1 / sum e and the position sums ms2, mc2 of the step's noise:
// dpi_c = (kappa/tau) y_c (sum_{j in S_c} P_j - sum_{j not in S_c} Q_j), P_j = (1 - M_j) u_j,
// Q_j = M_j u_j, u_j = G_j W_j - 2 lambda W_j^2 M_j.
__device__ __forceinline__ void grad_tail(const float2 w2[C2], float r, const float2 ms2[4], const float2 mc2[4],
                                          const float wt[8], const float gw[8], const StepScalars &sc,
                                          float *grow) {
    float P[8], Q[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // positions 2p, 2p+1
        const float2 ms = __fmul2_rn(ms2[p], f2(r)), mc = __fmul2_rn(mc2[p], f2(r));
        const float2 wj = make_float2(wt[2 * p], wt[2 * p + 1]), gj = make_float2(gw[2 * p], gw[2 * p + 1]);
        // fma(-(2 lambda W^2), M, G W)
        const float2 u = __ffma2_rn(__fmul2_rn(f2(-sc.two_lambda), __fmul2_rn(wj, wj)), ms, __fmul2_rn(gj, wj));
        const float2 pp = __fmul2_rn(mc, u), qq = __fmul2_rn(ms, u);
        P[2 * p] = pp.x; P[2 * p + 1] = pp.y;
        Q[2 * p] = qq.x; Q[2 * p + 1] = qq.y;
    }
    float DL[16], DH[16];
    half_diffs<0>(P, Q, DL);
    half_diffs<4>(P, Q, DH);
    const float cr = __fmul_rn(sc.kappa_over_tau, r);
    float2 *grow2 = reinterpret_cast<float2 *>(grow);  // rows are 280 B: 8-byte aligned
    static_for<0, C2>([&](auto I) {
        constexpr int k = decltype(I)::value;
        const float d0 = __fadd_rn(DL[lo4(2 * k)], DH[hi4(2 * k)]);
        const float d1 = __fadd_rn(DL[lo4(2 * k + 1)], DH[hi4(2 * k + 1)]);
        grow2[k] = __fmul2_rn(__fmul2_rn(f2(cr), w2[k]), make_float2(d0, d1));
    });
}

// The same from the block's logits (noise of step sc.step).
__device__ __forceinline__ void grad_row(const float *pi_row, const float wt[8], const float gw[8], uint64_t gid,
                                         const StepScalars &sc, const NlogCtx &L, float *grow) {
    float2 w2[C2], ms2[4], mc2[4];
    const float mx = perturbed(pi_row, gid, sc, L, w2);
    const float r = rcp_approx(soft_sums<true>(w2, mx, sc.c2, ms2, mc2));
    grad_tail(w2, r, ms2, mc2, wt, gw, sc, grow);
}

// Forward of one block (Eq.5-Eq.8) from r = 1 / sum e and the position sums ms2: soft mask
// ms[8] and soft-masked weights x[8] (fp32), regulariser partial added to acc.
__device__ __forceinline__ void fwd_tail(const float2 ms2[4], float r, const float wt[8], float ms[8], float x[8],
                                         float &acc) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 m = __fmul2_rn(ms2[p], f2(r));
        const float2 xx = __fmul2_rn(make_float2(wt[2 * p], wt[2 * p + 1]), m);
        ms[2 * p] = m.x; ms[2 * p + 1] = m.y;
        x[2 * p] = xx.x; x[2 * p + 1] = xx.y;
        acc = __fmaf_rn(xx.x, xx.x, acc);
        acc = __fmaf_rn(xx.y, xx.y, acc);
    }
}

// The same from the block's logits (noise of step sc.step).
__device__ __forceinline__ void fwd_row(const float *pi_row, const float wt[8], uint64_t gid, const StepScalars &sc,
                                        const NlogCtx &L, float ms[8], float x[8], float &acc) {
    float2 w2[C2], ms2[4], mc2[4];
    const float mx = perturbed(pi_row, gid, sc, L, w2);
    const float r = rcp_approx(soft_sums<false>(w2, mx, sc.c2, ms2, mc2));
    fwd_tail(ms2, r, wt, ms, x, acc);
}

// AdamW over a tile as one flat, coalesced array of float4: logits and gradients from shared
// memory, m and v from global memory (each thread first loads kUnroll vectors of each, so it
// keeps 2*kUnroll loads in flight). Updated logits, m, v (and the gradient when gout) are
// stored; with kKeep the updated logits are also written back to s_pi.
template <bool kKeep>
__device__ __forceinline__ void adam_tile(float *s_pi, const float *s_gr, int n, float *__restrict__ pi,
                                          float *__restrict__ mm, float *__restrict__ vv,
                                          float *__restrict__ gout, const StepScalars &sc) {
    const int n4 = n >> 2;
    constexpr int kUnroll = 6;
    for (int i0 = threadIdx.x; i0 < n4; i0 += kCtaThreads * kUnroll) {
        float4 m4[kUnroll], v4[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kCtaThreads;
            if (i < n4) {
                m4[u] = __ldcs(reinterpret_cast<const float4 *>(mm) + i);
                v4[u] = __ldcs(reinterpret_cast<const float4 *>(vv) + i);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kCtaThreads;
            if (i < n4) {
                float4 p4 = reinterpret_cast<const float4 *>(s_pi)[i];
                const float4 g4 = reinterpret_cast<const float4 *>(s_gr)[i];
                adamw4(p4, m4[u], v4[u], g4, sc);
                if (kKeep) reinterpret_cast<float4 *>(s_pi)[i] = p4;
                __stcs(reinterpret_cast<float4 *>(pi) + i, p4);
                __stcs(reinterpret_cast<float4 *>(mm) + i, m4[u]);
                __stcs(reinterpret_cast<float4 *>(vv) + i, v4[u]);
                if (gout) __stcs(reinterpret_cast<float4 *>(gout) + i, g4);
            }
        }
    }
    if ((n & 3) && threadIdx.x == 0) {  // 2-float tail of a tile with an odd block count
        for (int i = 4 * n4; i < n; ++i) {
            float p = s_pi[i], m = mm[i], v = vv[i];
            adamw(p, m, v, s_gr[i], sc);
            if (kKeep) s_pi[i] = p;
            pi[i] = p; mm[i] = m; vv[i] = v;
            if (gout) gout[i] = s_gr[i];
        }
    }
}

// AdamW over a tile whose gradients sit in s_buf (flat, coalesced float4s): the logits are
// read again from global memory (staged from there at the start of the tile, so they are
// still in L2), m and v from global memory (prefetched into L2); the updated logits overwrite
// the gradients in s_buf and are stored with m, v (and the gradient when gout). Each float4
// is read and rewritten by the same thread, so the update in place needs no barrier.
__device__ __forceinline__ void adam_tile_inplace(float *s_buf, int n, float *__restrict__ pi,
                                                  float *__restrict__ mm, float *__restrict__ vv,
                                                  float *__restrict__ gout, const StepScalars &sc) {
    const int n4 = n >> 2;
    constexpr int kUnroll = 4;
    for (int i0 = threadIdx.x; i0 < n4; i0 += kCtaThreads * kUnroll) {
        float4 p4[kUnroll], m4[kUnroll], v4[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kCtaThreads;
            if (i < n4) {
                p4[u] = __ldcg(reinterpret_cast<const float4 *>(pi) + i);
                m4[u] = __ldcs(reinterpret_cast<const float4 *>(mm) + i);
                v4[u] = __ldcs(reinterpret_cast<const float4 *>(vv) + i);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kCtaThreads;
            if (i < n4) {
                const float4 g4 = reinterpret_cast<const float4 *>(s_buf)[i];
                adamw4(p4[u], m4[u], v4[u], g4, sc);
                reinterpret_cast<float4 *>(s_buf)[i] = p4[u];
                __stcs(reinterpret_cast<float4 *>(pi) + i, p4[u]);
                __stcs(reinterpret_cast<float4 *>(mm) + i, m4[u]);
                __stcs(reinterpret_cast<float4 *>(vv) + i, v4[u]);
                if (gout) __stcs(reinterpret_cast<float4 *>(gout) + i, g4);
            }
        }
    }
    if ((n & 3) && threadIdx.x == 0) {  // 2-float tail of a tile with an odd block count
        for (int i = 4 * n4; i < n; ++i) {
            const float g = s_buf[i];
            float p = __ldcg(pi + i), m = mm[i], v = vv[i];
            adamw(p, m, v, g, sc);
            s_buf[i] = p;
            pi[i] = p; mm[i] = m; vv[i] = v;
            if (gout) gout[i] = g;
        }
    }
}

// CTA-level deterministic reduction of the regulariser partials, then the last CTA (ticket)
// combines all per-CTA partials in index order and resets the ticket. kThr: the CTA's threads.
template <int kThr = kCtaThreads>
__device__ __forceinline__ void reduce_reg(float acc, double *partials, unsigned int *ticket, double *reg_out,
                                           int accumulate) {
    __shared__ double s_w[kThr / 32];
    __shared__ bool s_last;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) s_w[warp] = (double)acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tt = 0.0;
        for (int i = 0; i < kThr / 32; ++i) tt += s_w[i];
        partials[blockIdx.x] = tt;
        __threadfence();
        s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    double tt = 0.0;
    for (unsigned int i = threadIdx.x; i < gridDim.x; i += kThr) tt += __ldcg(partials + i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tt += __shfl_xor_sync(0xFFFFFFFFu, tt, o);
    __syncthreads();
    if (lane == 0) s_w[warp] = tt;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (int i = 0; i < kThr / 32; ++i) tot += s_w[i];
        *reg_out = accumulate ? (*reg_out + tot) : tot;
        *ticket = 0u;
    }
}

// --------------------------------------------------------------------------- kernels

// Named barrier of half h (ids 1 and 2 as immediates; id 0 is the CTA-wide barrier).
__device__ __forceinline__ void half_sync(int h) {
    if (h) asm volatile("bar.sync 2, %0;" ::"n"(kCtaThreads) : "memory");
    else asm volatile("bar.sync 1, %0;" ::"n"(kCtaThreads) : "memory");
}

template <bool kW32>
__global__ void __launch_bounds__(kFwdThreads) fwd_kernel(const __grid_constant__ Group grp,
                                                          const StepScalars sc, double *partials,
                                                          unsigned int *ticket, double *reg_out,
                                                          int accumulate) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    extern __shared__ __align__(16) float s_dyn[];  // [kFwdHalves][kTileFloats] logits of each half's tile
    const int h = (int)threadIdx.x / kCtaThreads, lt = (int)threadIdx.x % kCtaThreads;
    float *s_pi = s_dyn + h * kTileFloats;
    load_tab(s_tab);
    __syncthreads();
    const NlogCtx L{s_tab};
    float acc = 0.f;
    int mi = 0;
    for (int64_t t = (int64_t)blockIdx.x * kFwdHalves + h; t < grp.total_work; t += (int64_t)gridDim.x * kFwdHalves) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t tb0 = (t - d.work_begin) * kBlocksPerCta;
        const int nb = (int)imin64(kBlocksPerCta, d.nblocks - tb0);
        half_sync(h);  // the half's previous tile's readers are done
        stage_in(s_pi, d.pi + tb0 * C, nb * C, lt);
        half_sync(h);
        if (lt < nb) {
            const int64_t b = tb0 + lt;
            float wt[8], ms[8], x[8];
            load8<kW32>(d.W, b, wt);
            fwd_row(s_pi + lt * C, wt, d.gid0 + b, sc, L, ms, x, acc);
            store8<kW32>(d.X, b, x);
            if (d.soft) {
                float4 *sp = reinterpret_cast<float4 *>(d.soft + b * 8);
                sp[0] = make_float4(ms[0], ms[1], ms[2], ms[3]);
                sp[1] = make_float4(ms[4], ms[5], ms[6], ms[7]);
            }
        }
    }
    if (reg_out) reduce_reg<kFwdThreads>(acc, partials, ticket, reg_out, accumulate);
}

template <bool kW32, bool kG32>
__global__ void __launch_bounds__(kCtaThreads) bwd_adam_kernel(const __grid_constant__ Group grp,
                                                               const StepScalars sc) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    extern __shared__ __align__(16) float s_dyn[];  // [2 * kTileFloats]: logits, gradients
    float *s_pi = s_dyn, *s_gr = s_dyn + kTileFloats;
    load_tab(s_tab);
    const NlogCtx L{s_tab};
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t tb0 = (t - d.work_begin) * kBlocksPerCta;
        const int nb = (int)imin64(kBlocksPerCta, d.nblocks - tb0);
        __syncthreads();
        if (threadIdx.x == 0) {
            prefetch_l2(d.m + tb0 * C, nb * C * 4);
            prefetch_l2(d.v + tb0 * C, nb * C * 4);
        }
        stage_in(s_pi, d.pi + tb0 * C, nb * C);
        __syncthreads();
        if ((int)threadIdx.x < nb) {
            const int64_t b = tb0 + threadIdx.x;
            float wt[8], gw[8];
            load8<kW32>(d.W, b, wt);
            load8<kG32>(d.G, b, gw);
            grad_row(s_pi + threadIdx.x * C, wt, gw, d.gid0 + b, sc, L, s_gr + threadIdx.x * C);
        }
        __syncthreads();
        adam_tile<false>(s_pi, s_gr, nb * C, d.pi + tb0 * C, d.m + tb0 * C, d.v + tb0 * C,
                         d.grad ? d.grad + tb0 * C : nullptr, sc);
    }
}

// Backward + AdamW of step t fused with the forward of step t+1 (mllm_sample_bwd_adam_fwd):
// per tile, the gradient of every block (noise of step t) written over the block's logits in
// the one tile buffer (each thread reads its whole row before it writes it), the flat AdamW
// pass (updated logits back into the buffer), then the forward of step t+1 from the updated
// logits. One 35.8 KB buffer per CTA lets three CTAs share an SM. The logits are read from
// HBM once: the AdamW pass reads them again from L2, and each tile start asks L2 for the
// tile's m and v and for the CTA's next tile of logits.
template <bool kW32, bool kG32>
__global__ void __launch_bounds__(kCtaThreads, 3) bwd_adam_fwd_kernel(const __grid_constant__ Group grp,
                                                                   const StepScalars sb, const StepScalars sf,
                                                                   double *partials, unsigned int *ticket,
                                                                   double *reg_out, int accumulate) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    extern __shared__ __align__(16) float s_buf[];  // [kTileFloats]: logits, gradients, updated logits
    load_tab(s_tab);
    const NlogCtx L{s_tab};
    float acc = 0.f;
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t tb0 = (t - d.work_begin) * kBlocksPerCta;
        const int nb = (int)imin64(kBlocksPerCta, d.nblocks - tb0);
        if (threadIdx.x == 0) {
            prefetch_l2(d.m + tb0 * C, nb * C * 4);
            prefetch_l2(d.v + tb0 * C, nb * C * 4);
            const int64_t tn = t + gridDim.x;
            if (tn < grp.total_work) {
                const MatDesc &dn = grp.d[next_mat(grp, mi, tn)];
                const int64_t nb0 = (tn - dn.work_begin) * kBlocksPerCta;
                prefetch_l2(dn.pi + nb0 * C, (int)imin64(kBlocksPerCta, dn.nblocks - nb0) * C * 4);
            }
        }
        __syncthreads();  // the previous tile's readers are done (and the table is loaded)
        stage_in(s_buf, d.pi + tb0 * C, nb * C);
        __syncthreads();
        const bool mine = (int)threadIdx.x < nb;
        const int64_t b = tb0 + threadIdx.x;
        if (mine) {
            float wt[8], gw[8];
            load8<kW32>(d.W, b, wt);
            load8<kG32>(d.G, b, gw);
            grad_row(s_buf + threadIdx.x * C, wt, gw, d.gid0 + b, sb, L, s_buf + threadIdx.x * C);
        }
        __syncthreads();
        adam_tile_inplace(s_buf, nb * C, d.pi + tb0 * C, d.m + tb0 * C, d.v + tb0 * C,
                          d.grad ? d.grad + tb0 * C : nullptr, sb);
        __syncthreads();  // updated logits in s_buf
        if (mine) {
            float wt[8], ms[8], x[8];
            load8<kW32>(d.W, b, wt);  // read again (from L2) rather than held through the tile
            fwd_row(s_buf + threadIdx.x * C, wt, d.gid0 + b, sf, L, ms, x, acc);
            store8<kW32>(d.X, b, x);
            if (d.soft) {
                float4 *sp = reinterpret_cast<float4 *>(d.soft + b * 8);
                sp[0] = make_float4(ms[0], ms[1], ms[2], ms[3]);
                sp[1] = make_float4(ms[4], ms[5], ms[6], ms[7]);
            }
        }
    }
    if (reg_out) reduce_reg(acc, partials, ticket, reg_out, accumulate);
}

// Prior initialisation; kFromIdx as for the 2:4 kernel (M0 = candidate d.prior[b], >= C: none).
template <bool kW32, bool kFromIdx>
__global__ void __launch_bounds__(kCtaThreads) prior_kernel(const __grid_constant__ Group grp,
                                                            float alpha, float init_std, uint64_t seed) {
    __shared__ __align__(16) float s_pi[kTileFloats];
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t tb0 = (t - d.work_begin) * kBlocksPerCta;
        const int nb = (int)imin64(kBlocksPerCta, d.nblocks - tb0);
        __syncthreads();
        if ((int)threadIdx.x < nb) {
            const int64_t b = tb0 + threadIdx.x;
            uint32_t m0 = 0;
            float shift = 2.0f;  // sim = |M0 & S_c| - N*N/M; no prior: every sim is 0
            if (kFromIdx) {
                const uint32_t k = d.prior[b];
                if (k < (uint32_t)C) m0 = g_cand48.m[k];
                else shift = 0.0f;
            } else {
                float wt[8], key[8];
                load8<kW32>(d.W, b, wt);
#pragma unroll
                for (int j = 0; j < 8; ++j) key[j] = (wt[j] != wt[j]) ? -1.0f : fabsf(wt[j]);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    int rank = 0;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        if (k != j && (key[k] > key[j] || (key[k] == key[j] && k < j))) ++rank;
                    if (rank < 4) m0 |= 1u << j;
                }
            }
            float *row = s_pi + threadIdx.x * C;
            if (init_std == 0.f) {
                static_for<0, C>([&](auto I) {
                    constexpr int c = decltype(I)::value;
                    row[c] = alpha * ((float)__popc(m0 & cand_mask(c)) - shift);
                });
            } else {
                float mu = 0.f;
#pragma unroll
                for (int gr = 0; gr < 12; ++gr) {
                    uint32_t f[6];
                    fields21(block_words(seed, d.gid0 + b, kInitStep, (uint32_t)gr), f);
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        const int c = 6 * gr + 2 * q;
                        if (c < C) {
                            const float u1 = uniform_from_field(f[2 * q]);
                            const float u2 = uniform_from_field(f[2 * q + 1]);
                            const float rad = sqrtf(-2.0f * logf(u1));
                            float sn, cs;
                            sincospif(2.0f * u2, &sn, &cs);
                            row[c] = init_std * (rad * cs);
                            row[c + 1] = init_std * (rad * sn);
                            mu += row[c] + row[c + 1];
                        }
                    }
                }
                mu *= (1.0f / C);
                float var = 0.f;
                for (int c = 0; c < C; ++c) var = fmaf(row[c] - mu, row[c] - mu, var);
                const float as = alpha * sqrtf(var * (1.0f / C));
                static_for<0, C>([&](auto I) {
                    constexpr int c = decltype(I)::value;
                    row[c] = fmaf(as, (float)__popc(m0 & cand_mask(c)) - shift, row[c]);
                });
            }
        }
        __syncthreads();
        const int n = nb * C, n4 = n >> 2;
        stage_out(d.pi + tb0 * C, s_pi, n);
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = threadIdx.x; i < n4; i += kCtaThreads) {
            if (d.m) __stcs(reinterpret_cast<float4 *>(d.m + tb0 * C) + i, z4);
            if (d.v) __stcs(reinterpret_cast<float4 *>(d.v + tb0 * C) + i, z4);
        }
        if ((n & 3) && threadIdx.x == 0) {
            for (int i = 4 * n4; i < n; ++i) {
                if (d.m) d.m[tb0 * C + i] = 0.f;
                if (d.v) d.v[tb0 * C + i] = 0.f;
            }
        }
    }
}

// Hard pack: one thread per block (tile staged through shared memory).
template <bool kW32>
__global__ void __launch_bounds__(kCtaThreads) pack_kernel(const __grid_constant__ Group grp) {
    __shared__ __align__(16) float s_pi[kTileFloats];
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t tb0 = (t - d.work_begin) * kBlocksPerCta;
        const int nb = (int)imin64(kBlocksPerCta, d.nblocks - tb0);
        __syncthreads();
        stage_in(s_pi, d.pi + tb0 * C, nb * C);
        __syncthreads();
        if ((int)threadIdx.x >= nb) continue;
        const int64_t b = tb0 + threadIdx.x;
        const float *row = s_pi + threadIdx.x * C;
        int k = -1;
        float best = 0.f;
        for (int c = 0; c < C; ++c) {
            const float p = row[c];
            if (p == p && (k < 0 || p > best)) { k = c; best = p; }
        }
        if (k < 0) k = 0;
        uint32_t mask = 0;
        static_for<0, C>([&](auto I) {
            constexpr int c = decltype(I)::value;
            if (c == k) mask = cand_mask(c);
        });
        int pos[4], n = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) if (mask & (1u << j)) pos[n++ & 3] = j;
        static_cast<uint16_t *>(d.pmeta)[b] = (uint16_t)(pos[0] | (pos[1] << 3) | (pos[2] << 6) | (pos[3] << 9));
        if (d.cidx) d.cidx[b] = (uint8_t)k;
        if (kW32) {
            const float *W = static_cast<const float *>(d.W) + b * 8;
            float4 o = make_float4(__ldcs(W + pos[0]), __ldcs(W + pos[1]), __ldcs(W + pos[2]), __ldcs(W + pos[3]));
            __stcs(reinterpret_cast<float4 *>(static_cast<float *>(d.pvals) + b * 4), o);
        } else {
            const uint4 a = ld_stream(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(d.W) + b * 8));
            const uint32_t wv[4] = {a.x, a.y, a.z, a.w};
            uint32_t h[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) h[q] = (wv[pos[q] >> 1] >> (16 * (pos[q] & 1))) & 0xFFFFu;
            __stcs(reinterpret_cast<uint2 *>(static_cast<uint16_t *>(d.pvals) + b * 4),
                   make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16)));
        }
    }
}

}  // namespace k48

// Gumbel noise of arbitrary blocks for inspection: one thread per block, C values each.
__global__ void __launch_bounds__(kThreads) noise_kernel(int C,
                                                         uint64_t seed, uint32_t step,
                                                         const uint64_t *__restrict__ gids,
                                                         int64_t n, float *__restrict__ out) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    load_tab(s_tab);
    __syncthreads();
    const NlogCtx L{s_tab};
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t gid = gids[i];
        for (int gr = 0; gr * 6 < C; ++gr) {
            // the samplers' own path: fields placed as the bits of 1 + eps, two draws per
            // paired evaluation (C is even)
            uint32_t u[6];
            fields21_unit(block_words(seed, gid, step, (uint32_t)gr), u);
            for (int k = 0; k < 6; k += 2) {
                const int c = 6 * gr + k;
                if (c < C) {
                    const float2 g = gumbel_unit2(u[k], u[k + 1], L);
                    out[i * C + c] = g.x;
                    out[i * C + c + 1] = g.y;
                }
            }
        }
    }
}

}  // namespace mllm
