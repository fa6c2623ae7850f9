// kernels_2of4.cuh -- the 2:4 sampler kernels (C = 6 candidates per block of 4 weights).
//
// MaskLLM (paper-graph-ui summary of arXiv 2409.17481): candidate set s.3.2 Eq.2; noise,
// soft index and soft mask s.3.4 Eq.5-Eq.7; regulariser Eq.8; prior Eq.9-Eq.10; hard mask
// s.3.2 "Information flow at inference".
//
// Work mapping: one thread owns a pair of consecutive blocks, so every per-pair access is a
// whole number of 16-byte vectors (W bf16: 16 B, logits/moments: 48 B = 3 x 16 B, X: 16 B).
// A CTA of kThreads threads covers a tile of kThreads pairs; a persistent grid strides over
// the tiles of all matrices of the group. A matrix with an odd block count ends in a
// single-block pair handled by the same code with scalar accesses.
//
// Candidate order (page listing): 0 {0,1}, 1 {0,2}, 2 {0,3}, 3 {1,3}, 4 {1,2}, 5 {2,3}.
#pragma once

#include "device_common.cuh"

namespace mllm {
namespace k24 {

constexpr int C = 6;

// --------------------------------------------------------------------------- pair I/O

template <bool kF32>
__device__ __forceinline__ void load_vals(const void *base, int64_t b0, bool two, float w[8]) {
    if (kF32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + b0 * 4);
        float4 a = ld_stream(p);
        float4 b = two ? ld_stream(p + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
        const uint16_t *q = static_cast<const uint16_t *>(base) + b0 * 4;
        uint4 a;
        if (two) {
            a = ld_stream(reinterpret_cast<const uint4 *>(q));
        } else {
            uint2 h = __ldcs(reinterpret_cast<const uint2 *>(q));
            a = make_uint4(h.x, h.y, 0u, 0u);
        }
        w[0] = bf16lo(a.x); w[1] = bf16hi(a.x); w[2] = bf16lo(a.y); w[3] = bf16hi(a.y);
        w[4] = bf16lo(a.z); w[5] = bf16hi(a.z); w[6] = bf16lo(a.w); w[7] = bf16hi(a.w);
    }
}

template <bool kF32>
__device__ __forceinline__ void store_vals(void *base, int64_t b0, bool two, const float x[8]) {
    if (kF32) {
        float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(base) + b0 * 4);
        st_stream(p, make_float4(x[0], x[1], x[2], x[3]));
        if (two) st_stream(p + 1, make_float4(x[4], x[5], x[6], x[7]));
    } else {
        uint16_t *q = static_cast<uint16_t *>(base) + b0 * 4;
        const uint32_t a = pack_bf16x2(x[0], x[1]), b = pack_bf16x2(x[2], x[3]);
        if (two) {
            st_stream(reinterpret_cast<uint4 *>(q),
                      make_uint4(a, b, pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7])));
        } else {
            __stcs(reinterpret_cast<uint2 *>(q), make_uint2(a, b));
        }
    }
}

// 12 floats of a pair's per-block array (6 when single), 16-byte aligned at even blocks.
__device__ __forceinline__ void load12(const float *base, int64_t b0, bool two, float v[12]) {
    const float4 *p = reinterpret_cast<const float4 *>(base + b0 * C);
    float4 a = ld_stream(p), b, c;
    if (two) {
        b = ld_stream(p + 1);
        c = ld_stream(p + 2);
    } else {
        float2 h = __ldcs(reinterpret_cast<const float2 *>(p + 1));
        b = make_float4(h.x, h.y, 0.f, 0.f);
        c = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y;
    v[6] = b.z; v[7] = b.w; v[8] = c.x; v[9] = c.y; v[10] = c.z; v[11] = c.w;
}

__device__ __forceinline__ void store12(float *base, int64_t b0, bool two, const float v[12]) {
    float4 *p = reinterpret_cast<float4 *>(base + b0 * C);
    st_stream(p, make_float4(v[0], v[1], v[2], v[3]));
    if (two) {
        st_stream(p + 1, make_float4(v[4], v[5], v[6], v[7]));
        st_stream(p + 2, make_float4(v[8], v[9], v[10], v[11]));
    } else {
        __stcs(reinterpret_cast<float2 *>(p + 1), make_float2(v[4], v[5]));
    }
}

// load12 / store12 as six pairs (elements 2k, 2k+1).
__device__ __forceinline__ void load12x2(const float *base, int64_t b0, bool two, float2 v[6]) {
    float t[12];
    load12(base, b0, two, t);
#pragma unroll
    for (int k = 0; k < 6; ++k) v[k] = make_float2(t[2 * k], t[2 * k + 1]);
}
__device__ __forceinline__ void store12x2(float *base, int64_t b0, bool two, const float2 v[6]) {
    float t[12];
#pragma unroll
    for (int k = 0; k < 6; ++k) { t[2 * k] = v[k].x; t[2 * k + 1] = v[k].y; }
    store12(base, b0, two, t);
}

// --------------------------------------------------------------------------- per-block math

// Gumbel noise of the block's six candidates at the step of sc: one Philox call, six fields.
__device__ __forceinline__ void noise6(const StepScalars &sc, uint64_t gid, const NlogCtx &L, float g[6]) {
    if (!sc.noise_on) {
#pragma unroll
        for (int i = 0; i < C; ++i) g[i] = 0.f;
        return;
    }
    uint32_t u[6];
    fields21_unit(block_words(sc, gid, 0u), u);
#pragma unroll
    for (int i = 0; i < C; ++i) g[i] = gumbel_unit(u[i], L);
}

// Unnormalised soft index e_i = 2^((w_i - max w) c2) with w_i = fma(kappa, pi_i, g_i), and
// r = 1 / sum e, so y_i = e_i r (Eq.6).
__device__ __forceinline__ void soft_index(const float *pi, const float g[6], float kappa, float c2,
                                           float e[6], float &r) {
    float w[6];
#pragma unroll
    for (int i = 0; i < C; ++i) w[i] = __fmaf_rn(kappa, pi[i], g[i]);
    const float mx = fmaxf(fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3])), fmaxf(w[4], w[5]));
    // (w_i - max) c2 as one fused step, w_i c2 - fl(max c2): the rounding of fl(max c2) is the
    // same for all six and cancels in the normalisation
    const float mc = __fmul_rn(mx, c2);
#pragma unroll
    for (int i = 0; i < C; ++i) e[i] = ex2_approx(__fmaf_rn(w[i], c2, -mc));
    const float s = __fadd_rn(__fadd_rn(__fadd_rn(e[0], e[1]), __fadd_rn(e[2], e[3])), __fadd_rn(e[4], e[5]));
    r = rcp_approx(s);
}

// Soft mask M_j = sum_{i: j in S_i} y_i (Eq.7) and its complement Mc_j = sum_{i: j not in S_i} y_i.
__device__ __forceinline__ void soft_mask(const float e[6], float r, float ms[4]) {
    ms[0] = (e[0] + e[1] + e[2]) * r;
    ms[1] = (e[0] + e[3] + e[4]) * r;
    ms[2] = (e[1] + e[4] + e[5]) * r;
    ms[3] = (e[2] + e[3] + e[5]) * r;
}
__device__ __forceinline__ void soft_mask_comp(const float e[6], float r, float mc[4]) {
    mc[0] = (e[3] + e[4] + e[5]) * r;
    mc[1] = (e[1] + e[2] + e[5]) * r;
    mc[2] = (e[0] + e[2] + e[3]) * r;
    mc[3] = (e[0] + e[1] + e[4]) * r;
}

// --------------------------------------------------------------------------- paired forms
// (bit-identical to the scalar helpers above; see the paired forms in device_common.cuh)

// noise6 as three pairs (g0 g1), (g2 g3), (g4 g5).
__device__ __forceinline__ void noise6x2(const StepScalars &sc, uint64_t gid, const NlogCtx &L, float2 g[3]) {
    if (!sc.noise_on) {
#pragma unroll
        for (int k = 0; k < 3; ++k) g[k] = make_float2(0.f, 0.f);
        return;
    }
    uint32_t u[6];
    fields21_unit(block_words(sc, gid, 0u), u);
#pragma unroll
    for (int k = 0; k < 3; ++k) g[k] = gumbel_unit2(u[2 * k], u[2 * k + 1], L);
}

// soft_index with the logits and noise as pairs (pi2[k] = (pi_2k, pi_2k+1)).
__device__ __forceinline__ void soft_index2(const float2 pi2[3], const float2 g[3], float kappa, float c2,
                                            float e[6], float &r) {
    float2 w[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) w[k] = __ffma2_rn(f2(kappa), pi2[k], g[k]);
    const float mx = fmaxf(fmaxf(fmaxf(w[0].x, w[0].y), fmaxf(w[1].x, w[1].y)), fmaxf(w[2].x, w[2].y));
    const float mc = __fmul_rn(mx, c2);
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const float2 a = __ffma2_rn(w[k], f2(c2), f2(-mc));
        e[2 * k] = ex2_approx(a.x);
        e[2 * k + 1] = ex2_approx(a.y);
    }
    const float s = __fadd_rn(__fadd_rn(__fadd_rn(e[0], e[1]), __fadd_rn(e[2], e[3])), __fadd_rn(e[4], e[5]));
    r = rcp_approx(s);
}

// AdamW, PyTorch step order, two elements.
__device__ __forceinline__ void adamw2(float2 &p, float2 &m, float2 &v, float2 g, const StepScalars &s) {
    const float2 pd = __fmul2_rn(p, f2(s.decay));
    m = __ffma2_rn(f2(s.beta1), m, __fmul2_rn(f2(s.one_minus_beta1), g));
    v = __ffma2_rn(f2(s.beta2), v, __fmul2_rn(f2(s.one_minus_beta2), __fmul2_rn(g, g)));
    const float2 denom = __ffma2_rn(make_float2(sqrt_approx(v.x), sqrt_approx(v.y)), f2(s.inv_sqrt_bc2), f2(s.eps));
    p = __ffma2_rn(f2(-s.step_size), make_float2(__fdividef(m.x, denom.x), __fdividef(m.y, denom.y)), pd);
}

// AdamW, PyTorch step order, one element.
__device__ __forceinline__ void adamw(float &p, float &m, float &v, float g, const StepScalars &s) {
    const float pd = __fmul_rn(p, s.decay);
    m = __fmaf_rn(s.beta1, m, __fmul_rn(s.one_minus_beta1, g));
    v = __fmaf_rn(s.beta2, v, __fmul_rn(s.one_minus_beta2, __fmul_rn(g, g)));
    const float denom = __fmaf_rn(sqrt_approx(v), s.inv_sqrt_bc2, s.eps);
    p = __fmaf_rn(-s.step_size, __fdividef(m, denom), pd);
}

// --------------------------------------------------------------------------- kernels

// Deterministic reduction of one double per CTA into *out: partials[blockIdx.x] is written,
// the last CTA to arrive (ticket) sums all partials in index order and resets the ticket.
__device__ __forceinline__ void reduce_to_global(float acc, double *partials, unsigned int *ticket,
                                                 double *out, int accumulate) {
    __shared__ double s_w[kThreads / 32];
    __shared__ bool s_last;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_w[warp] = (double)acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int i = 0; i < kThreads / 32; ++i) t += s_w[i];
        partials[blockIdx.x] = t;
        __threadfence();
        const unsigned int prev = atomicAdd(ticket, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    double t = 0.0;
    for (unsigned int i = threadIdx.x; i < gridDim.x; i += kThreads) t += __ldcg(partials + i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
    __syncthreads();
    if (lane == 0) s_w[warp] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (int i = 0; i < kThreads / 32; ++i) tot += s_w[i];
        *out = accumulate ? (*out + tot) : tot;
        *ticket = 0u;
    }
}

template <bool kW32>
__global__ void __launch_bounds__(kThreads) fwd_kernel(const __grid_constant__ Group grp,
                                                       const StepScalars sc, double *partials,
                                                       unsigned int *ticket, double *reg_out,
                                                       int accumulate) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    load_tab(s_tab);
    __syncthreads();
    const NlogCtx L{s_tab};
    float acc = 0.f;
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b0 = ((t - d.work_begin) * kThreads + threadIdx.x) * 2;
        if (b0 >= d.nblocks) continue;
        const bool two = b0 + 1 < d.nblocks;
        float w[8];
        float2 pi[6];
        load_vals<kW32>(d.W, b0, two, w);
        load12x2(d.pi, b0, two, pi);
        float x[8], msv[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 g[3];
            float e[6], r, ms[4];
            noise6x2(sc, d.gid0 + b0 + h, L, g);
            soft_index2(pi + 3 * h, g, sc.kappa, sc.c2, e, r);
            soft_mask(e, r, ms);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float2 xj = __fmul2_rn(make_float2(w[4 * h + 2 * k], w[4 * h + 2 * k + 1]),
                                             make_float2(ms[2 * k], ms[2 * k + 1]));
                x[4 * h + 2 * k] = xj.x;
                x[4 * h + 2 * k + 1] = xj.y;
                msv[4 * h + 2 * k] = ms[2 * k];
                msv[4 * h + 2 * k + 1] = ms[2 * k + 1];
                if (h == 0 || two) {
                    acc = __fmaf_rn(xj.x, xj.x, acc);
                    acc = __fmaf_rn(xj.y, xj.y, acc);
                }
            }
        }
        store_vals<kW32>(d.X, b0, two, x);
        if (d.soft) {
            float4 *sp = reinterpret_cast<float4 *>(d.soft + b0 * 4);
            sp[0] = make_float4(msv[0], msv[1], msv[2], msv[3]);
            if (two) sp[1] = make_float4(msv[4], msv[5], msv[6], msv[7]);
        }
    }
    if (reg_out) reduce_to_global(acc, partials, ticket, reg_out, accumulate);
}

template <bool kW32, bool kG32>
__global__ void __launch_bounds__(kThreads) bwd_adam_kernel(const __grid_constant__ Group grp,
                                                            const StepScalars sc) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    load_tab(s_tab);
    __syncthreads();
    const NlogCtx L{s_tab};
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b0 = ((t - d.work_begin) * kThreads + threadIdx.x) * 2;
        if (b0 >= d.nblocks) continue;
        const bool two = b0 + 1 < d.nblocks;
        float w[8], gw[8];
        float2 pi[6], mo[6], vo[6], grad[6];
        load_vals<kW32>(d.W, b0, two, w);
        load_vals<kG32>(d.G, b0, two, gw);
        load12x2(d.pi, b0, two, pi);
        load12x2(d.m, b0, two, mo);
        load12x2(d.v, b0, two, vo);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 g[3];
            float e[6], r, ms[4], mc[4], P[4], Q[4];
            noise6x2(sc, d.gid0 + b0 + h, L, g);
            soft_index2(pi + 3 * h, g, sc.kappa, sc.c2, e, r);
            soft_mask(e, r, ms);
            soft_mask_comp(e, r, mc);
#pragma unroll
            for (int k = 0; k < 2; ++k) {  // positions 2k, 2k+1
                const float2 wj = make_float2(w[4 * h + 2 * k], w[4 * h + 2 * k + 1]);
                const float2 gj = make_float2(gw[4 * h + 2 * k], gw[4 * h + 2 * k + 1]);
                const float2 msj = make_float2(ms[2 * k], ms[2 * k + 1]);
                const float2 mcj = make_float2(mc[2 * k], mc[2 * k + 1]);
                // u_j = G_j W_j - 2 lambda W_j^2 M_j (G_j W_j is exact for bf16 inputs)
                const float2 u = __ffma2_rn(__fmul2_rn(f2(-sc.two_lambda), __fmul2_rn(wj, wj)), msj, __fmul2_rn(gj, wj));
                const float2 pp = __fmul2_rn(mcj, u), qq = __fmul2_rn(msj, u);
                P[2 * k] = pp.x; P[2 * k + 1] = pp.y;
                Q[2 * k] = qq.x; Q[2 * k + 1] = qq.y;
            }
            float D[6];
            D[0] = (P[0] + P[1]) - (Q[2] + Q[3]);
            D[1] = (P[0] + P[2]) - (Q[1] + Q[3]);
            D[2] = (P[0] + P[3]) - (Q[1] + Q[2]);
            D[3] = (P[1] + P[3]) - (Q[0] + Q[2]);
            D[4] = (P[1] + P[2]) - (Q[0] + Q[3]);
            D[5] = (P[2] + P[3]) - (Q[0] + Q[1]);
            const float cr = __fmul_rn(sc.kappa_over_tau, r);
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                grad[3 * h + k] = __fmul2_rn(__fmul2_rn(f2(cr), make_float2(e[2 * k], e[2 * k + 1])),
                                             make_float2(D[2 * k], D[2 * k + 1]));
                adamw2(pi[3 * h + k], mo[3 * h + k], vo[3 * h + k], grad[3 * h + k], sc);
            }
        }
        store12x2(d.pi, b0, two, pi);
        store12x2(d.m, b0, two, mo);
        store12x2(d.v, b0, two, vo);
        if (d.grad) store12x2(d.grad, b0, two, grad);
    }
}

// Backward + AdamW of step t fused with the forward of step t+1 (mllm_sample_bwd_adam_fwd):
// per pair of blocks, the backward math of bwd_adam_kernel with step t's scalars (sb), then,
// from the updated logits still in registers, the forward math of fwd_kernel with step t+1's
// scalars (sf). W and the logits are read once for both; X of step t+1 is written.
template <bool kW32, bool kG32>
__global__ void __launch_bounds__(kThreads, 3) bwd_adam_fwd_kernel(const __grid_constant__ Group grp,
                                                                const StepScalars sb, const StepScalars sf,
                                                                double *partials, unsigned int *ticket,
                                                                double *reg_out, int accumulate) {
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    load_tab(s_tab);
    __syncthreads();
    const NlogCtx L{s_tab};
    float acc = 0.f;
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b0 = ((t - d.work_begin) * kThreads + threadIdx.x) * 2;
        if (b0 >= d.nblocks) continue;
        const bool two = b0 + 1 < d.nblocks;
        float w[8], gw[8], x[8], msv[8];
        float2 pi[6], mo[6], vo[6];  // pairs (2k, 2k+1); block h holds pairs 3h .. 3h+2
        load_vals<kW32>(d.W, b0, two, w);
        load_vals<kG32>(d.G, b0, two, gw);
        load12x2(d.pi, b0, two, pi);
        load12x2(d.m, b0, two, mo);
        load12x2(d.v, b0, two, vo);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint64_t gid = d.gid0 + b0 + h;
            {   // backward + AdamW, step t
                float2 g[3];
                float e[6], r, ms[4], mc[4], P[4], Q[4];
                noise6x2(sb, gid, L, g);
                soft_index2(pi + 3 * h, g, sb.kappa, sb.c2, e, r);
                soft_mask(e, r, ms);
                soft_mask_comp(e, r, mc);
#pragma unroll
                for (int k = 0; k < 2; ++k) {  // positions 2k, 2k+1
                    const float2 wj = make_float2(w[4 * h + 2 * k], w[4 * h + 2 * k + 1]);
                    const float2 gj = make_float2(gw[4 * h + 2 * k], gw[4 * h + 2 * k + 1]);
                    const float2 msj = make_float2(ms[2 * k], ms[2 * k + 1]);
                    const float2 mcj = make_float2(mc[2 * k], mc[2 * k + 1]);
                    // u_j = G_j W_j - 2 lambda W_j^2 M_j, as fma(-(2 lambda W_j^2), M_j, G_j W_j)
                    const float2 u = __ffma2_rn(__fmul2_rn(f2(-sb.two_lambda), __fmul2_rn(wj, wj)), msj, __fmul2_rn(gj, wj));
                    const float2 pp = __fmul2_rn(mcj, u), qq = __fmul2_rn(msj, u);
                    P[2 * k] = pp.x; P[2 * k + 1] = pp.y;
                    Q[2 * k] = qq.x; Q[2 * k + 1] = qq.y;
                }
                float D[6];
                D[0] = (P[0] + P[1]) - (Q[2] + Q[3]);
                D[1] = (P[0] + P[2]) - (Q[1] + Q[3]);
                D[2] = (P[0] + P[3]) - (Q[1] + Q[2]);
                D[3] = (P[1] + P[3]) - (Q[0] + Q[2]);
                D[4] = (P[1] + P[2]) - (Q[0] + Q[3]);
                D[5] = (P[2] + P[3]) - (Q[0] + Q[1]);
                const float cr = __fmul_rn(sb.kappa_over_tau, r);
                float2 grad[3];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    grad[k] = __fmul2_rn(__fmul2_rn(f2(cr), make_float2(e[2 * k], e[2 * k + 1])),
                                         make_float2(D[2 * k], D[2 * k + 1]));
                    adamw2(pi[3 * h + k], mo[3 * h + k], vo[3 * h + k], grad[k], sb);
                }
                if (d.grad && (h == 0 || two)) {
                    float2 *gp = reinterpret_cast<float2 *>(d.grad + (b0 + h) * C);
                    gp[0] = grad[0];
                    gp[1] = grad[1];
                    gp[2] = grad[2];
                }
            }
            {   // forward, step t+1, from the updated logits
                float2 g[3];
                float e[6], r, ms[4];
                noise6x2(sf, gid, L, g);
                soft_index2(pi + 3 * h, g, sf.kappa, sf.c2, e, r);
                soft_mask(e, r, ms);
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float2 xj = __fmul2_rn(make_float2(w[4 * h + 2 * k], w[4 * h + 2 * k + 1]),
                                                 make_float2(ms[2 * k], ms[2 * k + 1]));
                    x[4 * h + 2 * k] = xj.x;
                    x[4 * h + 2 * k + 1] = xj.y;
                    msv[4 * h + 2 * k] = ms[2 * k];
                    msv[4 * h + 2 * k + 1] = ms[2 * k + 1];
                    if (h == 0 || two) {
                        acc = __fmaf_rn(xj.x, xj.x, acc);
                        acc = __fmaf_rn(xj.y, xj.y, acc);
                    }
                }
            }
        }
        store12x2(d.pi, b0, two, pi);
        store12x2(d.m, b0, two, mo);
        store12x2(d.v, b0, two, vo);
        store_vals<kW32>(d.X, b0, two, x);
        if (d.soft) {
            float4 *sp = reinterpret_cast<float4 *>(d.soft + b0 * 4);
            sp[0] = make_float4(msv[0], msv[1], msv[2], msv[3]);
            if (two) sp[1] = make_float4(msv[4], msv[5], msv[6], msv[7]);
        }
    }
    if (reg_out) reduce_to_global(acc, partials, ticket, reg_out, accumulate);
}

// Prior candidate of one block: the two positions of largest |w| (ties: lower position;
// NaN ranks last) as a 4-bit keep mask.
__device__ __forceinline__ uint32_t top2_mask(const float *w) {
    float key[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) key[j] = (w[j] != w[j]) ? -1.0f : fabsf(w[j]);
    uint32_t mask = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        int rank = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k != j && (key[k] > key[j] || (key[k] == key[j] && k < j))) ++rank;
        if (rank < 2) mask |= 1u << j;
    }
    return mask;
}

// Keep masks of the candidates in the page's order (bit j = position j).
__device__ __forceinline__ uint32_t cand_mask(int i) {
    return (0xC6A953u >> (4 * i)) & 0xFu;  // 0x3, 0x5, 0x9, 0xA, 0x6, 0xC
}

// Prior initialisation. kFromIdx = false: M0 is the magnitude prior of the block's weights;
// kFromIdx = true: M0 is candidate d.prior[b] (an index >= C: no prior, sim = 0).
template <bool kW32, bool kFromIdx>
__global__ void __launch_bounds__(kThreads) prior_kernel(const __grid_constant__ Group grp,
                                                         float alpha, float init_std, uint64_t seed) {
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b0 = ((t - d.work_begin) * kThreads + threadIdx.x) * 2;
        if (b0 >= d.nblocks) continue;
        const bool two = b0 + 1 < d.nblocks;
        float w[8], pi[12], zero[12];
        if (!kFromIdx) load_vals<kW32>(d.W, b0, two, w);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float sim[6];
            if (kFromIdx) {
                const uint32_t k = (h == 0 || two) ? d.prior[b0 + h] : 255u;
                const uint32_t m0 = cand_mask(k < C ? (int)k : 0);
#pragma unroll
                for (int i = 0; i < C; ++i) sim[i] = (k < C) ? (float)__popc(m0 & cand_mask(i)) - 1.0f : 0.0f;
            } else {
                const uint32_t m0 = top2_mask(w + 4 * h);
#pragma unroll
                for (int i = 0; i < C; ++i) sim[i] = (float)__popc(m0 & cand_mask(i)) - 1.0f;  // N*N/M = 1
            }
            if (init_std == 0.f) {
#pragma unroll
                for (int i = 0; i < C; ++i) pi[6 * h + i] = alpha * sim[i];
            } else {
                uint32_t f[6];
                fields21(block_words(seed, d.gid0 + b0 + h, kInitStep, 0u), f);
                float p0[6];
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const float u1 = uniform_from_field(f[2 * q]);
                    const float u2 = uniform_from_field(f[2 * q + 1]);
                    const float rad = sqrtf(-2.0f * logf(u1));
                    float sn, cs;
                    sincospif(2.0f * u2, &sn, &cs);
                    p0[2 * q] = init_std * (rad * cs);
                    p0[2 * q + 1] = init_std * (rad * sn);
                }
                float mu = 0.f;
#pragma unroll
                for (int i = 0; i < C; ++i) mu += p0[i];
                mu *= (1.0f / 6.0f);
                float var = 0.f;
#pragma unroll
                for (int i = 0; i < C; ++i) var = fmaf(p0[i] - mu, p0[i] - mu, var);
                const float sigma = sqrtf(var * (1.0f / 6.0f));
#pragma unroll
                for (int i = 0; i < C; ++i) pi[6 * h + i] = fmaf(alpha * sigma, sim[i], p0[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 12; ++i) zero[i] = 0.f;
        store12(d.pi, b0, two, pi);
        if (d.m) store12(d.m, b0, two, zero);
        if (d.v) store12(d.v, b0, two, zero);
    }
}

// First index of the largest logit; NaN never wins; all-NaN gives 0.
__device__ __forceinline__ int argmax6(const float *p) {
    int k = -1;
    float best = 0.f;
#pragma unroll
    for (int i = 0; i < C; ++i) {
        const bool ok = (p[i] == p[i]) && (k < 0 || p[i] > best);
        if (ok) { k = i; best = p[i]; }
    }
    return k < 0 ? 0 : k;
}

// Hard pack: one thread per metadata word (8 blocks of one row).
template <bool kW32>
__global__ void __launch_bounds__(kThreads) pack_kernel(const __grid_constant__ Group grp) {
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t bpr = d.cols / 4, words = (bpr + 7) / 8;
        const int64_t widx = (t - d.work_begin) * kThreads + threadIdx.x;
        if (widx >= d.rows * words) continue;
        const int64_t row = widx / words, q0 = (widx % words) * 8;
        const int nb = (int)imin64(8, bpr - q0);
        uint32_t word = 0;
        for (int u = 0; u < nb; ++u) {
            const int64_t q = q0 + u, blk = row * bpr + q;
            const float2 *pp = reinterpret_cast<const float2 *>(d.pi + blk * C);
            const float2 a = __ldcs(pp), b = __ldcs(pp + 1), c = __ldcs(pp + 2);
            const float p[6] = {a.x, a.y, b.x, b.y, c.x, c.y};
            const int k = argmax6(p);
            const uint32_t km = cand_mask(k);
            const int p0 = __ffs(km) - 1, p1 = 31 - __clz(km);
            word |= (uint32_t)(p0 | (p1 << 2)) << (4 * u);
            if (d.cidx) d.cidx[blk] = (uint8_t)k;
            const int64_t src = row * d.cols + q * 4, dst = row * (bpr * 2) + q * 2;
            if (kW32) {
                const float *W = static_cast<const float *>(d.W);
                float *V = static_cast<float *>(d.pvals);
                V[dst] = __ldcs(W + src + p0);
                V[dst + 1] = __ldcs(W + src + p1);
            } else {
                const uint16_t *W = static_cast<const uint16_t *>(d.W);
                uint16_t *V = static_cast<uint16_t *>(d.pvals);
                V[dst] = W[src + p0];
                V[dst + 1] = W[src + p1];
            }
        }
        static_cast<uint32_t *>(d.pmeta)[widx] = word;
    }
}

// Hard pack when every row's block count is a multiple of 8, so each metadata word covers
// 8 consecutive blocks of one row and its index is (global block)/8: one thread per pair of
// blocks with whole-vector loads; four consecutive threads (lanes 4i..4i+3) assemble a word
// with two shuffles and the first of them stores it.
__device__ __forceinline__ uint32_t half_of(const uint4 &a, int idx) {  // bf16 idx of 8
    const uint32_t w = (idx & 4) ? ((idx & 2) ? a.w : a.z) : ((idx & 2) ? a.y : a.x);
    return (idx & 1) ? (w >> 16) : (w & 0xFFFFu);
}

template <bool kW32>
__global__ void __launch_bounds__(kThreads) pack_pairs_kernel(const __grid_constant__ Group grp) {
    const int lane = threadIdx.x & 31;
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b0 = ((t - d.work_begin) * kThreads + threadIdx.x) * 2;
        const bool valid = b0 < d.nblocks;  // nblocks is a multiple of 8 on this path
        uint32_t byte = 0;
        if (valid) {
            float pi[12];
            load12(d.pi, b0, true, pi);
            const int k0 = argmax6(pi), k1 = argmax6(pi + 6);
            const uint32_t m0 = cand_mask(k0), m1 = cand_mask(k1);
            const int a0 = __ffs(m0) - 1, c0 = 31 - __clz(m0);
            const int a1 = __ffs(m1) - 1, c1 = 31 - __clz(m1);
            byte = (uint32_t)(a0 | (c0 << 2)) | ((uint32_t)(a1 | (c1 << 2)) << 4);
            if (kW32) {
                const float *W = static_cast<const float *>(d.W) + b0 * 4;
                st_stream(reinterpret_cast<float4 *>(static_cast<float *>(d.pvals) + b0 * 2),
                          make_float4(__ldcs(W + a0), __ldcs(W + c0), __ldcs(W + 4 + a1), __ldcs(W + 4 + c1)));
            } else {
                const uint4 a = ld_stream(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(d.W) + b0 * 4));
                __stcs(reinterpret_cast<uint2 *>(static_cast<uint16_t *>(d.pvals) + b0 * 2),
                       make_uint2(half_of(a, a0) | (half_of(a, c0) << 16),
                                  half_of(a, 4 + a1) | (half_of(a, 4 + c1) << 16)));
            }
            if (d.cidx) *reinterpret_cast<uint16_t *>(d.cidx + b0) = (uint16_t)(k0 | (k1 << 8));
        }
        uint32_t word = byte << (8 * (lane & 3));
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
        word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
        if (valid && (lane & 3) == 0) static_cast<uint32_t *>(d.pmeta)[b0 / 8] = word;
    }
}

}  // namespace k24
}  // namespace mllm
