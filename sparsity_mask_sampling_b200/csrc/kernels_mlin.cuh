// kernels_mlin.cuh -- the sampler inside the frozen network's linear layer, on the
// fifth-generation tensor cores.
//
// MaskLLM trains only the logits: every linear layer of the frozen network multiplies its
// input by the soft-masked weight W . M on the forward pass, and the gradient that reaches the
// weight goes on to the logits (paper-graph-ui summary of arXiv 2409.17481, s.3.2 "Frozen LLM
// Backbone"; s.3.4 Eq.5-Eq.8). The kernels here do that layer's work without ever writing the
// soft-masked weight X = W . M or its gradient G = dL/dX to global memory:
//
//   masked_linear_fwd_kernel: Y = A X^T for activations A [T, cols]. Producer warps run the
//     sampler's forward (noise, soft index, soft mask, bf16 rounding: the same arithmetic as
//     the 2:4 forward kernel, so X is bit-identical to mllm_sample_fwd's) straight into the
//     MMA's shared-memory operand tile; the regulariser is reduced alongside.
//   masked_linear_bwd_adam_kernel: G = dY^T A, the layer's weight gradient, on the tensor
//     cores (both operands token-major in memory, i.e. MN-major for the MMA); its epilogue
//     moves each 128 x 128 tile of G from tensor memory to shared memory and runs the 2:4
//     backward + AdamW of the tile's blocks on it (the arithmetic of the 2:4 backward kernel
//     with G in fp32), so G never reaches global memory.
//
// Tile: 128 rows of W (the MMA's M) x all kN token columns (its N, the tokens rounded up) x
// 64 columns of W per pipeline stage (four MMAs of K = 16). Per stage the copy warp lands the
// kN x 64 box of A (128-byte swizzle, K-major) on the stage's "full" barrier; the 256 producer
// threads, once it has landed (which means the MMAs that last read the stage are complete),
// write the 128 x 64 bf16 tile of X in the same K-major 128-byte-swizzled layout, fence it
// for the tensor cores and arrive on the stage's "generated" barrier; the MMA warp then issues
// the stage's four MMAs and commits them to the stage's "empty" barrier, which releases the
// stage to the copy warp. At the end of a tile the producers read the accumulator from tensor
// memory and store Y (or a partial tile). Work split (stream-K over the 64-column chunks of
// all tiles of all matrices, partial tiles added by the last CTA to arrive), bounded waits,
// abort flag and wind-down follow the serving kernels of kernels_umma.cuh.
#pragma once

#include "kernels_2of4.cuh"
#include "kernels_umma.cuh"

namespace mllm {
namespace mlin {

using spl::fence_proxy_async;
using spl::globaltimer_ns;
using spl::kTmWaitNs;
using spl::mbar_arrive;
using spl::mbar_arrive_tx;
using spl::mbar_init;
using spl::mbar_try_wait;
using spl::tc_fence_after;
using spl::tc_fence_before;
using spl::tm_wait;
using spl::tma_load_2d;
using spl::tmem_ld16;
using spl::tmem_ld8;
using spl::um_bar;
using spl::um_bar_or;
using spl::um_desc;
using spl::um_wait;
using spl::umma_commit;
using spl::umma_dense;

constexpr int kRows = 128;          // MMA M: rows of W per tile
constexpr int kChunk = 64;          // columns of W per stage (one 128-byte atom of bf16)
constexpr int kProdWarps = 16;      // producer / epilogue warps
constexpr int kProd = 32 * kProdWarps;
constexpr int kThreads = kProd + 64;  // + the copy warp and the MMA warp
constexpr int kStages = 3;
constexpr int kMaxTokens = 256;     // one MMA's N (the forward)
constexpr int kMaxBwdTokens = 1 << 20;  // the backward's K: tokens in 64-token stages
constexpr int kMaxCtas = 160;       // grid cap (one CTA per SM); sizes the partial-tile workspace

template <int kN> constexpr int xbox_bytes() { return kN * 128; }
template <int kN> constexpr int stage_bytes() { return kRows * 128 + xbox_bytes<kN>(); }
template <int kN> constexpr int smem_bytes() { return kStages * stage_bytes<kN>() + 1024; }
template <int kN> constexpr unsigned tmem_cols() { return kN < 32 ? 32u : (unsigned)kN; }

// Workspace: partial tiles (two slots per CTA, 128 rows x kMaxTokens), one completion ticket
// per CTA, the regulariser's ticket and per-CTA partials, and the error word.
constexpr size_t kPartFloats = (size_t)kRows * kMaxTokens;
constexpr size_t kPartBytes = (size_t)kMaxCtas * 2 * kPartFloats * sizeof(float);
constexpr size_t kTicketOff = kPartBytes;
constexpr size_t kRegTicketOff = kTicketOff + (size_t)kMaxCtas * sizeof(unsigned int);
constexpr size_t kRegPartOff = kRegTicketOff + 16;
constexpr size_t kErrOff = kRegPartOff + (size_t)kMaxCtas * sizeof(double);
constexpr size_t kWorkspaceBytes = kErrOff + 16;

struct Op {
    const void *W;      // bf16 [rows, cols]
    float *pi;          // [rows*cols/4, 6] logits
    float *m, *v;       // AdamW moments (backward)
    float *y;           // fp32 [tokens, rows] (forward)
    void *X;            // bf16 [rows, cols] soft-masked weights (forward, optional, for inspection)
    float *soft;        // fp32 [rows, cols] soft mask (forward, optional)
    float *grad;        // fp32 [rows*cols/4, 6] logit gradient (backward, optional)
    uint64_t gid0;
    int64_t rows, cols;
    int64_t nch;          // 64-column chunks per tile
    int64_t ntiles;       // tiles of 128 rows
    int64_t chunk_begin;  // first chunk of this matrix in the launch's sequence
};

struct Group {
    int32_t n;
    int32_t tokens;
    int64_t total_chunks;
    Op d[kMaxMats];
    CUtensorMap x[kMaxMats];  // activations bf16 [tokens, cols], box 64 x kN, 128-byte swizzle
};

struct Cur {
    int op;
    int64_t tile, j;
};

__device__ __forceinline__ Cur decode(const Group &g, int64_t c) {
    int i = 0;
    while (i + 1 < g.n && c >= g.d[i + 1].chunk_begin) ++i;
    const int64_t r = c - g.d[i].chunk_begin;
    return Cur{i, r / g.d[i].nch, r % g.d[i].nch};
}

__device__ __forceinline__ void advance(const Group &g, Cur &c) {
    if (++c.j == g.d[c.op].nch) {
        c.j = 0;
        if (++c.tile == g.d[c.op].ntiles) {
            c.tile = 0;
            ++c.op;
        }
    }
}

// The producers' part of a stage: rows r0 + 64 i (i < 2) and pair slot c (columns 8c .. 8c+7
// of the chunk) of the 128 x 64 tile of X, computed by the 2:4 forward's arithmetic (k24) and
// written as one 16-byte chunk at its 128-byte-swizzled place. Rows past the matrix are zero.
constexpr int kRowStep = kProd / 8;            // rows a producer steps by (8 pair slots per row)
constexpr int kPairsPerThread = kRows / kRowStep;
__device__ __forceinline__ void gen_stage(unsigned char *tile, const Op &d, int64_t row_tile, int64_t j, int c,
                                          int r0, const StepScalars &sc, const NlogCtx &L, float &acc) {
    const int64_t bpr = d.cols >> 2;
#pragma unroll
    for (int i = 0; i < kPairsPerThread; ++i) {
        const int r = r0 + kRowStep * i;
        const int64_t row = row_tile * kRows + r;
        uint4 packed = make_uint4(0u, 0u, 0u, 0u);
        if (row < d.rows) {
            const int64_t b0 = row * bpr + ((j * kChunk + 8 * c) >> 2);  // even: a pair of blocks
            float w[8], x[8], msv[8];
            float2 pi[6];
            k24::load_vals<false>(d.W, b0, true, w);
            k24::load12x2(d.pi, b0, true, pi);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float2 g[3];
                float e[6], rr, ms[4];
                k24::noise6x2(sc, d.gid0 + b0 + h, L, g);
                k24::soft_index2(pi + 3 * h, g, sc.kappa, sc.c2, e, rr);
                k24::soft_mask(e, rr, ms);
#pragma unroll
                for (int q = 0; q < 4; q += 2) {
                    const float2 xq = __fmul2_rn(make_float2(w[4 * h + q], w[4 * h + q + 1]),
                                                 make_float2(ms[q], ms[q + 1]));
                    x[4 * h + q] = xq.x;
                    x[4 * h + q + 1] = xq.y;
                    msv[4 * h + q] = ms[q];
                    msv[4 * h + q + 1] = ms[q + 1];
                    acc = __fmaf_rn(xq.x, xq.x, acc);
                    acc = __fmaf_rn(xq.y, xq.y, acc);
                }
            }
            packed = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                pack_bf16x2(x[6], x[7]));
            if (d.X) st_stream(reinterpret_cast<uint4 *>(static_cast<uint16_t *>(d.X) + b0 * 4), packed);
            if (d.soft) {
                float4 *sp = reinterpret_cast<float4 *>(d.soft + b0 * 4);
                sp[0] = make_float4(msv[0], msv[1], msv[2], msv[3]);
                sp[1] = make_float4(msv[4], msv[5], msv[6], msv[7]);
            }
        }
        *reinterpret_cast<uint4 *>(tile + r * 128 + ((c ^ (r & 7)) << 4)) = packed;
    }
}

// Regulariser: per-thread fp32 partials -> one double per CTA (fixed order) -> the last CTA
// to arrive adds the per-CTA doubles in index order and resets the ticket. All threads call it.
__device__ __forceinline__ void reduce_reg(float acc, double *partials, unsigned int *ticket, double *out,
                                           int accumulate) {
    __shared__ double s_w[kThreads / 32];
    __shared__ bool s_last_reg;
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
        s_last_reg = (atomicAdd(ticket, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last_reg) return;
    __threadfence();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (unsigned int i = 0; i < gridDim.x; ++i) tot += __ldcg(partials + i);
        *out = accumulate ? (*out + tot) : tot;
        *ticket = 0u;
    }
}

template <int kN>
__device__ __forceinline__ void store_cols(const Op &d, int64_t tile, int q, int lane, int tok0, const float *v,
                                           int n, int tokens) {
    const int64_t r = tile * kRows + 32 * q + lane;
    if (r >= d.rows) return;
    for (int i = 0; i < n; ++i)
        if (tok0 + i < tokens) d.y[(int64_t)(tok0 + i) * d.rows + r] = v[i];
}

template <int kN>
__global__ void __launch_bounds__(kThreads, 1) masked_linear_fwd_kernel(const __grid_constant__ Group grp,
                                                                        const StepScalars sc, unsigned char *ws,
                                                                        double *reg_out, int accumulate) {
    static_assert(kN % 32 == 0 && kN >= 32 && kN <= kMaxTokens, "N of an M = 128 MMA");
    static_assert(kN % (8 * (kProdWarps / 4)) == 0, "each epilogue warp takes a multiple of 8 token columns");
    static_assert(smem_bytes<kN>() + 2 * kNlogEntries * 4 + 1024 <= 232448, "fits one SM");
    constexpr int kD = kStages, kStage = stage_bytes<kN>();
    constexpr uint32_t kIdesc = spl::u8_idesc<kN>();  // dense, f32 accumulator, bf16 K-major, M = 128
    constexpr int kSlices = kProdWarps / 4;              // epilogue warps per TMEM lane quarter
    constexpr int kHalf = kN / kSlices;                  // token columns per epilogue warp (a multiple of 8)
    extern __shared__ unsigned char s_dyn_ml[];
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    __shared__ __align__(8) unsigned long long s_full[kD], s_empty[kD], s_gen[kD], s_acc;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    __shared__ int s_last;
    float *part = reinterpret_cast<float *>(ws);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(ws + kTicketOff);
    unsigned int *err = reinterpret_cast<unsigned int *>(ws + kErrOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t total = grp.total_chunks;
    const int64_t G = gridDim.x, cta = blockIdx.x;  // the host launches at most total_chunks CTAs
    const int64_t lo = cta * total / G, hi = (cta + 1) * total / G;
    const int n = (int)(hi - lo);
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_ml);
    const unsigned pad = (1024u - (dyn_s & 1023u)) & 1023u;
    unsigned char *ring = s_dyn_ml + pad;
    const unsigned ring_s = dyn_s + pad;
    const unsigned full0 = (unsigned)__cvta_generic_to_shared(&s_full[0]);
    const unsigned empty0 = (unsigned)__cvta_generic_to_shared(&s_empty[0]);
    const unsigned gen0 = (unsigned)__cvta_generic_to_shared(&s_gen[0]);
    const unsigned accb = (unsigned)__cvta_generic_to_shared(&s_acc);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kD; ++s) {
            mbar_init(full0 + 8 * s, 1u);
            mbar_init(empty0 + 8 * s, 1u);
            mbar_init(gen0 + 8 * s, (unsigned)kProd);  // every producer thread arrives once per stage
        }
        mbar_init(accb, 1u);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    load_tab(s_tab);
    if (warp == 0) {
        const unsigned dst = (unsigned)__cvta_generic_to_shared(&s_tmem);
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                     "r"(tmem_cols<kN>())
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;
    float acc = 0.f;

    if (warp == kProdWarps) {
        // ------------------------------------------------------------ copy warp
        Cur ld = decode(grp, lo);
        int issued = 0;
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            if (f >= kD && !um_wait(empty0 + 8 * s, ((f / kD) - 1) & 1, &s_abort)) {
                if (lane == 0 && !s_abort) {
                    atomicOr(err, 1u);
                    s_abort = 1;
                }
                break;
            }
            if (lane == 0) {
                fence_proxy_async();
                mbar_arrive_tx(full0 + 8 * s, (unsigned)xbox_bytes<kN>());
                tma_load_2d(ring_s + s * kStage + kRows * 128, &grp.x[ld.op], (int)(kChunk * ld.j), 0, full0 + 8 * s);
            }
            ++issued;
            advance(grp, ld);
        }
        for (int s = 0; s < kD && s < issued; ++s) {  // every copy has landed (bounded) before exit
            const int last = s + ((issued - 1 - s) / kD) * kD;
            tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == kProdWarps + 1) {
        // ------------------------------------------------------------ MMA warp
        Cur cc = decode(grp, lo);
        bool fresh = true;
        int commits = 0;
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            if (!um_wait(gen0 + 8 * s, (f / kD) & 1, &s_abort)) {
                if (lane == 0 && !s_abort) {
                    atomicOr(err, 1u);
                    s_abort = 1;
                }
                break;
            }
            const Op &d = grp.d[cc.op];
            const bool piece_end = (cc.j == d.nch - 1) || (f == n - 1);
            if (lane == 0) {
                tc_fence_after();
                const unsigned st = ring_s + s * kStage;
                const uint64_t a0 = um_desc(st), b0 = um_desc(st + kRows * 128);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    umma_dense(tbase, a0 + (uint64_t)(2 * k), b0 + (uint64_t)(2 * k), kIdesc,
                               (fresh && k == 0) ? 0u : 1u);
                umma_commit(empty0 + 8 * s);
                if (piece_end) umma_commit(accb);
            }
            __syncwarp();
            ++commits;
            fresh = piece_end;
            advance(grp, cc);
        }
        if (commits > 0) {  // every MMA has completed (bounded) before the tensor memory is released
            const int f = commits - 1;
            tm_wait(empty0 + 8 * (f % kD), (f / kD) & 1);
        }
    } else {
        // ------------------------------------------------------------ producer / epilogue warps
        const NlogCtx L{s_tab};
        const int pc = threadIdx.x & 7, r0 = threadIdx.x >> 3;
        const int q = warp & 3, ch = warp >> 2;  // TMEM lane quarter, token slice of the epilogue
        const unsigned tq = tbase + ((unsigned)(32 * q) << 16) + (unsigned)(ch * kHalf);
        Cur cc = decode(grp, lo);
        unsigned acc_phase = 0u;
        bool failed = false;
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            const Op &d = grp.d[cc.op];
            if (!failed) {
                // the stage's activations have landed, so the MMAs that last read it are done
                if (um_wait(full0 + 8 * s, (f / kD) & 1, &s_abort)) {
                    gen_stage(ring + s * kStage, d, cc.tile, cc.j, pc, r0, sc, L, acc);
                    fence_proxy_async();  // the tile, written here, is read by the tensor cores
                    mbar_arrive(gen0 + 8 * s);
                } else {
                    failed = true;
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                }
            }
            const bool piece_end = (cc.j == d.nch - 1) || (f == n - 1);
            if (piece_end) {
                const bool acc_ok = !failed && um_wait(accb, acc_phase, &s_abort);
                acc_phase ^= 1u;
                if (um_bar_or<kProd>(!acc_ok)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                const int64_t a = d.chunk_begin + cc.tile * d.nch, b = a + d.nch;
                const int64_t c1 = ((a + 1) * G - 1) / total, c2 = (b * G - 1) / total;
                const int tok0 = ch * kHalf;
                if (c1 == c2) {
#pragma unroll 1
                    for (int k = 0; k < kHalf; k += 8) {
                        float v[8];
                        tmem_ld8(tq + k, v);
                        store_cols<kN>(d, cc.tile, q, lane, tok0 + k, v, 8, grp.tokens);
                    }
                    tc_fence_before();  // these reads precede the next piece's first MMA
                } else {
                    const int64_t lo1 = c1 * total / G;
                    const int slot = (cta == c1 && lo1 < a) ? 1 : 0;
                    float *mine = part + (size_t)(cta * 2 + slot) * kPartFloats + (size_t)tok0 * kRows + 32 * q + lane;
#pragma unroll 1
                    for (int k = 0; k < kHalf; k += 8) {
                        float v[8];
                        tmem_ld8(tq + k, v);
#pragma unroll
                        for (int i = 0; i < 8; ++i) __stcg(mine + (size_t)(k + i) * kRows, v[i]);
                    }
                    tc_fence_before();
                    __threadfence();
                    um_bar<kProd>();
                    if (threadIdx.x == 0) s_last = (atomicAdd(tickets + c1, 1u) == (unsigned int)(c2 - c1));
                    um_bar<kProd>();
                    if (s_last) {
                        __threadfence();
#pragma unroll 1
                        for (int k = 0; k < kHalf; k += 8) {
                            float sum[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) sum[i] = 0.f;
                            for (int64_t qq = c1; qq <= c2; ++qq) {
                                const int sid = (qq == c1 && lo1 < a) ? 1 : 0;
                                const float *p = part + (size_t)(qq * 2 + sid) * kPartFloats +
                                                 (size_t)(tok0 + k) * kRows + 32 * q + lane;
#pragma unroll
                                for (int i = 0; i < 8; ++i) sum[i] += __ldcg(p + (size_t)i * kRows);
                            }
                            store_cols<kN>(d, cc.tile, q, lane, tok0 + k, sum, 8, grp.tokens);
                        }
                        um_bar<kProd>();
                        if (threadIdx.x == 0) tickets[c1] = 0u;
                    }
                }
            }
            advance(grp, cc);
        }
        if (failed && threadIdx.x == 0 && !s_abort) {
            atomicOr(err, 1u);
            s_abort = 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(tmem_cols<kN>())
                     : "memory");
    }
    if (reg_out)
        reduce_reg(acc, reinterpret_cast<double *>(ws + kRegPartOff), reinterpret_cast<unsigned int *>(ws + kRegTicketOff),
                   reg_out, accumulate);
}

// ------------------------------------------------------------------ backward: G = dY^T A + AdamW

constexpr int kBwdCols = 128;                   // MMA N: columns of W per tile (32 blocks per row)
constexpr int kBwdK = 64;                       // tokens per stage (four MMAs of K = 16)
constexpr int kBwdStageBytes = 4 * 64 * 128;    // dY: two 64-row boxes, A: two 64-column boxes
constexpr int kGPitch = kBwdCols + 4;           // fp32 row pitch of the tile of G in shared memory
constexpr int kBwdSmem = kStages * kBwdStageBytes + kRows * kGPitch * 4 + 2048;
constexpr unsigned kBwdTmemCols = 128;

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle: 64 elements of
// M (or N) per 128-byte row, one row per k, eight k-rows per 1024-byte atom (stride between
// those 8-row groups: 1024 bytes), the second 64-element half of M (or N) 8192 bytes further.
__device__ __forceinline__ uint64_t mn_desc(unsigned saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(8192 >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16, dense, f32 accumulator, bf16 A and B, both MN-major, N = 128, M = 128.
constexpr uint32_t kBwdIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                               ((uint32_t)(kBwdCols >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);

struct BwdGroup {
    int32_t n;
    int32_t tokens;
    int64_t total_tiles;
    int64_t tile_begin[kMaxMats];   // first tile of each matrix in the launch's sequence
    int64_t ctiles[kMaxMats];       // column tiles per row tile
    Op d[kMaxMats];
    CUtensorMap dy[kMaxMats];       // bf16 [tokens, rows], box 64 rows x 64 tokens, 128-byte swizzle
    CUtensorMap x[kMaxMats];        // bf16 [tokens, cols], box 64 columns x 64 tokens
};

__device__ __forceinline__ void bwd_decode(const BwdGroup &g, int64_t t, int &op, int64_t &rt, int64_t &ct) {
    int i = 0;
    while (i + 1 < g.n && t >= g.tile_begin[i + 1]) ++i;
    const int64_t r = t - g.tile_begin[i];
    op = i;
    rt = r / g.ctiles[i];
    ct = r % g.ctiles[i];
}

// Backward + AdamW of one pair of blocks (row `row`, blocks b0, b0 + 1 of the matrix) with the
// pair's eight entries of G (fp32) from gp: the arithmetic of k24::bwd_adam_kernel.
__device__ __forceinline__ void pair_bwd_adam(const Op &d, int64_t b0, const float *gp, const StepScalars &sc,
                                              const NlogCtx &L) {
    float w[8], gw[8];
    float2 pi[6], mo[6], vo[6], grad[6];
    k24::load_vals<false>(d.W, b0, true, w);
    const float4 g0 = *reinterpret_cast<const float4 *>(gp), g1 = *reinterpret_cast<const float4 *>(gp + 4);
    gw[0] = g0.x; gw[1] = g0.y; gw[2] = g0.z; gw[3] = g0.w; gw[4] = g1.x; gw[5] = g1.y; gw[6] = g1.z; gw[7] = g1.w;
    k24::load12x2(d.pi, b0, true, pi);
    k24::load12x2(d.m, b0, true, mo);
    k24::load12x2(d.v, b0, true, vo);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float2 g[3];
        float e[6], r, ms[4], mc[4], P[4], Q[4];
        k24::noise6x2(sc, d.gid0 + b0 + h, L, g);
        k24::soft_index2(pi + 3 * h, g, sc.kappa, sc.c2, e, r);
        k24::soft_mask(e, r, ms);
        k24::soft_mask_comp(e, r, mc);
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // positions 2k, 2k+1
            const float2 wj = make_float2(w[4 * h + 2 * k], w[4 * h + 2 * k + 1]);
            const float2 gj = make_float2(gw[4 * h + 2 * k], gw[4 * h + 2 * k + 1]);
            const float2 msj = make_float2(ms[2 * k], ms[2 * k + 1]);
            const float2 mcj = make_float2(mc[2 * k], mc[2 * k + 1]);
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
            k24::adamw2(pi[3 * h + k], mo[3 * h + k], vo[3 * h + k], grad[3 * h + k], sc);
        }
    }
    k24::store12x2(d.pi, b0, true, pi);
    k24::store12x2(d.m, b0, true, mo);
    k24::store12x2(d.v, b0, true, vo);
    if (d.grad) k24::store12x2(d.grad, b0, true, grad);
}

__global__ void __launch_bounds__(kThreads, 1) masked_linear_bwd_adam_kernel(const __grid_constant__ BwdGroup grp,
                                                                             const StepScalars sc, unsigned char *ws) {
    static_assert(kBwdSmem + 2 * kNlogEntries * 4 + 1024 <= 232448, "fits one SM");
    constexpr int kD = kStages;
    extern __shared__ unsigned char s_dyn_mb[];
    __shared__ __align__(16) float2 s_tab[kNlogEntries];
    __shared__ __align__(8) unsigned long long s_full[kD], s_empty[kD], s_accf, s_acce;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    unsigned int *err = reinterpret_cast<unsigned int *>(ws + kErrOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = gridDim.x, cta = blockIdx.x;
    const int ntile = (int)((grp.total_tiles - cta + G - 1) / G);  // tiles cta, cta + G, ...
    const int kst = (grp.tokens + kBwdK - 1) / kBwdK;               // stages per tile
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_mb);
    const unsigned pad = (1024u - (dyn_s & 1023u)) & 1023u;
    unsigned char *ring = s_dyn_mb + pad;
    const unsigned ring_s = dyn_s + pad;
    float *s_g = reinterpret_cast<float *>(ring + kD * kBwdStageBytes);  // [kRows][kGPitch]
    const unsigned full0 = (unsigned)__cvta_generic_to_shared(&s_full[0]);
    const unsigned empty0 = (unsigned)__cvta_generic_to_shared(&s_empty[0]);
    const unsigned accf = (unsigned)__cvta_generic_to_shared(&s_accf);
    const unsigned acce = (unsigned)__cvta_generic_to_shared(&s_acce);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kD; ++s) {
            mbar_init(full0 + 8 * s, 1u);
            mbar_init(empty0 + 8 * s, 1u);
        }
        mbar_init(accf, 1u);
        mbar_init(acce, (unsigned)kProd);  // every epilogue thread, once it has read the accumulator
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    load_tab(s_tab);
    if (warp == 0) {
        const unsigned dst = (unsigned)__cvta_generic_to_shared(&s_tmem);
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                     "r"(kBwdTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;

    if (warp == kProdWarps) {
        // ------------------------------------------------------------ copy warp
        int f = 0, issued = 0;
        bool stop = false;
        for (int it = 0; it < ntile && !stop; ++it) {
            int op;
            int64_t rt, ct;
            bwd_decode(grp, cta + (int64_t)it * G, op, rt, ct);
            for (int k = 0; k < kst; ++k, ++f) {
                const int s = f % kD;
                if (f >= kD && !um_wait(empty0 + 8 * s, ((f / kD) - 1) & 1, &s_abort)) {
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    const unsigned st = ring_s + s * kBwdStageBytes, bar = full0 + 8 * s;
                    const int r0 = (int)(rt * kRows), c0 = (int)(ct * kBwdCols), t0 = k * kBwdK;
                    fence_proxy_async();
                    mbar_arrive_tx(bar, (unsigned)kBwdStageBytes);
                    tma_load_2d(st, &grp.dy[op], r0, t0, bar);
                    tma_load_2d(st + 8192, &grp.dy[op], r0 + 64, t0, bar);
                    tma_load_2d(st + 16384, &grp.x[op], c0, t0, bar);
                    tma_load_2d(st + 24576, &grp.x[op], c0 + 64, t0, bar);
                }
                ++issued;
            }
        }
        for (int s = 0; s < kD && s < issued; ++s) {
            const int last = s + ((issued - 1 - s) / kD) * kD;
            tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == kProdWarps + 1) {
        // ------------------------------------------------------------ MMA warp
        int f = 0, commits = 0;
        bool stop = false;
        for (int it = 0; it < ntile && !stop; ++it) {
            // the epilogue has read the previous tile's accumulator
            if (it > 0 && !um_wait(acce, (it - 1) & 1, &s_abort)) {
                if (lane == 0 && !s_abort) {
                    atomicOr(err, 1u);
                    s_abort = 1;
                }
                break;
            }
            for (int k = 0; k < kst; ++k, ++f) {
                const int s = f % kD;
                if (!um_wait(full0 + 8 * s, (f / kD) & 1, &s_abort)) {
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    tc_fence_after();
                    const unsigned st = ring_s + s * kBwdStageBytes;
                    const uint64_t a0 = mn_desc(st), b0 = mn_desc(st + 16384);
#pragma unroll
                    for (int q = 0; q < 4; ++q)  // K = 16 tokens = two 8-token groups = 2048 bytes
                        umma_dense(tbase, a0 + (uint64_t)(128 * q), b0 + (uint64_t)(128 * q), kBwdIdesc,
                                   (k == 0 && q == 0) ? 0u : 1u);
                    umma_commit(empty0 + 8 * s);
                    if (k == kst - 1) umma_commit(accf);
                }
                __syncwarp();
                ++commits;
            }
        }
        if (commits > 0) {
            const int ff = commits - 1;
            tm_wait(empty0 + 8 * (ff % kD), (ff / kD) & 1);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        const NlogCtx L{s_tab};
        constexpr int kCw = kBwdCols / (kProdWarps / 4);  // accumulator columns per epilogue warp
        const int q = warp & 3, ch = warp >> 2;  // TMEM lane quarter, column slice
        const unsigned tq = tbase + ((unsigned)(32 * q) << 16) + (unsigned)(ch * kCw);
        const int tid = threadIdx.x;
        bool failed = false;
        for (int it = 0; it < ntile; ++it) {
            const bool ok = !failed && um_wait(accf, it & 1, &s_abort);
            if (um_bar_or<kProd>(!ok)) {
                failed = true;
                break;
            }
            int op;
            int64_t rt, ct;
            bwd_decode(grp, cta + (int64_t)it * G, op, rt, ct);
            const Op &d = grp.d[op];
            tc_fence_after();
            float *grow = s_g + (32 * q + lane) * kGPitch + ch * kCw;
#pragma unroll 1
            for (int k = 0; k < kCw; k += 16) {
                float v[16];
                tmem_ld16(tq + k, v);
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4 *>(grow + k + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
            tc_fence_before();
            mbar_arrive(acce);  // the accumulator may take the next tile
            um_bar<kProd>();    // the whole tile of G is in shared memory
            const int64_t bpr = d.cols >> 2;
#pragma unroll 1
            for (int p = tid; p < kRows * 16; p += kProd) {
                const int r = p >> 4, pc = p & 15;
                const int64_t row = rt * kRows + r, bc = ct * 32 + 2 * pc;
                if (row < d.rows && bc < bpr) pair_bwd_adam(d, row * bpr + bc, s_g + r * kGPitch + 8 * pc, sc, L);
            }
            um_bar<kProd>();  // every pair has read G before the next tile overwrites it
        }
        if (failed && threadIdx.x == 0 && !s_abort) {
            atomicOr(err, 1u);
            s_abort = 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kBwdTmemCols)
                     : "memory");
    }
}

}  // namespace mlin
}  // namespace mllm
