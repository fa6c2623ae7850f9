// kernels_pf48.cuh -- the 4:8 serving product at prefill sizes (more than 64 tokens).
//
// y = x W*^T from the packed 4:8 hard mask (MaskLLM serves the masked network from its hard
// mask after training: paper-graph-ui summary of arXiv 2409.17481, s.3.2 "Information flow at
// inference"; s.5 Table 16 times 128- and 2048-token prompts). 4:8 has no hardware sparse
// mode, so each stage of compressed blocks is expanded to a dense bf16 tile in tensor memory
// (the byte-permute expansion of sparse_linear_umma48_kernel, same selector tables) and fed to
// dense tcgen05.mma (kind::f16) that reads A from tensor memory and the activations from
// shared memory. Unlike the decode kernel, which expands every weight once per group of at
// most 64 tokens, a stage here is expanded once for 256 tokens: the MMA's N is 256 and the
// accumulator (128 rows x 256 tokens of fp32) fills 256 tensor-memory columns (calls of at most
// 128 tokens use N = 128 and 128 columns, with six stages instead of four).
//
// A unit is (operand, 128-row tile, N-token chunk) over all columns, in stages of 64 columns
// (eight 4:8 blocks per row). Per stage the copy warp lands, on one mbarrier, the N x 64 box
// of x (128-byte swizzle, the MMA's K-major layout), the 128 x 32 box of compressed values
// (64-byte swizzle) and the 128 x 8 box of codes; each of the 16 expansion warps takes the 32
// rows of its tensor-memory lane quarter (warp % 4) and a quarter of the stage's columns
// (warp / 4), writes its rows' 8 dense columns with one tcgen05.st and arrives on the stage's
// "expanded" barrier; the MMA warp issues four MMAs (K = 16) and commits them to the stage's
// "empty" barrier, and at a unit's last stage to the accumulator barrier; then the same 16
// warps store the unit's y (warp w: TMEM lane quarter w % 4, a quarter of the unit's tokens).
// Tensor memory: the accumulator in columns 0 .. N-1, stage s's dense tile (32 columns) from
// column N + 32 s; a tile is rewritten only after its stage's MMAs have completed (the copy
// warp waits for that before it refills the stage). Units are dealt round-robin to one CTA
// per SM in the order of the 2:4 prefill kernel (row-tile groups, token chunk by token chunk),
// so a weight strip is read from HBM about once per launch. Rows and tokens past the call are
// zero-filled by the tensor maps and not stored. Every wait is bounded; a timeout sets the
// error word and the CTA winds down as the other tensor-memory kernels do.
#pragma once

#include "kernels_umma.cuh"

namespace mllm {
namespace spl {

// Tokens per unit (the MMA's N): 256, or 128 for calls of at most 128 tokens (a 256-token
// unit would compute half of its columns on zero-filled tokens).
template <int kTok> struct P8 {
    static constexpr int kXOff = 0;                              // x: kTok tokens x 64 columns (128-byte swizzle)
    static constexpr int kValOff = kTok * 128;                   // values: 128 rows x 32 bf16 (8 KB, 64-byte swizzle)
    static constexpr int kMetaOff = kValOff + kUmRows * 64;      // codes: 128 rows x 8 uint16 (2 KB)
    static constexpr int kStageTx = kTok * 128 + kUmRows * 64 + kUmRows * 16;  // bytes the copy engine lands
    static constexpr int kStage = (kMetaOff + kUmRows * 16 + 1023) / 1024 * 1024;
    static constexpr int kStages = kTok == 256 ? 4 : 6;
    static constexpr int kSmem = kStages * kStage + 8192 + kU8TabBytes;  // tables first, 8 KB aligned
    static constexpr unsigned kACol = kTok;                      // stage s's dense tile: 32 columns from kACol + 32 s
    static constexpr unsigned kTmemCols = 512;
    // Instruction descriptor of kind::f16: dense, f32 accumulator, bf16 A and B (K-major),
    // N = kTok, M = 128.
    static constexpr uint32_t kIdesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTok >> 3) << 17) | ((uint32_t)(kUmRows >> 4) << 24);
};
constexpr int kP8Threads = 32 * kU8Warps + 64;           // 16 expansion/epilogue warps, copy, MMA

template <int kTok>
__device__ __forceinline__ void p8_issue(const PfGroup &g, const PfCur &c, int64_t j, unsigned stage, unsigned bar) {
    using K = P8<kTok>;
    const TmMaps &mp = g.maps[c.op];
    const int row0 = (int)(c.pair * kUmRows), tok0 = (int)(c.tc * kTok);
    mbar_arrive_tx(bar, (unsigned)K::kStageTx);
    tma_load_2d(stage + K::kXOff, &mp.x, (int)(64 * j), tok0, bar);
    tma_load_2d(stage + K::kValOff, &mp.vals, (int)(32 * j), row0, bar);
    tma_load_2d(stage + K::kMetaOff, &mp.meta, (int)(8 * j), row0, bar);
}

// Thread (r, pt) of the stage: row r, blocks 2 pt and 2 pt + 1 (one 16-byte value chunk, one
// word of two codes) into the row's dense columns 8 pt .. 8 pt + 7 (two bf16 per column in K
// order). The values box lands with the 64-byte swizzle (16-byte chunk c of row r at chunk
// c ^ ((r >> 1) & 3)), so the 32 rows a warp reads at one pt fall on distinct banks in each
// quarter-warp; each thread reads its row's 16 bytes of codes whole and keeps word pt.
// ta / tb: shared-memory addresses of this lane's copy of entry 0 of the selector tables (8 KB
// aligned but for the copy's bits), the entry of pair code p at ta | p << 7 (u8_expand).
template <int kTok>
__device__ __forceinline__ void p8_expand(const unsigned char *st, unsigned ta, unsigned tb, int r, int pt,
                                          uint32_t (&w)[8]) {
    using K = P8<kTok>;
    const uint4 v = lds128(st + K::kValOff + r * 64 + ((pt ^ ((r >> 1) & 3)) << 4));
    const uint4 c4 = lds128(st + K::kMetaOff + r * 16);
    const uint32_t cw = pt == 0 ? c4.x : pt == 1 ? c4.y : pt == 2 ? c4.z : c4.w;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t lo = h ? v.z : v.x, hi = h ? v.w : v.y;
        const uint32_t ka = (h ? (cw >> 9) : (cw << 7)) & 0x1F80u;
        const uint32_t kb = (h ? (cw >> 15) : (cw << 1)) & 0x1F80u;
        const uint4 sa = lds128_at(ta | ka), sb = lds128_at(tb | kb);
        uint32_t *o = w + 4 * h;
        o[0] = __byte_perm(__byte_perm(lo, 0u, sa.x), hi, sb.x);
        o[1] = __byte_perm(__byte_perm(lo, 0u, sa.y), hi, sb.y);
        o[2] = __byte_perm(__byte_perm(lo, 0u, sa.z), hi, sb.z);
        o[3] = __byte_perm(__byte_perm(lo, 0u, sa.w), hi, sb.w);
    }
}

// 8 consecutive 32-bit columns of this thread's lane from w[8], then wait for the store.
__device__ __forceinline__ void tmem_st8(unsigned taddr, const uint32_t (&w)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(taddr),
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

template <int kTok>
__global__ void __launch_bounds__(kP8Threads, 1) sparse_linear_prefill48_kernel(const __grid_constant__ PfGroup pg,
                                                                              unsigned int *__restrict__ err) {
    using K = P8<kTok>;
    static_assert(K::kSmem + 1024 <= 232448, "fits one SM");
    static_assert(kU8Warps == 16, "four threads per row, 128 rows");
    static_assert(K::kACol + 32u * K::kStages <= K::kTmemCols, "accumulator and dense tiles fit tensor memory");
    static_assert(K::kValOff % 512 == 0 && K::kStage % 512 == 0, "64-byte-swizzled values box on a 512-byte boundary");
    constexpr int kD = K::kStages, kP8Stage = K::kStage, kQTok = kTok / 4;  // epilogue: tokens per warp
    constexpr int kBar = 32 * kU8Warps;
    constexpr uint32_t kIdesc = K::kIdesc;
    extern __shared__ unsigned char s_dyn_p8[];
    __shared__ __align__(8) unsigned long long s_full[kD], s_empty[kD], s_exp[kD], s_acc;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = gridDim.x, u0 = blockIdx.x, u1 = pg.total_units;
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_p8);
    const unsigned tab_s = (dyn_s + 8191u) & ~8191u;  // tables A, B: 8 KB each on 8 KB boundaries
    uint4 *tab = reinterpret_cast<uint4 *>(s_dyn_p8 + (tab_s - dyn_s));  // A: entries [0, 64), B: [64, 128), x copies
    const unsigned ring_s = tab_s + (unsigned)kU8TabBytes;  // 1 KB aligned
    unsigned char *ring = s_dyn_p8 + (ring_s - dyn_s);
    const unsigned full0 = (unsigned)__cvta_generic_to_shared(&s_full[0]);
    const unsigned empty0 = (unsigned)__cvta_generic_to_shared(&s_empty[0]);
    const unsigned exp0 = (unsigned)__cvta_generic_to_shared(&s_exp[0]);
    const unsigned accb = (unsigned)__cvta_generic_to_shared(&s_acc);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kD; ++s) {
            mbar_init(full0 + 8 * s, 1u);
            mbar_init(empty0 + 8 * s, 1u);
            mbar_init(exp0 + 8 * s, (unsigned)kBar);  // every expanding thread arrives once per stage
        }
        mbar_init(accb, 1u);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    for (int i = threadIdx.x; i < 2 * 64 * kU8TabCopies; i += blockDim.x)  // entry e, copy c at e * copies + c
        tab[i] = u8_table_entry((i / kU8TabCopies) & 63, i >= 64 * kU8TabCopies);
    if (warp == 0) {
        const unsigned dst = (unsigned)__cvta_generic_to_shared(&s_tmem);
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                     "r"(K::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;

    if (warp == kU8Warps) {
        // ------------------------------------------------------------ copy warp
        int f = 0, issued = 0;
        bool stop = false;
        for (int64_t u = u0; u < u1 && !stop; u += G) {
            const PfCur c = pf_decode(pg, u);
            const int64_t nch = pg.d[c.op].nch;
            for (int64_t j = 0; j < nch; ++j, ++f) {
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
                    fence_proxy_async();
                    p8_issue<kTok>(pg, c, j, ring_s + s * kP8Stage, full0 + 8 * s);
                }
                ++issued;
            }
        }
        for (int s = 0; s < kD && s < issued; ++s) {
            const int last = s + ((issued - 1 - s) / kD) * kD;
            tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == kU8Warps + 1) {
        // ------------------------------------------------------------ MMA warp
        int f = 0, commits = 0;
        bool stop = false;
        for (int64_t u = u0; u < u1 && !stop; u += G) {
            const PfCur c = pf_decode(pg, u);
            const int64_t nch = pg.d[c.op].nch;
            for (int64_t j = 0; j < nch; ++j, ++f) {
                const int s = f % kD;
                if (!um_wait(exp0 + 8 * s, (f / kD) & 1, &s_abort)) {
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    tc_fence_after();
                    const unsigned st = ring_s + s * kP8Stage;
                    const unsigned ta = tbase + K::kACol + 32u * (unsigned)s;  // the stage's dense tile
                    const uint64_t b0 = um_desc(st + K::kXOff);
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // K = 16 per MMA: 8 columns of A
                        umma_dense_ta(tbase, ta + 8u * (unsigned)k, b0 + (uint64_t)(2 * k), kIdesc,
                                      (j == 0 && k == 0) ? 0u : 1u);
                    umma_commit(empty0 + 8 * s);
                    if (j == nch - 1) umma_commit(accb);
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
        // ------------------------------------------------------------ expansion / epilogue warps
        const int q = warp & 3, sl = warp >> 2;                // TMEM lane quarter; token slice / part
        const int r = 32 * q + lane, pt = sl;                  // expansion: row (this lane), part
        const unsigned tq = tbase + ((unsigned)(32 * q) << 16) + (unsigned)(kQTok * sl);
        const unsigned tdense = tbase + ((unsigned)(32 * q) << 16) + K::kACol + 8u * (unsigned)pt;
        const unsigned tab_a = tab_s + 16u * (unsigned)(lane & (kU8TabCopies - 1)), tab_b = tab_a + 64u * 16u * kU8TabCopies;
        unsigned acc_phase = 0u;
        bool failed = false;
        int f = 0;
        for (int64_t u = u0; u < u1; u += G) {
            const PfCur c = pf_decode(pg, u);
            const PfOp &d = pg.d[c.op];
            for (int64_t j = 0; j < d.nch; ++j, ++f) {
                const int s = f % kD;
                if (!failed) {
                    if (um_wait(full0 + 8 * s, (f / kD) & 1, &s_abort)) {
                        uint32_t w[8];
                        p8_expand<kTok>(ring + s * kP8Stage, tab_a, tab_b, r, pt, w);
                        tmem_st8(tdense + 32u * (unsigned)s, w);  // into the stage's dense tile in tensor memory
                        tc_fence_before();
                        mbar_arrive(exp0 + 8 * s);
                    } else {
                        failed = true;
                        if (lane == 0 && !s_abort) {
                            atomicOr(err, 1u);
                            s_abort = 1;
                        }
                    }
                }
            }
            // ---------------------------------------------------- epilogue of the unit
            const bool acc_ok = !failed && um_wait(accb, acc_phase, &s_abort);
            acc_phase ^= 1u;
            if (um_bar_or<kBar>(!acc_ok)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const int tok0 = (int)(c.tc * kTok) + kQTok * sl;
            const int64_t row = c.pair * kUmRows + 32 * q + lane;
#pragma unroll 1
            for (int k = 0; k < kQTok; k += 16) {
                float v[16];
                tmem_ld16(tq + k, v);
                if (row < d.rows) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (tok0 + k + i < pg.tokens) d.y[(int64_t)(tok0 + k + i) * d.rows + row] = v[i];
                }
            }
            tc_fence_before();
            um_bar<kBar>();  // every read of the accumulator precedes the next unit's first arrival
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(K::kTmemCols)
                     : "memory");
    }
}

}  // namespace spl
}  // namespace mllm
