// kernels_umma.cuh -- the serving product on the fifth-generation tensor cores: 2:4 at 17-64
// tokens with tcgen05.mma.sp (operands in shared memory, sparsity metadata and accumulators in
// tensor memory), and 4:8 at 1-64 tokens with blocks expanded to a dense tile in tensor memory
// and dense tcgen05.mma (below, "4:8 on the dense tensor cores").
//
// The product is y = x W*^T with W* = W (.) M* in the form mllm_hard_pack writes (two kept
// bf16 values and one 4-bit position code per block of four weights); MaskLLM serves the
// masked network this way after training (paper-graph-ui summary of arXiv 2409.17481, s.3.2
// "Information flow at inference"). It is an HBM stream: every compressed weight is read once.
//
// Tile: 128 rows of W* (the MMA's M) x all kNTok tokens (its N, tokens rounded up to 16) x
// 128 columns per pipeline stage (four MMAs of K = 32). Per stage the tensor memory
// accelerator lands, on one mbarrier, the 128 x 64 box of compressed values and two kNTok x 64
// boxes of x (both with the 128-byte swizzle, the K-major layout the MMA's shared-memory
// descriptors name) and the 128 x 4 box of metadata words. Roles in a CTA of six warps:
//   warp 4       the copy warp: refills a stage when the MMAs that read it have completed
//                (their tcgen05.commit arrives on the stage's "empty" barrier);
//   warps 0-3    per stage, each thread builds the metadata word of its tensor-memory lane,
//                stores it with tcgen05.st and arrives on the stage's "metadata" barrier; at
//                the end of a tile each warp reads its 32 rows of the accumulator with
//                tcgen05.ld and stores y (or a partial tile);
//   warp 5       the MMA warp: once all 128 metadata threads have arrived, one lane issues
//                the stage's four MMAs and commits them.
// Metadata in tensor memory, M = 128, 16-bit types, one column per MMA (the address an MMA
// names is even; the descriptor's selector bits stay 0): lane
// L = (m % 8) + 8 h + 16 (m / 16) holds, for row m (m % 16 < 8) and K half h, the four
// 4-bit codes of blocks 4h .. 4h+3 in its low 16 bits and those of row m + 8 in its high 16
// bits -- the same per-quad distribution as the metadata of mma.sp m16n8k32, so a byte permute
// of the packed words of rows m and m + 8 gives it. Rows past the matrix are zero-filled by
// the copy engine; their zero words are replaced by a valid code (values there are zero).
// Tensor memory per CTA: 128 columns (accumulator at 0 .. kNTok-1, the metadata of MMA j of
// stage s at column 64 + 8s + 2j). A CTA takes more than a fifth of an SM's shared memory, so at most
// four are resident and their 512 columns fit; the allocation never waits on another CTA.
//
// Work split: the 128-column chunks of all tiles of all operands of a launch form one sequence,
// split into equal contiguous ranges over the CTAs (stream-K). A tile cut between CTAs leaves
// one partial tile per piece in the workspace (slot 1 for a CTA's last piece when that CTA
// also had earlier work, else slot 0); the last CTA to arrive (a ticket per tile, keyed by the
// tile's first CTA) adds the pieces in CTA order and stores y, so results are deterministic. Every wait is
// bounded (kTmWaitNs); a timeout sets the workspace's error word, the CTA stops issuing,
// waits (bounded) for the copies and MMAs it has in flight, frees its tensor memory and exits.
// arm_only_first (tests only) arms stage 0 without filling it, so that this path runs.
#pragma once

#include "kernels_spl.cuh"

namespace mllm {
namespace spl {

constexpr int kUmRows = kBatchRows;          // MMA M: rows of a tile (128)
constexpr int kUmStages = 3;
constexpr int kUmThreads = 192;              // 4 metadata/epilogue warps, the copy warp, the MMA warp
constexpr int kUmCtasPerSm = 2;              // resident CTAs the grid is sized for
constexpr unsigned kUmTmemCols = 128;
constexpr unsigned kUmMetaCol = 64;
constexpr size_t kUmPartFloats = kBatchPartFloats;  // one partial tile: 128 rows x 64 tokens

template <int kNTok> constexpr int um_xbox_bytes() { return kNTok * 128; }
template <int kNTok> constexpr int um_stage_tx() { return kUmRows * 128 + 2 * um_xbox_bytes<kNTok>() + kUmRows * 16; }
template <int kNTok> constexpr int um_stage_bytes() { return (um_stage_tx<kNTok>() + 1023) / 1024 * 1024; }
template <int kNTok> constexpr int um_smem_bytes() { return kUmStages * um_stage_bytes<kNTok>() + 1024; }

// Instruction descriptor of kind::f16: sparse, f32 accumulator, bf16 A and B (both
// K-major), N = kNTok, M = 128.
template <int kNTok> constexpr uint32_t um_idesc() {
    return (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kNTok >> 3) << 17) |
           ((uint32_t)(kUmRows >> 4) << 24);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t um_desc(unsigned saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void umma_sp(unsigned d_tmem, uint64_t adesc, uint64_t bdesc, unsigned e_tmem,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %5, 0;\n"
        " tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(unsigned bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// The metadata of a stage's four MMAs, one per even column (taddr, +2, +4, +6).
__device__ __forceinline__ void tmem_st_meta(unsigned taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %5, %2, %5, %3, %5, %4, %5};\n" ::"r"(taddr),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(0u)
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// 16 consecutive accumulator columns of this thread's lane; the wait names the registers so
// that no use is scheduled before the data is there.
__device__ __forceinline__ void tmem_ld16(unsigned taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Barrier (id 1) of the kCount threads that are not the copy warp, OR-reducing a predicate.
template <int kCount>
__device__ __forceinline__ bool um_bar_or(bool p) {
    unsigned r;
    asm volatile(
        "{\n .reg .pred a, b;\n setp.ne.u32 a, %1, 0;\n barrier.cta.red.or.pred b, 1, %2, a;\n"
        " selp.u32 %0, 1, 0, b;\n}\n"
        : "=r"(r)
        : "r"((unsigned)p), "n"(kCount)
        : "memory");
    return r != 0u;
}
template <int kCount>
__device__ __forceinline__ void um_bar() { asm volatile("barrier.cta.sync 1, %0;\n" ::"n"(kCount) : "memory"); }

// Warp-uniform bounded wait that also gives up once *abort is set. The clock and the abort
// flag are read once per 8 polls (each poll is a try_wait, which itself suspends the warp
// for a bounded time), so a waiting warp takes few issue slots from the working ones.
__device__ __forceinline__ bool um_wait(unsigned bar, unsigned parity, const volatile int *abort) {
    if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
    const unsigned long long t0 = __shfl_sync(0xFFFFFFFFu, globaltimer_ns(), 0);
    while (true) {
#pragma unroll 1
        for (int k = 0; k < 8; ++k)
            if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
        if (__any_sync(0xFFFFFFFFu, *abort != 0)) return false;
        if (__shfl_sync(0xFFFFFFFFu, globaltimer_ns(), 0) - t0 > kTmWaitNs) return false;
    }
}

template <int kNTok>
__device__ __forceinline__ void um_issue(const TmGroup &tg, const Cursor &c, unsigned stage, unsigned bar) {
    const TmMaps &mp = tg.maps[c.op];
    const int j = (int)c.j, row0 = (int)(c.tile * kUmRows);
    mbar_arrive_tx(bar, (unsigned)um_stage_tx<kNTok>());
    tma_load_2d(stage, &mp.vals, 64 * j, row0, bar);
    tma_load_2d(stage + kUmRows * 128, &mp.x, 128 * j, 0, bar);
    tma_load_2d(stage + kUmRows * 128 + um_xbox_bytes<kNTok>(), &mp.x, 128 * j + 64, 0, bar);
    tma_load_2d(stage + kUmRows * 128 + 2 * um_xbox_bytes<kNTok>(), &mp.meta, 4 * j, row0, bar);
}

template <int kNTok>
__device__ __forceinline__ void um_store(const SkOp &d, int64_t tile, int warp, int lane, const float (&v)[kNTok],
                                         int tokens) {
    const int64_t r = tile * kUmRows + 32 * warp + lane;
    if (r >= d.rows) return;
#pragma unroll
    for (int tok = 0; tok < kNTok; ++tok)
        if (tok < tokens) d.y[tok * d.rows + r] = v[tok];
}

template <int kNTok>
__global__ void __launch_bounds__(kUmThreads, kUmCtasPerSm) sparse_linear_umma_kernel(const __grid_constant__ TmGroup tg,
                                                                          float *__restrict__ part,
                                                                          unsigned int *__restrict__ tickets,
                                                                          unsigned int *__restrict__ err,
                                                                          int arm_only_first) {
    static_assert(kNTok % 16 == 0 && kNTok >= 16 && kNTok <= kMaxTokens, "N of an M = 128 MMA");
    static_assert(um_smem_bytes<kNTok>() * 5 > 233472, "at most four CTAs per SM: 4 x 128 TMEM columns");
    static_assert(kUmCtasPerSm * (um_smem_bytes<kNTok>() + 2048) <= 233472, "kUmCtasPerSm CTAs fit an SM");
    constexpr int kD = kUmStages, kStage = um_stage_bytes<kNTok>();
    constexpr uint32_t kIdesc = um_idesc<kNTok>();
    extern __shared__ unsigned char s_dyn_um[];
    __shared__ __align__(8) unsigned long long s_full[kD], s_empty[kD], s_meta[kD], s_acc;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    __shared__ int s_last;
    const SkGroup &grp = tg.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t total = grp.total_chunks;
    const int64_t G = imin64((int64_t)gridDim.x, total), cta = blockIdx.x;
    if (cta >= G) return;  // the whole CTA, before any barrier or allocation
    const int64_t lo = cta * total / G, hi = (cta + 1) * total / G;
    const int n = (int)(hi - lo);
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_um);
    const unsigned pad = (1024u - (dyn_s & 1023u)) & 1023u;
    const unsigned char *ring = s_dyn_um + pad;
    const unsigned ring_s = dyn_s + pad;
    const unsigned full0 = (unsigned)__cvta_generic_to_shared(&s_full[0]);
    const unsigned empty0 = (unsigned)__cvta_generic_to_shared(&s_empty[0]);
    const unsigned meta0 = (unsigned)__cvta_generic_to_shared(&s_meta[0]);
    const unsigned accb = (unsigned)__cvta_generic_to_shared(&s_acc);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kD; ++s) {
            mbar_init(full0 + 8 * s, 1u);
            mbar_init(empty0 + 8 * s, 1u);
            mbar_init(meta0 + 8 * s, 128u);  // every metadata thread arrives once per stage
        }
        mbar_init(accb, 1u);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        const unsigned dst = (unsigned)__cvta_generic_to_shared(&s_tmem);
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                     "r"(kUmTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;

    if (warp == 4) {
        // ------------------------------------------------------------ copy warp
        Cursor ld = sk_decode(grp, lo);
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
                if (f == 0 && arm_only_first)  // test of the bounded wait: a stage nothing fills
                    mbar_arrive_tx(full0, (unsigned)um_stage_tx<kNTok>());
                else {
                    fence_proxy_async();
                    um_issue<kNTok>(tg, ld, ring_s + s * kStage, full0 + 8 * s);
                }
            }
            ++issued;
            sk_advance(grp, ld);
        }
        // every copy this warp started has landed (bounded) before the CTA's memory is released
        for (int s = 0; s < kD && s < issued; ++s) {
            const int last = s + ((issued - 1 - s) / kD) * kD;  // the latest fill of stage s
            tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA warp
        Cursor cc = sk_decode(grp, lo);
        bool fresh = true;  // the next MMA starts a tile piece (overwrites the accumulator)
        int commits = 0;
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            if (!um_wait(meta0 + 8 * s, (f / kD) & 1, &s_abort)) {
                if (lane == 0 && !s_abort) {
                    atomicOr(err, 1u);
                    s_abort = 1;
                }
                break;
            }
            const SkOp &d = grp.d[cc.op];
            const bool piece_end = (cc.j == d.nch - 1) || (f == n - 1);
            if (lane == 0) {
                tc_fence_after();
                const unsigned st = ring_s + s * kStage;
                const uint64_t a0 = um_desc(st), b0 = um_desc(st + kUmRows * 128),
                               b1 = um_desc(st + kUmRows * 128 + um_xbox_bytes<kNTok>());
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    umma_sp(tbase, a0 + (uint64_t)(2 * j), ((j >> 1) ? b1 : b0) + (uint64_t)(4 * (j & 1)),
                            tbase + kUmMetaCol + 8 * s + 2 * j, kIdesc, (fresh && j == 0) ? 0u : 1u);
                umma_commit(empty0 + 8 * s);
                if (piece_end) umma_commit(accb);
            }
            __syncwarp();
            ++commits;
            fresh = piece_end;
            sk_advance(grp, cc);
        }
        if (commits > 0) {  // every MMA has completed (bounded) before the tensor memory is released
            const int f = commits - 1;
            tm_wait(empty0 + 8 * (f % kD), (f / kD) & 1);
        }
    } else {
        // ------------------------------------------------------------ metadata / epilogue warps
        const unsigned tlane = tbase + ((unsigned)(32 * warp) << 16);
        const int h = (lane >> 3) & 1;
        const int ra = 32 * warp + 16 * (lane >> 4) + (lane & 7);  // rows ra and ra + 8 of the tile
        const uint32_t esel = h ? 0x7632u : 0x5410u;
        Cursor cc = sk_decode(grp, lo);
        unsigned acc_phase = 0u;
        bool failed = false;
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            // A warp whose wait ran out stops working but keeps its place in the loop, so that
            // it meets the others at the end of the tile, where all of them leave together.
            if (!failed) {
                if (um_wait(full0 + 8 * s, (f / kD) & 1, &s_abort)) {
                    tc_fence_after();
                    const unsigned char *meta = ring + s * kStage + kUmRows * 128 + 2 * um_xbox_bytes<kNTok>();
                    const uint4 wa = lds128(meta + ra * 16), wb = lds128(meta + (ra + 8) * 16);
                    const uint32_t a4[4] = {wa.x, wa.y, wa.z, wa.w}, b4[4] = {wb.x, wb.y, wb.z, wb.w};
                    uint32_t e[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        e[j] = __byte_perm(a4[j] ? a4[j] : 0x44444444u, b4[j] ? b4[j] : 0x44444444u, esel);
                    tmem_st_meta(tlane + kUmMetaCol + 8 * s, e[0], e[1], e[2], e[3]);
                    tc_fence_before();
                    mbar_arrive(meta0 + 8 * s);
                } else {
                    failed = true;
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                }
            }
            const SkOp &d = grp.d[cc.op];
            const bool piece_end = (cc.j == d.nch - 1) || (f == n - 1);
            if (piece_end) {
                // ---------------------------------------------------- epilogue of a tile piece
                const bool acc_ok = !failed && um_wait(accb, acc_phase, &s_abort);
                acc_phase ^= 1u;
                if (um_bar_or<128>(!acc_ok)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float v[kNTok];
#pragma unroll
                for (int q = 0; q < kNTok / 16; ++q) tmem_ld16(tlane + 16 * q, v + 16 * q);
                tc_fence_before();  // these reads precede the next piece's first MMA (after its arrivals)
                const int64_t a = d.chunk_begin + cc.tile * d.nch, b = a + d.nch;
                const int64_t c1 = ((a + 1) * G - 1) / total, c2 = (b * G - 1) / total;
                if (c1 == c2) {
                    um_store<kNTok>(d, cc.tile, warp, lane, v, grp.tokens);
                } else {
                    const int64_t lo1 = c1 * total / G;
                    const int slot = (cta == c1 && lo1 < a) ? 1 : 0;
                    float *mine = part + (size_t)(cta * 2 + slot) * kUmPartFloats + 32 * warp + lane;
#pragma unroll
                    for (int tok = 0; tok < kNTok; ++tok) __stcg(mine + tok * kUmRows, v[tok]);
                    __threadfence();
                    um_bar<128>();
                    if (threadIdx.x == 0) s_last = (atomicAdd(tickets + c1, 1u) == (unsigned int)(c2 - c1));
                    um_bar<128>();
                    if (s_last) {
                        __threadfence();
                        float sum[kNTok];
#pragma unroll
                        for (int tok = 0; tok < kNTok; ++tok) sum[tok] = 0.f;
                        for (int64_t q = c1; q <= c2; ++q) {
                            const int sid = (q == c1 && lo1 < a) ? 1 : 0;
                            const float *p = part + (size_t)(q * 2 + sid) * kUmPartFloats + 32 * warp + lane;
#pragma unroll
                            for (int tok = 0; tok < kNTok; ++tok) sum[tok] += __ldcg(p + tok * kUmRows);
                        }
                        um_store<kNTok>(d, cc.tile, warp, lane, sum, grp.tokens);
                        um_bar<128>();
                        if (threadIdx.x == 0) tickets[c1] = 0u;
                    }
                }
            }
            sk_advance(grp, cc);
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kUmTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------ 2:4 prefill (more than 64 tokens)
//
// The same sparse MMA (M = 128 rows, K = 32 per instruction, metadata in tensor memory) with
// N = 128 tokens. A unit of work is (operand, pair of 128-row tiles, chunk of 128 tokens) over
// all the operand's columns: per 128-column stage the copy warp lands both tiles' compressed
// values and metadata and one 128-token box of the activations, and the MMA warp issues four
// MMAs per tile into two accumulators (TMEM columns 0-127 and 128-255) with the same
// activation operand, so every staged activation byte feeds two tiles. No unit is split
// between CTAs, so nothing is reduced across CTAs. CTA c takes units c, c + G, c + 2G, ... of a
// sequence ordered so that the G units in flight at any time share few weight strips and all
// token chunks: per operand, groups of R row-tile pairs (R = ceil(G / token chunks)), within
// a group token chunk by token chunk, within a chunk the group's pairs. The strips and chunks
// in flight then fit in L2, so a strip is read from HBM about once per group instead of once
// per token chunk. The host orders the operands by decreasing columns (the longest units
// first). Tokens past the call are zero-filled by the activations' tensor map, rows past the
// matrix by the weights' (their metadata words read zero and are replaced by a valid code),
// and the epilogue stores only rows and tokens inside the call. Warps 0-3 turn the first
// tile's metadata into TMEM, warps 4-7 the second tile's; warps 0-15 store the accumulators
// (4 per tile and half of the tokens; the MMA pipe idles while they drain, so more warps
// shorten the gap); warp 16 copies, warp 17 issues the MMAs. Barriers, bounded waits and
// wind-down as in sparse_linear_umma_kernel.

constexpr int kPfTok = 128;                   // MMA N: tokens per unit
constexpr int kPfThreads = 576;               // 16 metadata/epilogue warps (8 per tile), the copy warp, the MMA warp
constexpr int kPfMaxCtas = 160;
constexpr unsigned kPfTmemCols = 512;         // accumulators 0..255, metadata from column 256
constexpr unsigned kPfMetaCol = 256;
constexpr int kPfTileBytes = kUmRows * 128;   // one tile's compressed values in a stage (16 KB)
constexpr int kPfXOff = 2 * kPfTileBytes;     // the activations' two 128 x 64 boxes
constexpr int kPfMetaOff = kPfXOff + 2 * kPfTok * 128;  // both tiles' metadata (2 x 2 KB)
constexpr int kPfStageTx = kPfMetaOff + 2 * kUmRows * 16;
constexpr int kPfStage = (kPfStageTx + 1023) / 1024 * 1024;
constexpr int kPfSmem = kUmStages * kPfStage + 1024;

struct PfOp {
    const void *meta;
    float *y;
    int64_t rows, cols;
    int64_t nch;         // 128-column chunks
    int64_t npairs;      // pairs of row tiles
    int64_t nt;          // token chunks
    int64_t rgroup;      // row-tile pairs per group of the unit order
    int64_t unit_begin;  // first unit of this operand in the launch
};

struct PfGroup {
    int32_t n;
    int32_t tokens;
    int64_t total_units;
    PfOp d[kMaxMats];
    TmMaps maps[kMaxMats];  // vals and meta as for the batched kernel; x boxes 64 x 128 tokens
};

struct PfCur {
    int op;
    int64_t pair, tc;
};

__device__ __forceinline__ PfCur pf_decode(const PfGroup &g, int64_t u) {
    int i = 0;
    while (i + 1 < g.n && u >= g.d[i + 1].unit_begin) ++i;
    const PfOp &d = g.d[i];
    const int64_t idx = u - d.unit_begin, per = d.rgroup * d.nt;
    const int64_t grp = idx / per, rem = idx % per;
    const int64_t rg = d.npairs - grp * d.rgroup < d.rgroup ? d.npairs - grp * d.rgroup : d.rgroup;
    return PfCur{i, grp * d.rgroup + rem % rg, rem / rg};
}

__device__ __forceinline__ void pf_issue(const PfGroup &g, const PfCur &c, int64_t j, unsigned stage, unsigned bar) {
    const TmMaps &mp = g.maps[c.op];
    const int row0 = (int)(c.pair * 2 * kUmRows), tok0 = (int)(c.tc * kPfTok);
    mbar_arrive_tx(bar, (unsigned)kPfStageTx);
    tma_load_2d(stage, &mp.vals, (int)(64 * j), row0, bar);
    tma_load_2d(stage + kPfTileBytes, &mp.vals, (int)(64 * j), row0 + kUmRows, bar);
    tma_load_2d(stage + kPfXOff, &mp.x, (int)(128 * j), tok0, bar);
    tma_load_2d(stage + kPfXOff + kPfTok * 128, &mp.x, (int)(128 * j + 64), tok0, bar);
    tma_load_2d(stage + kPfMetaOff, &mp.meta, (int)(4 * j), row0, bar);
    tma_load_2d(stage + kPfMetaOff + kUmRows * 16, &mp.meta, (int)(4 * j), row0 + kUmRows, bar);
}

__global__ void __launch_bounds__(kPfThreads, 1) sparse_linear_prefill_kernel(const __grid_constant__ PfGroup pg,
                                                                            unsigned int *__restrict__ err) {
    static_assert(kPfSmem + 1024 <= 232448, "fits one SM");
    static_assert(kPfMetaCol + 2 * 8 * kUmStages <= kPfTmemCols, "metadata columns fit");
    constexpr int kD = kUmStages;
    constexpr uint32_t kIdesc = um_idesc<kPfTok>();
    extern __shared__ unsigned char s_dyn_pf[];
    __shared__ __align__(8) unsigned long long s_full[kD], s_empty[kD], s_meta[kD], s_acc;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t G = gridDim.x, u0 = blockIdx.x, u1 = pg.total_units;
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_pf);
    const unsigned pad = (1024u - (dyn_s & 1023u)) & 1023u;
    const unsigned char *ring = s_dyn_pf + pad;
    const unsigned ring_s = dyn_s + pad;
    const unsigned full0 = (unsigned)__cvta_generic_to_shared(&s_full[0]);
    const unsigned empty0 = (unsigned)__cvta_generic_to_shared(&s_empty[0]);
    const unsigned meta0 = (unsigned)__cvta_generic_to_shared(&s_meta[0]);
    const unsigned accb = (unsigned)__cvta_generic_to_shared(&s_acc);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kD; ++s) {
            mbar_init(full0 + 8 * s, 1u);
            mbar_init(empty0 + 8 * s, 1u);
            mbar_init(meta0 + 8 * s, 256u);  // every metadata thread of both tiles arrives once per stage
        }
        mbar_init(accb, 1u);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        const unsigned dst = (unsigned)__cvta_generic_to_shared(&s_tmem);
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                     "r"(kPfTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;

    if (warp == 16) {
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
                    pf_issue(pg, c, j, ring_s + s * kPfStage, full0 + 8 * s);
                }
                ++issued;
            }
        }
        for (int s = 0; s < kD && s < issued; ++s) {
            const int last = s + ((issued - 1 - s) / kD) * kD;
            tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == 17) {
        // ------------------------------------------------------------ MMA warp
        int f = 0, commits = 0;
        bool stop = false;
        for (int64_t u = u0; u < u1 && !stop; u += G) {
            const PfCur c = pf_decode(pg, u);
            const int64_t nch = pg.d[c.op].nch;
            for (int64_t j = 0; j < nch; ++j, ++f) {
                const int s = f % kD;
                if (!um_wait(meta0 + 8 * s, (f / kD) & 1, &s_abort)) {
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    tc_fence_after();
                    const unsigned st = ring_s + s * kPfStage;
                    const uint64_t b0 = um_desc(st + kPfXOff), b1 = um_desc(st + kPfXOff + kPfTok * 128);
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const uint64_t a0 = um_desc(st + t * kPfTileBytes);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            umma_sp(tbase + t * kPfTok, a0 + (uint64_t)(2 * q),
                                    ((q >> 1) ? b1 : b0) + (uint64_t)(4 * (q & 1)),
                                    tbase + kPfMetaCol + 8 * (kD * t + s) + 2 * q, kIdesc, (j == 0 && q == 0) ? 0u : 1u);
                    }
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
        // ------------------------------------------------------------ metadata / epilogue warps
        // warps 0-3 and 8-11 take row tile 0 of the pair, warps 4-7 and 12-15 row tile 1 (TMEM
        // lane quarter warp % 4); warps 0-7 also turn the metadata into TMEM. Each warp stores
        // half of its lanes' 128 accumulator columns (warps 0-7 the first half).
        const int t = (warp >> 2) & 1, wq = warp & 3, half = warp >> 3;
        const unsigned tlane = tbase + ((unsigned)(32 * wq) << 16);
        const int h = (lane >> 3) & 1;
        const int ra = 32 * wq + 16 * (lane >> 4) + (lane & 7);  // rows ra and ra + 8 of the tile
        const uint32_t esel = h ? 0x7632u : 0x5410u;
        unsigned acc_phase = 0u;
        bool failed = false;
        int f = 0;
        for (int64_t u = u0; u < u1; u += G) {
            const PfCur c = pf_decode(pg, u);
            const PfOp &d = pg.d[c.op];
            for (int64_t j = 0; j < d.nch && half == 0; ++j, ++f) {
                const int s = f % kD;
                if (!failed) {
                    if (um_wait(full0 + 8 * s, (f / kD) & 1, &s_abort)) {
                        tc_fence_after();
                        const unsigned char *meta = ring + s * kPfStage + kPfMetaOff + t * kUmRows * 16;
                        const uint4 wa = lds128(meta + ra * 16), wb = lds128(meta + (ra + 8) * 16);
                        const uint32_t a4[4] = {wa.x, wa.y, wa.z, wa.w}, b4[4] = {wb.x, wb.y, wb.z, wb.w};
                        uint32_t e[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            e[q] = __byte_perm(a4[q] ? a4[q] : 0x44444444u, b4[q] ? b4[q] : 0x44444444u, esel);
                        tmem_st_meta(tlane + kPfMetaCol + 8 * (kD * t + s), e[0], e[1], e[2], e[3]);
                        tc_fence_before();
                        mbar_arrive(meta0 + 8 * s);
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
            if (um_bar_or<512>(!acc_ok)) {
                failed = true;
                break;
            }
            tc_fence_after();
            const int tok0 = (int)(c.tc * kPfTok);
            const int64_t r = (c.pair * 2 + t) * kUmRows + 32 * wq + lane;
#pragma unroll 1
            for (int k = half * (kPfTok / 2); k < (half + 1) * (kPfTok / 2); k += 16) {
                float v[16];
                tmem_ld16(tlane + t * kPfTok + k, v);
                if (r < d.rows) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (tok0 + k + i < pg.tokens) d.y[(int64_t)(tok0 + k + i) * d.rows + r] = v[i];
                }
            }
            tc_fence_before();
            um_bar<512>();  // every read of the accumulators precedes the next unit's first arrival
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kPfTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------ 4:8 on the dense tensor cores
//
// 4:8 has no hardware sparse mode. Per 128-column stage, kU8Warps warps expand the compressed
// tile into a dense 128 x 128 bf16 tile in tensor memory (row m in lane m, 64 columns of two
// bf16 each in K order), and one thread issues eight dense tcgen05.mma (kind::f16, K = 16)
// that read A from tensor memory and the activations from shared memory. A 4:8 block (four
// kept values in position order and the code p0 | p1 << 3 | p2 << 6 | p3 << 9) expands into
// exactly four 32-bit columns. Column i of a block (positions 2i, 2i+1) is
// prmt(prmt(v0v1, 0, A[p0p1].i), v2v3, B[p2p3].i): table A places the first pair and
// zero-fills, table B places the second pair and keeps the rest (u8_table_entry). Each CTA
// builds both 64-entry tables in shared memory, 8 interleaved copies each, so that the
// 16-byte lookups of a quarter-warp never share a bank. Thread t expands row t % 128, part
// t / 128 of the stage (64 / kU8Warps blocks: 16 columns, one tcgen05.st of its own lane),
// and arrives on the stage's "expanded" barrier after its store has completed; a separate MMA
// warp waits for all arrivals and issues the stage's MMAs, so the expanding warps never wait
// on one another within a tile (they meet once per tile, for the epilogue). The dense tile
// never enters shared memory, so a stage is only what the copy engine lands: values 16 KB |
// x, two kNTok x 64 boxes | metadata, 128 rows x 16 codes (4 KB); five or six stages in
// flight. Tensor memory: the accumulator in columns 0-63, stage s's dense tile in columns
// 64 + 64 s (it is rewritten only after the stage's MMAs have completed, which the copy warp
// waits for before it refills the stage). One CTA per SM. Epilogue: warp w reads TMEM lanes
// 32 (w % 4) .. +31 and the token slice w / 4. Copy warp, bounded waits, work split and
// partial tiles as above; a warp whose wait runs out stops working and leaves with the others
// at the end of the tile.

constexpr int kU8Warps = 16;         // expansion / epilogue warps (a multiple of 4, at most 16)
constexpr int kU8Threads = 32 * kU8Warps + 64;  // + the copy warp and the MMA warp
constexpr int kU8NStep = 8 * (kU8Warps / 4) > 16 ? 8 * (kU8Warps / 4) : 16;  // N is a multiple of this
constexpr unsigned kU8TmemCols = 512;  // accumulator at 0 (N <= 64 columns), the stages' dense tiles from kU8ACol
constexpr unsigned kU8ACol = 64;       // a stage's dense 128 x 128 bf16 tile: 64 columns (2 values per column)

template <int kNTok> constexpr int u8_tx() { return kUmRows * 128 + 2 * um_xbox_bytes<kNTok>() + kUmRows * 32; }
template <int kNTok> constexpr int u8_stage_bytes() { return (u8_tx<kNTok>() + 1023) / 1024 * 1024; }
// Stages in flight: as many as shared memory holds beside the selector tables, at most six
// (six dense tiles fill tensor memory beside the accumulator).
template <int kNTok> constexpr int u8_stages() { return kNTok <= 48 ? 6 : 5; }
constexpr int kU8TabCopies = 8;      // one copy per lane of a quarter-warp: conflict-free 16-byte lookups
constexpr int kU8TabBytes = 2 * 64 * kU8TabCopies * 16;  // tables A and B
// The two 8 KB selector tables come first, on an 8 KB boundary (so that a lookup's address is
// the table's base OR'ed with the entry's and the copy's bits), then the stages.
template <int kNTok> constexpr int u8_smem_bytes() { return u8_stages<kNTok>() * u8_stage_bytes<kNTok>() + 8192 + kU8TabBytes; }

// Instruction descriptor of kind::f16: dense, f32 accumulator, bf16 A and B (K-major),
// N = kNTok, M = 128.
template <int kNTok> constexpr uint32_t u8_idesc() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kNTok >> 3) << 17) | ((uint32_t)(kUmRows >> 4) << 24);
}

__device__ __forceinline__ void umma_dense(unsigned d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same with A read from tensor memory (a_tmem: lane 0, first column of the K-slice; A
// K-major, two bf16 per 32-bit column).
__device__ __forceinline__ void umma_dense_ta(unsigned d_tmem, unsigned a_tmem, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 consecutive 32-bit columns of this thread's lane from w[16]; the store completes
// asynchronously (tmem_st_wait waits for all of the warp's earlier stores).
__device__ __forceinline__ void tmem_st16(unsigned taddr, const uint32_t (&w)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};\n" ::"r"(taddr),
        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]),
        "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// 8 consecutive accumulator columns of this thread's lane (see tmem_ld16).
__device__ __forceinline__ void tmem_ld8(unsigned taddr, float *v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Entry q = pa | pb << 3 of expansion table A (second = false) or B (second = true): the
// byte-permute selectors of the four words of a dense chunk (one per component) for a value
// pair at positions pa < pb. Table A places the first pair (v0 v1, bytes 0-3 of
// the permute's sources) and takes zero bytes (4-7, a zero operand) elsewhere; table B places
// the second pair (v2 v3, bytes 4-7) over that result and keeps its bytes (0-3) elsewhere.
__device__ __forceinline__ uint4 u8_table_entry(int q, bool second) {
    const int pa = q & 7, pb = q >> 3;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t sel = 0u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int pos = 2 * i + h;
            const uint32_t base = second ? 4u : 0u, other = second ? 2u * h : 4u;
            const uint32_t b0 = pos == pa ? base : (pos == pb ? base + 2u : other);  // first source byte
            sel |= (b0 | (b0 + 1u) << 4) << (8 * h);
        }
        w[i] = sel;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int kNTok>
__device__ __forceinline__ void u8_issue(const TmGroup &tg, const Cursor &c, unsigned stage, unsigned bar) {
    const TmMaps &mp = tg.maps[c.op];
    const int j = (int)c.j, row0 = (int)(c.tile * kUmRows);
    mbar_arrive_tx(bar, (unsigned)u8_tx<kNTok>());
    tma_load_2d(stage, &mp.vals, 64 * j, row0, bar);
    tma_load_2d(stage + kUmRows * 128, &mp.x, 128 * j, 0, bar);
    tma_load_2d(stage + kUmRows * 128 + um_xbox_bytes<kNTok>(), &mp.x, 128 * j + 64, 0, bar);
    tma_load_2d(stage + kUmRows * 128 + 2 * um_xbox_bytes<kNTok>(), &mp.meta, 16 * j, row0, bar);
}

// Row r, part pt of a stage (kBlk = 64 / kU8Warps blocks from block kBlk pt) expanded into
// its 4 kBlk 32-bit columns of the row's dense K-slice: block b's eight values are columns
// 4 (b - kBlk pt) .. +3, two bf16 per column in K order (the layout tcgen05.mma reads A in
// from tensor memory).
// 16-byte load from a shared-memory address.
__device__ __forceinline__ uint4 lds128_at(unsigned addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// Row r, part pt of a stage (kBlk = 64 / kU8Warps blocks from block kBlk pt) expanded into
// its 4 kBlk 32-bit columns of the row's dense K-slice: block b's eight values are columns
// 4 (b - kBlk pt) .. +3, two bf16 per column in K order (the layout tcgen05.mma reads A in
// from tensor memory). ta / tb: shared-memory addresses of this lane's copy of entry 0 of
// tables A and B (8 KB aligned but for the copy's bits 4-6), so that the entry of a 6-bit
// pair code p is ta | p << 7: each lookup address is one shift and one masked OR of the
// block's code word.
template <int kBlk>
__device__ __forceinline__ void u8_expand(const unsigned char *st, unsigned ta, unsigned tb,
                                          int meta_off, int r, int pt, uint32_t (&w)[4 * kBlk]) {
    const int b0 = kBlk * pt;
    uint32_t codes[kBlk / 2];
    if constexpr (kBlk == 8) {
        const uint4 cw = lds128(st + meta_off + r * 32 + b0 * 2);
        codes[0] = cw.x; codes[1] = cw.y; codes[2] = cw.z; codes[3] = cw.w;
    } else {
        const uint2 cw = *reinterpret_cast<const uint2 *>(st + meta_off + r * 32 + b0 * 2);
        codes[0] = cw.x; codes[1] = cw.y;
    }
#pragma unroll
    for (int c = 0; c < kBlk / 2; ++c) {
        const int cl = (b0 >> 1) + c;  // value chunk within the row
        const uint4 v = lds128(st + r * 128 + ((cl ^ (r & 7)) << 4));
        const uint32_t cw = codes[c];  // block 2c + 0 in bits 0-11, block 2c + 1 in bits 16-27
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t lo = h ? v.z : v.x, hi = h ? v.w : v.y;
            // pair codes p0p1 (code bits 0-5) and p2p3 (bits 6-11) placed at bits 7-12
            const uint32_t ka = (h ? (cw >> 9) : (cw << 7)) & 0x1F80u;
            const uint32_t kb = (h ? (cw >> 15) : (cw << 1)) & 0x1F80u;
            const uint4 sa = lds128_at(ta | ka), sb = lds128_at(tb | kb);
            uint32_t *o = w + 4 * (2 * c + h);
            o[0] = __byte_perm(__byte_perm(lo, 0u, sa.x), hi, sb.x);
            o[1] = __byte_perm(__byte_perm(lo, 0u, sa.y), hi, sb.y);
            o[2] = __byte_perm(__byte_perm(lo, 0u, sa.z), hi, sb.z);
            o[3] = __byte_perm(__byte_perm(lo, 0u, sa.w), hi, sb.w);
        }
    }
}

template <int kHalf>
__device__ __forceinline__ void u8_store(const SkOp &d, int64_t tile, int q, int lane, int tok0,
                                         const float (&v)[kHalf], int tokens) {
    const int64_t r = tile * kUmRows + 32 * q + lane;
    if (r >= d.rows) return;
#pragma unroll
    for (int i = 0; i < kHalf; ++i)
        if (tok0 + i < tokens) d.y[(tok0 + i) * d.rows + r] = v[i];
}

template <int kNTok>
__global__ void __launch_bounds__(kU8Threads, 1) sparse_linear_umma48_kernel(const __grid_constant__ TmGroup tg,
                                                                            float *__restrict__ part,
                                                                            unsigned int *__restrict__ tickets,
                                                                            unsigned int *__restrict__ err,
                                                                            int arm_only_first) {
    static_assert(kNTok % 16 == 0 && kNTok >= 16 && kNTok <= kMaxTokens, "N of an M = 128 MMA");
    static_assert(2 * (u8_smem_bytes<kNTok>() + 1024) > 233472, "one CTA per SM");
    static_assert(u8_smem_bytes<kNTok>() + 1024 <= 232448, "fits one SM");
    static_assert(kU8ACol >= (unsigned)kNTok && kU8ACol + 64u * u8_stages<kNTok>() <= kU8TmemCols,
                  "accumulator and dense tiles fit tensor memory");
    static_assert(kU8Warps == 16, "four threads per row, one x16 store of 16 columns each");
    static_assert(kU8Warps % 4 == 0 && kU8Warps <= 16 && kNTok % (8 * (kU8Warps / 4)) == 0,
                  "each epilogue warp takes a multiple of 8 token columns");
    constexpr int kD = u8_stages<kNTok>(), kStage = u8_stage_bytes<kNTok>();
    constexpr int kMetaOff = kUmRows * 128 + 2 * um_xbox_bytes<kNTok>();
    constexpr int kHalf = kNTok / (kU8Warps / 4);  // token columns per epilogue warp
    constexpr int kBar = 32 * kU8Warps;
    constexpr uint32_t kIdesc = u8_idesc<kNTok>();
    extern __shared__ unsigned char s_dyn_u8[];
    __shared__ __align__(8) unsigned long long s_full[kD], s_empty[kD], s_exp[kD], s_acc;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    __shared__ int s_last;
    const SkGroup &grp = tg.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t total = grp.total_chunks;
    const int64_t G = imin64((int64_t)gridDim.x, total), cta = blockIdx.x;
    if (cta >= G) return;  // the whole CTA, before any barrier or allocation
    const int64_t lo = cta * total / G, hi = (cta + 1) * total / G;
    const int n = (int)(hi - lo);
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_u8);
    const unsigned tab_s = (dyn_s + 8191u) & ~8191u;  // tables A, B: 8 KB each on 8 KB boundaries
    uint4 *tab = reinterpret_cast<uint4 *>(s_dyn_u8 + (tab_s - dyn_s));  // A: entries [0, 64), B: [64, 128), x copies
    const unsigned ring_s = tab_s + (unsigned)kU8TabBytes;  // 1 KB aligned
    unsigned char *ring = s_dyn_u8 + (ring_s - dyn_s);
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
                     "r"(kU8TmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;

    if (warp == kU8Warps) {
        // ------------------------------------------------------------ copy warp
        Cursor ld = sk_decode(grp, lo);
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
                if (f == 0 && arm_only_first)  // test of the bounded wait: a stage nothing fills
                    mbar_arrive_tx(full0, (unsigned)u8_tx<kNTok>());
                else {
                    fence_proxy_async();
                    u8_issue<kNTok>(tg, ld, ring_s + s * kStage, full0 + 8 * s);
                }
            }
            ++issued;
            sk_advance(grp, ld);
        }
        for (int s = 0; s < kD && s < issued; ++s) {
            const int last = s + ((issued - 1 - s) / kD) * kD;
            tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == kU8Warps + 1) {
        // ------------------------------------------------------------ MMA warp
        Cursor cc = sk_decode(grp, lo);
        bool fresh = true;
        int commits = 0;
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            if (!um_wait(exp0 + 8 * s, (f / kD) & 1, &s_abort)) {
                if (lane == 0 && !s_abort) {
                    atomicOr(err, 1u);
                    s_abort = 1;
                }
                break;
            }
            const SkOp &d = grp.d[cc.op];
            const bool piece_end = (cc.j == d.nch - 1) || (f == n - 1);
            if (lane == 0) {
                tc_fence_after();
                const unsigned sa = ring_s + s * kStage;
                const unsigned ta = tbase + kU8ACol + 64u * (unsigned)s;  // the stage's dense tile
                const uint64_t b0 = um_desc(sa + kUmRows * 128),
                               b1 = um_desc(sa + kUmRows * 128 + um_xbox_bytes<kNTok>());
#pragma unroll
                for (int j = 0; j < 8; ++j)  // K = 16 per MMA: 8 columns of A
                    umma_dense_ta(tbase, ta + 8u * (unsigned)j, ((j >> 2) ? b1 : b0) + (uint64_t)(2 * (j & 3)),
                                  kIdesc, (fresh && j == 0) ? 0u : 1u);
                umma_commit(empty0 + 8 * s);
                if (piece_end) umma_commit(accb);
            }
            __syncwarp();
            ++commits;
            fresh = piece_end;
            sk_advance(grp, cc);
        }
        if (commits > 0) {  // every MMA has completed (bounded) before the tensor memory is released
            const int f = commits - 1;
            tm_wait(empty0 + 8 * (f % kD), (f / kD) & 1);
        }
    } else {
        // ------------------------------------------------------------ expansion / epilogue warps
        const int r = threadIdx.x & (kUmRows - 1), pt = threadIdx.x >> 7;
        const int q = warp & 3, ch = warp >> 2;  // TMEM lane quarter, token slice of the epilogue
        const unsigned tq = tbase + ((unsigned)(32 * q) << 16) + (unsigned)(ch * kHalf);
        const unsigned tdense = tbase + ((unsigned)(32 * q) << 16) + kU8ACol + 16u * (unsigned)pt;  // row r's part
        const unsigned tab_a = tab_s + 16u * (unsigned)(lane & (kU8TabCopies - 1)), tab_b = tab_a + 64u * 16u * kU8TabCopies;
        Cursor cc = sk_decode(grp, lo);
        unsigned acc_phase = 0u;
        bool failed = false;
        // With six stages in flight, a stage's store into tensor memory is waited for (and the
        // stage handed to the MMA warp) only after the next stage's expansion, so the store's
        // latency overlaps it (1-32 tokens: 1 % faster); with five (above 48 tokens) the lost
        // stage costs more (2 %), so there each stage is handed over at once.
        constexpr bool kDefer = kD >= 6;
        int pending = -1;
        auto hand_over = [&]() {
            if (pending >= 0) {
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(exp0 + 8 * pending);
                pending = -1;
            }
        };
        for (int f = 0; f < n; ++f) {
            const int s = f % kD;
            unsigned char *st = ring + s * kStage;
            // A warp whose wait ran out stops working but keeps its place in the loop, so that
            // it meets the others at the end of the tile, where all of them leave together.
            if (!failed) {
                if (um_wait(full0 + 8 * s, (f / kD) & 1, &s_abort)) {
                    uint32_t w[16];
                    u8_expand<64 / kU8Warps>(st, tab_a, tab_b, kMetaOff, r, pt, w);
                    hand_over();
                    tmem_st16(tdense + 64u * (unsigned)s, w);  // into the stage's dense tile in tensor memory
                    pending = s;
                    if (!kDefer) hand_over();
                } else {
                    hand_over();
                    failed = true;
                    if (lane == 0 && !s_abort) {
                        atomicOr(err, 1u);
                        s_abort = 1;
                    }
                }
            }
            const SkOp &d = grp.d[cc.op];
            const bool piece_end = (cc.j == d.nch - 1) || (f == n - 1);
            if (piece_end) hand_over();
            if (piece_end) {
                const bool acc_ok = !failed && um_wait(accb, acc_phase, &s_abort);
                acc_phase ^= 1u;
                if (um_bar_or<kBar>(!acc_ok)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                float v[kHalf];
#pragma unroll
                for (int k = 0; k < kHalf / 8; ++k) tmem_ld8(tq + 8 * k, v + 8 * k);
                tc_fence_before();  // these reads precede the next piece's first MMA (after its arrivals)
                const int64_t a = d.chunk_begin + cc.tile * d.nch, b = a + d.nch;
                const int64_t c1 = ((a + 1) * G - 1) / total, c2 = (b * G - 1) / total;
                const int tok0 = ch * kHalf;
                if (c1 == c2) {
                    u8_store<kHalf>(d, cc.tile, q, lane, tok0, v, grp.tokens);
                } else {
                    const int64_t lo1 = c1 * total / G;
                    const int slot = (cta == c1 && lo1 < a) ? 1 : 0;
                    float *mine = part + (size_t)(cta * 2 + slot) * kUmPartFloats + (size_t)tok0 * kUmRows + 32 * q + lane;
#pragma unroll
                    for (int i = 0; i < kHalf; ++i) __stcg(mine + i * kUmRows, v[i]);
                    __threadfence();
                    um_bar<kBar>();
                    if (threadIdx.x == 0) s_last = (atomicAdd(tickets + c1, 1u) == (unsigned int)(c2 - c1));
                    um_bar<kBar>();
                    if (s_last) {
                        __threadfence();
                        float sum[kHalf];
#pragma unroll
                        for (int i = 0; i < kHalf; ++i) sum[i] = 0.f;
                        for (int64_t qq = c1; qq <= c2; ++qq) {
                            const int sid = (qq == c1 && lo1 < a) ? 1 : 0;
                            const float *p = part + (size_t)(qq * 2 + sid) * kUmPartFloats + (size_t)tok0 * kUmRows + 32 * q + lane;
#pragma unroll
                            for (int i = 0; i < kHalf; ++i) sum[i] += __ldcg(p + i * kUmRows);
                        }
                        u8_store<kHalf>(d, cc.tile, q, lane, tok0, sum, grp.tokens);
                        um_bar<kBar>();
                        if (threadIdx.x == 0) tickets[c1] = 0u;
                    }
                }
            }
            sk_advance(grp, cc);
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kU8TmemCols)
                     : "memory");
    }
}

}  // namespace spl
}  // namespace mllm
