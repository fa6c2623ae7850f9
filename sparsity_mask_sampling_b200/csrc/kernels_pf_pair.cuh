// kernels_pf_pair.cuh -- the 2:4 serving product at prefill sizes on pairs of SMs.
//
// The product y = x W*^T of sparse_linear_prefill_kernel (MaskLLM serves the masked network
// from its packed hard mask after training: paper-graph-ui summary of arXiv 2409.17481,
// s.3.2 "Information flow at inference"; s.5 Table 16 times 128- and 2048-token prompts),
// with the sparse MMA spread over the two CTAs of a cluster (tcgen05.mma.sp.cta_group::2,
// M = 256). In one instruction the tensor cores of both SMs compute a 256 x 128 tile: A is
// 128 rows from each CTA's shared memory, B (the 128-token activation box) is 64 tokens from
// each, and each CTA's tensor memory receives its own 128 rows x 128 tokens. Every staged
// activation byte therefore feeds twice the MMA work it feeds in the single-SM kernel:
// per 128-column stage a CTA stages 52 KB (two 128-row value tiles of 16 KB, a 64-token half
// of the activation box in two 8 KB pieces, 4 KB of metadata) where the single-SM kernel
// stages 68 KB for the same MMA work, and four stages fit where three did.
//
// A unit is (operand, four 128-row tiles, 128-token chunk) over all columns: CTA r of the
// pair holds row tiles 512 u + 256 t + 128 r (t = 0, 1), so MMA t covers the 256 rows
// 512 u + 256 t ... + 255 with the rows of CTA 0 first. Units are ordered and dealt to the
// clusters as in the single-SM kernel (groups of row units, token chunk by token chunk).
//
// Roles (per CTA, 18 warps): warp 16 copies, in both CTAs: the values and activation boxes
// land through the pair form of the tensor copy, which completes on the LEADER's (rank 0)
// "full" barrier; the metadata lands through the ordinary form on the CTA's own "metadata
// full" barrier. Warps 0-7 turn the CTA's metadata into its tensor memory (the layout of the
// single-SM kernel, same columns in both CTAs) and, one lane per warp, arrive on the
// leader's "metadata" barrier (16 arrivals per stage; the peer's are remote arrivals with
// release at cluster scope). Warp 17 of the leader waits for both barriers, issues the
// stage's eight pair MMAs and commits them to the "empty" barrier of both CTAs (a multicast
// commit); at a unit's last stage it commits the "accumulator" barrier of both CTAs. Warps
// 0-15 of each CTA store that CTA's rows. The leader's next unit cannot overwrite either
// accumulator before both CTAs' epilogues end: its MMAs wait for metadata arrivals that each
// CTA's metadata warps make only after their epilogue's reads.
//
// Tensor memory is allocated for the pair (cta_group::2, 512 columns in each CTA: the two
// accumulators at 0-255, stage metadata from 256). Every wait is bounded (kTmWaitNs); a
// timeout sets the error word and the CTA winds down as the single-SM kernel does; both CTAs
// meet at a cluster barrier before the pair frees its tensor memory and exits, so no copy,
// arrival or MMA of one CTA targets a CTA that has left.
#pragma once

#include "kernels_umma.cuh"

namespace mllm {
namespace spl {

constexpr int kP2Stages = 4;
constexpr int kP2Half = kPfTok / 2;                         // tokens of the activation box per CTA
constexpr int kP2XOff = 2 * kPfTileBytes;                   // after the two value tiles (32 KB)
constexpr int kP2XPiece = kP2Half * 128;                    // one 64-token x 64-column piece (8 KB)
constexpr int kP2MetaOff = kP2XOff + 2 * kP2XPiece;         // 48 KB
constexpr int kP2PairTx = kP2MetaOff;                       // bytes per CTA on the leader's barrier
constexpr int kP2MetaTx = 2 * kUmRows * 16;                 // metadata of both tiles (4 KB)
constexpr int kP2Stage = (kP2MetaOff + kP2MetaTx + 1023) / 1024 * 1024;
constexpr int kP2Smem = kP2Stages * kP2Stage + 1024;
constexpr int kP2RowUnit = 4 * kUmRows;                     // rows of a unit (512)
constexpr int kP2MaxPairs = 80;

// Instruction descriptor of the pair MMA: sparse, f32 accumulator, bf16 A and B (K-major),
// N = 128 tokens, M = 256 (128 rows in each CTA).
constexpr uint32_t p2_idesc() {
    return (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kPfTok >> 3) << 17) |
           ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ unsigned cluster_rank() {
    unsigned r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}

// The shared::cluster address of this CTA's shared-memory location saddr in CTA `rank`.
__device__ __forceinline__ unsigned cluster_addr(unsigned saddr, unsigned rank) {
    unsigned r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Arrival on another CTA's barrier. The data it publishes is tensor memory, ordered by the
// tcgen05 fences around the arrival, so the arrival needs no cluster-scope release (which
// would cost a memory barrier per arrival on the pipeline's critical path).
__device__ __forceinline__ void mbar_arrive_remote(unsigned caddr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];\n" ::"r"(caddr) : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// A tile copy of either CTA of the pair whose completion is counted on the leader's barrier
// (bar_caddr: its shared::cluster address); the data lands in the issuing CTA's memory.
__device__ __forceinline__ void tma_load_2d_pair(unsigned dst, const CUtensorMap *map, int x, int y, unsigned bar_caddr) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_caddr)
        : "memory");
}

__device__ __forceinline__ void umma_sp_pair(unsigned d_tmem, uint64_t adesc, uint64_t bdesc, unsigned e_tmem,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %5, 0;\n"
        " tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%3], %4, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at shared-memory offset `bar` of both CTAs when the pair MMAs
// issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(unsigned bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n" ::"r"(
            bar),
        "h"((unsigned short)3u)
        : "memory");
}

// One stage of a unit for CTA `rank`: its two value tiles and its half of the activation box
// on the leader's barrier (the leader also announces the pair's bytes there), its metadata on
// its own barrier.
__device__ __forceinline__ void p2_issue(const PfGroup &g, const PfCur &c, int64_t j, unsigned rank,
                                         unsigned stage, unsigned lead_full, unsigned own_full,
                                         unsigned own_mfull) {
    const TmMaps &mp = g.maps[c.op];
    const int row0 = (int)(c.pair * kP2RowUnit + rank * kUmRows), tok0 = (int)(c.tc * kPfTok + rank * kP2Half);
    mbar_arrive_tx(own_mfull, (unsigned)kP2MetaTx);
    tma_load_2d(stage + kP2MetaOff, &mp.meta, (int)(4 * j), row0, own_mfull);
    tma_load_2d(stage + kP2MetaOff + kUmRows * 16, &mp.meta, (int)(4 * j), row0 + 2 * kUmRows, own_mfull);
    if (rank == 0) mbar_arrive_tx(own_full, (unsigned)(2 * kP2PairTx));
    tma_load_2d_pair(stage, &mp.vals, (int)(64 * j), row0, lead_full);
    tma_load_2d_pair(stage + kPfTileBytes, &mp.vals, (int)(64 * j), row0 + 2 * kUmRows, lead_full);
    tma_load_2d_pair(stage + kP2XOff, &mp.x, (int)(128 * j), tok0, lead_full);
    tma_load_2d_pair(stage + kP2XOff + kP2XPiece, &mp.x, (int)(128 * j + 64), tok0, lead_full);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPfThreads, 1)
    sparse_linear_prefill_pair_kernel(const __grid_constant__ PfGroup pg, unsigned int *__restrict__ err) {
    static_assert(kP2Smem + 1024 <= 232448, "fits one SM");
    static_assert(kPfMetaCol + 2 * 8 * kP2Stages <= kPfTmemCols, "metadata columns fit");
    constexpr int kD = kP2Stages;
    constexpr uint32_t kIdesc = p2_idesc();
    extern __shared__ unsigned char s_dyn_p2[];
    __shared__ __align__(8) unsigned long long s_full[kD], s_mfull[kD], s_empty[kD], s_meta[kD], s_acc;
    __shared__ unsigned s_tmem;
    __shared__ volatile int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned rank = cluster_rank();
    const int64_t P = gridDim.x >> 1, u0 = blockIdx.x >> 1, u1 = pg.total_units;
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_p2);
    const unsigned pad = (1024u - (dyn_s & 1023u)) & 1023u;
    const unsigned char *ring = s_dyn_p2 + pad;
    const unsigned ring_s = dyn_s + pad;
    const unsigned full0 = (unsigned)__cvta_generic_to_shared(&s_full[0]);
    const unsigned mfull0 = (unsigned)__cvta_generic_to_shared(&s_mfull[0]);
    const unsigned empty0 = (unsigned)__cvta_generic_to_shared(&s_empty[0]);
    const unsigned meta0 = (unsigned)__cvta_generic_to_shared(&s_meta[0]);
    const unsigned accb = (unsigned)__cvta_generic_to_shared(&s_acc);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kD; ++s) {
            mbar_init(full0 + 8 * s, 1u);    // the leader's copy warp (with both CTAs' bytes)
            mbar_init(mfull0 + 8 * s, 1u);   // this CTA's copy warp (its metadata bytes)
            mbar_init(empty0 + 8 * s, 1u);   // the leader's commit
            mbar_init(meta0 + 8 * s, 16u);   // one lane of each metadata warp of both CTAs
        }
        mbar_init(accb, 1u);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    cluster_sync_all();  // both CTAs' barriers exist before any copy or arrival crosses the pair
    if (warp == 0) {
        const unsigned dst = (unsigned)__cvta_generic_to_shared(&s_tmem);
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
                     "r"(kPfTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const unsigned tbase = s_tmem;
    const unsigned lead_full0 = cluster_addr(full0, 0u), lead_meta0 = cluster_addr(meta0, 0u);

    if (warp == 16) {
        // ------------------------------------------------------------ copy warp (both CTAs)
        int f = 0, issued = 0;
        bool stop = false;
        for (int64_t u = u0; u < u1 && !stop; u += P) {
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
                    p2_issue(pg, c, j, rank, ring_s + s * kP2Stage, lead_full0 + 8 * s, full0 + 8 * s, mfull0 + 8 * s);
                }
                ++issued;
            }
        }
        // this CTA's metadata copies have landed (and, on the leader, both CTAs' other copies)
        for (int s = 0; s < kD && s < issued; ++s) {
            const int last = s + ((issued - 1 - s) / kD) * kD;
            tm_wait(mfull0 + 8 * s, (last / kD) & 1);
            if (rank == 0) tm_wait(full0 + 8 * s, (last / kD) & 1);
        }
    } else if (warp == 17) {
        // ------------------------------------------------------------ MMA warp (leader only)
        if (rank == 0) {
            int f = 0, commits = 0;
            bool stop = false;
            for (int64_t u = u0; u < u1 && !stop; u += P) {
                const PfCur c = pf_decode(pg, u);
                const int64_t nch = pg.d[c.op].nch;
                for (int64_t j = 0; j < nch; ++j, ++f) {
                    const int s = f % kD;
                    const unsigned ph = (f / kD) & 1;
                    if (!um_wait(full0 + 8 * s, ph, &s_abort) || !um_wait(meta0 + 8 * s, ph, &s_abort)) {
                        if (lane == 0 && !s_abort) {
                            atomicOr(err, 1u);
                            s_abort = 1;
                        }
                        stop = true;
                        break;
                    }
                    if (lane == 0) {
                        tc_fence_after();
                        const unsigned st = ring_s + s * kP2Stage;
                        const uint64_t b0 = um_desc(st + kP2XOff), b1 = um_desc(st + kP2XOff + kP2XPiece);
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            const uint64_t a0 = um_desc(st + t * kPfTileBytes);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                umma_sp_pair(tbase + t * kPfTok, a0 + (uint64_t)(2 * q),
                                             ((q >> 1) ? b1 : b0) + (uint64_t)(4 * (q & 1)),
                                             tbase + kPfMetaCol + 8 * (kD * t + s) + 2 * q, kIdesc,
                                             (j == 0 && q == 0) ? 0u : 1u);
                        }
                        umma_commit_pair(empty0 + 8 * s);
                        if (j == nch - 1) umma_commit_pair(accb);
                    }
                    __syncwarp();
                    ++commits;
                }
            }
            if (commits > 0) {
                const int ff = commits - 1;
                tm_wait(empty0 + 8 * (ff % kD), (ff / kD) & 1);
            }
        }
    } else {
        // ------------------------------------------------------------ metadata / epilogue warps
        // as in the single-SM kernel: warps 0-3 and 8-11 take row tile 0, warps 4-7 and 12-15
        // row tile 1 (TMEM lane quarter warp % 4); warps 0-7 also turn the metadata into TMEM
        const int t = (warp >> 2) & 1, wq = warp & 3, half = warp >> 3;
        const unsigned tlane = tbase + ((unsigned)(32 * wq) << 16);
        const int h = (lane >> 3) & 1;
        const int ra = 32 * wq + 16 * (lane >> 4) + (lane & 7);  // rows ra and ra + 8 of the tile
        const uint32_t esel = h ? 0x7632u : 0x5410u;
        unsigned acc_phase = 0u;
        bool failed = false;
        int f = 0;
        for (int64_t u = u0; u < u1; u += P) {
            const PfCur c = pf_decode(pg, u);
            const PfOp &d = pg.d[c.op];
            for (int64_t j = 0; j < d.nch && half == 0; ++j, ++f) {
                const int s = f % kD;
                if (!failed) {
                    if (um_wait(mfull0 + 8 * s, (f / kD) & 1, &s_abort)) {
                        tc_fence_after();
                        const unsigned char *meta = ring + s * kP2Stage + kP2MetaOff + t * kUmRows * 16;
                        const uint4 wa = lds128(meta + ra * 16), wb = lds128(meta + (ra + 8) * 16);
                        const uint32_t a4[4] = {wa.x, wa.y, wa.z, wa.w}, b4[4] = {wb.x, wb.y, wb.z, wb.w};
                        uint32_t e[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            e[q] = __byte_perm(a4[q] ? a4[q] : 0x44444444u, b4[q] ? b4[q] : 0x44444444u, esel);
                        tmem_st_meta(tlane + kPfMetaCol + 8 * (kD * t + s), e[0], e[1], e[2], e[3]);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if (rank == 0) mbar_arrive(meta0 + 8 * s);
                            else mbar_arrive_remote(lead_meta0 + 8 * s);
                        }
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
            const int64_t r = c.pair * kP2RowUnit + 2 * kUmRows * t + kUmRows * rank + 32 * wq + lane;
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
    cluster_sync_all();  // neither CTA frees its tensor memory or leaves while the other may use it
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kPfTmemCols)
                     : "memory");
    }
}

}  // namespace spl
}  // namespace mllm
