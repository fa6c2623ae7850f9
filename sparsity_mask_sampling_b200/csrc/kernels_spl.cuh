// kernels_spl.cuh -- product of activations with a hard-masked weight in its packed form.
//
// After training, MaskLLM applies the learned mask once and serves the sparse network
// (paper-graph-ui summary of arXiv 2409.17481, s.3.2 "Information flow at inference"). These
// kernels compute y = x W*^T for W* = W (.) M* stored as mllm_hard_pack writes it (N kept
// bf16 values per block of M consecutive weights plus their positions), for a few tokens per
// call (decode). At that size the product is bound by reading the compressed weight from
// HBM: 2:4 moves 2.25 bytes per weight pair instead of 4 dense.
//
// Operands with cols % 128 == 0 (every LLM shape) run on the fifth-generation tensor cores
// (kernels_umma.cuh) -- 2:4 above 16 tokens, 4:8 at any token count. The rest run here, up to
// 16 tokens per launch (more as groups of 16), on four kernels chosen per launch by the
// operands' widths (host side, mllm.cu):
//   sparse_linear_tma_kernel  2:4, cols % 128 == 0, 1-16 tokens: sparse tensor cores (mma.sp)
//                             fed by tiled tensor copies;
//   sparse_linear_sp_kernel   2:4, cols % 32 == 0: the same arithmetic fed by cp.async;
//   sparse_linear_sk_kernel   4:8 (no hardware sparse path) and 2:4 with cols % 16 == 0:
//                             blocks expanded to dense bf16 in registers, dense mma.sync;
//   sparse_linear_kernel      any cols % M == 0: the expansion with element-wise loads.
// The last three split the launch's chunks evenly over all warps (stream-K); the first
// kernel below splits whole row tiles over CTAs and is kept for the element-wise case.
//
// Mapping of the expansion kernels. A warp owns a tile of 16 rows; per chunk of 64 columns
// each thread (g = lane/4, t = lane%4) loads, for rows g and g+8 of the tile, the compressed
// values and metadata of columns 16t..16t+15 (one 16-byte vector and one 32-bit metadata word
// per row) and the same 16 columns of x for token g (and g+8). It expands its blocks to dense
// bf16 pairs in registers -- byte permutes whose selectors come from a small shared-memory
// table indexed by the metadata -- and issues four bf16 mma.sync m16n8k16 steps. The order of
// the k-sum is free, so the k-slots {2t, 2t+1, 2t+8, 2t+9} of step s are mapped to columns
// 16t+4s..16t+4s+3 of the chunk, for A and B alike: every thread then reads whole vectors of
// its own columns. In the tiled kernel the kWarps warps of a CTA work on kMT row tiles, kKS =
// kWarps/kMT warps per tile taking every kKS-th chunk; the partial tiles are added in shared
// memory in warp order, so the result is deterministic. 4:8 uses the same mapping (a thread
// owns two 4:8 blocks per chunk).
#pragma once

#include <cuda.h>  // CUtensorMap (type only; maps are encoded through the runtime's driver entry point)

#include "device_common.cuh"

namespace mllm {
namespace spl {

constexpr int kWarps = 8;
constexpr int kCtaThreads = 32 * kWarps;
constexpr int kChunk = 64;       // columns per k-chunk of a warp
constexpr int kMaxTokens = 64;   // per call; 17-64 tokens: the batched kernel (2:4) or groups of 16
constexpr int kMaxTileTokens = 16;  // two n8 tiles: the per-warp kernels

// One operand of a grouped call.
struct Op {
    const uint32_t *vals;    // packed values viewed as 32-bit words; cols/4 words per row
    const void *meta;        // 2:4: uint32 [rows, ceil(cols/32)]; 4:8: uint16 [rows, cols/8]
    const uint32_t *x;       // [tokens, cols] bf16, viewed as pairs
    float *y;                // [tokens, rows]
    int64_t rows, cols;
    int64_t task_begin;      // first task of this operand in the launch
};

struct OpGroup {
    int32_t n;
    int32_t tokens;
    int64_t total_tasks;
    Op d[kMaxMats];
};

__device__ __forceinline__ int find_op(const OpGroup &g, int64_t task) {
    int i = 0;
    while (i + 1 < g.n && task >= g.d[i + 1].task_begin) ++i;
    return i;
}

// ------------------------------------------------------------------ expansion tables

// 2:4: metadata nibble p0 | p1 << 2 -> byte-permute selectors that turn the block's value
// word (v0 in bytes 0-1, v1 in bytes 2-3; second operand 0) into dense positions (0,1) and
// (2,3). A position that is neither p0 nor p1 takes zero bytes (selector 4, 5).
struct Sel24Table {
    uint32_t lo[16], hi[16];
    static constexpr uint32_t src(int j, int p0, int p1) {
        return j == p0 ? 0x10u : (j == p1 ? 0x32u : 0x54u);  // two selector nibbles per bf16
    }
    constexpr Sel24Table() : lo(), hi() {
        for (int nib = 0; nib < 16; ++nib) {
            const int p0 = nib & 3, p1 = nib >> 2;
            lo[nib] = src(0, p0, p1) | src(1, p0, p1) << 8;
            hi[nib] = src(2, p0, p1) | src(3, p0, p1) << 8;
        }
    }
};
__device__ const Sel24Table g_sel24 = Sel24Table();

// 4:8: keep mask km (bit j = position j kept) -> for each dense pair (2i, 2i+1) a selector
// into the block's 8 value bytes (value r in bytes 2r, 2r+1, r = rank of the position among
// the kept ones) and a mask that zeroes the pruned half words.
struct Sel48Table {
    uint32_t sel[256][4], mask[256][4];
    static constexpr int rank(int km, int j) {
        int r = 0;
        for (int q = 0; q < j; ++q) r += (km >> q) & 1;
        return r;
    }
    constexpr Sel48Table() : sel(), mask() {
        for (int km = 0; km < 256; ++km)
            for (int i = 0; i < 4; ++i) {
                uint32_t s = 0, mk = 0;
                for (int h = 0; h < 2; ++h) {
                    const int j = 2 * i + h, r = rank(km, j);
                    if (((km >> j) & 1) && r < 4) {
                        s |= (uint32_t)(2 * r | (2 * r + 1) << 4) << (8 * h);
                        mk |= 0xFFFFu << (16 * h);
                    }
                }
                sel[km][i] = s;
                mask[km][i] = mk;
            }
    }
};
__device__ const Sel48Table g_sel48 = Sel48Table();

__device__ __forceinline__ uint32_t keep_mask48(uint32_t code) {
    return (1u << (code & 7u)) | (1u << ((code >> 3) & 7u)) | (1u << ((code >> 6) & 7u)) |
           (1u << ((code >> 9) & 7u));
}

// ------------------------------------------------------------------ tile pieces

template <int kNT>
struct Slab {
    uint4 v[2];        // compressed values of rows g, g+8: columns 16t..16t+15 of the chunk
    uint32_t m[2];     // their metadata: 2:4 four nibbles (low 16 bits), 4:8 two codes
    uint4 x[kNT][2];   // x of token g + 8*nt, the same 16 columns
};

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Loads the slab of columns col0..col0+15 (col0 = 64*chunk + 16t) of rows r0, r1, one block
// and one x element at a time with bounds checks (any cols % M == 0; zeros past the matrix).
template <int kN, int kNT>
__device__ __forceinline__ void load_slab(Slab<kNT> &s, const Op &d, int64_t r0, int64_t r1, int64_t col0,
                                          int g, int tokens) {
    const int64_t cols = d.cols, bpr = cols / (2 * kN);
    const int64_t wpr = cols >> 2;  // value words per row
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t r = h ? r1 : r0;
        uint32_t v[4] = {0u, 0u, 0u, 0u}, m = 0u;
        if (r < d.rows) {
            if constexpr (kN == 2) {
                const int64_t mw = (bpr + 7) >> 3;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int64_t b = (col0 >> 2) + q;
                    if (b < bpr) {
                        v[q] = d.vals[r * bpr + b];
                        const uint32_t w = static_cast<const uint32_t *>(d.meta)[r * mw + (b >> 3)];
                        m |= ((w >> (4 * (b & 7))) & 0xFu) << (4 * q);
                    }
                }
            } else {
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int64_t b = (col0 >> 3) + q;
                    if (b < bpr) {
                        v[2 * q] = d.vals[r * wpr + 2 * b];
                        v[2 * q + 1] = d.vals[r * wpr + 2 * b + 1];
                        m |= (uint32_t) static_cast<const uint16_t *>(d.meta)[r * bpr + b] << (16 * q);
                    }
                }
            }
        }
        s.v[h] = make_uint4(v[0], v[1], v[2], v[3]);
        s.m[h] = m;
    }
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
        const int tok = g + 8 * nt;
        uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (tok < tokens) {
            const uint16_t *xr = reinterpret_cast<const uint16_t *>(d.x) + tok * cols;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int64_t c = col0 + 2 * j;
                const uint32_t lo = c < cols ? xr[c] : 0u, hi = c + 1 < cols ? xr[c + 1] : 0u;
                w[j] = lo | hi << 16;
            }
        }
        s.x[nt][0] = make_uint4(w[0], w[1], w[2], w[3]);
        s.x[nt][1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// Expands the slab and accumulates its four k16 steps.
template <int kN, int kNT>
__device__ __forceinline__ void mma_slab(const Slab<kNT> &s, const uint2 *tab24, const uint4 *sel48,
                                         const uint4 *msk48, float (&acc)[kNT][4]) {
    if constexpr (kN == 2) {
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            const uint2 e0 = tab24[(s.m[0] >> (4 * st)) & 0xFu];
            const uint2 e1 = tab24[(s.m[1] >> (4 * st)) & 0xFu];
            const uint32_t w0 = word(s.v[0], st), w1 = word(s.v[1], st);
            const uint32_t a0 = __byte_perm(w0, 0u, e0.x), a2 = __byte_perm(w0, 0u, e0.y);
            const uint32_t a1 = __byte_perm(w1, 0u, e1.x), a3 = __byte_perm(w1, 0u, e1.y);
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt)
                mma_bf16_16816(acc[nt], a0, a1, a2, a3, word(s.x[nt][st >> 1], 2 * (st & 1)),
                               word(s.x[nt][st >> 1], 2 * (st & 1) + 1));
        }
    } else {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            uint32_t dn[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t km = keep_mask48((s.m[h] >> (16 * q)) & 0xFFFu);
                const uint4 sl = sel48[km], mk = msk48[km];
                const uint32_t lo = word(s.v[h], 2 * q), hi = word(s.v[h], 2 * q + 1);
                dn[h][0] = __byte_perm(lo, hi, sl.x) & mk.x;
                dn[h][1] = __byte_perm(lo, hi, sl.y) & mk.y;
                dn[h][2] = __byte_perm(lo, hi, sl.z) & mk.z;
                dn[h][3] = __byte_perm(lo, hi, sl.w) & mk.w;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int st = 2 * q + hh;
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
                    mma_bf16_16816(acc[nt], dn[0][2 * hh], dn[1][2 * hh], dn[0][2 * hh + 1], dn[1][2 * hh + 1],
                                   word(s.x[nt][st >> 1], 2 * (st & 1)), word(s.x[nt][st >> 1], 2 * (st & 1) + 1));
            }
        }
    }
}

// ------------------------------------------------------------------ kernel

// kNT n8 tiles of tokens (1: up to 8, 2: up to 16); kMT row tiles per CTA task; kDepth
// slabs in flight per warp.
template <int kN, int kNT, int kMT, int kDepth>
__global__ void __launch_bounds__(kCtaThreads) sparse_linear_kernel(const __grid_constant__ OpGroup grp) {
    constexpr int kKS = kWarps / kMT;
    static_assert(kWarps % kMT == 0, "row tiles must divide the warps");
    __shared__ uint2 s_tab24[16];
    __shared__ uint4 s_sel48[kN == 4 ? 256 : 1], s_msk48[kN == 4 ? 256 : 1];
    __shared__ float s_red[kWarps][4 * kNT][32];
    if constexpr (kN == 2) {
        if (threadIdx.x < 16) s_tab24[threadIdx.x] = make_uint2(g_sel24.lo[threadIdx.x], g_sel24.hi[threadIdx.x]);
    } else {
        for (int i = threadIdx.x; i < 256; i += kCtaThreads) {
            s_sel48[i] = make_uint4(g_sel48.sel[i][0], g_sel48.sel[i][1], g_sel48.sel[i][2], g_sel48.sel[i][3]);
            s_msk48[i] = make_uint4(g_sel48.mask[i][0], g_sel48.mask[i][1], g_sel48.mask[i][2], g_sel48.mask[i][3]);
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int mt = warp % kMT, ks = warp / kMT;
    for (int64_t task = blockIdx.x; task < grp.total_tasks; task += gridDim.x) {
        const Op &d = grp.d[find_op(grp, task)];
        const int64_t r0 = (task - d.task_begin) * (16 * kMT) + 16 * mt + g, r1 = r0 + 8;
        const int64_t nch = (d.cols + kChunk - 1) / kChunk;
        float acc[kNT][4];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        Slab<kNT> ring[kDepth];
#pragma unroll
        for (int i = 0; i < kDepth; ++i) {
            const int64_t c = ks + (int64_t)i * kKS;
            if (c < nch) load_slab<kN, kNT>(ring[i], d, r0, r1, c * kChunk + 16 * t, g, grp.tokens);
        }
        for (int64_t c0 = ks; c0 < nch; c0 += (int64_t)kDepth * kKS) {
#pragma unroll
            for (int i = 0; i < kDepth; ++i) {
                const int64_t c = c0 + (int64_t)i * kKS;
                if (c < nch) {
                    mma_slab<kN, kNT>(ring[i], s_tab24, s_sel48, s_msk48, acc);
                    const int64_t cn = c + (int64_t)kDepth * kKS;
                    if (cn < nch)
                        load_slab<kN, kNT>(ring[i], d, r0, r1, cn * kChunk + 16 * t, g, grp.tokens);
                }
            }
        }
        if constexpr (kKS > 1) {
            if (ks > 0) {
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) s_red[warp][4 * nt + q][lane] = acc[nt][q];
            }
            __syncthreads();
            if (ks == 0) {
#pragma unroll
                for (int k = 1; k < kKS; ++k)
#pragma unroll
                    for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[nt][q] += s_red[mt + k * kMT][4 * nt + q][lane];
            }
        }
        if (ks == 0) {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t r = h ? r1 : r0;
                    if (r >= d.rows) continue;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int tok = 8 * nt + 2 * t + e;
                        if (tok < grp.tokens) d.y[tok * d.rows + r] = acc[nt][2 * h + e];
                    }
                }
        }
        if constexpr (kKS > 1) __syncthreads();
    }
}

// ------------------------------------------------------------------ streamed kernel

// The kernel above holds its prefetched slabs in registers, which bounds the bytes each SM
// keeps in flight, and gives each CTA whole row tiles, so the long-k operands leave a tail.
// This one streams the compressed weight through a per-lane shared-memory ring with cp.async
// (kSkStages chunks in flight per warp, 32 rows per chunk) and splits the work evenly: the
// chunks of all tiles of all operands form one sequence, and warp w of W = min(warps,
// chunks) takes the non-empty contiguous range [w*total/W, (w+1)*total/W). A tile that lies inside one warp's range is
// stored straight from registers; a tile cut by range boundaries gets one partial tile per
// warp in a workspace slot, and the warp that arrives last (a ticket per tile, keyed by its
// first warp) adds the partials in warp order and stores y. Nothing waits on another warp,
// and the sum order depends only on the shapes and the grid. Needs cols % 16 == 0.

constexpr int kSkWarps = 8;
constexpr int kSkThreads = 32 * kSkWarps;
constexpr int kSkRows = 32;                 // rows per tile: two m16 tiles per warp
constexpr int kMaxSkWarps = 4096;
template <int kNT> constexpr int sk_lane_bytes() { return 80 + 32 * kNT; }  // v[4], x[kNT][2], m[4]
template <int kNT> constexpr int sk_stages() { return kNT == 1 ? 6 : 5; }
template <int kNT> constexpr int sk_smem_bytes() { return kSkWarps * sk_stages<kNT>() * 32 * sk_lane_bytes<kNT>(); }
// workspace: two partial tiles per warp (2 m-tiles x kNT x 4 floats per lane, kNT <= 2),
// then one ticket per warp, then an error word (set when a tensor copy never completes)
constexpr size_t kSkPartFloats = 2 * 2 * 4;
// batched kernel (17-64 tokens, kernels_umma.cuh): two partial tiles of 128 rows x 64 tokens
// per CTA, at most kBatchMaxCtas CTAs
constexpr int kBatchRows = 128, kBatchMaxCtas = 320;
constexpr size_t kBatchPartFloats = (size_t)kBatchRows * kMaxTokens;  // per CTA and slot
constexpr size_t kSpPartBytes = (size_t)kMaxSkWarps * 2 * 32 * kSkPartFloats * sizeof(float);
constexpr size_t kBatchPartBytes = (size_t)kBatchMaxCtas * 2 * kBatchPartFloats * sizeof(float);
constexpr size_t kPartBytes = kSpPartBytes > kBatchPartBytes ? kSpPartBytes : kBatchPartBytes;
constexpr size_t kSkWorkspaceBytes = kPartBytes + (size_t)kMaxSkWarps * sizeof(unsigned int) + 16;  // + error word

struct SkOp {
    const uint32_t *vals;
    const void *meta;
    const uint32_t *x;
    float *y;
    int64_t rows, cols;
    int64_t nch;          // chunks of 64 columns per tile
    int64_t ntiles;       // tiles of 32 rows
    int64_t chunk_begin;  // first chunk of this operand in the launch's sequence
};

struct SkGroup {
    int32_t n;
    int32_t tokens;
    int64_t total_chunks;
    SkOp d[kMaxMats];
};

struct Cursor {
    int op;
    int64_t tile, j;
};

__device__ __forceinline__ Cursor sk_decode(const SkGroup &g, int64_t c) {
    int i = 0;
    while (i + 1 < g.n && c >= g.d[i + 1].chunk_begin) ++i;
    const int64_t r = c - g.d[i].chunk_begin;
    return Cursor{i, r / g.d[i].nch, r % g.d[i].nch};
}

__device__ __forceinline__ void sk_advance(const SkGroup &g, Cursor &c) {
    if (++c.j == g.d[c.op].nch) {
        c.j = 0;
        if (++c.tile == g.d[c.op].ntiles) {
            c.tile = 0;
            ++c.op;
        }
    }
}

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, bool in) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(in ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(void *dst, const void *src, bool in) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src), "r"(in ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(kPending) : "memory"); }

// Copies this lane's share of chunk `c` into its ring slot: values and metadata of rows
// 32*tile + g + 8h (h = 0..3) at columns 64j + 16t .. +15, and x of tokens g + 8nt at the
// same columns. Out-of-range pieces are zero-filled (nothing is read for them).
template <int kN, int kNT>
__device__ __forceinline__ void sk_issue(const SkGroup &grp, const Cursor &c, unsigned char *slot, int g, int t) {
    const SkOp &d = grp.d[c.op];
    const int64_t col0 = c.j * kChunk + 16 * t;
    const bool colin = col0 < d.cols;
    const int64_t wpr = d.cols >> 2, bpr = d.cols / (2 * kN);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const int64_t r = c.tile * kSkRows + g + 8 * h;
        const bool in = colin && r < d.rows;
        const uint32_t *sv = in ? d.vals + r * wpr + (col0 >> 2) : d.vals;
        const void *sm;
        if constexpr (kN == 2)
            sm = in ? (const void *)(static_cast<const uint32_t *>(d.meta) + r * ((bpr + 7) >> 3) + (col0 >> 5)) : d.meta;
        else
            sm = in ? (const void *)(static_cast<const uint16_t *>(d.meta) + r * bpr + (col0 >> 3)) : d.meta;
        cp_async16_zfill(slot + 16 * h, sv, in);
        cp_async4_zfill(slot + 64 + 32 * kNT + 4 * h, sm, in);
    }
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
        const int tok = g + 8 * nt;
        const bool in = colin && tok < grp.tokens;
        const uint32_t *sx = in ? d.x + tok * (d.cols >> 1) + (col0 >> 1) : d.x;
        cp_async16_zfill(slot + 64 + 32 * nt, sx, in);
        cp_async16_zfill(slot + 64 + 32 * nt + 16, in ? sx + 4 : d.x, in);
    }
}

template <int kNT>
__device__ __forceinline__ void sk_store(const SkOp &d, int64_t tile, const float (&acc)[2][kNT][4], int g, int t,
                                         int tokens) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t r = tile * kSkRows + 16 * mt + 8 * h + g;
                if (r >= d.rows) continue;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = 8 * nt + 2 * t + e;
                    if (tok < tokens) d.y[tok * d.rows + r] = acc[mt][nt][2 * h + e];
                }
            }
}

// End of a warp's piece of a tile: store y if the warp owns the whole tile, else leave the
// partial tile in the workspace and, if this is the last piece to arrive, add all pieces in
// warp order and store y (then reset the tile's ticket for the next call).
template <int kNT>
__device__ __forceinline__ void sk_finish(const SkGroup &grp, const SkOp &d, int64_t tile, const float (&acc)[2][kNT][4],
                                          float *__restrict__ part, unsigned int *__restrict__ tickets, int64_t gw,
                                          int64_t GW, int64_t total, int lane, int g, int t) {
    const int64_t a = d.chunk_begin + tile * d.nch, b = a + d.nch;
    const int64_t w1 = ((a + 1) * GW - 1) / total, w2 = (b * GW - 1) / total;
    if (w1 == w2) {
        sk_store<kNT>(d, tile, acc, g, t, grp.tokens);
        return;
    }
    const int64_t lo1 = w1 * total / GW;
    const int slot_id = (gw == w1 && lo1 < a) ? 1 : 0;
    float4 *mine = reinterpret_cast<float4 *>(part) + ((gw * 2 + slot_id) * 32 + lane) * (2 * kNT);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
            __stcg(mine + mt * kNT + nt, make_float4(acc[mt][nt][0], acc[mt][nt][1], acc[mt][nt][2], acc[mt][nt][3]));
    __threadfence();
    __syncwarp();
    unsigned int old = 0;
    if (lane == 0) old = atomicAdd(tickets + w1, 1u);
    old = __shfl_sync(0xFFFFFFFFu, old, 0);
    if (old != (unsigned int)(w2 - w1)) return;
    __threadfence();
    float sum[2][kNT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) sum[mt][nt][0] = sum[mt][nt][1] = sum[mt][nt][2] = sum[mt][nt][3] = 0.f;
    for (int64_t w = w1; w <= w2; ++w) {
        const int sid = (w == w1 && lo1 < a) ? 1 : 0;
        const float4 *p = reinterpret_cast<const float4 *>(part) + ((w * 2 + sid) * 32 + lane) * (2 * kNT);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
                const float4 q = __ldcg(p + mt * kNT + nt);
                sum[mt][nt][0] += q.x;
                sum[mt][nt][1] += q.y;
                sum[mt][nt][2] += q.z;
                sum[mt][nt][3] += q.w;
            }
    }
    sk_store<kNT>(d, tile, sum, g, t, grp.tokens);
    __syncwarp();
    if (lane == 0) tickets[w1] = 0u;
}

template <int kN, int kNT>
__global__ void __launch_bounds__(kSkThreads, 1) sparse_linear_sk_kernel(const __grid_constant__ SkGroup grp,
                                                                         float *__restrict__ part,
                                                                         unsigned int *__restrict__ tickets) {
    constexpr int kD = sk_stages<kNT>();
    constexpr int kLane = sk_lane_bytes<kNT>();
    extern __shared__ __align__(16) unsigned char s_ring[];
    __shared__ uint2 s_tab24[16];
    __shared__ uint4 s_sel48[kN == 4 ? 256 : 1], s_msk48[kN == 4 ? 256 : 1];
    if constexpr (kN == 2) {
        if (threadIdx.x < 16) s_tab24[threadIdx.x] = make_uint2(g_sel24.lo[threadIdx.x], g_sel24.hi[threadIdx.x]);
    } else {
        for (int i = threadIdx.x; i < 256; i += kSkThreads) {
            s_sel48[i] = make_uint4(g_sel48.sel[i][0], g_sel48.sel[i][1], g_sel48.sel[i][2], g_sel48.sel[i][3]);
            s_msk48[i] = make_uint4(g_sel48.mask[i][0], g_sel48.mask[i][1], g_sel48.mask[i][2], g_sel48.mask[i][3]);
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    // the sequence is split between GW = min(warps, chunks) warps, so every range is
    // non-empty and the pieces of a tile come from the consecutive warps w1..w2
    const int64_t total = grp.total_chunks;
    const int64_t GW = imin64((int64_t)gridDim.x * kSkWarps, total), gw = (int64_t)blockIdx.x * kSkWarps + warp;
    if (gw >= GW) return;  // no block-wide barrier follows
    const int64_t lo = gw * total / GW, hi = (gw + 1) * total / GW;
    unsigned char *ring = s_ring + ((size_t)warp * kD * 32 + lane) * kLane;  // stage s at + s * 32 * kLane
    const int64_t n = hi - lo;
    Cursor ld = sk_decode(grp, lo), cc = ld;
#pragma unroll
    for (int s = 0; s < kD; ++s) {
        if (s < n) {
            sk_issue<kN, kNT>(grp, ld, ring + s * 32 * kLane, g, t);
            sk_advance(grp, ld);
        }
        cp_async_commit();
    }
    float acc[2][kNT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
    int s = 0;
    for (int64_t f = 0; f < n; ++f) {
        cp_async_wait<kD - 1>();  // this lane's copies of chunk f have landed
        unsigned char *slot = ring + s * 32 * kLane;
        const uint4 *sv = reinterpret_cast<const uint4 *>(slot);
        const uint4 mw = *reinterpret_cast<const uint4 *>(slot + 64 + 32 * kNT);
        Slab<kNT> sl[2];
        const uint32_t msh = kN == 2 ? 16 * (t & 1) : 0;
        sl[0].v[0] = sv[0];
        sl[0].v[1] = sv[1];
        sl[1].v[0] = sv[2];
        sl[1].v[1] = sv[3];
        sl[0].m[0] = mw.x >> msh;
        sl[0].m[1] = mw.y >> msh;
        sl[1].m[0] = mw.z >> msh;
        sl[1].m[1] = mw.w >> msh;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            sl[0].x[nt][0] = sl[1].x[nt][0] = sv[4 + 2 * nt];
            sl[0].x[nt][1] = sl[1].x[nt][1] = sv[5 + 2 * nt];
        }
        mma_slab<kN, kNT>(sl[0], s_tab24, s_sel48, s_msk48, acc[0]);
        mma_slab<kN, kNT>(sl[1], s_tab24, s_sel48, s_msk48, acc[1]);
        // the slot's contents are in registers and consumed: refill it with chunk f + kD
        if (f + kD < n) {
            sk_issue<kN, kNT>(grp, ld, slot, g, t);
            sk_advance(grp, ld);
        }
        cp_async_commit();
        s = (s + 1 == kD) ? 0 : s + 1;
        const SkOp &d = grp.d[cc.op];
        if (cc.j == d.nch - 1 || f == n - 1) {
            sk_finish<kNT>(grp, d, cc.tile, acc, part, tickets, gw, GW, total, lane, g, t);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
        }
        if (f + 1 < n) sk_advance(grp, cc);
    }
    cp_async_wait<0>();
}

// ------------------------------------------------------------------ 2:4 on sparse tensor cores

// mma.sp (m16n8k32, bf16, ordered metadata) takes the compressed operand as it is: per row
// and 32-column window, 8 blocks of 2 kept values (16 bf16) and 8 metadata nibbles p0 | p1 << 2
// -- exactly one metadata word of mllm_hard_pack. Register layout (lane g = lane/4,
// t = lane%4; measured on the device with distinct values per element and per nibble):
//   A reg0 / reg1 / reg2 / reg3 = the kept pair of block t of row g / of row g+8 /
//     of block t+4 of row g / of row g+8;
//   B reg q = x at columns 2t+8q, 2t+8q+1 of the window, token g;
//   metadata (selector 0): lane t = 0 holds blocks 0-3 of row g (bits 0-15) and of row g+8
//     (bits 16-31), lane t = 1 blocks 4-7; lanes 2, 3 are not read.
// So the kernel only moves data: a warp copies its 32 rows x 64 columns (two windows) of
// values and metadata and the chunk's x into a shared-memory stage with cp.async (rows padded
// to 80 bytes, tokens to 144, so that every fragment read is free of bank conflicts), reads
// the A and B fragments with ldmatrix (the x4 distribution is exactly the layout above), and
// issues 2 windows x 2 row tiles x kNT mma.sp per chunk. Work split and partial tiles as in
// the streamed kernel above. Needs cols % 32 == 0 (whole metadata words); metadata words
// that are zero-filled (rows or windows past the matrix, whose values and x are zero too)
// are replaced by a valid pattern.

constexpr int kSpRowBytes = 80;   // 64 bytes of values + 2 metadata words, padded
constexpr int kSpTokBytes = 144;  // 64 columns of x (128 bytes), padded
template <int kNT> constexpr int sp_stage_bytes() { return kSkRows * kSpRowBytes + 8 * kNT * kSpTokBytes; }
// 16 warps x 3 stages (up to 8 tokens) and 12 x 3 (16 tokens, more registers) keep ~110 KB
// per SM in flight; more warps with shallower rings measured faster than 8 x 6 (latency of
// each warp's own instruction chains, not bytes in flight, limited the deeper rings)
template <int kNT> constexpr int sp_warps() { return kNT == 1 ? 16 : 12; }
template <int kNT> constexpr int sp_stages() { return kNT == 1 ? 3 : 3; }
template <int kNT> constexpr int sp_smem_bytes() { return sp_warps<kNT>() * sp_stages<kNT>() * sp_stage_bytes<kNT>(); }

__device__ __forceinline__ void mma_sp_bf16_16832(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                  const uint32_t (&b)[4], uint32_t e) {
    asm("mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, 0x0;\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(e));
}

__device__ __forceinline__ uint32_t lds32(const unsigned char *p) { return *reinterpret_cast<const uint32_t *>(p); }

// Four 8x8 b16 matrices: lane L gives the address of row L%8 of matrix L/8; lane (g, t)
// receives elements 2t, 2t+1 of row g of matrix m in r[m].
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const unsigned char *p) {
    const unsigned a = (unsigned)__cvta_generic_to_shared(p);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

// Copy state of one lane for the chunk the load cursor points at: source byte pointers
// (advanced by one chunk per issue) and copy sizes (0 = zero-fill) of its pieces -- values of
// rows 32*tile + lane/4 + 8k (16-byte quarter lane%4), metadata of row 32*tile + lane (two
// words), x of tokens lane/8 + 4k (16-byte part lane%8).
template <int kNT>
struct SpLoad {
    int op, j, nch;
    int64_t tile;
    const char *v[4], *m, *x[2 * kNT];
    unsigned vsz[4], msz, xsz[2 * kNT];
};

// Positions the copy state at chunk j of tile `tile` of operand `op`.
template <int kNT>
__device__ __forceinline__ void sp_load_at(const SkGroup &grp, int op, int64_t tile, int j, int lane, SpLoad<kNT> &L) {
    const SkOp &d = grp.d[op];
    L.op = op;
    L.tile = tile;
    L.j = j;
    L.nch = (int)d.nch;
    const int64_t vrow = d.cols, mrow = d.cols >> 3, xrow = d.cols << 1;  // bytes per row (2:4)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t r = tile * kSkRows + (lane >> 2) + 8 * k;
        const bool in = r < d.rows;
        L.v[k] = reinterpret_cast<const char *>(d.vals) + (in ? r * vrow : 0) + 16 * (lane & 3) + 64 * j;
        L.vsz[k] = in ? 16u : 0u;
    }
    const int64_t rm = tile * kSkRows + lane;
    const bool min = rm < d.rows;
    L.m = static_cast<const char *>(d.meta) + (min ? rm * mrow : 0) + 8 * j;
    L.msz = min ? 4u : 0u;
#pragma unroll
    for (int k = 0; k < 2 * kNT; ++k) {
        const int tok = (lane >> 3) + 4 * k;
        const bool in = tok < grp.tokens;
        L.x[k] = reinterpret_cast<const char *>(d.x) + (in ? (int64_t)tok * xrow : 0) + 16 * (lane & 7) + 128 * j;
        L.xsz[k] = in ? 16u : 0u;
    }
}

// Issues the copies of the current chunk into `stage` (a shared-memory address) and moves
// the state to the next chunk of the sequence.
template <int kNT>
__device__ __forceinline__ void sp_issue(const SkGroup &grp, SpLoad<kNT> &L, unsigned stage, int lane) {
    const int cols = (int)grp.d[L.op].cols, col0 = L.j * kChunk;
    const bool whole = col0 + kChunk <= cols;  // only a row's last chunk can be partial
    const unsigned vdst = stage + (lane >> 2) * kSpRowBytes + 16 * (lane & 3);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const unsigned sz = (whole || col0 + 16 * (lane & 3) < cols) ? L.vsz[k] : 0u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(vdst + 8 * k * kSpRowBytes), "l"(L.v[k]),
                     "r"(sz) : "memory");
        L.v[k] += 64;
    }
    const unsigned mdst = stage + lane * kSpRowBytes + 64;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const unsigned sz = (whole || col0 + 32 * w < cols) ? L.msz : 0u;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(mdst + 4 * w), "l"(L.m + 4 * w), "r"(sz)
                     : "memory");
    }
    L.m += 8;
    const unsigned xdst = stage + kSkRows * kSpRowBytes + (lane >> 3) * kSpTokBytes + 16 * (lane & 7);
#pragma unroll
    for (int k = 0; k < 2 * kNT; ++k) {
        const unsigned sz = (whole || col0 + 8 * (lane & 7) < cols) ? L.xsz[k] : 0u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(xdst + 4 * k * kSpTokBytes), "l"(L.x[k]),
                     "r"(sz) : "memory");
        L.x[k] += 128;
    }
    if (++L.j == L.nch) {  // next tile (or next operand)
        const SkOp &d = grp.d[L.op];
        if (L.tile + 1 < d.ntiles) sp_load_at<kNT>(grp, L.op, L.tile + 1, 0, lane, L);
        else if (L.op + 1 < grp.n) sp_load_at<kNT>(grp, L.op + 1, 0, 0, lane, L);
    }
}

// One stage: 2 windows x 2 row tiles x kNT mma.sp. kEdge: the stage may hold zero-filled
// metadata words (rows past the matrix, or the window past its last column).
template <int kNT, bool kEdge>
__device__ __forceinline__ void sp_compute(const unsigned char *st, int lane, int g, int t, float (&acc)[2][kNT][4]) {
    const unsigned char *pa = st + ((lane & 7) + 8 * ((lane >> 3) & 1)) * kSpRowBytes + 16 * (lane >> 4);
    const unsigned char *pb = st + kSkRows * kSpRowBytes + (lane & 7) * kSpTokBytes + 16 * (lane >> 3);
    const uint32_t esel = (t & 1) ? 0x7632u : 0x5410u;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        uint32_t b[kNT][4];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) ldmatrix_x4(b[nt], pb + 8 * nt * kSpTokBytes + 64 * w);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            uint32_t a[4];
            ldmatrix_x4(a, pa + 16 * mt * kSpRowBytes + 32 * w);
            const unsigned char *ra = st + (16 * mt + g) * kSpRowBytes;
            uint32_t mg = lds32(ra + 64 + 4 * w), mg8 = lds32(ra + 8 * kSpRowBytes + 64 + 4 * w);
            if constexpr (kEdge) {
                mg = mg ? mg : 0x44444444u;
                mg8 = mg8 ? mg8 : 0x44444444u;
            }
            const uint32_t e = __byte_perm(mg, mg8, esel);
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) mma_sp_bf16_16832(acc[mt][nt], a[0], a[1], a[2], a[3], b[nt], e);
        }
    }
}

template <int kNT>
__global__ void __launch_bounds__(32 * sp_warps<kNT>(), 1) sparse_linear_sp_kernel(const __grid_constant__ SkGroup grp,
                                                                         float *__restrict__ part,
                                                                         unsigned int *__restrict__ tickets) {
    constexpr int kD = sp_stages<kNT>();
    constexpr int kStage = sp_stage_bytes<kNT>();
    extern __shared__ __align__(16) unsigned char s_ring[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t total = grp.total_chunks;
    constexpr int kW = sp_warps<kNT>();
    const int64_t GW = imin64((int64_t)gridDim.x * kW, total), gw = (int64_t)blockIdx.x * kW + warp;
    if (gw >= GW) return;
    const int64_t lo = gw * total / GW, hi = (gw + 1) * total / GW;
    const int n = (int)(hi - lo);  // chunks of this warp (< 2^31: a chunk holds > 2 KB of operands)
    unsigned char *ring = s_ring + (size_t)warp * kD * kStage;
    const unsigned ring_s = (unsigned)__cvta_generic_to_shared(ring);
    const Cursor c0 = sk_decode(grp, lo);
    SpLoad<kNT> L;
    sp_load_at<kNT>(grp, c0.op, c0.tile, (int)c0.j, lane, L);
#pragma unroll
    for (int s = 0; s < kD; ++s) {
        if (s < n) sp_issue<kNT>(grp, L, ring_s + s * kStage, lane);
        cp_async_commit();
    }
    // compute cursor
    int op = c0.op, j = (int)c0.j;
    int64_t tile = c0.tile;
    int nch = (int)grp.d[op].nch;
    bool rows_edge = (tile + 1) * kSkRows > grp.d[op].rows, cols_edge = (grp.d[op].cols & (kChunk - 1)) != 0;
    float acc[2][kNT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
    int s = 0;
    for (int f = 0; f < n; ++f) {
        cp_async_wait<kD - 1>();
        __syncwarp();  // every lane's copies of chunk f are visible to the warp
        const unsigned char *st = ring + s * kStage;
        if (rows_edge || (cols_edge && j == nch - 1)) sp_compute<kNT, true>(st, lane, g, t, acc);
        else sp_compute<kNT, false>(st, lane, g, t, acc);
        __syncwarp();  // the stage is read: it may be refilled
        if (f + kD < n) sp_issue<kNT>(grp, L, ring_s + s * kStage, lane);
        cp_async_commit();
        s = (s + 1 == kD) ? 0 : s + 1;
        if (j == nch - 1 || f == n - 1) {
            sk_finish<kNT>(grp, grp.d[op], tile, acc, part, tickets, gw, GW, total, lane, g, t);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
        }
        if (++j == nch && f + 1 < n) {
            j = 0;
            if (++tile == grp.d[op].ntiles) {
                tile = 0;
                ++op;
                nch = (int)grp.d[op].nch;
                cols_edge = (grp.d[op].cols & (kChunk - 1)) != 0;
            }
            rows_edge = (tile + 1) * kSkRows > grp.d[op].rows;
        }
    }
    cp_async_wait<0>();
}

// ------------------------------------------------------------------ 2:4, tensor copies (TMA)

// The same product for rows of whole 128-column stages (cols % 128 == 0, every LLM shape),
// fed by the tensor memory accelerator: per 32-row x 128-column stage one lane issues four
// tiled copies (cp.async.bulk.tensor.2d) -- the 32 x 64 box of compressed values, the 32 x 4
// box of metadata words and two 8kNT x 64 boxes of x -- completing on the stage's mbarrier.
// Boxes past the matrix (rows, tokens) are zero-filled by the copy engine. Values and x land
// with the 128-byte swizzle (16-byte chunk c of box row r at chunk c ^ (r % 8)), so the
// ldmatrix reads below are free of bank conflicts. Each tensor map describes one operand
// (values, metadata, x) and is passed with the launch. Waits are bounded (1 s): a copy that
// never lands sets the workspace's error word and the warp returns after a bounded wait for
// its other stages. arm_only_first (tests only) arms every warp's first stage without
// filling it, so that this path runs. Work split and partial tiles as in the kernels above, 128-column chunks.

constexpr int kTmChunk = 128;
constexpr unsigned long long kTmWaitNs = 1000000000ull;  // bound of one wait: 1 s (a stage lands in us)
// A stage's metadata box: 32 rows x 4 uint32 words.
template <int kNT> constexpr int tm_xbox_bytes() { return 8 * kNT * 128; }
template <int kNT> constexpr int tm_stage_tx() { return 32 * 128 + 2 * tm_xbox_bytes<kNT>() + 32 * 16; }
template <int kNT> constexpr int tm_stage_bytes() { return (tm_stage_tx<kNT>() + 1023) / 1024 * 1024; }
constexpr int kTmWarps = 8, kTmStages = 3;
template <int kNT> constexpr int tm_smem_bytes() { return kTmWarps * kTmStages * tm_stage_bytes<kNT>() + 1024; }

// Tensor maps of one operand. The per-warp kernel (2:4) uses 32-row boxes and x boxes of 8kNT
// tokens; the tensor-memory kernels (kernels_umma.cuh) 128-row boxes, x boxes of N tokens and,
// for 4:8, uint16 metadata [rows, cols/8] in boxes of 16 x 128.
struct TmMaps {
    CUtensorMap vals;  // bf16 [rows, cols/2], box 64 x rows, 128-byte swizzle
    CUtensorMap meta;  // 2:4: uint32 [rows, cols/32], box 4 x rows
    CUtensorMap x;     // bf16 [tokens, cols], box 64 x tokens, 128-byte swizzle
};

struct TmGroup {
    SkGroup g;
    TmMaps maps[kMaxMats];
};

__device__ __forceinline__ void mbar_init(unsigned bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(unsigned bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0u;
}
__device__ __forceinline__ void tma_load_2d(unsigned dst, const CUtensorMap *map, int x, int y, unsigned bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;\n" : "=l"(t));
    return t;
}

// Warp-uniform wait for phase `parity` of a stage's barrier, bounded by kTmWaitNs of lane
// 0's clock; false if it ran out.
__device__ __forceinline__ bool tm_wait(unsigned bar, unsigned parity) {
    if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
    const unsigned long long t0 = __shfl_sync(0xFFFFFFFFu, globaltimer_ns(), 0);
    while (true) {
        if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
        if (__shfl_sync(0xFFFFFFFFu, globaltimer_ns(), 0) - t0 > kTmWaitNs) return false;
    }
}

template <int kNT>
__device__ __forceinline__ void tm_issue(const TmGroup &tg, const Cursor &c, unsigned stage, unsigned bar) {
    const TmMaps &mp = tg.maps[c.op];
    const int j = (int)c.j, row0 = (int)(c.tile * kSkRows);
    mbar_arrive_tx(bar, (unsigned)tm_stage_tx<kNT>());
    tma_load_2d(stage, &mp.vals, 64 * j, row0, bar);
    tma_load_2d(stage + 4096, &mp.x, 128 * j, 0, bar);
    tma_load_2d(stage + 4096 + tm_xbox_bytes<kNT>(), &mp.x, 128 * j + 64, 0, bar);
    tma_load_2d(stage + 4096 + 2 * tm_xbox_bytes<kNT>(), &mp.meta, 4 * j, row0, bar);
}

__device__ __forceinline__ uint4 lds128(const unsigned char *p) { return *reinterpret_cast<const uint4 *>(p); }

template <int kNT, bool kEdge>
__device__ __forceinline__ void tm_compute(const unsigned char *st, int lane, int g, int t, float (&acc)[2][kNT][4]) {
    const unsigned char *meta = st + 4096 + 2 * tm_xbox_bytes<kNT>();
    const uint32_t esel = (t & 1) ? 0x7632u : 0x5410u;
    const int ar = (lane & 7) + 8 * ((lane >> 3) & 1);  // A box row of this lane (+16 mt)
    const int br = lane & 7;                             // x box row (token) of this lane (+8 nt)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const unsigned char *xb = st + 4096 + (w >> 1) * tm_xbox_bytes<kNT>();
        uint32_t b[kNT][4];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            const int r = br + 8 * nt, c = 4 * (w & 1) + (lane >> 3);
            ldmatrix_x4(b[nt], xb + r * 128 + ((c ^ (r & 7)) << 4));
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int r = ar + 16 * mt, c = 2 * w + (lane >> 4);
            uint32_t a[4];
            ldmatrix_x4(a, st + r * 128 + ((c ^ (r & 7)) << 4));
            const unsigned char *ra = meta + (16 * mt + g) * 16 + 4 * w;
            uint32_t mg = lds32(ra), mg8 = lds32(ra + 8 * 16);
            if constexpr (kEdge) {
                mg = mg ? mg : 0x44444444u;
                mg8 = mg8 ? mg8 : 0x44444444u;
            }
            const uint32_t e = __byte_perm(mg, mg8, esel);
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) mma_sp_bf16_16832(acc[mt][nt], a[0], a[1], a[2], a[3], b[nt], e);
        }
    }
}

template <int kNT>
__global__ void __launch_bounds__(32 * kTmWarps, 1) sparse_linear_tma_kernel(
    const __grid_constant__ TmGroup tg, float *__restrict__ part, unsigned int *__restrict__ tickets,
    unsigned int *__restrict__ err, int arm_only_first) {
    constexpr int kW = kTmWarps, kD = kTmStages, kStage = tm_stage_bytes<kNT>();
    extern __shared__ unsigned char s_dyn_tm[];
    __shared__ __align__(8) unsigned long long s_bar[kW][kD];
    const SkGroup &grp = tg.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t total = grp.total_chunks;
    const int64_t GW = imin64((int64_t)gridDim.x * kW, total), gw = (int64_t)blockIdx.x * kW + warp;
    if (gw >= GW) return;  // no block-wide barrier follows
    const int64_t lo = gw * total / GW, hi = (gw + 1) * total / GW;
    const int n = (int)(hi - lo);
    // 1024-byte aligned ring (the swizzle pattern repeats every 1024 bytes)
    const unsigned dyn_s = (unsigned)__cvta_generic_to_shared(s_dyn_tm);
    const unsigned pad = (1024u - (dyn_s & 1023u)) & 1023u;
    unsigned char *ring = s_dyn_tm + pad + (size_t)warp * kD * kStage;
    const unsigned ring_s = dyn_s + pad + (unsigned)(warp * kD * kStage);
    const unsigned bar0 = (unsigned)__cvta_generic_to_shared(&s_bar[warp][0]);
    if (lane == 0) {
        for (int s = 0; s < kD; ++s) mbar_init(bar0 + 8 * s, 1u);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    Cursor ld = sk_decode(grp, lo), cc = ld;
#pragma unroll
    for (int s = 0; s < kD; ++s)
        if (s < n) {
            if (lane == 0) {
                if (s == 0 && arm_only_first)  // test of the bounded wait: a stage nothing fills
                    mbar_arrive_tx(bar0, (unsigned)tm_stage_tx<kNT>());
                else
                    tm_issue<kNT>(tg, ld, ring_s + s * kStage, bar0 + 8 * s);
            }
            sk_advance(grp, ld);
        }
    bool rows_edge = (cc.tile + 1) * kSkRows > grp.d[cc.op].rows;
    float acc[2][kNT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
    unsigned phase = 0u;  // bit s: parity of the next phase of stage s
    int s = 0;
    for (int f = 0; f < n; ++f) {
        if (!tm_wait(bar0 + 8 * s, (phase >> s) & 1u)) {
            if (lane == 0) atomicOr(err, 1u);
            for (int q = 1; q < kD && f + q < n; ++q) {
                const int sq = (s + q) % kD;
                tm_wait(bar0 + 8 * sq, (phase >> sq) & 1u);
            }
            return;
        }
        phase ^= 1u << s;
        const unsigned char *st = ring + s * kStage;
        if (rows_edge) tm_compute<kNT, true>(st, lane, g, t, acc);
        else tm_compute<kNT, false>(st, lane, g, t, acc);
        __syncwarp();        // every lane has read the stage
        fence_proxy_async();  // generic reads before the stage's next asynchronous writes
        if (f + kD < n) {
            if (lane == 0) tm_issue<kNT>(tg, ld, ring_s + s * kStage, bar0 + 8 * s);
            sk_advance(grp, ld);
        }
        s = (s + 1 == kD) ? 0 : s + 1;
        const SkOp &d = grp.d[cc.op];
        if (cc.j == d.nch - 1 || f == n - 1) {
            sk_finish<kNT>(grp, d, cc.tile, acc, part, tickets, gw, GW, total, lane, g, t);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
        }
        if (f + 1 < n) {
            sk_advance(grp, cc);
            rows_edge = (cc.tile + 1) * kSkRows > grp.d[cc.op].rows;
        }
    }
}

}  // namespace spl
}  // namespace mllm
