// kernels_diag.cuh -- measurements of learned masks and a compact candidate-index code.
//
// MaskLLM (paper-graph-ui summary of arXiv 2409.17481) follows training with the mask
// difference between adjacent steps and between methods (s.3.4 Fig. 5a, Fig. 8), the mean
// maximum probability of the mask distributions (Fig. 5b) and the L1 norm of the kept
// weights relative to magnitude pruning (Fig. 6), and stores learned masks at 0.65 bits per
// parameter (Table 6 discussion). These kernels compute those quantities over the device
// arrays the sampler keeps, and pack candidate indices base C.
#pragma once

#include "device_common.cuh"
#include "kernels_2of4.cuh"
#include "kernels_4of8.cuh"

namespace mllm {
namespace diag {

constexpr int kMaxStatCtas = 1024;  // 4 doubles per CTA in the forward's workspace

// ------------------------------------------------------------------ mask difference

__global__ void __launch_bounds__(kThreads) mask_diff_kernel(const uint8_t *__restrict__ a,
                                                             const uint8_t *__restrict__ b, int64_t n,
                                                             unsigned long long *count) {
    unsigned long long c = 0;
    const int64_t n16 = n >> 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
        const uint4 x = __ldcs(reinterpret_cast<const uint4 *>(a) + i);
        const uint4 y = __ldcs(reinterpret_cast<const uint4 *>(b) + i);
        // __vcmpne4: 0xFF in every byte lane that differs
        c += __popc(__vcmpne4(x.x, y.x)) / 8 + __popc(__vcmpne4(x.y, y.y)) / 8 +
             __popc(__vcmpne4(x.z, y.z)) / 8 + __popc(__vcmpne4(x.w, y.w)) / 8;
    }
    for (int64_t i = 16 * n16 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        c += (a[i] != b[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    if ((threadIdx.x & 31) == 0 && c) atomicAdd(count, c);
}

// ------------------------------------------------------------------ mask statistics

// Deterministic reduction of 4 doubles per thread: per-CTA sums into partials[4 * cta + q],
// the last CTA sums the partials in index order into out[0..3] and resets the ticket.
__device__ __forceinline__ void reduce4(double v[4], double *partials, unsigned int *ticket, double *out) {
    __shared__ double s_w[kThreads / 32][4];
    __shared__ bool s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v[q] += __shfl_xor_sync(0xFFFFFFFFu, v[q], o);
        if (lane == 0) s_w[warp][q] = v[q];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int q = 0; q < 4; ++q) {
            double t = 0.0;
            for (int i = 0; i < kThreads / 32; ++i) t += s_w[i][q];
            partials[4 * blockIdx.x + q] = t;
        }
        __threadfence();
        s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x < 4) {
        double t = 0.0;
        for (unsigned int i = 0; i < gridDim.x; ++i) t += __ldcg(partials + 4 * i + threadIdx.x);
        out[threadIdx.x] = t;
    }
    __syncthreads();
    if (threadIdx.x == 0) *ticket = 0u;
}

// Per block: (max softmax(kappa pi), |W| kept by argmax pi, |W| kept by the magnitude mask,
// 1 if the two masks agree). 2:4: one thread per block pair.
template <bool kW32>
__global__ void __launch_bounds__(kThreads) stats24_kernel(const __grid_constant__ Group grp, float kappa,
                                                           double *partials, unsigned int *ticket, double *out) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b0 = ((t - d.work_begin) * kThreads + threadIdx.x) * 2;
        if (b0 >= d.nblocks) continue;
        const bool two = b0 + 1 < d.nblocks;
        float w[8], pi[12];
        k24::load_vals<kW32>(d.W, b0, two, w);
        k24::load12(d.pi, b0, two, pi);
        for (int h = 0; h < (two ? 2 : 1); ++h) {
            const float *p = pi + 6 * h;
            const int k = k24::argmax6(p);
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 6; ++i) mx = fmaxf(mx, kappa * p[i]);
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < 6; ++i) s += __expf(kappa * p[i] - mx);
            acc[0] += (double)__frcp_rn(s);  // the block's term in fp32, the sum over blocks in fp64
            const uint32_t mk = k24::cand_mask(k), m0 = k24::top2_mask(w + 4 * h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const double aw = fabs((double)w[4 * h + j]);
                if (mk & (1u << j)) acc[1] += aw;
                if (m0 & (1u << j)) acc[2] += aw;
            }
            acc[3] += (mk == m0) ? 1.0 : 0.0;
        }
    }
    reduce4(acc, partials, ticket, out);
}

// 4:8: one thread per block, the logit row read directly (70 floats, 8-byte aligned).
template <bool kW32>
__global__ void __launch_bounds__(kThreads) stats48_kernel(const __grid_constant__ Group grp, float kappa,
                                                           double *partials, unsigned int *ticket, double *out) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    int mi = 0;
    for (int64_t t = blockIdx.x; t < grp.total_work; t += gridDim.x) {
        mi = next_mat(grp, mi, t);
        const MatDesc &d = grp.d[mi];
        const int64_t b = (t - d.work_begin) * kThreads + threadIdx.x;
        if (b >= d.nblocks) continue;
        float w[8];
        k48::load8<kW32>(d.W, b, w);
        const float2 *row = reinterpret_cast<const float2 *>(d.pi + b * k48::C);
        int k = -1;
        float best = 0.f, mx = -INFINITY;
        for (int c2 = 0; c2 < k48::C / 2; ++c2) {
            const float2 v = __ldcs(row + c2);
            const float pv[2] = {v.x, v.y};
            for (int q = 0; q < 2; ++q) {
                if (pv[q] == pv[q] && (k < 0 || pv[q] > best)) { k = 2 * c2 + q; best = pv[q]; }
                mx = fmaxf(mx, kappa * pv[q]);
            }
        }
        if (k < 0) k = 0;
        float s = 0.f;
        for (int c2 = 0; c2 < k48::C / 2; ++c2) {
            const float2 v = __ldcs(row + c2);
            s += __expf(kappa * v.x - mx) + __expf(kappa * v.y - mx);
        }
        acc[0] += (double)__frcp_rn(s);  // the block's term in fp32, the sum over blocks in fp64
        float key[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) key[j] = (w[j] != w[j]) ? -1.0f : fabsf(w[j]);
        uint32_t m0 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int rank = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q != j && (key[q] > key[j] || (key[q] == key[j] && q < j))) ++rank;
            if (rank < 4) m0 |= 1u << j;
        }
        const uint32_t mk = k48::g_cand48.m[k];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const double aw = fabs((double)w[j]);
            if (mk & (1u << j)) acc[1] += aw;
            if (m0 & (1u << j)) acc[2] += aw;
        }
        acc[3] += (mk == m0) ? 1.0 : 0.0;
    }
    reduce4(acc, partials, ticket, out);
}

// ------------------------------------------------------------------ candidate-index codec

// D indices per uint32 word, base C, least significant digit first.
// Words w0 .. of the code (w0 > 0: the tail after encode4_kernel's groups).
__global__ void __launch_bounds__(kThreads) encode_kernel(const uint8_t *__restrict__ idx, int64_t n, int C,
                                                          int D, uint32_t *__restrict__ out, int64_t w0 = 0) {
    const int64_t words = (n + D - 1) / D;
    for (int64_t wi = w0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < words;
         wi += (int64_t)gridDim.x * blockDim.x) {
        uint32_t v = 0;
        for (int t = D - 1; t >= 0; --t) {  // Horner, most significant digit first
            const int64_t i = wi * D + t;
            v = v * (uint32_t)C + (i < n ? (uint32_t)idx[i] : 0u);
        }
        out[wi] = v;
    }
}

__global__ void __launch_bounds__(kThreads) decode_kernel(const uint32_t *__restrict__ in, int64_t n, int C,
                                                          int D, uint8_t *__restrict__ idx, int64_t w0 = 0) {
    const int64_t words = (n + D - 1) / D;
    for (int64_t wi = w0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < words;
         wi += (int64_t)gridDim.x * blockDim.x) {
        uint32_t v = in[wi];
        for (int t = 0; t < D; ++t) {
            const int64_t i = wi * D + t;
            if (i < n) idx[i] = (uint8_t)(v % (uint32_t)C);
            v /= (uint32_t)C;
        }
    }
}

// The same for whole groups of 4 words per thread with vector accesses (the digits of 4
// words, 4 D bytes, are read as D 32-bit words; the 4 words are written as one 16-byte
// store): group g covers indices 4 D g .. 4 D g + 4 D - 1. idx must be 4-byte aligned (16-byte
// when D % 4 == 0) and out 16-byte aligned; the caller runs the scalar kernel on the tail.
template <int C, int D>
__global__ void __launch_bounds__(kThreads) encode4_kernel(const uint8_t *__restrict__ idx, int64_t groups,
                                                           uint32_t *__restrict__ out) {
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
        uint32_t b[D];  // bytes 4 k .. 4 k + 3 of the group in b[k]
        if constexpr (D % 4 == 0) {
            const uint4 *p = reinterpret_cast<const uint4 *>(idx + 4 * D * g);
#pragma unroll
            for (int k = 0; k < D / 4; ++k) {
                const uint4 v = __ldcs(p + k);
                b[4 * k] = v.x; b[4 * k + 1] = v.y; b[4 * k + 2] = v.z; b[4 * k + 3] = v.w;
            }
        } else {
            const uint32_t *p = reinterpret_cast<const uint32_t *>(idx + 4 * D * g);
#pragma unroll
            for (int k = 0; k < D; ++k) b[k] = __ldcs(p + k);
        }
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t v = 0;
#pragma unroll
            for (int t = D - 1; t >= 0; --t) {  // Horner, most significant digit first
                const int byte = D * j + t;
                v = v * (uint32_t)C + __byte_perm(b[byte >> 2], 0u, 0x4440u | (uint32_t)(byte & 3));
            }
            w[j] = v;
        }
        __stcs(reinterpret_cast<uint4 *>(out) + g, make_uint4(w[0], w[1], w[2], w[3]));
    }
}

template <int C, int D>
__global__ void __launch_bounds__(kThreads) decode4_kernel(const uint32_t *__restrict__ in, int64_t groups,
                                                           uint8_t *__restrict__ idx) {
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += (int64_t)gridDim.x * blockDim.x) {
        const uint4 wv = __ldcs(reinterpret_cast<const uint4 *>(in) + g);
        const uint32_t wa[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t b[D];
#pragma unroll
        for (int k = 0; k < D; ++k) b[k] = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t v = wa[j];
#pragma unroll
            for (int t = 0; t < D; ++t) {
                const int byte = D * j + t;
                b[byte >> 2] |= (v % (uint32_t)C) << (8 * (byte & 3));
                v /= (uint32_t)C;
            }
        }
        if constexpr (D % 4 == 0) {
            uint4 *p = reinterpret_cast<uint4 *>(idx + 4 * D * g);
#pragma unroll
            for (int k = 0; k < D / 4; ++k) __stcs(p + k, make_uint4(b[4 * k], b[4 * k + 1], b[4 * k + 2], b[4 * k + 3]));
        } else {
            uint32_t *p = reinterpret_cast<uint32_t *>(idx + 4 * D * g);
#pragma unroll
            for (int k = 0; k < D; ++k) __stcs(p + k, b[k]);
        }
    }
}

}  // namespace diag
}  // namespace mllm
