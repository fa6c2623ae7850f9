// device_common.cuh -- launch descriptors and the random-number path shared by the kernels.
//
// The noise is part of the specification (bit for bit): Philox4x32-10 (Salmon, Moraes, Dror,
// Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) gives 128 bits per (seed,
// block, step, group); six 21-bit fields k give uniforms eps = (2k+1) 2^-22 and the Gumbel
// noise g = -nlog(-nlog(eps)) of MaskLLM's Eq.5 (paper-graph-ui summary, s.3.4 "Step 1").
// nlog is the fp32 table-driven logarithm of P.T.P. Tang (ACM TOMS 16(4), 1990): a 7-bit
// mantissa prefix j selects a breakpoint F_j in [0.75, 1.5) and x = 2^e mm, r = mm c_j - 1
// with c_j = fl32(1/F_j) and |r| < 2^-8; ln x = T[e][j] + (r - r^2/2 + r^3/3) with
// T[e][j] = fl32(e ln2 - ln c_j). Only correctly rounded fp32 operations (fma, mul, add) act
// on the data, so the bits are fixed by the definition on any IEEE machine. The noise takes
// logarithms of x in [2^-22, 16) only, so e runs over [-22, 4].
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace mllm {

constexpr int kMaxMats = 16;             // matrices per launch; larger groups are chunked
constexpr uint32_t kInitStep = 0xFFFFFFFFu;
constexpr int kThreads = 256;            // threads per CTA for every sampler kernel

// ---------------------------------------------------------------------------- nlog table

constexpr int kNlogEmin = -22, kNlogEmax = 4;
constexpr int kNlogRows = kNlogEmax - kNlogEmin + 1;  // 27
constexpr int kNlogEntries = kNlogRows * 128;        // 3456 (c_j, T[e][j]) pairs, 27 KB

// Natural logarithm in double, for building the table at compile time: x = m 2^k with m in
// [0.75, 1.5), ln m = 2 atanh((m-1)/(m+1)) by its series (|s| <= 0.2, 40 terms). Accurate to a
// few double ulps; every table entry lies more than 2^-20 fp32 ulp from a rounding boundary,
// so rounding this to fp32 gives the correctly rounded entry.
constexpr double kLn2 = 0.693147180559945309417232121458176568;
constexpr double cx_ln(double x) {
    int k = 0;
    while (x >= 1.5) { x *= 0.5; ++k; }
    while (x < 0.75) { x *= 2.0; --k; }
    const double s = (x - 1.0) / (x + 1.0), s2 = s * s;
    double term = s, sum = 0.0;
    for (int i = 1; i < 80; i += 2) { sum += term / i; term *= s2; }
    return 2.0 * sum + k * kLn2;
}

// The table in the order the kernels index it. With ib2 = bits(x) + 0x408000 (rounding the
// mantissa at its 7-bit prefix, plus half a binade), ib2 >> 23 = e + 127 and bits 16..22 of
// ib2 are j ^ 64 (prefixes j >= 64 carry into the exponent), so entry (ib2 >> 16) - 105*128
// = (e + 22)*128 + (j ^ 64) holds (c_j 2^-e, T[e][j]). Storing c_j scaled by 2^-e (exact)
// lets the kernel form r = fma(x, c_j 2^-e, -1), which equals fma(x 2^-e, c_j, -1) bit for
// bit, without reconstructing the reduced argument x 2^-e.
constexpr double cx_pow2(int e) {
    double p = 1.0;
    for (; e > 0; --e) p *= 2.0;
    for (; e < 0; ++e) p *= 0.5;
    return p;
}

struct NoiseTable {
    float2 cT[kNlogEntries];
    constexpr NoiseTable() : cT{} {
        for (int row = 0; row < kNlogRows; ++row) {
            const int e = row + kNlogEmin;
            for (int jr = 0; jr < 128; ++jr) {
                const int j = jr ^ 64;
                const double F = (j < 64) ? (1.0 + j / 128.0) : (1.0 + j / 128.0) * 0.5;
                const float c = (float)(1.0 / F);
                cT[row * 128 + jr] = float2{(float)((double)c * cx_pow2(-e)),
                                            (float)((double)e * kLn2 - cx_ln((double)c))};
            }
        }
    }
};
__device__ const NoiseTable g_noise_table{};
constexpr uint32_t kNlogIndexBias = (uint32_t)(127 + kNlogEmin) * 128u;  // 13440
constexpr float kOneThird = (float)(1.0 / 3.0);

// One matrix of a grouped launch. work_begin/work_count are in the kernel's work units
// (tiles of kThreads pairs of blocks, or of packed words).
struct MatDesc {
    const void *W;
    void *X;
    const void *G;
    float *pi, *m, *v;
    float *soft, *grad;
    void *pvals, *pmeta;
    uint8_t *cidx;
    const uint8_t *prior;  // prior candidate index per block (prior init from a given mask)
    int64_t rows, cols, nblocks;
    uint64_t gid0;
    int64_t work_begin, work_count;
    int32_t w_f32, g_f32;
};

struct Group {
    int32_t n;
    int32_t pad;
    int64_t total_work;
    MatDesc d[kMaxMats];
};

// Scalars of one forward / backward launch, derived on the host from mllm_hparams.
struct StepScalars {
    float kappa;         // logit scale
    float c2;            // fl32(log2(e) / tau): exp((w - max)/tau) = 2^((w - max) * c2)
    float kappa_over_tau;// fl32(kappa / tau), the z -> pi chain factor
    float two_lambda;    // 2 lambda
    float decay;         // fl32(1 - lr * wd)
    float beta1, one_minus_beta1, beta2, one_minus_beta2;
    float step_size;     // fl32(lr / (1 - beta1^t))
    float inv_sqrt_bc2;  // fl32(1 / sqrt(1 - beta2^t))
    float eps;
    uint32_t step;
    uint32_t noise_on;
    uint64_t seed;
    uint32_t rk[20];     // Philox round keys of the seed: rk[2r], rk[2r+1] = k0 + r W0, k1 + r W1
};

__device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// Index of the matrix that owns work unit t (uniform across the CTA).
__device__ __forceinline__ int find_mat(const Group &g, int64_t t) {
    int i = 0;
    while (i + 1 < g.n && t >= g.d[i + 1].work_begin) ++i;
    return i;
}

// The same searching forward from matrix i, the owner of a smaller unit: a CTA's grid-stride
// walk visits its units in increasing order, so the search resumes where the last one ended.
__device__ __forceinline__ int next_mat(const Group &g, int i, int64_t t) {
    while (i + 1 < g.n && t >= g.d[i + 1].work_begin) ++i;
    return i;
}

// ---------------------------------------------------------------------------- Philox

// One Philox round: the two 32 x 32 -> 64-bit products (one wide multiply each), then the
// S-box and the round key.
__device__ __forceinline__ uint4 philox_round(uint4 c, uint32_t rk0, uint32_t rk1) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c.x, p1 = (uint64_t)0xCD9E8D57u * c.z;
    return make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ rk0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ rk1, (uint32_t)p0);
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r)  // Weyl key schedule
        c = philox_round(c, k0 + (uint32_t)r * 0x9E3779B9u, k1 + (uint32_t)r * 0xBB67AE85u);
    return c;
}

// The same with the round keys of the launch's seed precomputed on the host (StepScalars::rk):
// in an unrolled loop they are read straight from the kernel's parameters.
__device__ __forceinline__ uint4 philox4x32_10_rk(uint4 c, const uint32_t (&rk)[20]) {
#pragma unroll
    for (int r = 0; r < 10; ++r) c = philox_round(c, rk[2 * r], rk[2 * r + 1]);
    return c;
}

// The six 21-bit fields of the 128-bit output (x as a little-endian integer).
__device__ __forceinline__ void fields21(uint4 x, uint32_t f[6]) {
    constexpr uint32_t M21 = 0x1FFFFFu;
    f[0] = x.x & M21;
    f[1] = __funnelshift_r(x.x, x.y, 21) & M21;
    f[2] = (x.y >> 10) & M21;
    f[3] = __funnelshift_r(x.y, x.z, 31) & M21;
    f[4] = __funnelshift_r(x.z, x.w, 20) & M21;
    f[5] = (x.w >> 9) & M21;
}

// The same six fields k, each already placed as the float bits of 1 + (2k+1) 2^-22: the
// field shifted to bits 2..22 (one funnel shift two places short of the field's offset)
// merged with the constant bits 0x3F800002 (one three-input logic op).
__device__ __forceinline__ void fields21_unit(uint4 x, uint32_t u[6]) {
    constexpr uint32_t MK = 0x7FFFFCu, ONE = 0x3F800002u;
    u[0] = ((x.x << 2) & MK) | ONE;
    u[1] = (__funnelshift_r(x.x, x.y, 19) & MK) | ONE;
    u[2] = ((x.y >> 8) & MK) | ONE;
    u[3] = (__funnelshift_r(x.y, x.z, 29) & MK) | ONE;
    u[4] = (__funnelshift_r(x.z, x.w, 18) & MK) | ONE;
    u[5] = ((x.w >> 7) & MK) | ONE;
}

__device__ __forceinline__ uint4 block_words(uint64_t seed, uint64_t gid, uint32_t step, uint32_t group) {
    return philox4x32_10(make_uint4((uint32_t)gid, (uint32_t)(gid >> 32), step, group),
                         (uint32_t)seed, (uint32_t)(seed >> 32));
}

// block_words for a launch's step (seed and step from the step's scalars).
__device__ __forceinline__ uint4 block_words(const StepScalars &sc, uint64_t gid, uint32_t group) {
    return philox4x32_10_rk(make_uint4((uint32_t)gid, (uint32_t)(gid >> 32), sc.step, group), sc.rk);
}

// eps = (2k+1) 2^-22: the bit pattern of 1 + (2k+1) 2^-22 minus 1 (both exact).
__device__ __forceinline__ float uniform_from_field(uint32_t k) {
    return __fadd_rn(__uint_as_float(0x3F800002u | (k << 2)), -1.0f);
}

// ---------------------------------------------------------------------------- nlog

// nlog(x) for x in [2^-22, 16). Both logarithms of the noise stay in that domain: the first
// takes eps in [2^-22, 1), and its result t = -nlog(eps), the second's argument, lies in
// [2^-22 + 2^-45, 15.25] for every one of the 2^21 fields (an exhaustive property of the
// definition), so the table index needs no clamp.
__device__ __forceinline__ float nlog(float x, const float2 *__restrict__ tab) {
    const uint32_t ib2 = __float_as_uint(x) + 0x408000u;
    const uint32_t idx = (ib2 >> 16) - kNlogIndexBias;
    const float2 cT = tab[idx];
    const float r = __fmaf_rn(x, cT.x, -1.0f);  // = fma(x 2^-e, c_j, -1)
    const float q = __fmaf_rn(r, kOneThird, -0.5f);
    const float rq = __fmul_rn(r, q);
    const float p = __fmaf_rn(rq, r, r);
    return __fadd_rn(cT.y, p);
}

struct NlogCtx {
    const float2 *tab;
};

// g = -log(-log eps) for field k (the negations are exact).
__device__ __forceinline__ float gumbel(uint32_t k, const NlogCtx &L) {
    const float eps = uniform_from_field(k);
    const float t = -nlog(eps, L.tab);
    return -nlog(t, L.tab);
}

// The same from the bits of 1 + eps (fields21_unit): eps = that - 1, exact.
__device__ __forceinline__ float gumbel_unit(uint32_t unit_bits, const NlogCtx &L) {
    const float eps = __fadd_rn(__uint_as_float(unit_bits), -1.0f);
    const float t = -nlog(eps, L.tab);
    return -nlog(t, L.tab);
}

// ---------------------------------------------------------------------------- paired forms
//
// The same arithmetic on two independent values at once with the fp32x2 instructions of
// sm_100 (__ffma2_rn, __fmul2_rn, __fadd2_rn: each component rounds exactly as __fmaf_rn,
// __fmul_rn, __fadd_rn), so every result is bit-identical to the scalar form while a pair
// costs one instruction where the scalar form costs two. Table lookups, integer steps and
// the special-function instructions stay per value.
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// (-nlog(x.x), -nlog(x.y)): the negation folded into the last add, (-T) + (-p) = -(T + p).
__device__ __forceinline__ float2 neg_nlog2(float2 x, const float2 *__restrict__ tab) {
    const float2 ca = tab[((__float_as_uint(x.x) + 0x408000u) >> 16) - kNlogIndexBias];
    const float2 cb = tab[((__float_as_uint(x.y) + 0x408000u) >> 16) - kNlogIndexBias];
    const float2 r = make_float2(__fmaf_rn(x.x, ca.x, -1.0f), __fmaf_rn(x.y, cb.x, -1.0f));
    const float2 q = __ffma2_rn(r, f2(kOneThird), f2(-0.5f));
    const float2 rq = __fmul2_rn(r, q);
    const float2 p = __ffma2_rn(rq, r, r);
    return make_float2(__fadd_rn(-ca.y, -p.x), __fadd_rn(-cb.y, -p.y));
}

// gumbel_unit of two fields.
__device__ __forceinline__ float2 gumbel_unit2(uint32_t ua, uint32_t ub, const NlogCtx &L) {
    const float2 eps = __fadd2_rn(make_float2(__uint_as_float(ua), __uint_as_float(ub)), f2(-1.0f));
    return neg_nlog2(neg_nlog2(eps, L.tab), L.tab);
}

// Copy the table into shared memory (all threads; __syncthreads() before use).
__device__ __forceinline__ void load_tab(float2 *s_tab) {
    const float4 *src = reinterpret_cast<const float4 *>(g_noise_table.cT);
    float4 *dst = reinterpret_cast<float4 *>(s_tab);
    for (int i = threadIdx.x; i < kNlogEntries / 2; i += blockDim.x) dst[i] = src[i];
}

// ---------------------------------------------------------------------------- misc

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Square root to about one ulp in one instruction (keeps denormals; sqrt(0) = 0). The
// AdamW denominator needs no correctly rounded root: its result is compared at 1e-4.
__device__ __forceinline__ float sqrt_approx(float x) {
    float y;
    asm("sqrt.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t *>(&h);
}

// Streaming (evict-first) global accesses for data touched once per call.
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }
__device__ __forceinline__ void st_stream(uint4 *p, uint4 v) { __stcs(p, v); }

}  // namespace mllm
