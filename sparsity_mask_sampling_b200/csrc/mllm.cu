// mllm.cu -- host side of libmllm: argument validation, grouping, launch configuration and
// the extern "C" entry points declared in include/mllm.h.
#include <algorithm>
#include <cudaTypedefs.h>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "mllm.h"
#include "device_common.cuh"
#include "kernels_2of4.cuh"
#include "kernels_4of8.cuh"
#include "kernels_diag.cuh"
#include "kernels_spl.cuh"
#include "kernels_umma.cuh"
#include "kernels_pf48.cuh"
#include "kernels_mlin.cuh"

namespace mllm {
namespace {

thread_local int32_t g_last_cuda = 0;

// Workspace layout of the forward's regulariser reduction: a ticket word, then one double
// per CTA of the launch (the forward grid is capped at kMaxReduceCtas).
constexpr int kMaxReduceCtas = 4096;
constexpr size_t kWsPartialsOffset = 16;
constexpr size_t kWorkspaceBytes = kWsPartialsOffset + sizeof(double) * kMaxReduceCtas;

// ------------------------------------------------------------------------ device info

struct OccKey {
    int dev;
    const void *fn;
};
std::mutex g_occ_mu;
std::vector<std::pair<OccKey, int>> g_occ;  // (device, kernel) -> resident CTAs per SM
std::vector<int> g_sms;

int sm_count(int dev) {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    if ((int)g_sms.size() <= dev) g_sms.resize(dev + 1, 0);
    if (!g_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 1;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

// Resident CTAs per SM of a kernel on a device (first use also sets the kernel's dynamic
// shared-memory limit to what its launches request).
int resident_ctas(int dev, const void *fn, int threads, int dyn_smem) {
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        for (auto &e : g_occ)
            if (e.first.dev == dev && e.first.fn == fn) return e.second;
    }
    if (dyn_smem > 0) cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, dyn_smem) != cudaSuccess || n <= 0) n = 1;
    std::lock_guard<std::mutex> lk(g_occ_mu);
    g_occ.push_back({OccKey{dev, fn}, n});
    return n;
}

int64_t grid_for(const void *fn, int threads, int dyn_smem, int64_t work, int64_t cap) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int64_t g = (int64_t)sm_count(dev) * resident_ctas(dev, fn, threads, dyn_smem);
    return std::max<int64_t>(1, std::min<int64_t>({work, g, cap}));
}

// CTAs the 4:8 forward can use on a group: each CTA's two halves take one tile each.
int64_t k48_fwd_ctas(const Group &g) { return (g.total_work + k48::kFwdHalves - 1) / k48::kFwdHalves; }

mllm_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MLLM_OK;
    g_last_cuda = (int32_t)e;
    return MLLM_ERR_CUDA;
}

// ------------------------------------------------------------------------ validation

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

enum Need : unsigned {
    kNeedW = 1, kNeedX = 2, kNeedG = 4, kNeedPi = 8, kNeedMV = 16, kNeedPack = 32,
};

int num_cand(mllm_nm nm) {
    if (nm.n == 2 && nm.m == 4) return 6;
    if (nm.n == 4 && nm.m == 8) return 70;
    return 0;
}

mllm_status check_ptr(const void *p, bool required) {
    if (!p) return required ? MLLM_ERR_INVALID_ARG : MLLM_OK;
    return aligned16(p) ? MLLM_OK : MLLM_ERR_MISALIGNED;
}

mllm_status validate_mats(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, unsigned need) {
    if (!num_cand(nm)) return MLLM_ERR_UNSUPPORTED;
    if (!mats || n_mats <= 0) return MLLM_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_mats; ++i) {
        const mllm_matrix &a = mats[i];
        if (a.rows < 0 || a.cols < 0 || a.cols % nm.m) return MLLM_ERR_INVALID_ARG;
        if (a.rows > 0 && a.cols > ((int64_t)1 << 62) / a.rows) return MLLM_ERR_INVALID_ARG;
        if (a.w_dtype != MLLM_BF16 && a.w_dtype != MLLM_F32) return MLLM_ERR_UNSUPPORTED;
        if (a.w_dtype != mats[0].w_dtype) return MLLM_ERR_UNSUPPORTED;
        if (need & kNeedG) {
            if (a.g_dtype != MLLM_BF16 && a.g_dtype != MLLM_F32) return MLLM_ERR_UNSUPPORTED;
            if (a.g_dtype != mats[0].g_dtype) return MLLM_ERR_UNSUPPORTED;
        }
        const bool any = a.rows > 0 && a.cols > 0;
        mllm_status s;
        if ((s = check_ptr(a.W, any && (need & kNeedW))) != MLLM_OK) return s;
        if ((s = check_ptr(a.X_out, any && (need & kNeedX))) != MLLM_OK) return s;
        if ((s = check_ptr(a.G, any && (need & kNeedG))) != MLLM_OK) return s;
        if ((s = check_ptr(a.logits, any && (need & kNeedPi))) != MLLM_OK) return s;
        if ((s = check_ptr(a.adam_m, any && (need & kNeedMV))) != MLLM_OK) return s;
        if ((s = check_ptr(a.adam_v, any && (need & kNeedMV))) != MLLM_OK) return s;
        if ((s = check_ptr(a.soft_mask_out, false)) != MLLM_OK) return s;
        if ((s = check_ptr(a.grad_logits_out, false)) != MLLM_OK) return s;
        if ((s = check_ptr(a.pack_values, any && (need & kNeedPack))) != MLLM_OK) return s;
        if ((s = check_ptr(a.pack_meta, any && (need & kNeedPack))) != MLLM_OK) return s;
        if ((s = check_ptr(a.cand_idx_out, false)) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

bool finite(float x) { return std::isfinite(x); }

mllm_status validate_fwd_hp(const mllm_hparams *hp) {
    if (!hp) return MLLM_ERR_INVALID_ARG;
    if (!finite(hp->kappa) || !(hp->kappa > 0.f)) return MLLM_ERR_INVALID_ARG;
    if (!finite(hp->tau) || !(hp->tau > 0.f)) return MLLM_ERR_INVALID_ARG;
    if (hp->step == kInitStep || hp->reserved != 0) return MLLM_ERR_INVALID_ARG;
    const double c2 = 1.4426950408889634 / (double)hp->tau;
    const double kt = (double)hp->kappa / (double)hp->tau;
    if (!std::isfinite((float)c2) || !std::isfinite((float)kt)) return MLLM_ERR_INVALID_ARG;
    return MLLM_OK;
}

mllm_status validate_bwd_hp(const mllm_hparams *hp) {
    mllm_status s = validate_fwd_hp(hp);
    if (s != MLLM_OK) return s;
    if (!finite(hp->lambda) || hp->lambda < 0.f) return MLLM_ERR_INVALID_ARG;
    if (!finite(hp->lr) || hp->lr < 0.f) return MLLM_ERR_INVALID_ARG;
    if (!(hp->beta1 >= 0.f && hp->beta1 < 1.f)) return MLLM_ERR_INVALID_ARG;
    if (!(hp->beta2 >= 0.f && hp->beta2 < 1.f)) return MLLM_ERR_INVALID_ARG;
    if (!finite(hp->eps) || !(hp->eps > 0.f)) return MLLM_ERR_INVALID_ARG;
    if (!finite(hp->weight_decay) || hp->weight_decay < 0.f) return MLLM_ERR_INVALID_ARG;
    if (hp->adam_step < 1) return MLLM_ERR_INVALID_ARG;
    return MLLM_OK;
}

StepScalars make_scalars(const mllm_hparams &hp) {
    StepScalars s{};
    const double t = (double)hp.adam_step;
    s.kappa = hp.kappa;
    s.c2 = (float)(1.4426950408889634 / (double)hp.tau);
    s.kappa_over_tau = (float)((double)hp.kappa / (double)hp.tau);
    s.two_lambda = 2.0f * hp.lambda;
    s.decay = (float)(1.0 - (double)hp.lr * (double)hp.weight_decay);
    s.beta1 = hp.beta1;
    s.one_minus_beta1 = (float)(1.0 - (double)hp.beta1);
    s.beta2 = hp.beta2;
    s.one_minus_beta2 = (float)(1.0 - (double)hp.beta2);
    const double bc1 = 1.0 - std::pow((double)hp.beta1, t);
    const double bc2 = 1.0 - std::pow((double)hp.beta2, t);
    s.step_size = (bc1 > 0.0) ? (float)((double)hp.lr / bc1) : 0.f;
    s.inv_sqrt_bc2 = (bc2 > 0.0) ? (float)(1.0 / std::sqrt(bc2)) : 0.f;
    s.eps = hp.eps;
    s.step = hp.step;
    s.noise_on = hp.noise_on ? 1u : 0u;
    s.seed = hp.seed;
    for (int r = 0; r < 10; ++r) {  // Philox4x32-10 key schedule (Weyl sequence), mod 2^32
        s.rk[2 * r] = (uint32_t)hp.seed + (uint32_t)r * 0x9E3779B9u;
        s.rk[2 * r + 1] = (uint32_t)(hp.seed >> 32) + (uint32_t)r * 0xBB67AE85u;
    }
    return s;
}

// ------------------------------------------------------------------------ grouping

MatDesc make_desc(const mllm_matrix &a, int M) {
    MatDesc d{};
    d.W = a.W; d.X = a.X_out; d.G = a.G;
    d.pi = a.logits; d.m = a.adam_m; d.v = a.adam_v;
    d.soft = a.soft_mask_out; d.grad = a.grad_logits_out;
    d.pvals = a.pack_values; d.pmeta = a.pack_meta; d.cidx = a.cand_idx_out;
    d.rows = a.rows; d.cols = a.cols;
    d.nblocks = (a.rows > 0 && a.cols > 0) ? a.rows * (a.cols / M) : 0;
    d.gid0 = a.block_offset;
    d.w_f32 = a.w_dtype == MLLM_F32;
    d.g_f32 = a.g_dtype == MLLM_F32;
    return d;
}

// Work units of one matrix for a kernel kind.
enum class Kind { Sample24, Pack24, Sample48, Pack48 };

int64_t work_units(const MatDesc &d, Kind k) {
    if (d.nblocks == 0) return 0;
    switch (k) {
        case Kind::Sample24: {
            const int64_t pairs = (d.nblocks + 1) / 2;
            return (pairs + kThreads - 1) / kThreads;
        }
        case Kind::Pack24: {
            const int64_t bpr = d.cols / 4, words = d.rows * ((bpr + 7) / 8);
            return (words + kThreads - 1) / kThreads;
        }
        case Kind::Sample48:
            return (d.nblocks + k48::kBlocksPerCta - 1) / k48::kBlocksPerCta;
        case Kind::Pack48:
            return (d.nblocks + k48::kBlocksPerCta - 1) / k48::kBlocksPerCta;
    }
    return 0;
}

// Split the call into groups of at most kMaxMats matrices with their work prefix sums.
std::vector<Group> make_groups(const mllm_matrix *mats, int32_t n_mats, int M, Kind k) {
    std::vector<Group> out;
    for (int32_t i0 = 0; i0 < n_mats; i0 += kMaxMats) {
        Group g{};
        const int32_t n = std::min<int32_t>(kMaxMats, n_mats - i0);
        int64_t acc = 0;
        for (int32_t i = 0; i < n; ++i) {
            MatDesc d = make_desc(mats[i0 + i], M);
            d.work_begin = acc;
            d.work_count = work_units(d, k);
            acc += d.work_count;
            g.d[i] = d;
        }
        g.n = n;
        g.total_work = acc;
        out.push_back(g);
    }
    return out;
}

// ------------------------------------------------------------------------ sparse linear

constexpr int kMaxCallTokens = 16384;  // tokens per mllm_sparse_linear call
constexpr int kSplRowTiles = 2;   // row tiles of 16 per CTA task (4 warps per tile split k)
constexpr int kSplDepth = 2;      // slabs in flight per warp

mllm_status validate_operands(const mllm_sparse_operand *ops, int32_t n_ops, mllm_nm nm, int32_t tokens) {
    if (!num_cand(nm)) return MLLM_ERR_UNSUPPORTED;
    if (!ops || n_ops <= 0 || tokens < 1 || tokens > kMaxCallTokens) return MLLM_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_ops; ++i) {
        const mllm_sparse_operand &o = ops[i];
        if (o.rows < 0 || o.cols < 0 || o.cols % nm.m || o.rows > INT32_MAX || o.cols > INT32_MAX)
            return MLLM_ERR_INVALID_ARG;
        if (o.rows == 0) continue;
        mllm_status s;
        if ((s = check_ptr(o.y, true)) != MLLM_OK) return s;
        const bool any = o.cols > 0;
        if ((s = check_ptr(o.pack_values, any)) != MLLM_OK) return s;
        if ((s = check_ptr(o.pack_meta, any)) != MLLM_OK) return s;
        if ((s = check_ptr(o.x, any)) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

template <int kN, int kNT>
mllm_status launch_spl_sk(const spl::SkGroup &g, float *part, unsigned int *tickets, cudaStream_t st) {
    auto fn = spl::sparse_linear_sk_kernel<kN, kNT>;
    constexpr int smem = spl::sk_smem_bytes<kNT>();
    const int64_t grid = grid_for((const void *)fn, spl::kSkThreads, smem, INT32_MAX,
                                  spl::kMaxSkWarps / spl::kSkWarps);
    fn<<<(unsigned)grid, spl::kSkThreads, smem, st>>>(g, part, tickets);
    return cuda_status(cudaGetLastError());
}

template <int kNT>
mllm_status launch_spl_sp(const spl::SkGroup &g, float *part, unsigned int *tickets, cudaStream_t st) {
    auto fn = spl::sparse_linear_sp_kernel<kNT>;
    constexpr int smem = spl::sp_smem_bytes<kNT>(), threads = 32 * spl::sp_warps<kNT>();
    const int64_t grid = grid_for((const void *)fn, threads, smem, INT32_MAX, spl::kMaxSkWarps / spl::sp_warps<kNT>());
    fn<<<(unsigned)grid, threads, smem, st>>>(g, part, tickets);
    return cuda_status(cudaGetLastError());
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A 2-D row-major tensor [outer, inner] with rows of row_bytes, copied in boxes of
// box_outer x box_inner elements.
bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    const auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The three maps of an operand for the TMA kernel (cols % 128 == 0).
bool encode_operand(spl::TmMaps *mp, const mllm_sparse_operand &o, int32_t tokens, int kNT) {
    const uint64_t rows = (uint64_t)o.rows, cols = (uint64_t)o.cols;
    return encode_2d(&mp->meta, CU_TENSOR_MAP_DATA_TYPE_UINT32, o.pack_meta, cols / 32, rows, cols / 8, 4, 32,
                     CU_TENSOR_MAP_SWIZZLE_NONE) &&
           encode_2d(&mp->vals, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.pack_values, cols / 2, rows, cols, 64, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B) &&
           encode_2d(&mp->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.x, cols, (uint64_t)tokens, 2 * cols, 64,
                     (uint32_t)(8 * kNT), CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int kNT>
mllm_status launch_spl_tma(const spl::TmGroup &g, float *part, unsigned int *tickets, unsigned int *err,
                           cudaStream_t st, int arm_only_first = 0) {
    auto fn = spl::sparse_linear_tma_kernel<kNT>;
    constexpr int smem = spl::tm_smem_bytes<kNT>(), threads = 32 * spl::kTmWarps;
    const int64_t grid = grid_for((const void *)fn, threads, smem, INT32_MAX, spl::kMaxSkWarps / spl::kTmWarps);
    fn<<<(unsigned)grid, threads, smem, st>>>(g, part, tickets, err, arm_only_first);
    return cuda_status(cudaGetLastError());
}

template <int kNTok>
mllm_status launch_spl_umma(const spl::TmGroup &g, float *part, unsigned int *tickets, unsigned int *err,
                            cudaStream_t st, int arm_only_first = 0) {
    auto fn = spl::sparse_linear_umma_kernel<kNTok>;
    constexpr int smem = spl::um_smem_bytes<kNTok>();
    // The occupancy query reports one resident CTA per SM for this kernel, although its launch
    // bounds and shared memory admit kUmCtasPerSm (and a profile of a launch shows that
    // limit); the grid is sized from those limits. No CTA waits on another, so any grid is correct.
    int dev = 0;
    cudaGetDevice(&dev);
    resident_ctas(dev, (const void *)fn, spl::kUmThreads, smem);  // sets the dynamic shared-memory limit
    const int64_t grid = std::min<int64_t>((int64_t)sm_count(dev) * spl::kUmCtasPerSm, spl::kBatchMaxCtas);
    fn<<<(unsigned)grid, spl::kUmThreads, smem, st>>>(g, part, tickets, err, arm_only_first);
    return cuda_status(cudaGetLastError());
}

template <int kNTok>
mllm_status launch_spl_umma48(const spl::TmGroup &g, float *part, unsigned int *tickets, unsigned int *err,
                              cudaStream_t st, int arm_only_first = 0) {
    auto fn = spl::sparse_linear_umma48_kernel<kNTok>;
    constexpr int smem = spl::u8_smem_bytes<kNTok>();
    int dev = 0;
    cudaGetDevice(&dev);
    resident_ctas(dev, (const void *)fn, spl::kU8Threads, smem);  // sets the dynamic shared-memory limit
    const int64_t grid = std::min<int64_t>((int64_t)sm_count(dev), spl::kBatchMaxCtas);  // one CTA per SM
    fn<<<(unsigned)grid, spl::kU8Threads, smem, st>>>(g, part, tickets, err, arm_only_first);
    return cuda_status(cudaGetLastError());
}

template <int kN, int kNT>
mllm_status launch_spl(const spl::OpGroup &g, cudaStream_t st) {
    auto fn = spl::sparse_linear_kernel<kN, kNT, kSplRowTiles, kSplDepth>;
    const int64_t grid = grid_for((const void *)fn, spl::kCtaThreads, 0, g.total_tasks, INT32_MAX);
    fn<<<(unsigned)grid, spl::kCtaThreads, 0, st>>>(g);
    return cuda_status(cudaGetLastError());
}

// ------------------------------------------------------------------------ prior launcher

template <bool kFromIdx>
mllm_status launch_prior(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, const uint8_t *const *prior_idx,
                         float alpha, float init_std, uint64_t seed, void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool w32 = mats[0].w_dtype == MLLM_F32;
    const bool is24 = nm.m == 4;
    int32_t i0 = 0;
    for (Group g : make_groups(mats, n_mats, nm.m, is24 ? Kind::Sample24 : Kind::Sample48)) {
        if (kFromIdx)
            for (int32_t i = 0; i < g.n; ++i) g.d[i].prior = prior_idx[i0 + i];
        i0 += g.n;
        if (g.total_work == 0) continue;
        if (is24) {
            const void *fn = w32 ? (const void *)k24::prior_kernel<true, kFromIdx> : (const void *)k24::prior_kernel<false, kFromIdx>;
            const int64_t grid = grid_for(fn, kThreads, 0, g.total_work, INT32_MAX);
            if (w32) k24::prior_kernel<true, kFromIdx><<<(unsigned)grid, kThreads, 0, st>>>(g, alpha, init_std, seed);
            else k24::prior_kernel<false, kFromIdx><<<(unsigned)grid, kThreads, 0, st>>>(g, alpha, init_std, seed);
        } else {
            const void *fn = w32 ? (const void *)k48::prior_kernel<true, kFromIdx> : (const void *)k48::prior_kernel<false, kFromIdx>;
            const int64_t grid = grid_for(fn, k48::kCtaThreads, 0, g.total_work, INT32_MAX);
            if (w32) k48::prior_kernel<true, kFromIdx><<<(unsigned)grid, k48::kCtaThreads, 0, st>>>(g, alpha, init_std, seed);
            else k48::prior_kernel<false, kFromIdx><<<(unsigned)grid, k48::kCtaThreads, 0, st>>>(g, alpha, init_std, seed);
        }
        mllm_status s = cuda_status(cudaGetLastError());
        if (s != MLLM_OK) return s;
    }
    return MLLM_OK;
}

// ------------------------------------------------------------------------ no-alloc scratch

// Scratch of mllm_sample_fwd_noalloc: the ticket word at offset 0, per-CTA partial sums from
// offset kWsPartialsOffset. A file-scope device array, so no allocation is ever made. Host
// code cannot use the symbol itself (it names a host-side stand-in), so the array's device
// address on the current device is looked up with cudaGetSymbolAddress. That is done on every
// call rather than cached: a device reset or a new context may place the module, and with it
// the array, elsewhere, and a stale address would make the launch touch memory it does not own.
// Once the module is loaded on a device the lookup is a host-side table query.
constexpr int kNoallocMaxCtas = 2048;
constexpr size_t kNoallocBytes = kWsPartialsOffset + sizeof(double) * kNoallocMaxCtas;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

mllm_status noalloc_scratch(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    if (!p) return MLLM_ERR_CUDA;
    *out = p;
    return MLLM_OK;
}

// 2:4 operands with cols % 128 == 0 above 64 tokens on the prefill kernel, 16 operands per
// launch (longest rows first): units (operand, pair of 128-row tiles, 128-token chunk) dealt
// round-robin over the CTAs in the kernel's group order. False if a tensor map cannot be encoded (nothing
// is launched then).
bool sparse_linear_prefill(const std::vector<mllm_sparse_operand> &ops_in, int32_t tokens, unsigned int *err,
                           cudaStream_t st, mllm_status *status) {
    std::vector<mllm_sparse_operand> ops = ops_in;
    std::stable_sort(ops.begin(), ops.end(),
                     [](const mllm_sparse_operand &a, const mllm_sparse_operand &b) { return a.cols > b.cols; });
    auto fn = spl::sparse_linear_prefill_kernel;
    constexpr int smem = spl::kPfSmem;
    int dev = 0;
    cudaGetDevice(&dev);
    resident_ctas(dev, (const void *)fn, spl::kPfThreads, smem);  // sets the dynamic shared-memory limit
    for (size_t i0 = 0; i0 < ops.size(); i0 += kMaxMats) {
        const size_t n = std::min<size_t>(kMaxMats, ops.size() - i0);
        static thread_local spl::PfGroup pg;
        pg = spl::PfGroup{};
        pg.tokens = tokens;
        const int64_t nt = (tokens + spl::kPfTok - 1) / spl::kPfTok;
        const int64_t G0 = std::min<int64_t>((int64_t)sm_count(dev), (int64_t)spl::kPfMaxCtas);
        int64_t units = 0;
        for (size_t k = 0; k < n; ++k) {
            const mllm_sparse_operand &o = ops[i0 + k];
            spl::PfOp &d = pg.d[k];
            d.meta = o.pack_meta;
            d.y = o.y;
            d.rows = o.rows;
            d.cols = o.cols;
            d.nch = o.cols / spl::kTmChunk;
            d.npairs = (o.rows + 2 * spl::kUmRows - 1) / (2 * spl::kUmRows);
            d.nt = nt;
            d.rgroup = std::max<int64_t>(1, (G0 + nt - 1) / nt);
            d.unit_begin = units;
            units += d.npairs * nt;
            const uint64_t rows = (uint64_t)o.rows, cols = (uint64_t)o.cols;
            if (!(encode_2d(&pg.maps[k].vals, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.pack_values, cols / 2, rows, cols, 64,
                            spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  encode_2d(&pg.maps[k].meta, CU_TENSOR_MAP_DATA_TYPE_UINT32, o.pack_meta, cols / 32, rows, cols / 8, 4,
                            spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  encode_2d(&pg.maps[k].x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.x, cols, (uint64_t)tokens, 2 * cols, 64,
                            (uint32_t)spl::kPfTok, CU_TENSOR_MAP_SWIZZLE_128B)))
                return false;
        }
        pg.n = (int32_t)n;
        pg.total_units = units;
        const int64_t G = std::min<int64_t>(G0, units);
        fn<<<(unsigned)G, spl::kPfThreads, smem, st>>>(pg, err);
        if ((*status = cuda_status(cudaGetLastError())) != MLLM_OK) return true;
    }
    *status = MLLM_OK;
    return true;
}

// 4:8 at prefill sizes: units of (operand, 128 rows, kTok tokens) over 64-column stages, each
// stage expanded to dense once; operand and unit order as for the 2:4 prefill kernel. Returns
// false when a tensor map cannot be encoded (the caller then runs 64-token groups).
template <int kTok>
bool sparse_linear_prefill48_n(const std::vector<mllm_sparse_operand> &ops_in, int32_t tokens, unsigned int *err,
                               cudaStream_t st, mllm_status *status) {
    std::vector<mllm_sparse_operand> ops = ops_in;
    std::stable_sort(ops.begin(), ops.end(),
                     [](const mllm_sparse_operand &a, const mllm_sparse_operand &b) { return a.cols > b.cols; });
    auto fn = spl::sparse_linear_prefill48_kernel<kTok>;
    constexpr int smem = spl::P8<kTok>::kSmem;
    int dev = 0;
    cudaGetDevice(&dev);
    resident_ctas(dev, (const void *)fn, spl::kP8Threads, smem);  // sets the dynamic shared-memory limit
    for (size_t i0 = 0; i0 < ops.size(); i0 += kMaxMats) {
        const size_t n = std::min<size_t>(kMaxMats, ops.size() - i0);
        static thread_local spl::PfGroup pg;
        pg = spl::PfGroup{};
        pg.tokens = tokens;
        const int64_t nt = (tokens + kTok - 1) / kTok;
        const int64_t G0 = std::min<int64_t>((int64_t)sm_count(dev), (int64_t)spl::kPfMaxCtas);
        int64_t units = 0;
        for (size_t k = 0; k < n; ++k) {
            const mllm_sparse_operand &o = ops[i0 + k];
            spl::PfOp &d = pg.d[k];
            d.meta = o.pack_meta;
            d.y = o.y;
            d.rows = o.rows;
            d.cols = o.cols;
            d.nch = o.cols / 64;                                   // 64-column stages
            d.npairs = (o.rows + spl::kUmRows - 1) / spl::kUmRows;  // 128-row tiles
            d.nt = nt;
            d.rgroup = std::max<int64_t>(1, (G0 + nt - 1) / nt);
            d.unit_begin = units;
            units += d.npairs * nt;
            const uint64_t rows = (uint64_t)o.rows, cols = (uint64_t)o.cols;
            if (!(encode_2d(&pg.maps[k].vals, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.pack_values, cols / 2, rows, cols, 32,
                            spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_64B) &&
                  encode_2d(&pg.maps[k].meta, CU_TENSOR_MAP_DATA_TYPE_UINT16, o.pack_meta, cols / 8, rows, cols / 4, 8,
                            spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                  encode_2d(&pg.maps[k].x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.x, cols, (uint64_t)tokens, 2 * cols, 64,
                            (uint32_t)kTok, CU_TENSOR_MAP_SWIZZLE_128B)))
                return false;
        }
        pg.n = (int32_t)n;
        pg.total_units = units;
        const int64_t G = std::min<int64_t>(G0, units);
        fn<<<(unsigned)G, spl::kP8Threads, smem, st>>>(pg, err);
        if ((*status = cuda_status(cudaGetLastError())) != MLLM_OK) return true;
    }
    *status = MLLM_OK;
    return true;
}

bool sparse_linear_prefill48(const std::vector<mllm_sparse_operand> &ops, int32_t tokens, unsigned int *err,
                             cudaStream_t st, mllm_status *status) {
    return tokens <= 128 ? sparse_linear_prefill48_n<128>(ops, tokens, err, st, status)
                         : sparse_linear_prefill48_n<256>(ops, tokens, err, st, status);
}

// The per-warp kernels for up to 16 tokens; every operand has rows > 0 and cols > 0.
mllm_status sparse_linear_small(const std::vector<mllm_sparse_operand> &ops, mllm_nm nm, int32_t tokens, float *part,
                                unsigned int *tickets, unsigned int *err, cudaStream_t st) {
    mllm_status s = MLLM_OK;
    std::vector<int32_t> order(ops.size());
    for (size_t i = 0; i < ops.size(); ++i) order[i] = (int32_t)i;
    // operands grouped by the kernel their width allows (so that a launch of 16 does not fall
    // back for one odd operand), then the longest rows first (the tiled kernel's first wave
    // takes them)
    auto width_class = [&](int64_t cols) {
        if (cols % spl::kTmChunk == 0) return 0;
        if (cols % 32 == 0) return 1;
        return cols % 16 == 0 ? 2 : 3;
    };
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
        const int ca = width_class(ops[a].cols), cb = width_class(ops[b].cols);
        return ca != cb ? ca < cb : ops[a].cols > ops[b].cols;
    });
    const bool is24 = nm.m == 4, two = tokens > 8;
    for (size_t i0 = 0; i0 < order.size(); i0 += kMaxMats) {
        const size_t n = std::min<size_t>(kMaxMats, order.size() - i0);
        bool vec = true, words = true, stages = true;
        for (size_t k = 0; k < n; ++k) {
            vec = vec && (ops[order[i0 + k]].cols % 16 == 0);
            words = words && (ops[order[i0 + k]].cols % 32 == 0);
            stages = stages && (ops[order[i0 + k]].cols % spl::kTmChunk == 0);
        }
        if (vec) {  // streamed kernels: the launch's chunks split evenly over all warps
            // 2:4 in whole 128-column stages: tensor copies (falls back if a map cannot be
            // encoded); other 2:4 with whole metadata words: sparse tensor cores via cp.async;
            // else (and 4:8 whose maps could not be encoded for the tensor-memory kernel)
            // block expansion
            const bool tma = stages && is24;
            auto group_of = [&](int64_t chunk) {
                spl::SkGroup g{};
                g.tokens = tokens;
                int64_t acc = 0;
                for (size_t k = 0; k < n; ++k) {
                    const mllm_sparse_operand &o = ops[order[i0 + k]];
                    spl::SkOp &d = g.d[k];
                    d.vals = static_cast<const uint32_t *>(o.pack_values);
                    d.meta = o.pack_meta;
                    d.x = static_cast<const uint32_t *>(o.x);
                    d.y = o.y;
                    d.rows = o.rows;
                    d.cols = o.cols;
                    d.nch = (o.cols + chunk - 1) / chunk;
                    d.ntiles = (o.rows + spl::kSkRows - 1) / spl::kSkRows;
                    d.chunk_begin = acc;
                    acc += d.nch * d.ntiles;
                }
                g.n = (int32_t)n;
                g.total_chunks = acc;
                return g;
            };
            if (tma) {
                static thread_local spl::TmGroup tg;
                tg.g = group_of(spl::kTmChunk);
                bool ok = true;
                for (size_t k = 0; k < n && ok; ++k)
                    ok = encode_operand(&tg.maps[k], ops[order[i0 + k]], tokens, two ? 2 : 1);
                if (ok) {
                    s = two ? launch_spl_tma<2>(tg, part, tickets, err, st) : launch_spl_tma<1>(tg, part, tickets, err, st);
                    if (s != MLLM_OK) return s;
                    continue;
                }
            }
            const spl::SkGroup g = group_of(spl::kChunk);
            if (is24 && words) s = two ? launch_spl_sp<2>(g, part, tickets, st) : launch_spl_sp<1>(g, part, tickets, st);
            else if (is24) s = two ? launch_spl_sk<2, 2>(g, part, tickets, st) : launch_spl_sk<2, 1>(g, part, tickets, st);
            else s = two ? launch_spl_sk<4, 2>(g, part, tickets, st) : launch_spl_sk<4, 1>(g, part, tickets, st);
            if (s != MLLM_OK) return s;
            continue;
        }
        spl::OpGroup g{};
        g.tokens = tokens;
        int64_t acc = 0;
        const int64_t rows_per_task = 16 * kSplRowTiles;
        for (size_t k = 0; k < n; ++k) {
            const mllm_sparse_operand &o = ops[order[i0 + k]];
            spl::Op &d = g.d[k];
            d.vals = static_cast<const uint32_t *>(o.pack_values);
            d.meta = o.pack_meta;
            d.x = static_cast<const uint32_t *>(o.x);
            d.y = o.y;
            d.rows = o.rows;
            d.cols = o.cols;
            d.task_begin = acc;
            acc += (o.rows + rows_per_task - 1) / rows_per_task;
        }
        g.n = (int32_t)n;
        g.total_tasks = acc;
        if (is24) s = two ? launch_spl<2, 2>(g, st) : launch_spl<2, 1>(g, st);
        else s = two ? launch_spl<4, 2>(g, st) : launch_spl<4, 1>(g, st);
        if (s != MLLM_OK) return s;
    }
    return MLLM_OK;
}


// Operands with cols % 128 == 0 on the tensor-memory kernels (2:4 sparse MMA above 16 tokens,
// 4:8 expanded to dense at any token count), 16 operands per launch (false if a tensor map
// cannot be encoded; nothing is launched then).
bool sparse_linear_batched(const std::vector<mllm_sparse_operand> &ops, mllm_nm nm, int32_t tokens, float *part,
                           unsigned int *tickets, unsigned int *err, cudaStream_t st, mllm_status *status,
                           int arm_only_first = 0) {
    const bool is24 = nm.m == 4;
    const int step = is24 ? 16 : spl::kU8NStep;  // the MMA's N: tokens rounded up to a step, at least 32
    const int ntok = (tokens + step - 1) / step * step < 32 ? 32 : (tokens + step - 1) / step * step;
    for (size_t i0 = 0; i0 < ops.size(); i0 += kMaxMats) {
        const size_t n = std::min<size_t>(kMaxMats, ops.size() - i0);
        static thread_local spl::TmGroup tg;
        tg.g = spl::SkGroup{};
        tg.g.tokens = tokens;
        int64_t acc = 0;
        for (size_t k = 0; k < n; ++k) {
            const mllm_sparse_operand &o = ops[i0 + k];
            spl::SkOp &d = tg.g.d[k];
            d.vals = static_cast<const uint32_t *>(o.pack_values);
            d.meta = o.pack_meta;
            d.x = static_cast<const uint32_t *>(o.x);
            d.y = o.y;
            d.rows = o.rows;
            d.cols = o.cols;
            d.nch = o.cols / spl::kTmChunk;
            d.ntiles = (o.rows + spl::kUmRows - 1) / spl::kUmRows;
            d.chunk_begin = acc;
            acc += d.nch * d.ntiles;
            const uint64_t rows = (uint64_t)o.rows, cols = (uint64_t)o.cols;
            if (!(encode_2d(&tg.maps[k].vals, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.pack_values, cols / 2, rows, cols, 64,
                            spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  (is24 ? encode_2d(&tg.maps[k].meta, CU_TENSOR_MAP_DATA_TYPE_UINT32, o.pack_meta, cols / 32, rows,
                                    cols / 8, 4, spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_NONE)
                        : encode_2d(&tg.maps[k].meta, CU_TENSOR_MAP_DATA_TYPE_UINT16, o.pack_meta, cols / 8, rows,
                                    cols / 4, 16, spl::kUmRows, CU_TENSOR_MAP_SWIZZLE_NONE)) &&
                  encode_2d(&tg.maps[k].x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.x, cols, (uint64_t)tokens, 2 * cols, 64,
                            (uint32_t)ntok, CU_TENSOR_MAP_SWIZZLE_128B)))
                return false;
        }
        tg.g.n = (int32_t)n;
        tg.g.total_chunks = acc;
        if (is24)
            *status = ntok == 64   ? launch_spl_umma<64>(tg, part, tickets, err, st, arm_only_first)
                      : ntok == 48 ? launch_spl_umma<48>(tg, part, tickets, err, st, arm_only_first)
                                   : launch_spl_umma<32>(tg, part, tickets, err, st, arm_only_first);
        else if (ntok == 64)
            *status = launch_spl_umma48<64>(tg, part, tickets, err, st, arm_only_first);
        else if constexpr (48 % spl::kU8NStep == 0)
            *status = ntok == 48 ? launch_spl_umma48<48>(tg, part, tickets, err, st, arm_only_first)
                                 : launch_spl_umma48<32>(tg, part, tickets, err, st, arm_only_first);
        else
            *status = launch_spl_umma48<32>(tg, part, tickets, err, st, arm_only_first);
        if (*status != MLLM_OK) return true;
    }
    *status = MLLM_OK;
    return true;
}

// ------------------------------------------------------------------------ masked linear layer

// Tokens rounded up to the MMA's N (32, 64, 128 or 256).
int mlin_n(int32_t tokens) { return tokens <= 32 ? 32 : tokens <= 64 ? 64 : tokens <= 128 ? 128 : 256; }

mllm_status validate_mlin(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats, mllm_nm nm,
                          int32_t tokens, unsigned need, bool fwd) {
    mllm_status s = validate_mats(mats, n_mats, nm, need);
    if (s != MLLM_OK) return s;
    if (nm.m != 4) return MLLM_ERR_UNSUPPORTED;
    // the forward's tokens are one MMA's N; the backward's are the MMA's K, in 64-token stages
    if (!io || tokens < 1 || tokens > (fwd ? mlin::kMaxTokens : mlin::kMaxBwdTokens)) return MLLM_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_mats; ++i) {
        const mllm_matrix &a = mats[i];
        if (a.w_dtype != MLLM_BF16) return MLLM_ERR_UNSUPPORTED;
        if (a.cols % mlin::kChunk) return MLLM_ERR_UNSUPPORTED;
        if (a.rows > INT32_MAX || a.cols > INT32_MAX) return MLLM_ERR_INVALID_ARG;
        const bool any = a.rows > 0 && a.cols > 0;
        if ((s = check_ptr(io[i].x, any)) != MLLM_OK) return s;
        if ((s = check_ptr(fwd ? (const void *)io[i].y : io[i].dy, any)) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

// The call's matrices in groups of at most kMaxMats, each with its chunk sequence and the
// activations' tensor maps (box 64 columns x N tokens, 128-byte swizzle). False if a map
// cannot be encoded.
bool mlin_groups(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats, int32_t tokens, int N,
                 std::vector<mlin::Group> *out) {
    for (int32_t i0 = 0; i0 < n_mats; i0 += kMaxMats) {
        mlin::Group g{};
        g.tokens = tokens;
        int64_t acc = 0;
        int32_t k = 0;
        for (int32_t i = i0; i < std::min<int32_t>(n_mats, i0 + kMaxMats); ++i) {
            const mllm_matrix &a = mats[i];
            if (a.rows == 0 || a.cols == 0) continue;
            mlin::Op &d = g.d[k];
            d.W = a.W; d.pi = a.logits; d.m = a.adam_m; d.v = a.adam_v;
            d.y = io[i].y; d.X = a.X_out; d.soft = a.soft_mask_out; d.grad = a.grad_logits_out;
            d.gid0 = a.block_offset;
            d.rows = a.rows; d.cols = a.cols;
            d.nch = a.cols / mlin::kChunk;
            d.ntiles = (a.rows + mlin::kRows - 1) / mlin::kRows;
            d.chunk_begin = acc;
            acc += d.nch * d.ntiles;
            if (!encode_2d(&g.x[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, io[i].x, (uint64_t)a.cols, (uint64_t)tokens,
                           2 * (uint64_t)a.cols, 64, (uint32_t)N, CU_TENSOR_MAP_SWIZZLE_128B))
                return false;
            ++k;
        }
        g.n = k;
        g.total_chunks = acc;
        if (k > 0) out->push_back(g);
    }
    return true;
}

template <int kN>
mllm_status launch_mlin_fwd(const mlin::Group &g, const StepScalars &sc, unsigned char *ws, double *reg,
                            int accumulate, cudaStream_t st) {
    auto fn = mlin::masked_linear_fwd_kernel<kN>;
    constexpr int smem = mlin::smem_bytes<kN>();
    int dev = 0;
    cudaGetDevice(&dev);
    resident_ctas(dev, (const void *)fn, mlin::kThreads, smem);  // sets the dynamic shared-memory limit
    const int64_t grid = std::min<int64_t>({(int64_t)sm_count(dev), g.total_chunks, (int64_t)mlin::kMaxCtas});
    fn<<<(unsigned)grid, mlin::kThreads, smem, st>>>(g, sc, ws, reg, accumulate);
    return cuda_status(cudaGetLastError());
}

bool mlin_bwd_groups(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats, int32_t tokens,
                     std::vector<mlin::BwdGroup> *out) {
    for (int32_t i0 = 0; i0 < n_mats; i0 += kMaxMats) {
        mlin::BwdGroup g{};
        g.tokens = tokens;
        int64_t acc = 0;
        int32_t k = 0;
        for (int32_t i = i0; i < std::min<int32_t>(n_mats, i0 + kMaxMats); ++i) {
            const mllm_matrix &a = mats[i];
            if (a.rows == 0 || a.cols == 0) continue;
            mlin::Op &d = g.d[k];
            d.W = a.W; d.pi = a.logits; d.m = a.adam_m; d.v = a.adam_v; d.grad = a.grad_logits_out;
            d.gid0 = a.block_offset;
            d.rows = a.rows; d.cols = a.cols;
            g.ctiles[k] = (a.cols + mlin::kBwdCols - 1) / mlin::kBwdCols;
            g.tile_begin[k] = acc;
            acc += g.ctiles[k] * ((a.rows + mlin::kRows - 1) / mlin::kRows);
            if (!encode_2d(&g.dy[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, io[i].dy, (uint64_t)a.rows, (uint64_t)tokens,
                           2 * (uint64_t)a.rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
                !encode_2d(&g.x[k], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, io[i].x, (uint64_t)a.cols, (uint64_t)tokens,
                           2 * (uint64_t)a.cols, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
                return false;
            ++k;
        }
        g.n = k;
        g.total_tiles = acc;
        if (k > 0) out->push_back(g);
    }
    return true;
}

}  // namespace
}  // namespace mllm

using namespace mllm;

extern "C" {

int32_t mllm_num_candidates(mllm_nm nm) { return num_cand(nm); }

size_t mllm_workspace_bytes(void) { return kWorkspaceBytes; }

mllm_status mllm_noise_table(float *c_out, float *t_out) {
    if (!c_out || !t_out) return MLLM_ERR_INVALID_ARG;
    static constexpr NoiseTable tab{};  // the same compile-time table as g_noise_table
    constexpr int row0 = -kNlogEmin;    // e = 0, where the stored c_j 2^-e is c_j itself
    for (int row = 0; row < kNlogRows; ++row)
        for (int jr = 0; jr < 128; ++jr) {
            const int j = jr ^ 64;
            if (row == row0) c_out[j] = tab.cT[row * 128 + jr].x;
            t_out[row * 128 + j] = tab.cT[row * 128 + jr].y;
        }
    return MLLM_OK;
}

int32_t mllm_abi_version(void) { return MLLM_ABI_VERSION; }
size_t mllm_sizeof_matrix(void) { return sizeof(mllm_matrix); }
size_t mllm_sizeof_hparams(void) { return sizeof(mllm_hparams); }
int32_t mllm_last_cuda_error(void) { return g_last_cuda; }

const char *mllm_status_string(mllm_status s) {
    switch (s) {
        case MLLM_OK: return "ok";
        case MLLM_ERR_INVALID_ARG: return "invalid argument";
        case MLLM_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
        case MLLM_ERR_UNSUPPORTED: return "unsupported N:M pattern or dtype";
        case MLLM_ERR_WORKSPACE: return "workspace missing or too small";
        case MLLM_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

mllm_status mllm_prior_init(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, float alpha,
                            float init_std, uint64_t seed, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedPi);
    if (s != MLLM_OK) return s;
    if (!finite(alpha) || alpha < 0.f || !finite(init_std) || init_std < 0.f) return MLLM_ERR_INVALID_ARG;
    return launch_prior<false>(mats, n_mats, nm, nullptr, alpha, init_std, seed, stream);
}

mllm_status mllm_prior_init_from_mask(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                      const uint8_t *const *prior_idx, float alpha, float init_std,
                                      uint64_t seed, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedPi);
    if (s != MLLM_OK) return s;
    if (!finite(alpha) || alpha < 0.f || !finite(init_std) || init_std < 0.f) return MLLM_ERR_INVALID_ARG;
    if (!prior_idx) return MLLM_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_mats; ++i) {
        const bool any = mats[i].rows > 0 && mats[i].cols > 0;
        if ((s = check_ptr(prior_idx[i], any)) != MLLM_OK) return s;
    }
    return launch_prior<true>(mats, n_mats, nm, prior_idx, alpha, init_std, seed, stream);
}

mllm_status mllm_sample_fwd(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                            const mllm_hparams *hp, double *reg_sum_out, void *workspace,
                            size_t workspace_bytes, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedX | kNeedPi);
    if (s != MLLM_OK) return s;
    if ((s = validate_fwd_hp(hp)) != MLLM_OK) return s;
    if (reg_sum_out) {
        if ((reinterpret_cast<uintptr_t>(reg_sum_out) & 7u) != 0) return MLLM_ERR_MISALIGNED;
        if (!workspace || workspace_bytes < kWorkspaceBytes) return MLLM_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StepScalars sc = make_scalars(*hp);
    const bool w32 = mats[0].w_dtype == MLLM_F32;
    const bool is24 = nm.m == 4;
    unsigned int *ticket = reg_sum_out ? static_cast<unsigned int *>(workspace) : nullptr;
    double *partials = reg_sum_out ? reinterpret_cast<double *>(static_cast<char *>(workspace) + kWsPartialsOffset) : nullptr;
    bool wrote_reg = false;
    for (const Group &g : make_groups(mats, n_mats, nm.m, is24 ? Kind::Sample24 : Kind::Sample48)) {
        if (g.total_work == 0) continue;
        const int accumulate = wrote_reg ? 1 : 0;
        if (is24) {
            const void *fn = w32 ? (const void *)k24::fwd_kernel<true> : (const void *)k24::fwd_kernel<false>;
            const int64_t grid = grid_for(fn, kThreads, 0, g.total_work, kMaxReduceCtas);
            if (w32) k24::fwd_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
            else k24::fwd_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
        } else {
            const void *fn = w32 ? (const void *)k48::fwd_kernel<true> : (const void *)k48::fwd_kernel<false>;
            const int64_t grid = grid_for(fn, k48::kFwdThreads, k48::kFwdDynSmem, k48_fwd_ctas(g), kMaxReduceCtas);
            if (w32) k48::fwd_kernel<true><<<(unsigned)grid, k48::kFwdThreads, k48::kFwdDynSmem, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
            else k48::fwd_kernel<false><<<(unsigned)grid, k48::kFwdThreads, k48::kFwdDynSmem, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
        }
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
        wrote_reg = true;
    }
    if (reg_sum_out && !wrote_reg) {
        if ((s = cuda_status(cudaMemsetAsync(reg_sum_out, 0, sizeof(double), st))) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_sample_fwd_noalloc(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                    const mllm_hparams *hp, double *reg_sum_out, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedX | kNeedPi);
    if (s != MLLM_OK) return s;
    if ((s = validate_fwd_hp(hp)) != MLLM_OK) return s;
    if (!reg_sum_out) return MLLM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(reg_sum_out) & 7u) != 0) return MLLM_ERR_MISALIGNED;
    const bool w32 = mats[0].w_dtype == MLLM_F32;
    const bool is24 = nm.m == 4;
    const void *fn = is24 ? (w32 ? (const void *)k24::fwd_kernel<true> : (const void *)k24::fwd_kernel<false>)
                          : (w32 ? (const void *)k48::fwd_kernel<true> : (const void *)k48::fwd_kernel<false>);
    const int threads = is24 ? kThreads : k48::kFwdThreads;
    const int dyn_smem = is24 ? 0 : k48::kFwdDynSmem;
    auto ctas_wanted = [&](const Group &g) { return is24 ? g.total_work : k48_fwd_ctas(g); };
    const std::vector<Group> groups = make_groups(mats, n_mats, nm.m, is24 ? Kind::Sample24 : Kind::Sample48);
    // every launch's scratch need (one partial per CTA) is checked before anything runs
    for (const Group &g : groups) {
        if (g.total_work == 0) continue;
        if (grid_for(fn, threads, dyn_smem, ctas_wanted(g), kMaxReduceCtas) > kNoallocMaxCtas) return MLLM_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != MLLM_OK) return s;
    unsigned int *ticket = static_cast<unsigned int *>(scratch);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(scratch) + kWsPartialsOffset);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StepScalars sc = make_scalars(*hp);
    bool wrote_reg = false;
    for (const Group &g : groups) {
        if (g.total_work == 0) continue;
        if ((s = cuda_status(cudaMemsetAsync(ticket, 0, sizeof(unsigned int), st))) != MLLM_OK) return s;
        const int accumulate = wrote_reg ? 1 : 0;
        const int64_t grid = grid_for(fn, threads, dyn_smem, ctas_wanted(g), kMaxReduceCtas);
        if (is24) {
            if (w32) k24::fwd_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
            else k24::fwd_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
        } else {
            if (w32) k48::fwd_kernel<true><<<(unsigned)grid, k48::kFwdThreads, k48::kFwdDynSmem, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
            else k48::fwd_kernel<false><<<(unsigned)grid, k48::kFwdThreads, k48::kFwdDynSmem, st>>>(g, sc, partials, ticket, reg_sum_out, accumulate);
        }
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
        wrote_reg = true;
    }
    if (!wrote_reg) {
        if ((s = cuda_status(cudaMemsetAsync(reg_sum_out, 0, sizeof(double), st))) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_sample_bwd_adam(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                 const mllm_hparams *hp, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedG | kNeedPi | kNeedMV);
    if (s != MLLM_OK) return s;
    if ((s = validate_bwd_hp(hp)) != MLLM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StepScalars sc = make_scalars(*hp);
    const bool w32 = mats[0].w_dtype == MLLM_F32, g32 = mats[0].g_dtype == MLLM_F32;
    const bool is24 = nm.m == 4;
    for (const Group &g : make_groups(mats, n_mats, nm.m, is24 ? Kind::Sample24 : Kind::Sample48)) {
        if (g.total_work == 0) continue;
#define MLLM_LAUNCH_BWD(NS, THREADS, SMEM, W32, G32)                                              \
    do {                                                                                         \
        const void *fn = (const void *)NS::bwd_adam_kernel<W32, G32>;                            \
        const int64_t grid = grid_for(fn, THREADS, SMEM, g.total_work, INT32_MAX);                 \
        NS::bwd_adam_kernel<W32, G32><<<(unsigned)grid, THREADS, SMEM, st>>>(g, sc); \
    } while (0)
        if (is24) {
            if (w32 && g32) MLLM_LAUNCH_BWD(k24, kThreads, 0, true, true);
            else if (w32) MLLM_LAUNCH_BWD(k24, kThreads, 0, true, false);
            else if (g32) MLLM_LAUNCH_BWD(k24, kThreads, 0, false, true);
            else MLLM_LAUNCH_BWD(k24, kThreads, 0, false, false);
        } else {
            if (w32 && g32) MLLM_LAUNCH_BWD(k48, k48::kCtaThreads, k48::kBwdDynSmem, true, true);
            else if (w32) MLLM_LAUNCH_BWD(k48, k48::kCtaThreads, k48::kBwdDynSmem, true, false);
            else if (g32) MLLM_LAUNCH_BWD(k48, k48::kCtaThreads, k48::kBwdDynSmem, false, true);
            else MLLM_LAUNCH_BWD(k48, k48::kCtaThreads, k48::kBwdDynSmem, false, false);
        }
#undef MLLM_LAUNCH_BWD
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_sample_bwd_adam_fwd(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                     const mllm_hparams *hp, const mllm_hparams *hp_next,
                                     double *reg_sum_out, void *workspace, size_t workspace_bytes,
                                     void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedX | kNeedG | kNeedPi | kNeedMV);
    if (s != MLLM_OK) return s;
    if ((s = validate_bwd_hp(hp)) != MLLM_OK) return s;
    if ((s = validate_fwd_hp(hp_next)) != MLLM_OK) return s;
    if (reg_sum_out) {
        if ((reinterpret_cast<uintptr_t>(reg_sum_out) & 7u) != 0) return MLLM_ERR_MISALIGNED;
        if (!workspace || workspace_bytes < kWorkspaceBytes) return MLLM_ERR_WORKSPACE;
        if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StepScalars sb = make_scalars(*hp), sf = make_scalars(*hp_next);
    const bool w32 = mats[0].w_dtype == MLLM_F32, g32 = mats[0].g_dtype == MLLM_F32;
    const bool is24 = nm.m == 4;
    unsigned int *ticket = reg_sum_out ? static_cast<unsigned int *>(workspace) : nullptr;
    double *partials = reg_sum_out ? reinterpret_cast<double *>(static_cast<char *>(workspace) + kWsPartialsOffset) : nullptr;
    bool wrote_reg = false;
    for (const Group &g : make_groups(mats, n_mats, nm.m, is24 ? Kind::Sample24 : Kind::Sample48)) {
        if (g.total_work == 0) continue;
        const int accumulate = wrote_reg ? 1 : 0;
#define MLLM_LAUNCH_FUSED(NS, THREADS, SMEM, W32, G32)                                                 \
    do {                                                                                                 \
        const void *fn = (const void *)NS::bwd_adam_fwd_kernel<W32, G32>;                                \
        const int64_t grid = grid_for(fn, THREADS, SMEM, g.total_work, kMaxReduceCtas);                   \
        NS::bwd_adam_fwd_kernel<W32, G32><<<(unsigned)grid, THREADS, SMEM, st>>>(g, sb, sf, partials, ticket, \
                                                                               reg_sum_out, accumulate); \
    } while (0)
        if (is24) {
            if (w32 && g32) MLLM_LAUNCH_FUSED(k24, kThreads, 0, true, true);
            else if (w32) MLLM_LAUNCH_FUSED(k24, kThreads, 0, true, false);
            else if (g32) MLLM_LAUNCH_FUSED(k24, kThreads, 0, false, true);
            else MLLM_LAUNCH_FUSED(k24, kThreads, 0, false, false);
        } else {
            if (w32 && g32) MLLM_LAUNCH_FUSED(k48, k48::kCtaThreads, k48::kStepDynSmem, true, true);
            else if (w32) MLLM_LAUNCH_FUSED(k48, k48::kCtaThreads, k48::kStepDynSmem, true, false);
            else if (g32) MLLM_LAUNCH_FUSED(k48, k48::kCtaThreads, k48::kStepDynSmem, false, true);
            else MLLM_LAUNCH_FUSED(k48, k48::kCtaThreads, k48::kStepDynSmem, false, false);
        }
#undef MLLM_LAUNCH_FUSED
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
        wrote_reg = true;
    }
    if (reg_sum_out && !wrote_reg) {
        if ((s = cuda_status(cudaMemsetAsync(reg_sum_out, 0, sizeof(double), st))) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_hard_pack(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedPi | kNeedPack);
    if (s != MLLM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool w32 = mats[0].w_dtype == MLLM_F32;
    const bool is24 = nm.m == 4;
    // 2:4 rows of whole metadata words (cols % 32 == 0, every LLM shape) take the pair kernel
    bool words_aligned = true;
    for (int32_t i = 0; i < n_mats; ++i) words_aligned = words_aligned && ((mats[i].cols / 4) % 8 == 0);
    if (is24 && words_aligned) {
        for (const Group &g : make_groups(mats, n_mats, nm.m, Kind::Sample24)) {
            if (g.total_work == 0) continue;
            const void *fn = w32 ? (const void *)k24::pack_pairs_kernel<true> : (const void *)k24::pack_pairs_kernel<false>;
            const int64_t grid = grid_for(fn, kThreads, 0, g.total_work, INT32_MAX);
            if (w32) k24::pack_pairs_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(g);
            else k24::pack_pairs_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(g);
            if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
        }
        return MLLM_OK;
    }
    for (const Group &g : make_groups(mats, n_mats, nm.m, is24 ? Kind::Pack24 : Kind::Pack48)) {
        if (g.total_work == 0) continue;
        if (is24) {
            const void *fn = w32 ? (const void *)k24::pack_kernel<true> : (const void *)k24::pack_kernel<false>;
            const int64_t grid = grid_for(fn, kThreads, 0, g.total_work, INT32_MAX);
            if (w32) k24::pack_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(g);
            else k24::pack_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(g);
        } else {
            const void *fn = w32 ? (const void *)k48::pack_kernel<true> : (const void *)k48::pack_kernel<false>;
            const int64_t grid = grid_for(fn, k48::kCtaThreads, 0, g.total_work, INT32_MAX);
            if (w32) k48::pack_kernel<true><<<(unsigned)grid, k48::kCtaThreads, 0, st>>>(g);
            else k48::pack_kernel<false><<<(unsigned)grid, k48::kCtaThreads, 0, st>>>(g);
        }
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_mask_diff(const uint8_t *a, const uint8_t *b, int64_t n, unsigned long long *count_out,
                           void *stream) {
    if (n < 0) return MLLM_ERR_INVALID_ARG;
    mllm_status s;
    if ((s = check_ptr(count_out, true)) != MLLM_OK) return s;
    if ((s = check_ptr(a, n > 0)) != MLLM_OK) return s;
    if ((s = check_ptr(b, n > 0)) != MLLM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = cuda_status(cudaMemsetAsync(count_out, 0, sizeof(unsigned long long), st))) != MLLM_OK) return s;
    if (n == 0) return MLLM_OK;
    const int64_t grid = grid_for((const void *)diag::mask_diff_kernel, kThreads, 0,
                                  (n / 16 + kThreads - 1) / kThreads + 1, INT32_MAX);
    diag::mask_diff_kernel<<<(unsigned)grid, kThreads, 0, st>>>(a, b, n, count_out);
    return cuda_status(cudaGetLastError());
}

mllm_status mllm_mask_stats(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, float kappa, double *out,
                            void *workspace, size_t workspace_bytes, void *stream) {
    mllm_status s = validate_mats(mats, n_mats, nm, kNeedW | kNeedPi);
    if (s != MLLM_OK) return s;
    if (!finite(kappa) || !(kappa > 0.f)) return MLLM_ERR_INVALID_ARG;
    if ((s = check_ptr(out, true)) != MLLM_OK) return s;
    if (!workspace || workspace_bytes < kWorkspaceBytes) return MLLM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    if (n_mats > kMaxMats) return MLLM_ERR_UNSUPPORTED;  // one launch: one deterministic sum
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool w32 = mats[0].w_dtype == MLLM_F32, is24 = nm.m == 4;
    Group g = make_groups(mats, n_mats, nm.m, Kind::Sample24)[0];
    if (!is24) {  // 4:8: one block per thread
        int64_t acc = 0;
        for (int32_t i = 0; i < g.n; ++i) {
            g.d[i].work_begin = acc;
            g.d[i].work_count = (g.d[i].nblocks + kThreads - 1) / kThreads;
            acc += g.d[i].work_count;
        }
        g.total_work = acc;
    }
    if (g.total_work == 0) return cuda_status(cudaMemsetAsync(out, 0, 4 * sizeof(double), st));
    unsigned int *ticket = static_cast<unsigned int *>(workspace);
    double *partials = reinterpret_cast<double *>(static_cast<char *>(workspace) + kWsPartialsOffset);
    const void *fn = is24 ? (w32 ? (const void *)diag::stats24_kernel<true> : (const void *)diag::stats24_kernel<false>)
                          : (w32 ? (const void *)diag::stats48_kernel<true> : (const void *)diag::stats48_kernel<false>);
    const int64_t grid = grid_for(fn, kThreads, 0, g.total_work, diag::kMaxStatCtas);
    if (is24) {
        if (w32) diag::stats24_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(g, kappa, partials, ticket, out);
        else diag::stats24_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(g, kappa, partials, ticket, out);
    } else {
        if (w32) diag::stats48_kernel<true><<<(unsigned)grid, kThreads, 0, st>>>(g, kappa, partials, ticket, out);
        else diag::stats48_kernel<false><<<(unsigned)grid, kThreads, 0, st>>>(g, kappa, partials, ticket, out);
    }
    return cuda_status(cudaGetLastError());
}

static mllm_status codec_args(mllm_nm nm, const void *src, const void *dst, int64_t n, int *C, int *D) {
    *C = num_cand(nm);
    if (!*C) return MLLM_ERR_UNSUPPORTED;
    *D = (nm.m == 4) ? 12 : 5;
    if (n < 0) return MLLM_ERR_INVALID_ARG;
    mllm_status s;
    if ((s = check_ptr(src, n > 0)) != MLLM_OK) return s;
    return check_ptr(dst, n > 0);
}

// The codec's vector kernels read or write the indices as 32-bit (D % 4 == 0: 16-byte) words
// and the code as 16-byte vectors (the entry points' pointer checks already ask for 16-byte
// alignment; this keeps the kernels' own requirement next to them).
static bool codec_vector_ok(const void *idx, const void *words, int D) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(idx), b = reinterpret_cast<uintptr_t>(words);
    return (b & 15u) == 0 && (a & ((D % 4 == 0) ? 15u : 3u)) == 0;
}

mllm_status mllm_encode_candidates(mllm_nm nm, const uint8_t *idx, int64_t n, uint32_t *words, void *stream) {
    int C, D;
    mllm_status s = codec_args(nm, idx, words, n, &C, &D);
    if (s != MLLM_OK || n == 0) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t w = (n + D - 1) / D;
    // whole groups of 4 words with vector accesses where the pointers allow, the rest word by word
    const int64_t groups = codec_vector_ok(idx, words, D) ? n / (4 * (int64_t)D) : 0;
    if (groups > 0) {
        const int64_t grid = std::min<int64_t>((groups + kThreads - 1) / kThreads, 65535 * 16);
        if (C == 6) diag::encode4_kernel<6, 12><<<(unsigned)grid, kThreads, 0, st>>>(idx, groups, words);
        else diag::encode4_kernel<70, 5><<<(unsigned)grid, kThreads, 0, st>>>(idx, groups, words);
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
    }
    if (4 * groups < w) {
        const int64_t grid = std::min<int64_t>((w - 4 * groups + kThreads - 1) / kThreads, 65535 * 16);
        diag::encode_kernel<<<(unsigned)grid, kThreads, 0, st>>>(idx, n, C, D, words, 4 * groups);
    }
    return cuda_status(cudaGetLastError());
}

mllm_status mllm_decode_candidates(mllm_nm nm, const uint32_t *words, int64_t n, uint8_t *idx, void *stream) {
    int C, D;
    mllm_status s = codec_args(nm, words, idx, n, &C, &D);
    if (s != MLLM_OK || n == 0) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t w = (n + D - 1) / D;
    const int64_t groups = codec_vector_ok(idx, words, D) ? n / (4 * (int64_t)D) : 0;
    if (groups > 0) {
        const int64_t grid = std::min<int64_t>((groups + kThreads - 1) / kThreads, 65535 * 16);
        if (C == 6) diag::decode4_kernel<6, 12><<<(unsigned)grid, kThreads, 0, st>>>(words, groups, idx);
        else diag::decode4_kernel<70, 5><<<(unsigned)grid, kThreads, 0, st>>>(words, groups, idx);
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
    }
    if (4 * groups < w) {
        const int64_t grid = std::min<int64_t>((w - 4 * groups + kThreads - 1) / kThreads, 65535 * 16);
        diag::decode_kernel<<<(unsigned)grid, kThreads, 0, st>>>(words, n, C, D, idx, 4 * groups);
    }
    return cuda_status(cudaGetLastError());
}

mllm_status mllm_sparse_linear(const mllm_sparse_operand *ops, int32_t n_ops, mllm_nm nm, int32_t tokens,
                               void *workspace, size_t workspace_bytes, void *stream) {
    mllm_status s = validate_operands(ops, n_ops, nm, tokens);
    if (s != MLLM_OK) return s;
    if (!workspace || workspace_bytes < spl::kSkWorkspaceBytes) return MLLM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *part = static_cast<float *>(workspace);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(static_cast<char *>(workspace) + spl::kPartBytes);
    unsigned int *err = tickets + spl::kMaxSkWarps;
    std::vector<mllm_sparse_operand> act, batched;
    for (int32_t i = 0; i < n_ops; ++i) {
        if (ops[i].rows == 0) continue;
        if (ops[i].cols == 0) {  // y = 0
            s = cuda_status(cudaMemsetAsync(ops[i].y, 0, sizeof(float) * (size_t)tokens * (size_t)ops[i].rows, st));
            if (s != MLLM_OK) return s;
            continue;
        }
        // the tensor-memory kernels: 2:4 above 16 tokens, 4:8 (expanded to dense) at any count
        if (ops[i].cols % spl::kTmChunk == 0 && (tokens > spl::kMaxTileTokens || nm.m == 8)) batched.push_back(ops[i]);
        else act.push_back(ops[i]);
    }
    if (tokens > spl::kMaxTokens) {
        // prefill-sized calls: on the prefill kernels (2:4 sparse MMA, 4:8 expanded once per
        // stage for 256 tokens); if a tensor map cannot be encoded, 4:8 through the batched
        // kernel in groups of 64 tokens (x and y rows offset)
        bool grouped = false;
        if (!batched.empty() && nm.m == 4) {
            if (!sparse_linear_prefill(batched, tokens, err, st, &s)) act.insert(act.end(), batched.begin(), batched.end());
            if (s != MLLM_OK) return s;
        } else if (!batched.empty()) {
            grouped = !sparse_linear_prefill48(batched, tokens, err, st, &s);
            if (s != MLLM_OK) return s;
        }
        if (grouped) {
            for (int32_t t0 = 0; t0 < tokens; t0 += spl::kMaxTokens) {
                std::vector<mllm_sparse_operand> grp = batched;
                for (mllm_sparse_operand &o : grp) {
                    o.x = static_cast<const char *>(o.x) + (size_t)t0 * (size_t)o.cols * 2;
                    o.y = o.y + (size_t)t0 * (size_t)o.rows;
                }
                if (!sparse_linear_batched(grp, nm, std::min<int32_t>(spl::kMaxTokens, tokens - t0), part, tickets, err,
                                           st, &s)) {
                    act.insert(act.end(), batched.begin(), batched.end());
                    break;
                }
                if (s != MLLM_OK) return s;
            }
        }
    } else if (!batched.empty() && !sparse_linear_batched(batched, nm, tokens, part, tickets, err, st, &s)) {
        act.insert(act.end(), batched.begin(), batched.end());  // maps not encodable: token groups
    }
    if (s != MLLM_OK) return s;
    if (act.empty()) return MLLM_OK;
    if (tokens <= spl::kMaxTileTokens) return sparse_linear_small(act, nm, tokens, part, tickets, err, st);
    // more tokens than the per-warp kernels take: groups of 16 tokens (x and y rows offset)
    for (int32_t t0 = 0; t0 < tokens; t0 += spl::kMaxTileTokens) {
        std::vector<mllm_sparse_operand> grp = act;
        for (mllm_sparse_operand &o : grp) {
            o.x = static_cast<const char *>(o.x) + (size_t)t0 * (size_t)o.cols * 2;
            o.y = o.y + (size_t)t0 * (size_t)o.rows;
        }
        s = sparse_linear_small(grp, nm, std::min<int32_t>(spl::kMaxTileTokens, tokens - t0), part, tickets, err, st);
        if (s != MLLM_OK) return s;
    }
    return MLLM_OK;
}

size_t mllm_sparse_linear_workspace_bytes(void) { return spl::kSkWorkspaceBytes; }

mllm_status mllm_sparse_linear_check_timeout(const mllm_sparse_operand *op, mllm_nm nm, int32_t tokens,
                                             void *workspace, size_t workspace_bytes, void *stream) {
    mllm_status s = validate_operands(op, 1, nm, tokens);
    if (s != MLLM_OK) return s;
    if (!workspace || workspace_bytes < spl::kSkWorkspaceBytes) return MLLM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    if (op->rows == 0 || op->cols == 0 || op->cols % spl::kTmChunk || tokens > spl::kMaxTokens)
        return MLLM_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *part = static_cast<float *>(workspace);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(static_cast<char *>(workspace) + spl::kPartBytes);
    unsigned int *err = tickets + spl::kMaxSkWarps;
    if (tokens > spl::kMaxTileTokens || nm.m == 8) {  // the tensor-memory kernel
        const std::vector<mllm_sparse_operand> ops(1, *op);
        if (!sparse_linear_batched(ops, nm, tokens, part, tickets, err, st, &s, 1)) return MLLM_ERR_UNSUPPORTED;
        return s;
    }
    static thread_local spl::TmGroup tg;
    tg.g = spl::SkGroup{};
    tg.g.tokens = tokens;
    spl::SkOp &d = tg.g.d[0];
    d.vals = static_cast<const uint32_t *>(op->pack_values);
    d.meta = op->pack_meta;
    d.x = static_cast<const uint32_t *>(op->x);
    d.y = op->y;
    d.rows = op->rows;
    d.cols = op->cols;
    d.nch = op->cols / spl::kTmChunk;
    d.ntiles = (op->rows + spl::kSkRows - 1) / spl::kSkRows;
    d.chunk_begin = 0;
    tg.g.n = 1;
    tg.g.total_chunks = d.nch * d.ntiles;
    const int nt = tokens > 8 ? 2 : 1;  // 2:4 up to 16 tokens: the per-warp kernel
    if (!encode_operand(&tg.maps[0], *op, tokens, nt)) return MLLM_ERR_UNSUPPORTED;
    return nt == 2 ? launch_spl_tma<2>(tg, part, tickets, err, st, 1) : launch_spl_tma<1>(tg, part, tickets, err, st, 1);
}

size_t mllm_sizeof_sparse_operand(void) { return sizeof(mllm_sparse_operand); }
size_t mllm_sizeof_linear_io(void) { return sizeof(mllm_linear_io); }

size_t mllm_masked_linear_workspace_bytes(void) { return mlin::kWorkspaceBytes; }

mllm_status mllm_masked_linear_bwd_adam(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats,
                                        mllm_nm nm, int32_t tokens, const mllm_hparams *hp, void *workspace,
                                        size_t workspace_bytes, void *stream) {
    mllm_status s = validate_mlin(mats, io, n_mats, nm, tokens, kNeedW | kNeedPi | kNeedMV, false);
    if (s != MLLM_OK) return s;
    if ((s = validate_bwd_hp(hp)) != MLLM_OK) return s;
    for (int32_t i = 0; i < n_mats; ++i)
        if (mats[i].rows % 8) return MLLM_ERR_UNSUPPORTED;  // dY rows are whole 16-byte units
    if (!workspace || workspace_bytes < mlin::kWorkspaceBytes) return MLLM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    std::vector<mlin::BwdGroup> groups;
    if (!mlin_bwd_groups(mats, io, n_mats, tokens, &groups)) return MLLM_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StepScalars sc = make_scalars(*hp);
    auto fn = mlin::masked_linear_bwd_adam_kernel;
    int dev = 0;
    cudaGetDevice(&dev);
    resident_ctas(dev, (const void *)fn, mlin::kThreads, mlin::kBwdSmem);  // sets the dynamic shared-memory limit
    for (const mlin::BwdGroup &g : groups) {
        const int64_t grid = std::min<int64_t>({(int64_t)sm_count(dev), g.total_tiles, (int64_t)mlin::kMaxCtas});
        fn<<<(unsigned)grid, mlin::kThreads, mlin::kBwdSmem, st>>>(g, sc, static_cast<unsigned char *>(workspace));
        if ((s = cuda_status(cudaGetLastError())) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_masked_linear_fwd(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats, mllm_nm nm,
                                   int32_t tokens, const mllm_hparams *hp, double *reg_sum_out, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    mllm_status s = validate_mlin(mats, io, n_mats, nm, tokens, kNeedW | kNeedPi, true);
    if (s != MLLM_OK) return s;
    if ((s = validate_fwd_hp(hp)) != MLLM_OK) return s;
    if (reg_sum_out && (reinterpret_cast<uintptr_t>(reg_sum_out) & 7u) != 0) return MLLM_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < mlin::kWorkspaceBytes) return MLLM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MLLM_ERR_MISALIGNED;
    const int N = mlin_n(tokens);
    std::vector<mlin::Group> groups;
    if (!mlin_groups(mats, io, n_mats, tokens, N, &groups)) return MLLM_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const StepScalars sc = make_scalars(*hp);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    bool wrote_reg = false;
    for (const mlin::Group &g : groups) {
        const int accumulate = wrote_reg ? 1 : 0;
        s = N == 32    ? launch_mlin_fwd<32>(g, sc, ws, reg_sum_out, accumulate, st)
            : N == 64  ? launch_mlin_fwd<64>(g, sc, ws, reg_sum_out, accumulate, st)
            : N == 128 ? launch_mlin_fwd<128>(g, sc, ws, reg_sum_out, accumulate, st)
                       : launch_mlin_fwd<256>(g, sc, ws, reg_sum_out, accumulate, st);
        if (s != MLLM_OK) return s;
        wrote_reg = true;
    }
    if (reg_sum_out && !wrote_reg) {
        if ((s = cuda_status(cudaMemsetAsync(reg_sum_out, 0, sizeof(double), st))) != MLLM_OK) return s;
    }
    return MLLM_OK;
}

mllm_status mllm_noise(mllm_nm nm, uint64_t seed, uint32_t step, const uint64_t *gids,
                       int64_t n_blocks, float *g_out, void *stream) {
    const int C = num_cand(nm);
    if (!C) return MLLM_ERR_UNSUPPORTED;
    if (n_blocks < 0) return MLLM_ERR_INVALID_ARG;
    if (n_blocks == 0) return MLLM_OK;
    mllm_status s;
    if ((s = check_ptr(gids, true)) != MLLM_OK) return s;
    if ((s = check_ptr(g_out, true)) != MLLM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t grid = std::min<int64_t>((n_blocks + kThreads - 1) / kThreads, INT32_MAX);
    noise_kernel<<<(unsigned)grid, kThreads, 0, st>>>(C, seed, step, gids, n_blocks, g_out);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
