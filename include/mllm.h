/*
 * mllm.h -- C ABI of libmllm, the B200 (sm_100a) implementation of MaskLLM's per-block
 * differentiable N:M mask sampler.
 *
 * Source of the method: "MaskLLM: Learnable Semi-Structured Sparsity for Large Language
 * Models" (arXiv 2409.17481), as summarised on the paper-graph-ui page; sections below are
 * that page's. Every weight matrix is frozen; each block of M consecutive weights along a
 * row carries C = C(M,N) learnable logits, one per candidate N:M mask (s.3.2). One
 * training step calls mllm_sample_fwd for every matrix, the caller's network consumes the
 * soft-masked weights and returns their gradient, then mllm_sample_bwd_adam updates the
 * logits in place (s.3.4, Algorithm 1 step 2). mllm_prior_init runs once before training
 * (Algorithm 1 step 1) and mllm_hard_pack once after it (Algorithm 1 step 3).
 *
 * Conventions shared by every call
 *   Layout. A matrix is row-major [rows, cols] with cols % M == 0. Block b (0-based, in
 *     row-major order) covers elements [b*M, b*M + M) of the flattened matrix, i.e. M
 *     consecutive weights of one row. B = rows*cols/M blocks. Per-block arrays (logits and
 *     the AdamW moments) are row-major [B, C] fp32. The candidate order is fixed:
 *       2:4 (C = 6): [1,1,0,0] [1,0,1,0] [1,0,0,1] [0,1,0,1] [0,1,1,0] [0,0,1,1]
 *                    (the page's listing, s.3.2 Eq.2; 1 = keep);
 *       4:8 (C = 70): the 4-subsets of positions 0..7 in lexicographic order of their
 *                    ascending index tuples, (0,1,2,3), (0,1,2,4), ..., (4,5,6,7).
 *   Ownership. Every pointer inside mllm_matrix, and reg_sum_out / workspace, is device
 *     memory owned by the caller and borrowed for the duration of the enqueued work. The
 *     `mats` and `hp` arrays themselves are host memory, read during the call only. The
 *     library allocates nothing and keeps no state between calls, except the fixed scratch
 *     array of mllm_sample_fwd_noalloc (described there).
 *   Streams. `stream` is a cudaStream_t (NULL = the legacy default stream). All work is
 *     enqueued asynchronously on it; the call returns once enqueued.
 *   Alignment. Every device pointer must be 16-byte aligned (MLLM_ERR_MISALIGNED).
 *   Errors. Arguments are validated on the host before anything is enqueued; on any error
 *     nothing is launched and no output is touched. A failed launch returns MLLM_ERR_CUDA
 *     (mllm_last_cuda_error() gives the cudaError_t). No call waits on the device, so no
 *     call can hang; device-side faults surface at the caller's next synchronisation.
 *   Grouping. `n_mats > 1` processes all matrices of one layer in a single launch; each
 *     matrix keeps its own buffers. Matrices with rows == 0 or cols == 0 are allowed and
 *     contribute nothing.
 *   Random numbers. Noise for candidate c of block b of a matrix at sampling step s comes
 *     from Philox4x32-10 (Salmon et al., SC'11) with key (seed lo32, seed hi32) and counter
 *     (gid lo32, gid hi32, s, c/6), gid = block_offset + b; field c%6 = bits [21(c%6),
 *     21(c%6)+21) of the 128-bit output (word 0 least significant) is k, eps =
 *     (2k+1)*2^-22, and g = -nlog(-nlog(eps)) with nlog the fp32 table-driven logarithm
 *     fixed by the specification (Tang's method: x = 2^e mm, a 7-bit mantissa prefix j,
 *     r = fma(mm, c_j, -1), ln x = T[e][j] + (r - r^2/2 + r^3/3); see mllm_noise_table).
 *     Step 0xFFFFFFFF is reserved for mllm_prior_init. The same (seed, step) gives
 *     bit-identical noise in forward and backward; noise is recomputed, never stored.
 */
#ifndef MLLM_H
#define MLLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLLM_ABI_VERSION 1

typedef enum {
    MLLM_OK = 0,
    MLLM_ERR_INVALID_ARG = 1, /* null pointer, bad size, non-finite or out-of-range scalar */
    MLLM_ERR_MISALIGNED = 2,  /* a device pointer is not 16-byte aligned */
    MLLM_ERR_UNSUPPORTED = 3, /* N:M other than 2:4 or 4:8, or an unsupported dtype */
    MLLM_ERR_WORKSPACE = 4,   /* workspace missing or smaller than mllm_workspace_bytes() */
    MLLM_ERR_CUDA = 5         /* a CUDA launch or runtime call failed */
} mllm_status;

typedef enum {
    MLLM_BF16 = 0, /* bfloat16 */
    MLLM_F32 = 1   /* IEEE binary32 */
} mllm_dtype;

typedef struct {
    int32_t n; /* weights kept per block: 2 or 4 */
    int32_t m; /* block length: 4 or 8 */
} mllm_nm;

/* One frozen weight matrix and its buffers. Fields a call does not use may be NULL. */
typedef struct {
    const void *W;          /* [rows, cols] w_dtype, frozen weights (all calls) */
    void *X_out;            /* [rows, cols] w_dtype, soft-masked weights W . M (fwd) */
    const void *G;          /* [rows, cols] g_dtype, dL/dX from the network (bwd) */
    int32_t w_dtype;        /* mllm_dtype of W and X_out */
    int32_t g_dtype;        /* mllm_dtype of G */
    int64_t rows, cols;     /* cols % M == 0 */
    float *logits;          /* [B, C] fp32 logits pi (init writes; fwd reads; bwd updates) */
    float *adam_m;          /* [B, C] fp32 AdamW first moment (init zeroes; bwd updates) */
    float *adam_v;          /* [B, C] fp32 AdamW second moment (init zeroes; bwd updates) */
    uint64_t block_offset;  /* global id of block 0, the Philox counter base */
    float *soft_mask_out;   /* [rows, cols] fp32 soft mask M (fwd, optional, for inspection) */
    float *grad_logits_out; /* [B, C] fp32 dL/dpi before AdamW (bwd, optional) */
    void *pack_values;      /* [rows, cols*N/M] w_dtype kept weights (pack) */
    void *pack_meta;        /* pack: 2:4 uint32 [rows, ceil(cols/32)]; 4:8 uint16 [rows, cols/8] */
    uint8_t *cand_idx_out;  /* [B] uint8 argmax candidate index (pack, optional) */
} mllm_matrix;

/* Per-step scalars (s.3.4 Table 7 values in brackets; the schedules are the caller's). */
typedef struct {
    float kappa;        /* logit scale, > 0 (100 -> 500 linearly) */
    float tau;          /* Gumbel-softmax temperature, > 0 (4 -> 0.05 linearly) */
    float lambda;       /* sparse-weight regulariser strength, >= 0 (1e-5), Eq.8 */
    float lr;           /* AdamW learning rate, >= 0 (5e-4 LLaMA-2, 1e-3 GPT-3) */
    float beta1, beta2; /* AdamW betas in [0, 1) (0.9, 0.999) */
    float eps;          /* AdamW epsilon, > 0 (1e-8) */
    float weight_decay; /* decoupled weight decay, >= 0 (0.1) */
    uint32_t adam_step; /* 1-based AdamW step t for the bias corrections 1 - beta^t */
    uint32_t step;      /* sampling step s, the Philox counter word 2; != 0xFFFFFFFF */
    uint64_t seed;      /* Philox key */
    int32_t noise_on;   /* 0 replaces the Gumbel noise by zero */
    int32_t reserved;   /* must be 0 */
} mllm_hparams;

/* Number of candidate masks C(M, N) (6 or 70), or 0 if unsupported. */
int32_t mllm_num_candidates(mllm_nm nm);

/* Mask-prior initialisation (s.3.4 "Mask Prior", Eq.9 and Eq.10; Algorithm 1 step 1).
 * Per block: M0 = the N positions of largest |W| (equal magnitudes: lower position first;
 * NaN ranks last); sim_i = M0.S_i - (mean over k of M0.S_k) = M0.S_i - N*N/M;
 * pi0_i = init_std * n_i with n_i standard normal (Box-Muller: candidates 2p and 2p+1 take
 * radius sqrt(-2 ln u_2p) and angle 2*pi*u_(2p+1), u_c the reserved-step uniform of
 * candidate c); pi_i = pi0_i + alpha * sigma * sim_i with sigma the population standard
 * deviation of pi0 over the block's C logits. init_std == 0 selects a deterministic mode
 * (an addition, not on the pages): pi_i = alpha * sim_i, so argmax pi is the prior mask.
 * Writes logits, and zeroes adam_m and adam_v when they are non-NULL.
 * Reads W; needs logits. alpha >= 0 and init_std >= 0, both finite. */
mllm_status mllm_prior_init(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, float alpha,
                            float init_std, uint64_t seed, void *stream);

/* Mask-prior initialisation from a given prior mask (the transfer prior: s.3.4 "Mask
 * Prior" takes M0 from any one-shot method or from a previous MaskLLM run; Table 5's
 * domain-transfer masks start from the general mask). Exactly mllm_prior_init with M0 of
 * block b = candidate prior_idx[i][b] of matrix i instead of the magnitude prior, where
 * prior_idx is a host array of n_mats device pointers to uint8 [B] (for instance the
 * cand_idx_out of an earlier mllm_hard_pack). An index >= C gives that block no prior
 * (sim = 0: pi = pi0, or 0 in the deterministic mode). W is not read. */
mllm_status mllm_prior_init_from_mask(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                      const uint8_t *const *prior_idx, float alpha,
                                      float init_std, uint64_t seed, void *stream);

/* Forward of the sampler (s.3.4 Eq.5-Eq.8, Algorithm 1 lines 1-5). Per block:
 *   w_i = fma(kappa, pi_i, g_i) in fp32 (one rounding); y = softmax(w / tau) (Eq.6);
 *   M_j = sum_i y_i S_ij (Eq.7); X_j = W_j * M_j rounded to nearest-even in w_dtype;
 *   reg += sum_j (W_j M_j)^2 (Eq.8 without lambda, before rounding X).
 * Writes X_out (and soft_mask_out when non-NULL). When reg_sum_out is non-NULL it receives
 * the sum over all blocks of all matrices as one double; this needs a workspace of
 * mllm_workspace_bytes() bytes, zero-filled before its first use (each call leaves it
 * zero-filled when its work completes; calls sharing a workspace must be stream-ordered).
 * The sum is deterministic for a given device. reg_sum_out == NULL skips the reduction and
 * the workspace may be NULL. Reads W, logits. */
mllm_status mllm_sample_fwd(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                            const mllm_hparams *hp, double *reg_sum_out, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Forward for callers that cannot allocate device memory (no counterpart in the paper;
 * an addition of this library). Some callers own no allocator: a plugin whose host
 * framework hands it only the tensors of the step and forbids cudaMalloc/cudaFree after
 * start-up (they synchronise the device and fragment a fixed memory budget), or a runtime
 * that exposes device memory to it only as the call's inputs and outputs. For them the
 * scratch of the regulariser reduction (a ticket word and one double per CTA) lives in a
 * fixed array inside this library instead of the `workspace` argument of mllm_sample_fwd.
 * Semantics, outputs and arguments are otherwise those of mllm_sample_fwd.
 *   Limit: the array holds 2048 per-CTA partial sums (16,400 bytes, 256-byte aligned); a
 *     launch that would need more (a device with more than 2048 resident CTAs of the
 *     kernel) is rejected with MLLM_ERR_WORKSPACE before anything is enqueued.
 *   Set-up: every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress), so an address never outlives a device reset or a context;
 *     the first call on a device may load the library's device code there, so make that
 *     first call before any stream capture. Every GPU that loads the library holds the
 *     array until exit.
 *   Sharing: all calls on a device share the one array and each call clears its ticket
 *     word before launching; calls whose work overlaps on the GPU (different streams
 *     without ordering between them) race on the array and must not be issued.
 *   reg_sum_out must be non-NULL. Nothing is allocated: no cudaMalloc, no cudaFree. */
mllm_status mllm_sample_fwd_noalloc(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                    const mllm_hparams *hp, double *reg_sum_out, void *stream);

/* Backward to the logits fused with AdamW (s.3.2 "Frozen LLM Backbone"; s.3.4 Eq.8 and
 * Algorithm 1 step 2; AdamW as in PyTorch, Loshchilov & Hutter decoupled decay).
 * Recomputes the forward's noise, y and M for the same (seed, step), then per block:
 *   u_j = G_j W_j - 2 lambda W_j^2 M_j                 (dL/dM for L = L_LM - lambda R)
 *   dpi_i = (kappa/tau) y_i sum_j (S_ij - M_j) u_j     (1 - M_j formed as a sum of y)
 *   pi <- pi (1 - lr wd); m <- b1 m + (1-b1) dpi; v <- b2 v + (1-b2) dpi^2;
 *   pi <- pi - lr/(1-b1^t) * m / (sqrt(v)/sqrt(1-b2^t) + eps),  t = adam_step.
 * Updates logits, adam_m, adam_v in place; writes grad_logits_out when non-NULL.
 * Reads W, G. */
mllm_status mllm_sample_bwd_adam(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                 const mllm_hparams *hp, void *stream);

/* Backward + AdamW of step t fused with the forward of step t+1 (an addition of this
 * library, not on the pages). A training step runs the forward of every layer, then the
 * backward in reverse; the next step's forward of a layer needs exactly the logits this
 * step's backward just wrote. This call does, for every block, mllm_sample_bwd_adam with
 * `hp` followed by mllm_sample_fwd with `hp_next` on the updated logits, reading W and the
 * logits once: logits, adam_m, adam_v get step t's update, X_out receives step t+1's
 * soft-masked weights, grad_logits_out (optional) step t's gradient, soft_mask_out
 * (optional) step t+1's soft mask, and reg_sum_out (optional, with the workspace as in
 * mllm_sample_fwd) step t+1's regulariser. A loop then calls mllm_sample_fwd once for the
 * first step and this call for every step after it. Results are identical to the two calls
 * in sequence. One launch per group of matrices for both patterns.
 * Reads W, G. hp is validated as for mllm_sample_bwd_adam, hp_next as for mllm_sample_fwd. */
mllm_status mllm_sample_bwd_adam_fwd(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm,
                                     const mllm_hparams *hp, const mllm_hparams *hp_next,
                                     double *reg_sum_out, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Activations of one matrix's linear layer for the mllm_masked_linear_* calls (device
 * memory, caller-owned, 16-byte aligned). */
typedef struct {
    const void *x;  /* [tokens, cols] bf16: the layer's input A, row-major                  */
    float *y;       /* [tokens, rows] fp32: the layer's output Y = A X^T (forward; overwritten) */
    const void *dy; /* [tokens, rows] bf16: dL/dY, the gradient of the output (backward)     */
} mllm_linear_io;

/* The sampler's forward inside the frozen network's linear layer (s.3.2 "Frozen LLM
 * Backbone": every linear layer multiplies by the soft-masked weight; s.3.4 Eq.5-Eq.8):
 *   Y[t, r] = sum_k A[t, k] X[r, k],  X = W (.) M in bf16, exactly the X of mllm_sample_fwd
 * (same noise, same arithmetic, bit for bit), for 1 <= tokens <= 256, with the products on the
 * tensor cores (bf16 operands, fp32 accumulation). X is made tile by tile in shared memory
 * and never written to global memory (unless X_out is non-NULL, for inspection; soft_mask_out
 * likewise). reg_sum_out (optional) receives the regulariser sum of the call as in
 * mllm_sample_fwd. Matrix i uses io[i]; its W is bf16, cols % 64 == 0; 2:4 only
 * (MLLM_ERR_UNSUPPORTED otherwise). workspace: mllm_masked_linear_workspace_bytes() bytes,
 * zero-filled before its first use; every call leaves it zero-filled (partial tiles of rows
 * split between CTAs, completion tickets, the regulariser's partials and an error word -- the
 * uint32 at byte offset mllm_masked_linear_workspace_bytes() - 16 -- that a call sets if one of
 * its bounded waits ran out, in which case its outputs are invalid; never expected). Calls sharing a workspace must
 * be stream-ordered. Deterministic for a given device. Reads W, logits, x. */
mllm_status mllm_masked_linear_fwd(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats,
                                   mllm_nm nm, int32_t tokens, const mllm_hparams *hp, double *reg_sum_out,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* The weight side of the same layer's backward fused with the logits' backward and AdamW
 * (s.3.2 "Frozen LLM Backbone": the frozen weights take no update, the gradient reaching the
 * soft-masked weight goes to the logits; s.3.4 Eq.8, Algorithm 1 step 2): per matrix
 *   G[r, k] = sum_t dY[t, r] A[t, k]     (dL/dX of Y = A X^T; tensor cores, fp32 accumulation)
 * and then, per block, exactly mllm_sample_bwd_adam with G in fp32 in place of the upstream
 * gradient: the noise of hp's step recomputed, dpi through Eq.7 and Eq.6 with the
 * regulariser's term, AdamW on logits, adam_m, adam_v in place (grad_logits_out receives dpi
 * when non-NULL). G is formed tile by tile in tensor and shared memory and never written to
 * global memory. io[i].x and io[i].dy are the forward's activations and dL/dY; 1 <= tokens
 * <= 1048576 (the tokens are the products' summation index, run in stages of 64 tokens, so a
 * whole batch's tokens can go in one call); W bf16, cols % 64 == 0, rows % 8 == 0, 2:4 only
 * (MLLM_ERR_UNSUPPORTED otherwise).
 * workspace as for mllm_masked_linear_fwd (only its error word is used here). Reads W, x, dy. */
mllm_status mllm_masked_linear_bwd_adam(const mllm_matrix *mats, const mllm_linear_io *io, int32_t n_mats,
                                        mllm_nm nm, int32_t tokens, const mllm_hparams *hp, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* Workspace bytes of the mllm_masked_linear_* calls (independent of sizes). */
size_t mllm_masked_linear_workspace_bytes(void);

/* Hard-mask extraction and compressed export (s.3.2 "Information flow at inference";
 * Algorithm 1 step 3). Per block: k = first index of the largest logit (NaN never wins;
 * all-NaN gives 0), kept positions p_0 < ... < p_{N-1} of S_k;
 *   pack_values[r, q*N + t] = W[r, q*M + p_t] (bit copy), for block q of row r;
 *   2:4 pack_meta: nibble p_0 | p_1 << 2 in bits [4(q%8), 4(q%8)+4) of uint32 word q/8 of
 *     row r; a row has ceil((cols/4)/8) words; unused high nibbles are written as zero;
 *   4:8 pack_meta: uint16 per block, p_0 | p_1 << 3 | p_2 << 6 | p_3 << 9;
 *   cand_idx_out[b] = k when non-NULL.
 * Reads W, logits. */
mllm_status mllm_hard_pack(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, void *stream);

/* Mask difference (s.3.4 Fig. 5a between adjacent steps, Fig. 8 between methods):
 * *count_out (device, uint64) = number of i < n with a[i] != b[i], for two device arrays of
 * candidate indices (e.g. cand_idx_out of two mllm_hard_pack calls). Exact. */
mllm_status mllm_mask_diff(const uint8_t *a, const uint8_t *b, int64_t n,
                           unsigned long long *count_out, void *stream);

/* Mask statistics over all blocks of the matrices (at most 16 per call), into out[0..3]
 * (device doubles): out[0] = sum over blocks of max_i softmax(kappa pi)_i (mean maximum
 * probability, Fig. 5b, is out[0]/B); out[1] = sum of |W| kept by the hard mask argmax pi;
 * out[2] = sum of |W| kept by the magnitude mask (out[1]/out[2]: relative L1 norm of the
 * kept weights, Fig. 6); out[3] = number of blocks whose hard mask is the magnitude mask.
 * Needs the mllm_sample_fwd workspace; deterministic for a given device. Reads W, logits. */
mllm_status mllm_mask_stats(const mllm_matrix *mats, int32_t n_mats, mllm_nm nm, float kappa,
                            double *out, void *workspace, size_t workspace_bytes, void *stream);

/* Compact code of hard masks (the page stores learned 2:4 masks at 0.65 bits/param, the
 * entropy log2(6)/4 of a candidate index): D candidate indices per uint32 word, word w =
 * sum_{t<D} idx[wD + t] C^t (missing tail digits 0); 2:4: D = 12 (0.667 bits per weight),
 * 4:8: base 70, D = 5 (0.8 bits per weight). words has ceil(n/D) entries. */
mllm_status mllm_encode_candidates(mllm_nm nm, const uint8_t *idx, int64_t n, uint32_t *words,
                                   void *stream);
mllm_status mllm_decode_candidates(mllm_nm nm, const uint32_t *words, int64_t n, uint8_t *idx,
                                   void *stream);

/* One operand of mllm_sparse_linear: a hard-masked weight W* = W (.) M* [rows, cols] in the
 * compressed form mllm_hard_pack writes for a bf16 matrix, and the activations it multiplies.
 * All four pointers are caller-owned device memory, 16-byte aligned. */
typedef struct {
    const void *pack_values;  /* [rows, cols*N/M] bf16: pack_values of mllm_hard_pack        */
    const void *pack_meta;    /* pack_meta of mllm_hard_pack (2:4 uint32 words, 4:8 uint16)  */
    const void *x;            /* [tokens, cols] bf16 activations, row-major                  */
    float *y;                 /* [tokens, rows] fp32 output, row-major (overwritten)          */
    int64_t rows, cols;       /* of the dense matrix; cols % M == 0                           */
} mllm_sparse_operand;

/* Serving the learned sparse network (s.3.2 "Information flow at inference": the mask is
 * applied once and the N:M-sparse weights are used from then on): for every operand,
 *   y[t, r] = sum over blocks q of row r and kept slots i < N of
 *             pack_values[r, qN + i] * x[t, qM + p_i],
 * i.e. y = x W*^T, with bf16 products accumulated in fp32 (tensor cores), for 1 <= tokens
 * <= 16384. Decode-sized calls (up to 64 tokens) are bound by reading the compressed weight,
 * which operands whose cols are a multiple of 128 read once per call (above 16 tokens the
 * others run as groups of 16 tokens). Above 64 tokens (prefill), operands whose cols are a
 * multiple of 128 run in units over all columns, no unit split between CTAs: 2:4 on the
 * sparse tensor cores (two 128-row tiles x 128 tokens), 4:8 expanded to dense once per
 * 64-column stage for 256 tokens (128 for calls of at most 128 tokens); other widths run as
 * groups of 16 tokens.
 * Operands may differ in shape and are processed in one launch per 16 of them; rows == 0
 * operands are skipped and cols == 0 gives y = 0 (pointers other than y may then be NULL).
 * workspace: device memory of mllm_sparse_linear_workspace_bytes() bytes, zero-filled by the
 * caller before its first use; every call leaves it zero-filled again (partial tiles of rows
 * whose columns are split between warps, one completion counter per warp, and an error word
 * -- the uint32 at byte offset workspace_bytes - 16 -- that a call sets to nonzero if one of
 * its asynchronous copies never completed within a bounded wait, in which case that call's
 * y is invalid; it is never expected to be set). Calls that may run concurrently need
 * separate workspaces. Deterministic on a given device: the
 * summation order depends only on the shapes and the launch size. Works for 2:4 and 4:8. */
mllm_status mllm_sparse_linear(const mllm_sparse_operand *ops, int32_t n_ops, mllm_nm nm, int32_t tokens,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes mllm_sparse_linear needs (independent of sizes). */
size_t mllm_sparse_linear_workspace_bytes(void);

/* Test of the bounded waits of mllm_sparse_linear's copy pipeline (no counterpart in the
 * paper): one launch of the 2:4 or 4:8 kernel for one operand (cols % 128 == 0,
 * 1 <= tokens <= 64: the per-warp kernel up to 16 tokens, the tensor-memory kernel above) in which
 * the first pipeline stage of every warp (per-warp kernel) or CTA (tensor-memory kernel) is
 * armed but never filled, so that its wait runs out after the 1 s bound, sets the workspace's
 * error word and the kernel winds down (bounded waits for what it has in flight) and returns.
 * Takes one to two seconds; y is left invalid and the workspace must be zero-filled again
 * afterwards. Nothing faults and the context stays usable. MLLM_ERR_UNSUPPORTED for other
 * shapes. */
mllm_status mllm_sparse_linear_check_timeout(const mllm_sparse_operand *op, mllm_nm nm, int32_t tokens,
                                             void *workspace, size_t workspace_bytes, void *stream);

/* The Gumbel noise itself, for inspection and statistical tests: g_out[i*C + c] = noise
 * of candidate c of the block with global id gids[i] at (seed, step). gids and g_out are
 * device arrays of n_blocks and n_blocks*C entries; step may be any value, including the
 * reserved one. */
mllm_status mllm_noise(mllm_nm nm, uint64_t seed, uint32_t step, const uint64_t *gids,
                       int64_t n_blocks, float *g_out, void *stream);

/* The logarithm table the noise uses, as compiled into the kernels (host memory, for
 * inspection and tests): c_out[j] = fl32(1/F_j), j = 0..127, and t_out[(e + 22)*128 + j] =
 * fl32(e ln2 - ln c_j) for e = -22..4 (27*128 entries). No device work. */
mllm_status mllm_noise_table(float *c_out, float *t_out);

/* Workspace bytes mllm_sample_fwd needs for its regulariser sum (independent of sizes). */
size_t mllm_workspace_bytes(void);

/* Static description of a status code. */
const char *mllm_status_string(mllm_status s);

/* cudaError_t of the most recent MLLM_ERR_CUDA on the calling thread (0 if none). */
int32_t mllm_last_cuda_error(void);

/* ABI guards for bindings: MLLM_ABI_VERSION and the sizes of the structs. */
int32_t mllm_abi_version(void);
size_t mllm_sizeof_matrix(void);
size_t mllm_sizeof_hparams(void);
size_t mllm_sizeof_sparse_operand(void);
size_t mllm_sizeof_linear_io(void);

#ifdef __cplusplus
}
#endif

#endif /* MLLM_H */
