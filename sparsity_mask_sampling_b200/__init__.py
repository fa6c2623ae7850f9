"""MaskLLM's differentiable N:M mask sampler on B200 (sm_100a).

The computation lives in libmllm.so (hand-written CUDA kernels behind the C ABI of
include/mllm.h); this package is its ctypes binding plus host-side plumbing (buffer
allocation, workload shapes and schedules, seeded synthetic inputs).
"""
from ._mllm import (  # noqa: F401
    INIT_STEP, MLLM_BF16, MLLM_F32, Hparams, MatrixArray, MatrixBuffers, MllmError,
    mllm_decode_candidates, mllm_encode_candidates, mllm_hard_pack, mllm_last_cuda_error,
    mllm_mask_diff, mllm_mask_stats, mllm_noise, mllm_num_candidates, mllm_prior_init, mllm_prior_init_from_mask,
    mllm_sample_bwd_adam, mllm_sample_bwd_adam_fwd, mllm_sample_fwd, mllm_sample_fwd_noalloc, mllm_sparse_linear, mllm_sparse_linear_check_timeout, mllm_sparse_linear_workspace_bytes,
    sparse_linear_workspace, mllm_masked_linear_fwd, mllm_masked_linear_workspace_bytes,
    masked_linear_workspace, mllm_masked_linear_bwd_adam,
    mllm_status_string, mllm_workspace_bytes, lib, SparseOperandArray,
)
from .buffers import alloc_matrix, pack_shapes  # noqa: F401
from .configs import WORKLOADS, Workload, linear_schedule  # noqa: F401
