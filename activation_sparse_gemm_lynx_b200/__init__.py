"""B200-native (sm_100a) RT-Lynx online 2:4 activation-sparse linear layer.

    Y = S(X) W^T + bias + (X A^T) B^T

S(X) keeps, per token row, the 2 largest magnitudes of every 4 consecutive
values (ties to the lower position), rescaled by the fp32 norm-compensation
factor sum|x| / sum|kept| and rounded to bf16; the product runs on sparse
tensor cores (tcgen05.mma.sp) and the rank-r LoRA residual on the dense X
plus the bias are added in the same accumulator before one bf16 store.

The public entry points mirror the C ABI of ``include/lynx.h``; see
:mod:`activation_sparse_gemm_lynx_b200.lynx`.  ``workloads`` holds the seeded
synthetic inputs used by the tests and the benchmark.
"""
from .lynx import (  # noqa: F401
    LYNX_ACT_GELU_TANH,
    LYNX_ACT_NONE,
    LynxError,
    lynx_check_error,
    lynx_debug_set_stall,
    lynx_linear,
    lynx_linear_act,
    lynx_linear_begin,
    lynx_linear_dense,
    lynx_linear_finish,
    lynx_linear_fused,
    lynx_linear_host,
    lynx_linear_host_act,
    lynx_linear_host_workspace_bytes,
    lynx_lora_rank,
    lynx_lora_rank_supported,
    lynx_meta_bytes,
    lynx_meta_canonical_to_hw,
    lynx_meta_hw_to_canonical,
    lynx_profile_set_part,
    lynx_profile_set_split_event,
    lynx_sparse_gemm,
    lynx_sparsify,
    lynx_sparsify_noalloc,
    lynx_sparsify_noalloc_max_rows,
    lynx_sparsify_workspace_bytes,
    lynx_status_string,
    lynx_vals_bytes,
    lynx_version,
    lynx_workspace_bytes,
    library,
)
