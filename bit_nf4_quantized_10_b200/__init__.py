"""QLoRA NF4 hot path for B200 (sm_100a): NF4 quantize / double quant /
dequant, the frozen-4-bit + LoRA linear (forward and backward) and the
adapter merge.

The compute lives in libqlora_nf4.so (hand-written CUDA; C ABI declared in
include/qlora_nf4.h).  This package only loads it and marshals arguments.
"""
from ._lib import (  # noqa: F401
    LIB_PATH, QLoraError, NF4Weight, quantize_weight,
    nf4_quantize, nf4_double_quant, nf4_dequant, qlora_linear_fwd, qlora_linear_bwd,
    qlora_silu_gate_fwd, qlora_silu_gate_bwd, qlora_merge,
    nf4_double_quant_level1, nf4_double_quant_finish, qlora_workspace_size, nf4_storage_bytes,
    nvfp4_quantize, mxfp4_quantize, nvfp4_dequant, mxfp4_dequant, qlora_adamw_step, qlora_paged_prefetch,
    nvfp4_scale_atoms_bytes, nvfp4_scale_atoms, nvfp4_gemm, mxfp4_scale_atoms_bytes, mxfp4_scale_atoms, mxfp4_gemm,
    nf4_codebook, qlora_get_status, status_string, qlora_selftest_wait_timeout,
    QL_F32, QL_BF16, QL_OP_DOUBLE_QUANT, QL_OP_FWD, QL_OP_BWD, QL_OP_NVFP4, QL_PAGE_DEVICE, QL_PAGE_HOST,
    QL_OK, QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED, QL_ERR_WORKSPACE, QL_ERR_CUDA, QL_ERR_NONFINITE, QL_ERR_TIMEOUT,
)
