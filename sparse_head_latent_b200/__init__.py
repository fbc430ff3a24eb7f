"""B200 (sm_100a) sparse MLA prefill attend block.

The C ABI (include/mla.h, libmla_b200.so) runs the whole block in CUDA
kernels: W_kvb up-projection (tcgen05 GEMM), top-k selection bitmap,
fused sparse-causal attention (block-dense, or absorbed over each row's
gathered latent keys for long rows), W_o output projection (tcgen05 GEMM).
This package is its thin ctypes binding; the library is loaded on first
use and a missing build is an error, never a fallback.
"""
from .mla import (  # noqa: F401
    MLA_ACT_BF16,
    MLA_ACT_E4M3_DYNAMIC,
    MLA_ENTRY_ATTEND,
    MLA_ENTRY_DECODE,
    MLA_ENTRY_KV_UPPROJECT,
    MLA_ENTRY_OUT_PROJECT,
    MLA_ENTRY_PREFILL,
    MLA_PATH_ABSORBED,
    MLA_PATH_AUTO,
    MLA_PATH_BLOCK_DENSE,
    MlaDims,
    MlaError,
    PrefillPipeline,
    library_path,
    load_library,
    make_dims,
    mla_attend,
    mla_attend_static,
    mla_decode,
    mla_device_status,
    mla_kv_upproject,
    mla_out_project,
    mla_prefill,
    mla_profile_begin,
    mla_profile_end,
    mla_quantize_act,
    mla_set_e4m3_weight_conversion,
    mla_set_wait_timeout_ns,
    mla_status_str,
    mla_test_withhold_attention_loads,
    mla_workspace_bytes,
)
