"""block_sparse_chunked_b200 — CompactAttention's Block-Union KV selection and
paged chunk attention on NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libcompactattn.so`` (C ABI in
``include/compactattn.h``).  Every step of the computation runs in the
library's CUDA kernels; this module only checks tensor metadata, allocates
outputs with torch and passes pointers and the current CUDA stream.  There is
no CPU fallback: importing this package without the built library raises.
"""
from ._capi import (  # noqa: F401
    CA_OK,
    CA_ERR_ARG,
    CA_ERR_ALIGN,
    CA_ERR_DTYPE,
    CA_ERR_LAUNCH,
    CA_ERR_BOUNDS,
    CA_ERR_TIMEOUT,
    CA_ERR_WORKSPACE,
    CompactAttnError,
    LIB_PATH,
    EXPORTS,
    lib,
    version,
    build_tables,
    build_tables_batched,
    build_tables_bits,
    workspace_size,
    chunk_attention,
    chunk_attention_varlen,
    chunk_attention_masked,
    chunk_attention_fp8,
    append_kv,
    check,
    wait_probe,
    last_error,
)
from .accounting import (  # noqa: F401
    selected_pairs,
    selected_flops,
    selected_pairs_pl,
    selected_flops_pl,
    dense_flops,
    builder_bytes,
)
