"""nvpa: paged-KV attention for NVIDIA B200 (sm_100a).

The computation lives in libnvpa.so (hand-written CUDA kernels behind the C ABI of
include/nvpa.h).  This package is its thin Python binding: `_lib` holds the ctypes
declarations, `api` the torch-tensor marshalling.
"""

from ._lib import (  # noqa: F401
    LIB_PATH,
    NVPA_FLAG_BAD_BLOCK_ID,
    NVPA_FLAG_BAD_LENGTH,
    NVPA_FLAG_BAD_SLOT,
    NVPA_FLAG_TIMEOUT,
    NvpaError,
    lib,
)
from .api import (  # noqa: F401
    check_bounded_wait,
    decode_shared_prefix_workspace_size,
    decode_step,
    decode_step_shared_prefix,
    gather_kv,
    lse_combine,
    paged_decode_attention,
    paged_decode_partial,
    paged_decode_workspace_size,
    store_kvcache,
    varlen_prefill_attention,
    varlen_prefill_workspace_size,
)
