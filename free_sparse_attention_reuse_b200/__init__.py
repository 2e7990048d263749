"""MC-Sparse token-sparse attention with metadata reuse, for NVIDIA B200 (sm_100a).

The compute lives in libmcs.so (hand-written CUDA, C ABI in include/mcs.h); this package is
its Python binding.  Importing it does not load the library; the first call does, and fails
loudly if the library is missing.
"""

from .api import (  # noqa: F401
    Metadata,
    Schedule,
    anchor,
    dense_attn,
    group,
    host_staging,
    perquery_attn,
    residual,
    select,
    select_blocks,
    select_noalloc,
    sparse_attn,
    sparse_attn_host,
    sync_status,
    workspace,
    workspace_size,
)
from ._lib import EXPORTS, LIB_PATH, MCSError, load  # noqa: F401
