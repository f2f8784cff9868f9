"""Compressed paged KV cache for B200: quantize-and-pack write and paged decode attention.

The compute runs in libtq.so (CUDA, sm_100a; C ABI in include/tq.h). This
package only marshals arguments (``tq``) and draws seeded synthetic inputs
(``workloads``).
"""

from .tq import (  # noqa: F401
    Codec, UnsupportedFormatError, TQTimeoutError, TQCudaError, codec_host_tables, load_recipe_metadata,
    page_pool, pack_kv, decode_workspace_bytes, alloc_workspace, decode_paged, byte_ledger, host_ledger, lib,
    TQ_DERR_SLOT, TQ_DERR_BLOCK, TQ_DERR_TIMEOUT, HEAD_DIM,
)
