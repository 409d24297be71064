"""Block-DCT int8 KV-cache codec and coefficient-domain decode attention for
NVIDIA B200 (sm_100a).

The compute lives in ``libfc.so`` (C ABI declared in ``include/fc.h``,
``include/fc_view.h`` and ``include/fc_state.h``); ``_lib`` is its ctypes
binding and ``archive`` the host bookkeeping of one layer's compressed K/V
streams (raw tail, capacity-doubling archive, reconstructed view, crop,
batch gather, reset, save / restore) plus the multi-layer decode step.
"""

from . import _lib
from ._lib import (FcArchive, FcError, FcTail, fc_append_step,
                   fc_archive_copy_prefix, fc_combine, fc_compress_blocks,
                   fc_decode_attention, fc_decode_attention_noalloc,
                   fc_decode_kernel, fc_decode_plan, fc_decode_step,
                   fc_decode_step_layers, fc_decode_workspace_bytes,
                   fc_noalloc_status, fc_status_string, fc_storage_bytes,
                   fc_workspace_status, fc_read_view, fc_crop,
                   fc_select_batch, fc_state_bytes, fc_state_save,
                   fc_state_restore)
from .archive import (CodecKVCache, CodecStream, decode_step_layers,
                      grown_capacity)

__all__ = [
    "CodecKVCache", "CodecStream", "decode_step_layers", "grown_capacity",
    "FcArchive", "FcTail", "FcError", "fc_compress_blocks", "fc_append_step",
    "fc_archive_copy_prefix", "fc_decode_plan", "fc_decode_workspace_bytes",
    "fc_decode_kernel", "fc_decode_attention", "fc_decode_attention_noalloc",
    "fc_noalloc_status", "fc_decode_step", "fc_decode_step_layers",
    "fc_combine", "fc_workspace_status", "fc_storage_bytes",
    "fc_status_string", "fc_read_view", "fc_crop", "fc_select_batch",
    "fc_state_bytes", "fc_state_save", "fc_state_restore",
]
