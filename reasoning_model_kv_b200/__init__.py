"""B200-native compressed-KV decode step (thought-adaptive quantisation, decode
attention with attention-mass scores, budgeted and segment-level eviction).  The
compute path is libtkv.so (hand-written sm_100a CUDA behind a C ABI, include/tkv.h);
this package is its thin Python binding."""
from .tkv import (TkvCache, TkvError, lib, make_config, tkv_decode_attention, tkv_decode_step,  # noqa: F401
                  tkv_evict_compact, tkv_evict_compact_window, tkv_evict_segments, tkv_evict_tam,
                  tkv_quantize_append, tkv_tbe_schedule, tkv_workspace_bytes)
