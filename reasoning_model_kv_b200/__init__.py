"""B200-native compressed-KV decode step (thought-adaptive quantisation, decode
attention with attention-mass scores, budgeted eviction).  The compute path is
libtkv.so (hand-written sm_100a CUDA behind a C ABI, include/tkv.h); this package
is its thin Python binding."""
from .tkv import (TkvCache, TkvError, tkv_decode_attention, tkv_evict_compact,  # noqa: F401
                  tkv_quantize_append, lib, make_config, tkv_workspace_bytes)
