"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/tkv.h declares, sizes workspaces and rejects bad arguments on the
host without launching anything."""
import ctypes
import re
from pathlib import Path

import pytest

from reasoning_model_kv_b200 import tkv

ROOT = Path(__file__).resolve().parents[1]


def declared_functions():
    text = (ROOT / "include" / "tkv.h").read_text()
    return sorted(set(re.findall(r"TKV_API\s+[\w\s\*]*?\b(tkv_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(tkv.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = tkv.lib()
    for name in declared_functions():
        assert hasattr(L, name), name


def _cfg(**kw):
    args = dict(B=2, Hkv=2, G=4, cap=[8, 16, 16, 16], n_protect=4, max_append=64)
    args.update(kw)
    return tkv.make_config(**args)


def test_workspace_bytes_valid_and_invalid():
    n = tkv.tkv_workspace_bytes(_cfg())
    assert n > 0 and n % 256 == 0
    bigger = tkv.tkv_workspace_bytes(_cfg(cap=[8, 32, 16, 16]))
    assert bigger > n
    for bad in (dict(G=3), dict(B=0), dict(cap=[1, -1, 0, 0]), dict(max_append=0)):
        assert tkv.tkv_workspace_bytes(_cfg(**bad)) == 0
    cfg = _cfg()
    cfg.D = 64
    assert tkv.tkv_workspace_bytes(cfg) == 0
    cfg = _cfg()
    cfg.bits[1] = 6
    assert tkv.tkv_workspace_bytes(cfg) == 0


def test_layout_is_aligned_and_inside_workspace():
    L = tkv.lib()
    cfg = _cfg()
    n = L.tkv_workspace_bytes(ctypes.byref(cfg))
    h = ctypes.c_void_p()
    # tkv_create only records the pointer: a fake aligned address is fine on the host
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == 0
    lay = tkv.TkvLayout()
    assert L.tkv_get_layout(h, ctypes.byref(lay)) == 0
    offs = [lay.n, lay.ft, lay.hw, lay.err] + [getattr(lay, f)[c] for f in
                                               ("handle", "pos", "score", "fs", "pool") for c in range(4)]
    assert all(o % 256 == 0 for o in offs)
    assert lay.state_bytes <= lay.total_bytes == n
    assert list(lay.rec_bytes) == [512, 288, 160, 96]
    assert L.tkv_destroy(h) == 0


def test_create_rejects_bad_workspace():
    L = tkv.lib()
    cfg = _cfg()
    n = L.tkv_workspace_bytes(ctypes.byref(cfg))
    h = ctypes.c_void_p()
    assert L.tkv_create(ctypes.byref(cfg), None, n, ctypes.byref(h)) == tkv.TKV_ERR_INVALID
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(4096 + 16), n, ctypes.byref(h)) == tkv.TKV_ERR_INVALID
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(4096), n - 1, ctypes.byref(h)) == tkv.TKV_ERR_INVALID
    assert b"small" in L.tkv_last_error_string()


def test_calls_reject_bad_arguments_without_launching():
    L = tkv.lib()
    cfg = _cfg()
    n = L.tkv_workspace_bytes(ctypes.byref(cfg))
    h = ctypes.c_void_p()
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == 0
    p = ctypes.c_void_p(1 << 24)
    INV = tkv.TKV_ERR_INVALID
    assert L.tkv_quantize_append(h, None, p, p, p, 1, None) == INV
    assert L.tkv_quantize_append(h, p, p, p, p, 0, None) == INV
    assert L.tkv_quantize_append(h, p, p, p, p, 65, None) == INV          # > max_append
    assert L.tkv_quantize_append(h, ctypes.c_void_p((1 << 24) + 8), p, p, p, 1, None) == INV
    assert L.tkv_decode_attention(h, None, 0.1, p, None) == INV
    assert L.tkv_decode_attention(h, p, 0.1, ctypes.c_void_p((1 << 24) + 4), None) == INV
    odd = ctypes.c_void_p((1 << 24) + 8)
    assert L.tkv_decode_step(None, p, p, p, p, p, 0.1, p, None) == INV
    for i in range(6):                                   # each NULL pointer, in argument order
        args = [p] * 6
        args[i] = None
        assert L.tkv_decode_step(h, *args[:5], 0.1, args[5], None) == INV, i
    for i in (0, 1, 3, 4, 5):                            # k, v, pos, q, out must be 16-byte aligned
        args = [p] * 6
        args[i] = odd
        assert L.tkv_decode_step(h, *args[:5], 0.1, args[5], None) == INV, i
    assert L.tkv_evict_compact(h, -1, None) == INV
    assert L.tkv_evict_compact(None, 3, None) == INV
    assert L.tkv_selftest_wait_timeout(None, 1000, None) == INV
    assert L.tkv_selftest_wait_timeout(h, 0, None) == INV
    assert L.tkv_selftest_wait_timeout(h, (1 << 31) + 1, None) == INV
    assert L.tkv_launch_count(h) == 0
    assert L.tkv_destroy(h) == 0


def test_evict_segments_rejects_bad_arguments_without_launching():
    L = tkv.lib()
    cfg = _cfg()
    n = L.tkv_workspace_bytes(ctypes.byref(cfg))
    h = ctypes.c_void_p()
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == 0
    p = ctypes.c_void_p(1 << 24)
    INV = tkv.TKV_ERR_INVALID
    assert L.tkv_evict_segments(None, p, p, p, p, 4, None) == INV
    assert L.tkv_evict_segments(h, p, p, p, p, -1, None) == INV
    assert L.tkv_evict_segments(h, p, p, p, p, 4097, None) == INV
    assert L.tkv_evict_segments(h, None, p, p, p, 4, None) == INV
    assert L.tkv_evict_segments(h, p, p, p, None, 4, None) == INV
    assert L.tkv_evict_segments(h, ctypes.c_void_p((1 << 24) + 2), p, p, p, 4, None) == INV
    assert L.tkv_evict_segments(h, None, None, None, None, 0, None) == tkv.TKV_OK   # no segments: no-op
    assert L.tkv_launch_count(h) == 0
    assert L.tkv_destroy(h) == 0


def test_tbe_schedule_host_function_matches_the_oracle():
    """The library's schedule (host code, one backward sweep) against the oracle's
    (a forward count per segment) on the golden rows and random label sequences."""
    import numpy as np

    from oracle import oracle as orc
    from tests.test_oracle_tbe import _golden_rows

    for labels, expected in _golden_rows():
        assert tkv.tkv_tbe_schedule(labels, 64, 16) == expected
    rng = np.random.default_rng(11)
    for _ in range(300):
        labels = rng.integers(0, 4, size=int(rng.integers(0, 40))).tolist()
        r0, t_keep = int(rng.integers(0, 200)), int(rng.integers(0, 40))
        assert tkv.tkv_tbe_schedule(labels, r0, t_keep) == orc.tbe_schedule(labels, r0, t_keep).tolist()


def test_tbe_schedule_rejects_bad_arguments():
    for labels, r0, t_keep in (([1, 4], 64, 16), ([1, 3], -1, 16), ([1, 3], 64, -2)):
        with pytest.raises(tkv.TkvError):
            tkv.tkv_tbe_schedule(labels, r0, t_keep)
    assert tkv.lib().tkv_tbe_schedule(None, -1, 64, 16, None) == tkv.TKV_ERR_INVALID
    assert tkv.lib().tkv_tbe_schedule(None, 3, 64, 16, None) == tkv.TKV_ERR_INVALID


def test_evict_tam_rejects_bad_arguments_without_launching():
    L = tkv.lib()
    cfg = _cfg()
    n = L.tkv_workspace_bytes(ctypes.byref(cfg))
    h = ctypes.c_void_p()
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == 0
    p = ctypes.c_void_p(1 << 24)
    INV = tkv.TKV_ERR_INVALID
    assert L.tkv_evict_tam(None, p, p, p, 4, 10, 1.0, None) == INV
    assert L.tkv_evict_tam(h, p, p, p, 4097, 10, 1.0, None) == INV
    assert L.tkv_evict_tam(h, p, p, p, 4, -1, 1.0, None) == INV
    assert L.tkv_evict_tam(h, p, p, p, 4, 10, -0.5, None) == INV
    assert L.tkv_evict_tam(h, p, p, p, 4, 10, float("nan"), None) == INV
    assert L.tkv_evict_tam(h, p, p, p, 4, 10, float("inf"), None) == INV
    assert L.tkv_evict_tam(h, None, p, p, 4, 10, 1.0, None) == INV
    assert L.tkv_evict_tam(h, p, p, ctypes.c_void_p((1 << 24) + 1), 4, 10, 1.0, None) == INV
    assert L.tkv_evict_tam(h, None, None, None, 0, 10, 1.0, None) == tkv.TKV_OK   # no segments: no-op
    assert L.tkv_launch_count(h) == 0
    assert L.tkv_destroy(h) == 0


def test_evict_compact_window_rejects_bad_arguments_without_launching():
    L = tkv.lib()
    cfg = _cfg()
    n = L.tkv_workspace_bytes(ctypes.byref(cfg))
    h = ctypes.c_void_p()
    assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == 0
    assert L.tkv_evict_compact_window(None, 3, 100, None) == tkv.TKV_ERR_INVALID
    assert L.tkv_evict_compact_window(h, -1, 100, None) == tkv.TKV_ERR_INVALID
    assert L.tkv_launch_count(h) == 0
    assert L.tkv_destroy(h) == 0


def test_every_config_rule_is_enforced_on_the_host():
    """Each rule of the configuration check, one violation at a time (no device needed)."""
    assert tkv.tkv_workspace_bytes(_cfg(dense=True)) > 0
    assert tkv.tkv_workspace_bytes(_cfg(dense=True, attn_kernel=1)) > 0
    assert tkv.tkv_workspace_bytes(_cfg(dense=True, attn_kernel=2)) > 0
    assert tkv.tkv_workspace_bytes(_cfg(cap=[(1 << 24) - 1] * 4)) > 0      # largest legal capacities
    for kw in (dict(Hkv=0), dict(G=16), dict(n_protect=-1), dict(max_append=(1 << 24) + 1),
               dict(B=256, Hkv=256),                  # B * Hkv above 65535
               dict(cap=[0, 1 << 24, 0, 0]),          # a class capacity of 2^24
               dict(attn_kernel=1),                   # the tensor-memory kernel needs dense placement
               dict(attn_kernel=2),                   # so does the persistent warp-tile kernel
               dict(dense=True, attn_kernel=1, codec=1)):   # FP codes: the warp-tile kernel only
        assert tkv.tkv_workspace_bytes(_cfg(**kw)) == 0, kw
    for field, value in (("group", 16), ("dense", 2), ("attn_kernel", 3), ("codec", 2)):
        cfg = _cfg()
        setattr(cfg, field, value)
        assert tkv.tkv_workspace_bytes(cfg) == 0, field
    cfg = _cfg()
    cfg.bits[0] = 8
    assert tkv.tkv_workspace_bytes(cfg) == 0


def test_fp_codec_record_sizes_in_the_layout():
    """codec 1: class records of 272 (FP8), 144 (NVFP4) and 80 (ternary) bytes, as the
    header documents and the oracle packs them; codec 0 keeps 288 / 160 / 96."""
    from oracle import oracle as orc
    for codec, want in ((0, [512, 288, 160, 96]), (1, [512, 272, 144, 80])):
        cfg = _cfg(codec=codec)
        n = tkv.tkv_workspace_bytes(cfg)
        assert n > 0
        L = tkv.lib()
        h = ctypes.c_void_p()
        assert L.tkv_create(ctypes.byref(cfg), ctypes.c_void_p(1 << 20), n, ctypes.byref(h)) == 0
        lay = tkv.TkvLayout()
        assert L.tkv_get_layout(h, ctypes.byref(lay)) == 0
        assert list(lay.rec_bytes) == want
        assert want[1:] == [orc.record_bytes_fmt(orc.class_format(b, codec)) for b in (8, 4, 2)]
        assert L.tkv_destroy(h) == 0
