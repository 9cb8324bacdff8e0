"""tkv_quantize_append_noalloc: the append variant for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the
library instead of the workspace).  Its results must equal the regular
tkv_quantize_append's bit for bit, call after call, since every later call
reads the state the earlier ones wrote.

Kept in a file of its own, collected last, so that a run stopping at the first
failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import synth
from reasoning_model_kv_b200 import TkvCache, TkvError, tkv
from tests.conftest import gpu_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"


def _inputs(B, Hkv, p0, T, seed=11):
    k = synth.normal_bf16(seed, 0, synth.TID_K, B, Hkv, p0, T, 128).to(DEV)
    v = synth.normal_bf16(seed, 0, synth.TID_V, B, Hkv, p0, T, 128).to(DEV)
    cls = synth.class_ids(seed, B, p0 + T, 0.4, 0.4)[:, p0:].contiguous().to(DEV)
    pos = synth.positions(B, p0, T).to(DEV)
    return k, v, cls, pos


def _same_state(a: TkvCache, b: TkvCache):
    ga, gb = a.export_state(), b.export_state()
    for key in ("n", "ft", "hw"):
        assert np.array_equal(ga[key], gb[key]), key
    for c in range(4):
        for s in range(a.S):
            n, ft = ga["n"][s, c], ga["ft"][s, c]
            for f in ("handle", "pos", "score"):
                assert np.array_equal(ga[f"{f}{c}"][s, :n].view(np.int32),
                                      gb[f"{f}{c}"][s, :n].view(np.int32)), (f, c, s)
            assert np.array_equal(ga[f"fs{c}"][s, :ft], gb[f"fs{c}"][s, :ft])
            hs = ga[f"handle{c}"][s, :n]
            assert np.array_equal(ga[f"pool{c}"][s, hs], gb[f"pool{c}"][s, hs]), (c, s)


def test_noalloc_append_matches_regular_append_on_consecutive_calls():
    B, Hkv, G = 3, 2, 4
    cap = [40, 400, 400, 400]
    reg = TkvCache(B, Hkv, G, cap, n_protect=16, max_append=512)
    noa = TkvCache(B, Hkv, G, cap, n_protect=16, max_append=512)
    p0 = 0
    for T in (301, 77, 1):                      # consecutive calls on the same caches
        k, v, cls, pos = _inputs(B, Hkv, p0, T)
        reg.quantize_append(k, v, cls, pos)
        noa.quantize_append_noalloc(k, v, cls, pos)
        torch.cuda.synchronize()
        _same_state(reg, noa)
        p0 += T
    # after an eviction the free stacks are non-empty: the ranks now pick popped slots
    q = synth.normal_bf16(11, 0, synth.TID_Q, B, Hkv * G, p0, 1, 128)[:, :, 0].contiguous().to(DEV)
    for cache in (reg, noa):
        cache.decode_attention(q, 128 ** -0.5)
        cache.evict_compact(100)
    for T in (45, 130):
        k, v, cls, pos = _inputs(B, Hkv, p0, T)
        reg.quantize_append(k, v, cls, pos)
        noa.quantize_append_noalloc(k, v, cls, pos)
        torch.cuda.synchronize()
        _same_state(reg, noa)
        p0 += T
    assert reg.poll_error() == tkv.TKV_OK and noa.poll_error() == tkv.TKV_OK


def test_noalloc_append_rejects_appends_beyond_its_scratch():
    B, Hkv = 64, 1
    cache = TkvCache(B, Hkv, 4, [4, 9000, 9000, 9000], n_protect=0, max_append=9000)
    T = 524288 // B - 3                         # B * (T + 4) = 524352 > 524288
    k = torch.zeros((B, Hkv, T, 128), dtype=torch.bfloat16, device=DEV)
    cls = torch.ones((B, T), dtype=torch.uint8, device=DEV)
    pos = torch.zeros((B, T), dtype=torch.int32, device=DEV)
    before = cache.launch_count()
    with pytest.raises(TkvError) as e:
        cache.quantize_append_noalloc(k, k, cls, pos)
    assert e.value.status == tkv.TKV_ERR_INVALID
    assert cache.launch_count() == before
    assert int(cache.export_state()["n"].sum()) == 0
    # the largest append that fits is accepted
    T = 524288 // B - 4
    cache.quantize_append_noalloc(k[:, :, :T].contiguous(), k[:, :, :T].contiguous(),
                                  cls[:, :T].contiguous(), pos[:, :T].contiguous())
    assert cache.poll_error() == tkv.TKV_OK
    assert int(cache.export_state()["n"].sum()) == B * Hkv * T
