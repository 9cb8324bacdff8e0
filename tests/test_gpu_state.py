"""Checkpoint / restore through the C ABI (tkv_export_state / tkv_import_state).

The block table is the cache's whole state (ThinKV, "Implementacao do Sistema":
the Continuous Thinking block table tracks every entry's thought type, position
and slot), so a cache restored from an exported state must continue exactly as
the cache it was taken from."""
import numpy as np
import pytest
import torch

import synth
from reasoning_model_kv_b200 import TkvCache, TkvError, tkv
from tests.conftest import gpu_available
from tests.gpu_harness import MODES, OUT_ATOL, build_pair, compare_states, np_bits

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCALE = 128 ** -0.5


@pytest.mark.parametrize("mode", list(MODES))
def test_export_import_round_trip_continues_bit_identically(mode):
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, steps=3, **MODES[mode])
    w["cls"] = synth.class_ids(0, w["B"], w["ctx"] + 3, w["p_r"], w["p_e"])
    k, v, cls, pos, q = synth.decode_inputs(w, 0, device=DEV)
    gpu.quantize_append(k, v, cls, pos)
    gpu.decode_attention(q, SCALE)
    gpu.evict_compact(w["budget"])
    st = gpu.export_state()
    fresh = TkvCache(gpu.B, gpu.Hkv, gpu.G, gpu.cap, gpu.n_protect, max_append=gpu.max_append, **MODES[mode])
    fresh.import_state(st)
    back = fresh.export_state()
    for key, arr in st.items():   # bytes: unused slots may hold NaN patterns
        assert np.array_equal(back[key].view(np.uint8), arr.view(np.uint8)), key
    gpu.import_state(st)           # both caches restored from the same checkpoint
    outs, states = [], []
    for step in (1, 2):
        k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
        pair = []
        for c in (gpu, fresh):
            c.quantize_append(k, v, cls, pos)
            pair.append(c.decode_attention(q, SCALE))
        assert torch.equal(pair[0], pair[1]), f"step {step}: outputs differ"
    a, b = gpu.export_state(), fresh.export_state()
    for key in a:
        assert np.array_equal(a[key].view(np.uint8), b[key].view(np.uint8)), key
    o.load_state(b)
    k, v, cls, pos, q = synth.decode_inputs(w, 2)
    ref = o.attend(np_bits(q), SCALE)          # the restored state still matches the oracle
    got = fresh.decode_attention(q.to(DEV), SCALE).cpu().numpy()
    assert float(np.max(np.abs(got - ref))) <= OUT_ATOL
    assert fresh.poll_error() == tkv.TKV_OK and gpu.poll_error() == tkv.TKV_OK


def test_import_rejects_wrong_shapes_and_keys():
    gpu = TkvCache(1, 2, 4, cap=[4, 4, 4, 4], n_protect=0)
    st = gpu.export_state()
    with pytest.raises(TkvError):
        gpu.import_state({"n": np.zeros((3, 4), dtype=np.int32)})
    with pytest.raises(TkvError):
        gpu.import_state({"nope": st["n"]})
    gpu.import_state({"n": st["n"]})
