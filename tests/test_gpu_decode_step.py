"""The decode step (tkv_decode_step) against its definition: one T = 1
tkv_quantize_append followed by tkv_decode_attention.  A twin cache that takes the
two calls must end every step with the same state (tables, counters, free stacks,
records, scores) and the same output, bit for bit, and the same device errors; the
oracle's append + attention over the new token bounds the output and the scores as
in the other parity tests."""
import numpy as np
import pytest
import torch

import synth
from reasoning_model_kv_b200 import TkvCache, tkv
from tests.conftest import gpu_available
from tests.gpu_harness import MODES, OUT_ATOL, build_pair, compare_states, np_bits, rows_streams

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCALE = 128 ** -0.5
STATE_KEYS = ("n", "ft", "hw") + tuple(f"{a}{c}" for a in ("handle", "pos", "score", "fs", "pool") for c in range(4))


def _twin(gpu: TkvCache) -> TkvCache:
    t = TkvCache(gpu.B, gpu.Hkv, gpu.G, gpu.cap, gpu.n_protect, max_append=gpu.max_append, dense=gpu.dense,
                 attn_kernel=gpu.attn_kernel, codec=gpu.codec)
    t.import_state(gpu.export_state())
    return t


def _same_state(a: TkvCache, b: TkvCache, what: str):
    sa, sb = a.export_state(), b.export_state()
    for key in STATE_KEYS:
        assert np.array_equal(sa[key].view(np.uint8), sb[key].view(np.uint8)), f"{what}: {key} differs"


def _step_inputs(w, step):
    k, v, cls, pos, q = synth.decode_inputs(w, step)
    return (k.to(DEV), v.to(DEV), cls.to(DEV), pos.to(DEV), q.to(DEV))


def _step_and_twin(gpu, twin, k, v, cls, pos, q, what):
    out = gpu.decode_step(k[:, :, 0].contiguous(), v[:, :, 0].contiguous(), cls[:, 0].contiguous(),
                          pos[:, 0].contiguous(), q, SCALE)
    twin.quantize_append(k, v, cls, pos)
    ref = twin.decode_attention(q, SCALE)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int32), ref.view(torch.int32)), f"{what}: outputs differ"
    _same_state(gpu, twin, what)
    e1, e2 = gpu.poll_error(), twin.poll_error()
    assert e1 == e2, f"{what}: device errors {e1} vs {e2}"
    return out, e1


CASES = [(m, 0) for m in MODES] + [("reuse", 1), ("dense", 1)]


@pytest.mark.parametrize("mode,codec", CASES)
def test_decode_step_equals_append_then_attention_and_the_oracle(mode, codec):
    """2k-token workload (two streams, each split over a cluster of CTAs by the warp-tile
    kernel): three steps, an eviction, and two more steps that refill evicted slots; the
    oracle checks steps 0 and 3."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", codec=codec, steps=6, **MODES[mode])
    twin = _twin(gpu)
    sub = rows_streams(gpu, rows)
    for step in range(5):
        k, v, cls, pos, q = _step_inputs(w, step)
        check_oracle = step in (0, 3)
        if check_oracle:
            o.load_state(gpu.export_state(sub))
        out, err = _step_and_twin(gpu, twin, k, v, cls, pos, q, f"{mode} codec {codec} step {step}")
        assert err == tkv.TKV_OK
        if check_oracle:
            assert o.append(np_bits(k.cpu()[rows]), np_bits(v.cpu()[rows]), cls.cpu()[rows].numpy(),
                            pos.cpu()[rows].numpy()) == 0
            ref = o.attend(np_bits(q.cpu()[rows]), SCALE)
            e = float(np.max(np.abs(out[rows].cpu().numpy() - ref)))
            assert e <= OUT_ATOL, f"step {step}: max-abs {e}"
            compare_states(gpu.export_state(sub), o.state, scores="tol", what=f"decode step {step}")
        if step == 2:
            gpu.evict_compact(w["budget"])
            twin.evict_compact(w["budget"])
            _same_state(gpu, twin, "eviction")


@pytest.mark.parametrize("dense", [False, True], ids=["reuse", "dense"])
def test_decode_step_few_long_streams(dense):
    """Two 24k-token streams: the attention splits each over more CTAs than a cluster holds
    and merges them in a second pass; two steps against the two calls, bit for bit."""
    w = synth.prefill_inputs("tiny_b1_ctx2k", B=1, Hkv=2, Hq=8, ctx=24000, n_protect=4, steps=2)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], dense=dense)
    gpu.quantize_append(w["k"].to(DEV), w["v"].to(DEV), w["cls"][:, :w["ctx"]].contiguous().to(DEV),
                        w["pos"].to(DEV))
    twin = _twin(gpu)
    for step in range(2):
        _step_and_twin(gpu, twin, *_step_inputs(w, step), f"long streams step {step}")


@pytest.mark.parametrize("G", [1, 2, 8])
def test_decode_step_gqa_widths(G):
    """Other GQA group widths (one CTA per stream at 8 streams)."""
    w = synth.prefill_inputs("tiny_b1_ctx2k", Hkv=8, Hq=8 * G, ctx=512, steps=2)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], dense=True)
    gpu.quantize_append(w["k"].to(DEV), w["v"].to(DEV), w["cls"][:, :w["ctx"]].contiguous().to(DEV),
                        w["pos"].to(DEV))
    twin = _twin(gpu)
    for step in range(2):
        _step_and_twin(gpu, twin, *_step_inputs(w, step), f"G {G} step {step}")


@pytest.mark.parametrize("dense", [False, True])
def test_decode_step_device_errors(dense):
    """A full class and an invalid class id: the token is dropped and the same error
    is latched as by the separate append; the attention still runs on the rest."""
    gpu = TkvCache(2, 2, 4, cap=[2, 3, 3, 3], n_protect=1, max_append=8, dense=dense)
    k = synth.normal_bf16(0, 0, synth.TID_K, 2, 2, 0, 4, 128).to(DEV)
    v = synth.normal_bf16(0, 0, synth.TID_V, 2, 2, 0, 4, 128).to(DEV)
    gpu.quantize_append(k, v, torch.tensor([[0, 1, 1, 1], [0, 2, 3, 1]], dtype=torch.uint8, device=DEV),
                        torch.arange(4, dtype=torch.int32, device=DEV).repeat(2, 1).contiguous())
    assert gpu.poll_error() == tkv.TKV_OK
    twin = _twin(gpu)
    q = synth.normal_bf16(0, 0, synth.TID_Q, 2, 8, 4, 1, 128)[:, :, 0].contiguous().to(DEV)
    kn = synth.normal_bf16(0, 0, synth.TID_K, 2, 2, 4, 1, 128).to(DEV)
    vn = synth.normal_bf16(0, 0, synth.TID_V, 2, 2, 4, 1, 128).to(DEV)
    pos = torch.full((2, 1), 4, dtype=torch.int32, device=DEV)
    # row 0: class 1 is full (capacity error); row 1: a valid class-2 token
    cls = torch.tensor([[1], [2]], dtype=torch.uint8, device=DEV)
    _, err = _step_and_twin(gpu, twin, kn, vn, cls, pos, q, "capacity")
    assert err == tkv.TKV_ERR_CAPACITY
    # row 0: class id 9 (invalid); row 1: class 3
    cls = torch.tensor([[9], [3]], dtype=torch.uint8, device=DEV)
    pos = pos + 1
    _, err = _step_and_twin(gpu, twin, kn, vn, cls, pos, q, "invalid class")
    assert err == tkv.TKV_ERR_INVALID
    n = gpu.export_state()["n"]
    assert n[:2].tolist() == [[1, 3, 0, 0], [1, 3, 0, 0]]      # row 0 unchanged by both steps
    assert n[2:].tolist() == [[1, 1, 2, 2], [1, 1, 2, 2]]


def test_decode_step_on_an_empty_cache():
    """The first token of every stream arrives through the decode step."""
    gpu = TkvCache(2, 2, 4, cap=[4, 4, 4, 4], n_protect=0, dense=True)
    twin = _twin(gpu)
    k = synth.normal_bf16(1, 0, synth.TID_K, 2, 2, 0, 1, 128).to(DEV)
    v = synth.normal_bf16(1, 0, synth.TID_V, 2, 2, 0, 1, 128).to(DEV)
    q = synth.normal_bf16(1, 0, synth.TID_Q, 2, 8, 0, 1, 128)[:, :, 0].contiguous().to(DEV)
    cls = torch.tensor([[1], [3]], dtype=torch.uint8, device=DEV)
    pos = torch.zeros((2, 1), dtype=torch.int32, device=DEV)
    out, err = _step_and_twin(gpu, twin, k, v, cls, pos, q, "empty cache")
    assert err == tkv.TKV_OK
    assert torch.isfinite(out).all()
