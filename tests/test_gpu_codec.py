"""Parity of the floating-point class records (codec 1: class 1 FP8 E4M3, class 2
NVFP4, class 3 ternary; ThinKV page, Metodologia, TBQ) with the oracle, through the C
ABI: the append writes the oracle's records bit for bit, decode attention over them
stays within the output tolerance, eviction and compaction match bit for bit, in both
placements."""
import numpy as np
import pytest
import torch

import synth
from reasoning_model_kv_b200 import TkvCache, TkvError, tkv
from tests.conftest import gpu_available
from tests.gpu_harness import OUT_ATOL, build_pair, compare_states, np_bits, rows_streams
from tests.test_gpu_parity import _evict_lockstep

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCALE = 128 ** -0.5


def _step(w, gpu, o, rows, step):
    k, v, cls, pos, q = synth.decode_inputs(w, step)
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    gpu.quantize_append(k.to(DEV), v.to(DEV), cls.to(DEV), pos.to(DEV))
    assert o.append(np_bits(k[rows]), np_bits(v[rows]), cls[rows].numpy(), pos[rows].numpy()) == 0
    compare_states(gpu.export_state(sub), o.state, what=f"fp append step {step}")
    out = gpu.decode_attention(q.to(DEV), SCALE)
    ref = o.attend(np_bits(q[rows]), SCALE)
    err = float(np.max(np.abs(out[rows].cpu().numpy() - ref)))
    assert err <= OUT_ATOL, f"step {step}: max-abs {err}"
    compare_states(gpu.export_state(sub), o.state, scores="tol", what=f"fp attention step {step}")
    assert gpu.poll_error() == tkv.TKV_OK
    return err


@pytest.mark.parametrize("dense", [False, True], ids=["reuse", "dense"])
@pytest.mark.parametrize("G,ctx,n_protect,outliers", [(4, 2000, 128, True), (8, 709, 4, False), (1, 1500, 0, True)])
def test_fp_codec_prefill_decode_evict(dense, G, ctx, n_protect, outliers):
    """Prefill records bit-exact, three decode steps, an eviction to 300 (bit-exact
    tables, free stacks and moved records) and two more steps on the compacted cache."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, Hq=2 * G, Hkv=2, ctx=ctx, n_protect=n_protect,
                                 outliers=outliers, steps=6, dense=dense, codec=1)
    compare_states(gpu.export_state(), o.state, what="fp prefill")
    errs = [_step(w, gpu, o, rows, s) for s in range(3)]
    _evict_lockstep(gpu, o, rows, 300)
    errs += [_step(w, gpu, o, rows, s) for s in range(3, 5)]
    print(f"codec 1 G={G} ctx={ctx} dense={dense}: max-abs output errors {max(errs):.2e}")


def test_fp_codec_extreme_magnitudes():
    """Keys and values scaled by 2^12 and 2^-12 around a unit query: FP8 / NVFP4 scales
    and ternary magnitudes cover both ends without overflow or flush."""
    for sc in (2.0 ** 12, 2.0 ** -12):
        w = synth.prefill_inputs("tiny_b1_ctx2k", B=1, Hq=4, Hkv=1, ctx=600, n_protect=4, steps=2)
        w["k"] = (w["k"].float() * sc).to(torch.bfloat16)
        w["v"] = (w["v"].float() * sc).to(torch.bfloat16)
        gpu = TkvCache(1, 1, 4, w["cap"], 4, max_append=w["ctx"], dense=True, codec=1)
        from oracle import oracle as orc
        o = orc.OracleCache(1, 1, 4, cap=w["cap"], n_protect=4, dense=True, codec=1)
        gpu.quantize_append(w["k"].to(DEV), w["v"].to(DEV), w["cls"][:, :w["ctx"]].contiguous().to(DEV),
                            w["pos"].to(DEV))
        assert o.append(np_bits(w["k"]), np_bits(w["v"]), w["cls"][:, :w["ctx"]].numpy(), w["pos"].numpy()) == 0
        compare_states(gpu.export_state(), o.state, what=f"fp prefill x{sc}")
        q = synth.decode_inputs(w, 0)[4]
        out = gpu.decode_attention(q.to(DEV), SCALE).cpu().numpy().astype(np.float64)
        ref = o.attend(np_bits(q), SCALE)
        err = np.abs(out - ref) / np.maximum(1.0, np.abs(ref))
        assert float(err.max()) <= OUT_ATOL, (sc, float(err.max()))
        assert gpu.poll_error() == tkv.TKV_OK


def test_fp_codec_rejects_the_tensor_core_kernel():
    with pytest.raises(TkvError):
        TkvCache(1, 1, 4, [8, 16, 16, 16], 4, dense=True, attn_kernel=1, codec=1)
