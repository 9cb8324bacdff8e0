"""Free-running kept-set parity: the GPU and the oracle each decode and evict on
their own accumulated scores, with no state copied between them, and the kept sets
are compared at every eviction.

The rule (the benchmark spec of the method): kept-token sets are bit-exact except
at score ties within 1e-6 relative, the lower index winning.  A token kept by one
side and evicted by the other is therefore allowed only when its (oracle) score lies
within 1e-6 relative of the eviction threshold -- the budget-th highest candidate
score.  Scores accumulate the attention mass of every decode step (cumulative,
H2O-style: "Back from the Future", problem statement), so the check also covers the
drift of many steps of fp32 accumulation against the oracle's fp64 sums.

Each eviction prints how many kept tokens differ and how far the farthest one sits
from the threshold."""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as orc
from reasoning_model_kv_b200 import TkvCache, tkv
from tests.conftest import gpu_available
from tests.gpu_harness import MODES, np_bits, rows_streams

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCALE = 128 ** -0.5
TIE_RTOL = 1e-6


def _kept(state, s):
    return set(np.concatenate([state[f"pos{c}"][s, :state["n"][s, c]] for c in range(4)]).tolist())


def _scores(state, s):
    sc = {}
    for c in range(4):
        n = state["n"][s, c]
        sc.update(zip(state[f"pos{c}"][s, :n].tolist(), state[f"score{c}"][s, :n].astype(np.float64).tolist()))
    return sc


def _free_run(name, rows, steps, evict_every, modes, **over):
    w = synth.prefill_inputs(name, device=DEV, steps=steps, **over)
    cls0 = w["cls"][:, :w["ctx"]].contiguous().to(DEV)
    gpus = {}
    for mode in modes:
        g = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
        g.quantize_append(w["k"], w["v"], cls0, w["pos"].to(DEV))
        gpus[mode] = g
    first = gpus[modes[0]]
    sub = rows_streams(first, rows)
    o = orc.OracleCache(len(rows), w["Hkv"], w["G"], cap=w["cap"], n_protect=w["n_protect"],
                        dense=first.dense)
    o.load_state(first.export_state(sub))      # the prefill is bit-exact (tested elsewhere)
    del w["k"], w["v"]
    report = []
    for step in range(steps):
        k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
        for g in gpus.values():
            g.quantize_append(k, v, cls, pos)
            g.decode_attention(q, SCALE)
        kc, vc, clc, pc, qc = k.cpu(), v.cpu(), cls.cpu(), pos.cpu(), q.cpu()
        assert o.append(np_bits(kc[rows]), np_bits(vc[rows]), clc[rows].numpy(), pc[rows].numpy()) == 0
        o.attend(np_bits(qc[rows]), SCALE)
        if (step + 1) % evict_every:
            continue
        before = o.copy_state()
        assert o.evict(w["budget"]) == 0
        for mode, g in gpus.items():
            g.evict_compact(w["budget"])
            st = g.export_state(sub)
            ndiff, worst = 0, 0.0
            for s in range(len(sub)):
                diff = _kept(st, s) ^ _kept(o.state, s)
                if not diff:
                    continue
                sc = _scores(before, s)
                cand = sorted((v_ for p_, v_ in sc.items() if p_ >= w["n_protect"]), reverse=True)
                thr = cand[w["budget"] - 1]
                for p_ in diff:
                    rel = abs(sc[p_] - thr) / thr
                    ndiff += 1
                    worst = max(worst, rel)
                    assert rel <= TIE_RTOL, (f"{mode} step {step} stream {sub[s]}: position {p_} kept by one side "
                                             f"only, {rel:.3e} relative from the threshold")
            report.append((mode, step, ndiff, worst))
            assert g.poll_error() == tkv.TKV_OK
    for mode, step, ndiff, worst in report:
        print(f"kept sets {name} {mode} eviction after step {step}: {ndiff} tokens differ, "
              f"farthest {worst:.2e} relative from the threshold")
    return report


def test_kept_sets_free_running_2k():
    """The 2k single-layer workload: 24 decode steps, eviction to 512 every 8 steps."""
    _free_run("tiny_b1_ctx2k", [0], steps=24, evict_every=8, modes=list(MODES))


@pytest.mark.slow
def test_kept_sets_free_running_16k():
    """Batch 8 x 32/8 heads, 16k context, 256 decode steps with eviction to 1638 every
    128 steps (all rows on the GPU; the oracle follows two rows)."""
    _free_run("b8_ctx16k_256steps", [2, 6], steps=256, evict_every=128, modes=list(MODES))
