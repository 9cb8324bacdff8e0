"""Parity of the CUDA segment-level eviction (tkv_evict_segments, ThinKV TBE) with
the oracle, called through the C ABI.  Before every eviction the oracle loads the
GPU's state, so tables, free stacks and (dense placement) moved records must match
bit for bit; decode steps on the evicted caches are checked like every other step.
The GPU side takes its retentions from the library's schedule (tkv_tbe_schedule),
the oracle from its own, so a schedule mismatch fails the state comparison too."""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as orc
from reasoning_model_kv_b200 import TkvCache, TkvError, tkv
from tests.conftest import gpu_available
from tests.gpu_harness import MODES, build_pair, compare_states, oracle_for, rows_streams
from tests.test_gpu_parity import _assert_dense, _decode_step

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCALE = 128 ** -0.5


def _tables(w, upto, max_seg=None):
    st, lb, ns = synth.segment_table(w["seed"], w["B"], upto, w["p_r"], w["p_e"], b0=w.get("b0", 0),
                                     max_seg=max_seg)
    kg = np.full(st.shape, -1, np.int32)
    ko = np.full(st.shape, -1, np.int32)
    for b in range(w["B"]):
        n = int(ns[b])
        kg[b, :n] = tkv.tkv_tbe_schedule(lb[b, :n].tolist(), 64, 16)
        ko[b, :n] = orc.tbe_schedule(lb[b, :n], 64, 16)
    return st, lb, kg, ko, ns


def _tbe_lockstep(w, gpu, o, rows, upto):
    st, lb, kg, ko, ns = _tables(w, upto)
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    gpu.evict_segments(dev(st), dev(lb), dev(kg), dev(ns))
    assert o.evict_segments(st[rows], lb[rows], ko[rows], ns[rows]) == 0
    compare_states(gpu.export_state(sub), o.state, what=f"segment eviction at {upto}")
    assert gpu.poll_error() == tkv.TKV_OK


def _transition_starts(w, lo, hi):
    """Positions in [lo, hi) where some batch row starts a Transition segment."""
    st, lb, ns = synth.segment_table(w["seed"], w["B"], hi, w["p_r"], w["p_e"], b0=w.get("b0", 0))
    out = set()
    for b in range(w["B"]):
        for j in range(int(ns[b])):
            if lb[b, j] == synth.CLS_T and lo <= st[b, j] < hi:
                out.add(int(st[b, j]))
    return sorted(out)


@pytest.mark.parametrize("mode", list(MODES))
def test_small_decode_loop_with_segment_eviction_at_every_transition(mode):
    """4 rows x 8/2 heads, 2k prefill, 800 decode steps (R/E/T 0.25/0.25/0.5);
    whenever a row starts a Transition segment the schedule is applied (lock-step
    state check), and the decode step that follows is checked against the oracle."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=4, steps=800, p_r=0.25, p_e=0.25, **MODES[mode])
    ctx = w["ctx"]
    _tbe_lockstep(w, gpu, o, rows, ctx - 1)            # after the prefill (scores all 0)
    _decode_step(w, gpu, o, rows, 0)
    trig = set(_transition_starts(w, ctx + 1, ctx + w["steps"]))
    assert len(trig) >= 3
    checked = 0
    for step in range(1, w["steps"]):
        p = ctx + step
        if p in trig:
            _tbe_lockstep(w, gpu, o, rows, p)           # the new T segment is open, still empty
            _decode_step(w, gpu, o, rows, step)
            checked += 1
        else:
            k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
            gpu.quantize_append(k, v, cls, pos)
            gpu.decode_attention(q, SCALE)
            if step % 50 == 0:
                o.load_state(gpu.export_state(rows_streams(gpu, rows)))
    assert checked >= 3
    if MODES[mode]["dense"]:
        _assert_dense(gpu)
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_b8_ctx16k_segment_eviction_sampled_row(mode):
    """Batch 8 x 32/8 heads, 16k prefill and a scoring step, then the schedule at the
    first transitions of the decode loop; lock-step on row 3 (about 110 segments,
    most R/E segments cut to 64/32/16 at the first call)."""
    rows = [3]
    w = synth.prefill_inputs("b8_ctx16k_256steps", device=DEV)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
    gpu.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(DEV), w["pos"].to(DEV))
    o = oracle_for(gpu, gpu.export_state(rows_streams(gpu, rows)), B=1)
    trig = _transition_starts(w, w["ctx"], w["ctx"] + w["steps"])
    before = gpu.export_state()["n"].sum()
    done = 0
    for step in range(w["steps"]):
        p = w["ctx"] + step
        if p in trig and done < 3:
            _tbe_lockstep(w, gpu, o, rows, p)
            _decode_step(w, gpu, o, rows, step)
            done += 1
        else:
            k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
            gpu.quantize_append(k, v, cls, pos)
            gpu.decode_attention(q, SCALE)
    assert done >= 1
    assert gpu.export_state()["n"].sum() < before      # the schedule did evict
    if MODES[mode]["dense"]:
        _assert_dense(gpu)
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_segment_edge_cases(mode):
    """Retention 0 and whole-segment keeps, segments starting inside the protected
    window (those tokens are bf16, foreign to the segment's label: kept), a row
    with no segments, and a call with no segment columns (no-op)."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, **MODES[mode], n_protect=100)
    _decode_step(w, gpu, o, rows, 0)
    ctx = w["ctx"]
    st, lb, ns = synth.segment_table(w["seed"], w["B"], ctx, w["p_r"], w["p_e"])
    keep = np.full(st.shape, -1, np.int32)
    keep[:, 0::3] = 0
    keep[:, 1::3] = 5
    ns = ns.copy()
    ns[1] = 0                                            # row 1: no segments, nothing evicted
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    n1 = gpu.export_state()["n"][gpu.Hkv:].copy()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    gpu.evict_segments(dev(st), dev(lb), dev(keep), dev(ns))
    assert o.evict_segments(st, lb, keep, ns) == 0
    g = gpu.export_state(sub)
    compare_states(g, o.state, what="edge cases")
    assert np.array_equal(g["n"][gpu.Hkv:], n1)
    before = gpu.export_state()
    empty = torch.zeros((w["B"], 0), dtype=torch.int32, device=DEV)
    gpu.evict_segments(empty, empty.to(torch.uint8), empty, torch.zeros(w["B"], dtype=torch.int32, device=DEV))
    after = gpu.export_state()
    for key in before:
        assert np.array_equal(before[key], after[key]), key
    with pytest.raises(TkvError):
        gpu.evict_segments(dev(st), dev(lb), dev(keep), dev(ns[:1]))
    assert gpu.poll_error() == tkv.TKV_OK


# ----------------------------------------------------------------------------
# thought-aware budgets with pivotal tokens (tkv_evict_tam)
# ----------------------------------------------------------------------------
def _tam_lockstep(w, gpu, o, rows, upto, budget, c):
    st, lb, ns = synth.segment_table(w["seed"], w["B"], upto, w["p_r"], w["p_e"], b0=w.get("b0", 0))
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    gpu.evict_tam(dev(st), dev(lb), dev(ns), budget, c)
    assert o.evict_tam(st[rows], lb[rows], ns[rows], budget, c) == 0
    compare_states(gpu.export_state(sub), o.state, what=f"tam at {upto}")
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_periodic_tam_small(mode):
    """4 rows x 8/2 heads, 2k prefill; every 64 decode steps the thought-aware
    budgets (512 per stream, pivotal above 3x the mean score) are applied and
    checked against the oracle, three times (the page's periodic compaction), with
    a checked decode step after each."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=4, steps=200, **MODES[mode])
    ctx = w["ctx"]
    for step in range(w["steps"]):
        if step in (64, 128, 192):
            _tam_lockstep(w, gpu, o, rows, ctx + step - 1, 512, 3.0)
            _decode_step(w, gpu, o, rows, step)          # checked step on the compacted cache
        else:
            k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
            gpu.quantize_append(k, v, cls, pos)
            gpu.decode_attention(q, SCALE)
    if MODES[mode]["dense"]:
        _assert_dense(gpu)
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_b8_ctx16k_tam_sampled_row(mode):
    """Batch 8 x 32/8 heads, 16k prefill, 16 decode steps for scores, then budgets of
    1638 per stream with pivotal tokens above 4x the mean; lock-step on row 6."""
    rows = [6]
    w = synth.prefill_inputs("b8_ctx16k_256steps", device=DEV)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
    gpu.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(DEV), w["pos"].to(DEV))
    for step in range(16):
        k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
        gpu.quantize_append(k, v, cls, pos)
        gpu.decode_attention(q, SCALE)
    o = oracle_for(gpu, gpu.export_state(rows_streams(gpu, rows)), B=1)
    before = gpu.export_state()["n"].sum()
    _tam_lockstep(w, gpu, o, rows, w["ctx"] + 15, w["budget"], 4.0)
    assert gpu.export_state()["n"].sum() < before
    _decode_step(w, gpu, o, rows, 16)
    if MODES[mode]["dense"]:
        _assert_dense(gpu)
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_tam_degenerate_cases(mode):
    """c = 0 makes every candidate pivotal (nothing leaves); budget 0 with no pivotal
    token keeps only protected, foreign and unsegmented entries."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, **MODES[mode], n_protect=100)
    _decode_step(w, gpu, o, rows, 0)
    before = gpu.export_state()
    st, lb, ns = synth.segment_table(w["seed"], w["B"], w["ctx"], w["p_r"], w["p_e"])
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    gpu.evict_tam(dev(st), dev(lb), dev(ns), 0, 0.0)
    after = gpu.export_state()
    for key in before:
        assert np.array_equal(before[key], after[key]), key
    _tam_lockstep(w, gpu, o, rows, w["ctx"], 0, 1e30)
    g = gpu.export_state()
    assert g["n"][:, 1:].sum() == 0                     # every R/E/T candidate left
    assert (g["n"][:, 0] == 100).all()                  # the bf16 window stays


@pytest.mark.parametrize("mode", list(MODES))
def test_tam_wide_scores_bit_exact(mode):
    """Scores spread over 2^-40 .. 2^30: fp64 sums taken in different orders would round
    differently here; the exact sums make the budgets, and so the kept sets, bit-exact
    with the oracle (both sides start from the same state)."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, **MODES[mode])
    _decode_step(w, gpu, o, rows, 0)
    state = gpu.export_state()
    rng = np.random.default_rng(77)
    for c in range(4):
        sc = state[f"score{c}"]
        sc[...] = np.ldexp(rng.random(sc.shape) + 0.5, rng.integers(-40, 31, sc.shape)).astype(np.float32)
    gpu.import_state(state)
    for budget, c in ((300, 2.0), (120, 0.7), (700, 5.0)):
        _tam_lockstep(w, gpu, o, rows, w["ctx"], budget, c)
    assert gpu.poll_error() == tkv.TKV_OK
