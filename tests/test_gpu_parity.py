"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Every comparison hands the oracle the GPU's pre-call state, so a difference is
always attributable to one call: codes/scales/zeros/tables/free stacks are
compared bit for bit, attention output within max-abs 2e-3, scores within the
fp32 dot-product bound stated in tests/gpu_harness.py.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as orc
from reasoning_model_kv_b200 import TkvCache, TkvError, tkv
from tests.conftest import gpu_available
from tests.gpu_harness import (MODES, OUT_ATOL, build_pair, compare_states, np_bits, oracle_for,
                               rows_streams)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCALE = 128 ** -0.5


def _decode_step(w, gpu, o, rows, step, check=True):
    """Lock-step append + attention on GPU and oracle (oracle first loads the GPU state)."""
    k, v, cls, pos, q = synth.decode_inputs(w, step)
    sub = rows_streams(gpu, rows)
    pre = gpu.export_state(sub)
    o.load_state(pre)
    gpu.quantize_append(k.to(DEV), v.to(DEV), cls.to(DEV), pos.to(DEV))
    assert o.append(np_bits(k[rows]), np_bits(v[rows]), cls[rows].numpy(), pos[rows].numpy()) == 0
    if check:
        compare_states(gpu.export_state(sub), o.state, what=f"append step {step}")
    out = gpu.decode_attention(q.to(DEV), SCALE)
    ref = o.attend(np_bits(q[rows]), SCALE)
    got = out[rows].cpu().numpy()
    err = float(np.max(np.abs(got - ref)))
    assert err <= OUT_ATOL, f"step {step}: max-abs {err}"
    if check:
        compare_states(gpu.export_state(sub), o.state, scores="tol", what=f"attention step {step}")
    assert gpu.poll_error() == tkv.TKV_OK
    return err


def _evict_lockstep(gpu, o, rows, budget):
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    gpu.evict_compact(budget)
    assert o.evict(budget) == 0
    compare_states(gpu.export_state(sub), o.state, what=f"evict {budget}")


def _assert_dense(gpu):
    """Dense placement invariant: entry i of every class table lives in slot i."""
    g = gpu.export_state()
    assert (g["ft"] == 0).all() and np.array_equal(g["hw"], g["n"])
    for c in range(4):
        for s in range(gpu.S):
            n = g["n"][s, c]
            assert np.array_equal(g[f"handle{c}"][s, :n], np.arange(n)), (c, s)


# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", list(MODES))
def test_tiny_prefill_decode_evict_reuse(mode):
    """2k-token single-layer workload: prefill, decode step, eviction to 512, and
    a second step that reuses evicted slots (dense placement: appends after the
    moved records)."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", **MODES[mode])
    dense = gpu.dense
    compare_states(gpu.export_state(), o.state, what="prefill")
    _decode_step(w, gpu, o, rows, 0)
    _evict_lockstep(gpu, o, rows, w["budget"])
    n = gpu.export_state()["n"]
    assert (n[:, 1:].sum(axis=1) == w["budget"]).all()
    w2 = dict(w, steps=2)
    w2["cls"] = synth.class_ids(0, w["B"], w["ctx"] + 2, w["p_r"], w["p_e"])
    _decode_step(w2, gpu, o, rows, 1)
    assert gpu.launch_count() > 0
    if dense:
        _assert_dense(gpu)


def test_kept_sets_free_running_match_up_to_near_ties():
    """GPU and oracle each evict on their own accumulated scores; kept sets agree
    except for entries whose oracle scores tie the threshold within the score
    tolerance."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k")
    for step in range(3):
        k, v, cls, pos, q = synth.decode_inputs(dict(w, cls=synth.class_ids(0, 1, w["ctx"] + 3, 0.4, 0.4)), step)
        gpu.quantize_append(k.to(DEV), v.to(DEV), cls.to(DEV), pos.to(DEV))
        o.append(np_bits(k), np_bits(v), cls.numpy(), pos.numpy())
        gpu.decode_attention(q.to(DEV), SCALE)
        o.attend(np_bits(q), SCALE)
    g_before = gpu.export_state()
    gpu.evict_compact(w["budget"])
    o_before = o.copy_state()
    o.evict(w["budget"])
    g = gpu.export_state()
    for s in range(gpu.S):
        kept_g = set(np.concatenate([g[f"pos{c}"][s, :g["n"][s, c]] for c in range(4)]).tolist())
        kept_o = set(np.concatenate([o.state[f"pos{c}"][s, :o.state["n"][s, c]] for c in range(4)]).tolist())
        diff = kept_g ^ kept_o
        if diff:
            sc = {}
            for c in range(4):
                n = o_before["n"][s, c]
                sc.update(zip(o_before[f"pos{c}"][s, :n].tolist(), o_before[f"score{c}"][s, :n].tolist()))
            thr = sorted((v for p, v in sc.items() if p >= w["n_protect"]), reverse=True)[w["budget"] - 1]
            for p in diff:
                assert abs(sc[p] - thr) <= 1e-4 * thr, (p, sc[p], thr)


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("G,n_protect,outliers", [(1, 4, False), (2, 128, True), (4, 4, True),
                                                  (8, 128, False)])
def test_gqa_widths_and_windows(G, n_protect, outliers, mode):
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, Hq=2 * G, Hkv=2, ctx=709,
                                 n_protect=n_protect, outliers=outliers, steps=2, **MODES[mode])
    compare_states(gpu.export_state(), o.state, what="prefill")
    _decode_step(w, gpu, o, rows, 0)
    _evict_lockstep(gpu, o, rows, 300)
    _decode_step(w, gpu, o, rows, 1)


@pytest.mark.parametrize("mode,codec", [("reuse", 0), ("dense", 0), ("reuse", 1), ("dense", 1)])
@pytest.mark.parametrize("G", [4, 8])
def test_few_long_streams_split_beyond_a_cluster(G, mode, codec):
    """Two 24k-token streams: the warp-tile kernel gives each stream more CTAs than a
    cluster holds (23 here) and a second pass merges their partials and adds the scores;
    a ragged tail (24000 + 1 entries) and a step after an eviction to 3000 (8 CTAs: the
    cluster path again)."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=1, Hq=2 * G, Hkv=2, ctx=24000, n_protect=4,
                                 outliers=True, steps=2, codec=codec, **MODES[mode])
    _decode_step(w, gpu, o, rows, 0)
    _evict_lockstep(gpu, o, rows, 3000)
    _decode_step(w, gpu, o, rows, 1)


@pytest.mark.parametrize("mode", list(MODES))
def test_clusters_shrunk_to_one_wave(mode):
    """72 streams of 2048 entries: eight CTAs per stream would fill the SMs' slots, but
    clusters live within one GPC and a B200 holds only 71 clusters of eight such CTAs, so
    the launcher takes the largest cluster size that keeps every stream resident at once
    (seven here: a size that is not a power of two), compared on three sampled rows."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=9, Hq=32, Hkv=8, ctx=2048, n_protect=4, outliers=True,
                                 steps=2, rows=[0, 4, 8], **MODES[mode])
    _decode_step(w, gpu, o, rows, 0)
    _evict_lockstep(gpu, o, rows, 1200)
    _decode_step(w, gpu, o, rows, 1)


@pytest.mark.parametrize("dense", [False, True], ids=["reuse", "dense"])
def test_multi_token_append_after_eviction_reuses_slots_in_order(dense):
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", ctx=600, steps=80, dense=dense)
    gpu.decode_attention(synth.decode_inputs(w, 0)[4].to(DEV), SCALE)
    _evict_lockstep(gpu, o, rows, 100)
    T = 77
    p0 = w["ctx"]
    k = synth.normal_bf16(0, 0, synth.TID_K, 1, 2, p0, T, 128)
    v = synth.normal_bf16(0, 0, synth.TID_V, 1, 2, p0, T, 128)
    cls = w["cls"][:, p0:p0 + T].contiguous()
    pos = synth.positions(1, p0, T)
    o.load_state(gpu.export_state())
    gpu.quantize_append(k.to(DEV), v.to(DEV), cls.to(DEV), pos.to(DEV))
    assert o.append(np_bits(k), np_bits(v), cls.numpy(), pos.numpy()) == 0
    compare_states(gpu.export_state(), o.state, what="append T=77 after eviction")


@pytest.mark.parametrize("mode", list(MODES))
def test_empty_cache_and_single_token(mode):
    gpu = TkvCache(1, 2, 4, cap=[4, 4, 4, 4], n_protect=0, **MODES[mode])
    q = synth.normal_bf16(0, 0, synth.TID_Q, 1, 8, 0, 1, 128)[:, :, 0].contiguous()
    out = gpu.decode_attention(q.to(DEV), SCALE)
    assert not out.any()
    k = synth.normal_bf16(0, 0, synth.TID_K, 1, 2, 0, 1, 128)
    cls = torch.tensor([[3]], dtype=torch.uint8)
    pos = torch.zeros((1, 1), dtype=torch.int32)
    gpu.quantize_append(k.to(DEV), k.to(DEV), cls.to(DEV), pos.to(DEV))
    o = orc.OracleCache(1, 2, 4, cap=[4, 4, 4, 4], n_protect=0, dense=MODES[mode]["dense"])
    o.append(np_bits(k), np_bits(k), cls.numpy(), pos.numpy())
    out = gpu.decode_attention(q.to(DEV), SCALE).cpu().numpy()
    ref = o.attend(np_bits(q), SCALE)
    assert np.max(np.abs(out - ref)) <= OUT_ATOL
    g = gpu.export_state()
    assert abs(g["score3"][0, 0] - 4.0) < 1e-6 and abs(g["score3"][1, 0] - 4.0) < 1e-6


@pytest.mark.parametrize("mode", list(MODES))
def test_budget_edge_cases(mode):
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", ctx=300, n_protect=17, **MODES[mode])
    gpu.decode_attention(synth.decode_inputs(w, 0)[4].to(DEV), SCALE)
    before = gpu.export_state()
    gpu.evict_compact(300)                     # budget >= candidates: untouched
    after = gpu.export_state()
    for key in before:
        assert np.array_equal(before[key], after[key]), key
    _evict_lockstep(gpu, o, rows, 0)           # evict every unprotected token
    g = gpu.export_state()
    assert (g["n"].sum(axis=1) == 17).all()


@pytest.mark.parametrize("ctx", [500, 3000])
def test_all_scores_equal_keep_lowest_positions(ctx):
    """Equal scores: every key differs only in its position bits, so the radix
    select runs through all score digits with every candidate still in play."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", ctx=ctx)
    views = gpu.state_views()
    for c in range(4):
        views[f"score{c}"].fill_(0.5)
    _evict_lockstep(gpu, o, rows, 40)
    g = gpu.export_state()
    for s in range(gpu.S):
        kept = sorted(np.concatenate([g[f"pos{c}"][s, :g["n"][s, c]] for c in range(4)]).tolist())
        assert kept == list(range(44))


@pytest.mark.parametrize("dense", [False, True], ids=["reuse", "dense"])
def test_exact_key_ties_resolved_by_class_then_index(dense):
    """Duplicate positions with equal scores: the 64-bit key ties, so class then table
    index decide (same rule on both sides)."""
    B, Hkv, T = 1, 1, 40
    gpu = TkvCache(B, Hkv, 4, cap=[4, 40, 40, 40], n_protect=0, max_append=T, dense=dense)
    o = orc.OracleCache(B, Hkv, 4, cap=[4, 40, 40, 40], n_protect=0, dense=dense)
    k = synth.normal_bf16(3, 0, synth.TID_K, B, Hkv, 0, T, 128)
    cls = torch.tensor([[1 + (t % 3) for t in range(T)]], dtype=torch.uint8)
    pos = torch.tensor([[t // 4 for t in range(T)]], dtype=torch.int32)   # duplicates
    gpu.quantize_append(k.to(DEV), k.to(DEV), cls.to(DEV), pos.to(DEV))
    views = gpu.state_views()
    for c in range(4):
        views[f"score{c}"].copy_((views[f"pos{c}"] % 3).float() * 0.25)
    o.load_state(gpu.export_state())
    for budget in (13, 7, 1):
        gpu.evict_compact(budget)
        o.evict(budget)
        compare_states(gpu.export_state(), o.state, what=f"tie budget {budget}")


def test_device_errors_capacity_and_invalid_class():
    gpu = TkvCache(1, 2, 4, cap=[1, 2, 2, 2], n_protect=1, max_append=8)
    k = synth.normal_bf16(0, 0, synth.TID_K, 1, 2, 0, 5, 128).to(DEV)
    cls = torch.tensor([[1, 1, 1, 1, 2]], dtype=torch.uint8, device=DEV)
    pos = torch.arange(5, dtype=torch.int32, device=DEV).view(1, 5)
    gpu.quantize_append(k, k, cls, pos)        # class 1 gets 4 tokens but has 2 slots
    assert gpu.poll_error() == tkv.TKV_ERR_CAPACITY
    assert gpu.poll_error() == tkv.TKV_OK      # cleared by the poll
    g = gpu.export_state()
    assert g["n"][0].tolist() == [1, 2, 1, 0] and g["hw"][0].tolist() == [1, 2, 1, 0]
    gpu2 = TkvCache(1, 1, 4, cap=[4, 4, 4, 4], n_protect=0)
    gpu2.quantize_append(k[:, :1, :1].contiguous(), k[:, :1, :1].contiguous(),
                         torch.tensor([[9]], dtype=torch.uint8, device=DEV),
                         torch.zeros((1, 1), dtype=torch.int32, device=DEV))
    assert gpu2.poll_error() == tkv.TKV_ERR_INVALID
    assert gpu2.export_state()["n"].sum() == 0


def test_binding_rejects_wrong_tensors():
    gpu = TkvCache(1, 2, 4, cap=[4, 4, 4, 4], n_protect=0)
    q = torch.zeros((1, 8, 128), dtype=torch.float32, device=DEV)
    with pytest.raises(TkvError):
        gpu.decode_attention(q, SCALE)
    with pytest.raises(TkvError):
        gpu.decode_attention(q.to(torch.bfloat16)[:, :4], SCALE)


# ----------------------------------------------------------------------------
# The workload shapes of the decode configurations, lock-step on sampled rows/steps
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", list(MODES))
def test_b64_ctx32k_timed_step_sampled_rows(mode):
    """Batch 64 x 32/8 heads, 32k context, K outliers, 5 % budget + 128-token bf16
    window: prefill, scoring step, eviction to 1638, then the timed step
    (append + attention), compared on three sampled batch rows."""
    rows = [0, 37, 63]
    w = synth.prefill_inputs("b64_ctx32k_evict5pct", device=DEV, steps=2)
    w["cls"] = synth.class_ids(0, w["B"], w["ctx"] + 2, w["p_r"], w["p_e"])
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
    dense = gpu.dense
    gpu.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(DEV), w["pos"].to(DEV))
    del w["k"], w["v"]
    torch.cuda.empty_cache()
    o = oracle_for(gpu, gpu.export_state(rows_streams(gpu, rows)), B=len(rows))
    _decode_step(w, gpu, o, rows, 0)                 # scoring step
    _evict_lockstep(gpu, o, rows, w["budget"])
    err = _decode_step(w, gpu, o, rows, 1)           # the timed step's work
    assert err <= OUT_ATOL
    if dense:
        _assert_dense(gpu)


@pytest.mark.parametrize("mode", list(MODES))
def test_b8_ctx16k_decode_loop_sampled_steps(mode):
    """Batch 8 x 32/8 heads, 16k context, 256 decode steps with eviction to 1638
    every 128 steps; lock-step checks on one row at steps 0, 127, 128, 255."""
    rows = [5]
    w = synth.prefill_inputs("b8_ctx16k_256steps", device=DEV)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
    gpu.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(DEV), w["pos"].to(DEV))
    o = oracle_for(gpu, gpu.export_state(rows_streams(gpu, rows)), B=1)
    for step in range(w["steps"]):
        if step in (0, 127, 128, 255):
            _decode_step(w, gpu, o, rows, step)
        else:
            k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
            gpu.quantize_append(k, v, cls, pos)
            gpu.decode_attention(q, SCALE)
        if (step + 1) % w["evict_every"] == 0:
            if step == 127:
                _evict_lockstep(gpu, o, rows, w["budget"])
            else:
                gpu.evict_compact(w["budget"])
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_b1_ctx131k_long_decode_sampled_steps(mode):
    """Batch 1 x 64/8 heads (G = 8), 131k context, transition-heavy segments,
    eviction to 4096 every 64 steps; lock-step at steps 0, 63, 64 and 200."""
    rows = [0]
    w = synth.prefill_inputs("b1_ctx131k_512steps", device=DEV, steps=201)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
    gpu.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(DEV), w["pos"].to(DEV))
    o = oracle_for(gpu, gpu.export_state(), B=1)
    for step in range(201):
        if step in (0, 63, 64, 200):
            _decode_step(w, gpu, o, rows, step)
        else:
            k, v, cls, pos, q = synth.decode_inputs(w, step, device=DEV)
            gpu.quantize_append(k, v, cls, pos)
            gpu.decode_attention(q, SCALE)
        if (step + 1) % w["evict_every"] == 0:
            if step == 63:
                _evict_lockstep(gpu, o, rows, w["budget"])
            else:
                gpu.evict_compact(w["budget"])
    assert gpu.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("mode", list(MODES))
def test_l32_b32_ctx32k_decode_loop_sampled_layers_and_steps(mode):
    """32 layers x batch 32 x 32/8 heads, 32k context with K outliers and a 128-token
    bf16 window, 1024 decode steps with eviction to 1638 every 64 steps.  Every layer
    runs every step; lock-step oracle checks on one batch row of layers 0 and 31 at
    steps 0, 63 (and the eviction after it), 64 and 1023."""
    name = "l32_b32_ctx32k_1024steps"
    spec = synth.WORKLOADS[name]
    L, steps, E = spec["layers"], spec["steps"], spec["evict_every"]
    rows, check_layers, check_steps = [3], (0, L - 1), (0, 63, 64, steps - 1)
    caches, ws, oracles = [], [], {}
    for layer in range(L):
        w = synth.prefill_inputs(name, layer=layer, device=DEV)
        cache = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"],
                         **MODES[mode])
        cache.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(DEV),
                              w["pos"].to(DEV))
        del w["k"], w["v"]
        caches.append(cache)
        ws.append(w)
        if layer in check_layers:
            oracles[layer] = oracle_for(cache, cache.export_state(rows_streams(cache, rows)), B=1)
    torch.cuda.synchronize()
    B, Hkv, Hq, D, ctx = spec["B"], spec["Hkv"], spec["Hq"], spec["D"], spec["ctx"]
    cls_dev = ws[0]["cls"][:, ctx:ctx + steps].contiguous().to(DEV)
    for c0 in range(0, steps, 64):
        chunk = []
        for layer in range(L):
            seed = ws[layer]["seed"]
            k = synth.normal_bf16(seed, layer, synth.TID_K, B, Hkv, ctx + c0, 64, D, DEV)
            k = synth.apply_k_outliers(k, seed, layer)
            v = synth.normal_bf16(seed, layer, synth.TID_V, B, Hkv, ctx + c0, 64, D, DEV)
            q = synth.normal_bf16(seed, layer, synth.TID_Q, B, Hq, ctx + c0, 64, D, DEV)
            chunk.append((k, v, q))
        for j in range(64):
            step = c0 + j
            pos = torch.full((B, 1), ctx + step, dtype=torch.int32, device=DEV)
            cls = cls_dev[:, step:step + 1].contiguous()
            for layer in range(L):
                if layer in check_layers and step in check_steps:
                    _decode_step(ws[layer], caches[layer], oracles[layer], rows, step)
                    continue
                k, v, q = chunk[layer]
                caches[layer].quantize_append(k[:, :, j:j + 1].contiguous(), v[:, :, j:j + 1].contiguous(),
                                              cls, pos)
                caches[layer].decode_attention(q[:, :, j].contiguous(), SCALE)
            if (step + 1) % E == 0:
                for layer in range(L):
                    if layer in check_layers and step == 63:
                        _evict_lockstep(caches[layer], oracles[layer], rows, spec["budget"])
                    else:
                        caches[layer].evict_compact(spec["budget"])
    for cache in caches:
        assert cache.poll_error() == tkv.TKV_OK


@pytest.mark.parametrize("dense", [False, True], ids=["reuse", "dense"])
def test_local_window_eviction(dense):
    """Top-k with a local window of the 200 most recent positions (DYNTS 2.3): the
    window and the protected sinks stay, the budget applies to the rest; a window
    past every position is the plain eviction."""
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=2, dense=dense)
    _decode_step(w, gpu, o, rows, 0)
    keep_from = w["ctx"] + 1 - 200
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    gpu.evict_compact_window(300, keep_from)
    assert o.evict_window(300, keep_from) == 0
    g = gpu.export_state(sub)
    compare_states(g, o.state, what="local window")
    assert (g["n"].sum(axis=1) == w["n_protect"] + 300 + 200).all()
    before = gpu.export_state()
    gpu.evict_compact_window(300, keep_from)     # the same window again: nothing to evict
    after = gpu.export_state()
    for key in before:
        assert np.array_equal(before[key], after[key]), key
    o.load_state(gpu.export_state(sub))          # window past every position: plain top-k
    gpu.evict_compact_window(100, 1 << 30)
    assert o.evict(100) == 0
    compare_states(gpu.export_state(sub), o.state, what="window past every position")
    assert gpu.poll_error() == tkv.TKV_OK


def _scaled_case(mode, k_scale, v_scale, q_fn):
    """The 709-token two-row workload with its 4 bf16 sink tokens' K / V scaled by
    k_scale / v_scale (exactly, in bf16) and the query transformed by q_fn."""
    w = synth.prefill_inputs("tiny_b1_ctx2k", B=2, Hq=8, Hkv=2, ctx=709, n_protect=4, steps=2)
    w["k"][:, :, :4] = (w["k"][:, :, :4].float() * k_scale).to(torch.bfloat16)
    w["v"][:, :, :4] = (w["v"][:, :, :4].float() * v_scale).to(torch.bfloat16)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], **MODES[mode])
    gpu.quantize_append(w["k"].to(DEV), w["v"].to(DEV), w["cls"][:, :w["ctx"]].contiguous().to(DEV),
                        w["pos"].to(DEV))
    o = oracle_for(gpu, gpu.export_state())
    q = q_fn(synth.decode_inputs(w, 0)[4].float()).to(torch.bfloat16)
    out = gpu.decode_attention(q.to(DEV), SCALE).cpu().numpy()
    ref = o.attend(np_bits(q), SCALE)
    assert np.isfinite(out).all(), "non-finite output"
    # an fp32 output of magnitude |ref| >> 1 cannot be closer than its own rounding, so
    # the 2e-3 bound applies to max(1, |ref|)
    err = np.abs(out.astype(np.float64) - ref) / np.maximum(1.0, np.abs(ref))
    assert float(err.max()) <= OUT_ATOL, float(err.max())
    assert gpu.poll_error() == tkv.TKV_OK
    return float(err.max())


@pytest.mark.parametrize("mode", list(MODES))
def test_extreme_magnitudes_sinks_and_query(mode):
    """bf16 sink keys / values around 1e5 (beyond f16's range), query entries around
    +-1e5 in one dim per head, and a query scaled below 2^-14 (f16-subnormal) against
    sink keys scaled up by 2^20: every path keeps bf16 values and the query without
    narrowing them (ThinKV, TBQ: protected tokens stay at full precision)."""
    _scaled_case(mode, 1e5, 1e5, lambda q: q)

    def spike(q):
        q = q.clone()
        q[:, :, 17] = 1e5
        q[:, ::2, 90] = -1e5
        return q
    _scaled_case(mode, 1.0, 1.0, spike)
    _scaled_case(mode, 2.0 ** 20, 8.0, lambda q: q * 2.0 ** -20)


SPARSITY_ATOL = 2e-5


SPARSITY_MODES = {"warp_dense": dict(dense=True), "warp_reuse": dict(dense=False),
                  "tc": dict(dense=True, attn_kernel=1)}


@pytest.mark.parametrize("mode", list(SPARSITY_MODES))
@pytest.mark.parametrize("G,ctx,n_protect,B,Hkv", [(4, 2000, 128, 2, 2), (8, 709, 4, 2, 2), (1, 3000, 0, 2, 2),
                                                   (4, 24000, 4, 1, 2), (4, 300, 4, 40, 8)])
def test_attention_sparsity_statistic(G, ctx, n_protect, B, Hkv, mode):
    """tkv_decode_attention_sparsity: the step's output and scores as in a plain decode
    call, plus per (stream, head) 1 - H(p) / ln N against the oracle's fp64 value and
    the thought class under the thresholds (ThinKV, Metodologia: thought types differ in
    the sparsity of their attention).  The warp-tile kernel's three layouts: clusters
    (4 streams), the split with the merge pass (2 streams of 24k) and one CTA per stream
    (320 streams)."""
    rows = [0, 1] if B > 1 else [0]
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", rows=rows, B=B, Hq=Hkv * G, Hkv=Hkv, ctx=ctx,
                                 n_protect=n_protect, steps=2, **SPARSITY_MODES[mode])
    k, v, cls, pos, q = synth.decode_inputs(w, 0)
    sub = rows_streams(gpu, rows)
    o.load_state(gpu.export_state(sub))
    gpu.quantize_append(k.to(DEV), v.to(DEV), cls.to(DEV), pos.to(DEV))
    assert o.append(np_bits(k[rows]), np_bits(v[rows]), cls[rows].numpy(), pos[rows].numpy()) == 0
    ref_sp = o.attention_sparsity(np_bits(q[rows]), SCALE).reshape(len(rows), -1)
    th_r, th_t = float(np.quantile(ref_sp, 0.3)), float(np.quantile(ref_sp, 0.7))
    out, sp, thought = gpu.decode_attention_sparsity(q.to(DEV), SCALE, th_r, th_t)
    ref = o.attend(np_bits(q[rows]), SCALE)
    assert float(np.max(np.abs(out[rows].cpu().numpy() - ref))) <= OUT_ATOL
    compare_states(gpu.export_state(sub), o.state, scores="tol", what="sparsity step")
    got = sp[rows].cpu().numpy().astype(np.float64)
    assert float(np.max(np.abs(got - ref_sp))) <= SPARSITY_ATOL
    th = thought[rows].cpu().numpy()
    for i in np.ndindex(ref_sp.shape):
        near = min(abs(ref_sp[i] - th_r), abs(ref_sp[i] - th_t)) <= SPARSITY_ATOL
        if not near:
            assert th[i] == orc.classify_sparsity(ref_sp[i], th_r, th_t), i
    assert gpu.poll_error() == tkv.TKV_OK


def test_attention_sparsity_rejects_the_persistent_pipeline_and_bad_thresholds():
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=1, dense=True, attn_kernel=2)
    q = synth.decode_inputs(w, 0)[4].to(DEV)
    with pytest.raises(TkvError):
        gpu.decode_attention_sparsity(q, SCALE)
    for kernel in (0, 1):
        w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=1, dense=True, attn_kernel=kernel)
        q = synth.decode_inputs(w, 0)[4].to(DEV)
        with pytest.raises(TkvError):
            gpu.decode_attention_sparsity(q, SCALE, 0.8, 0.2)   # th_r > th_t



@pytest.mark.parametrize("mode", ["dense", "dense_tc", "dense_ws"])
@pytest.mark.parametrize("seed", [0, 1])
def test_ragged_streams_with_empty_classes_and_streams(mode, seed):
    """Dense caches whose streams hold very different numbers of entries per class --
    empty classes, empty streams, single entries, full tiles plus a ragged tail -- so the
    persistent kernels' byte-balanced split puts several streams in one CTA, one stream
    over several CTAs, and leaves CTAs with no tile at all."""
    rng = np.random.default_rng(900 + seed)
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", B=6, Hq=16, Hkv=4, ctx=700, n_protect=5, steps=2,
                                 **MODES[mode])
    st = gpu.export_state()
    for s_ in range(gpu.S):
        for c in range(4):
            n = int(st["n"][s_, c])
            pick = rng.choice([0, 1, n // 3, n, max(n - 1, 0), int(rng.integers(0, n + 1))])
            st["n"][s_, c] = min(n, pick)
            st["hw"][s_, c] = st["n"][s_, c]
    st["n"][3] = 0                     # one empty stream
    st["hw"][3] = 0
    gpu.import_state(st)
    o.load_state(gpu.export_state(rows_streams(gpu, rows)))
    for step in range(2):
        _decode_step(w, gpu, o, rows, step)
    assert gpu.poll_error() == tkv.TKV_OK
