"""Lock-step comparison of the CUDA path (through the C ABI) with the CPU oracle.

The oracle is always handed the GPU's pre-call state for the streams under test,
applies the same call, and the post-call states are compared: codes, scales,
zeros, tables, counters and free stacks bit for bit; scores and outputs within
the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import oracle as orc
from reasoning_model_kv_b200 import TkvCache
from tests.helpers import bits_of

# Attention output: max-abs tolerance fixed by the target (fp32 output).
OUT_ATOL = 2e-3
# Scores: fp32 logits from 128-term dot products carry a relative error of at most
# ~128 * 2^-24 * sum|q_d k_d| / |q.k| in the worst case; with the magnitudes of
# these workloads that bounds the relative error of p, hence of a score, by 1e-4.
SCORE_RTOL = 1e-4
SCORE_ATOL = 1e-7


def oracle_for(gpu: TkvCache, state: dict, B: int | None = None) -> orc.OracleCache:
    """An oracle cache holding `state` (exported from `gpu`, possibly a subset of
    whole batch rows: B rows x Hkv streams)."""
    Bn = B if B is not None else gpu.B
    o = orc.OracleCache(Bn, gpu.Hkv, gpu.G, cap=gpu.cap, n_protect=gpu.n_protect, dense=gpu.dense,
                        codec=gpu.codec)
    o.load_state(state)
    return o


def rows_streams(gpu: TkvCache, rows):
    return [b * gpu.Hkv + h for b in rows for h in range(gpu.Hkv)]


def compare_states(g: dict, o: dict, *, scores="exact", what=""):
    S = g["n"].shape[0]
    for key in ("n", "ft", "hw"):
        assert np.array_equal(g[key], o[key]), f"{what}: {key} differs"
    bad_scores = 0
    for c in range(4):
        for s in range(S):
            n = o["n"][s, c]
            ft = o["ft"][s, c]
            assert np.array_equal(g[f"handle{c}"][s, :n], o[f"handle{c}"][s, :n]), f"{what}: handle{c} s={s}"
            assert np.array_equal(g[f"pos{c}"][s, :n], o[f"pos{c}"][s, :n]), f"{what}: pos{c} s={s}"
            assert np.array_equal(g[f"fs{c}"][s, :ft], o[f"fs{c}"][s, :ft]), f"{what}: fs{c} s={s}"
            hs = o[f"handle{c}"][s, :n]
            gr, orr = g[f"pool{c}"][s, hs], o[f"pool{c}"][s, hs]
            if not np.array_equal(gr, orr):
                i = int(np.nonzero((gr != orr).any(axis=1))[0][0])
                raise AssertionError(f"{what}: record class {c} stream {s} entry {i} slot {hs[i]} "
                                     f"differs at bytes {np.nonzero(gr[i] != orr[i])[0][:8]}")
            gs, os_ = g[f"score{c}"][s, :n], o[f"score{c}"][s, :n]
            if scores == "exact":
                assert np.array_equal(gs.view(np.int32), os_.view(np.int32)), f"{what}: score{c} s={s}"
            else:
                err = np.abs(gs.astype(np.float64) - os_.astype(np.float64))
                bad_scores += int((err > SCORE_RTOL * np.abs(os_) + SCORE_ATOL).sum())
    assert bad_scores == 0, f"{what}: {bad_scores} scores outside tolerance"


def score_error(g: dict, o: dict):
    worst = 0.0
    for c in range(4):
        for s in range(g["n"].shape[0]):
            n = o["n"][s, c]
            os_ = o[f"score{c}"][s, :n].astype(np.float64)
            gs = g[f"score{c}"][s, :n].astype(np.float64)
            if n:
                worst = max(worst, float(np.max(np.abs(gs - os_) / np.maximum(np.abs(os_), 1e-30))))
    return worst


def np_bits(t: torch.Tensor) -> np.ndarray:
    return bits_of(t)


# Cache modes the parity tests run in: placement and decode-attention kernel.
MODES = {"reuse": dict(dense=False), "dense": dict(dense=True),
         "dense_tc": dict(dense=True, attn_kernel=1), "dense_ws": dict(dense=True, attn_kernel=2)}


def build_pair(name: str, device="cuda", rows=None, dense=False, attn_kernel=0, codec=0, **over):
    """Prefill a GPU cache with a workload, and an oracle cache with the same
    inputs for batch rows `rows` (default: all); `dense` selects dense placement
    on both sides, `attn_kernel` the GPU's decode-attention kernel.  Returns
    (w, gpu, oracle, rows)."""
    w = synth.prefill_inputs(name, **over)
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], dense=dense,
                   attn_kernel=attn_kernel, codec=codec)
    k, v = w["k"].to(device), w["v"].to(device)
    cls = w["cls"][:, :w["ctx"]].contiguous().to(device)
    pos = w["pos"].to(device)
    gpu.quantize_append(k, v, cls, pos)
    rows = list(range(w["B"])) if rows is None else list(rows)
    o = orc.OracleCache(len(rows), w["Hkv"], w["G"], cap=w["cap"], n_protect=w["n_protect"], dense=dense,
                        codec=codec)
    st = o.append(np_bits(w["k"][rows]), np_bits(w["v"][rows]), w["cls"][rows, :w["ctx"]].numpy(),
                  w["pos"][rows].numpy())
    assert st == orc.ORC_OK
    return w, gpu, o, rows
