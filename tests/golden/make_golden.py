"""Writes tiny_b1_ctx2k.json: digests of the oracle's state and output on the
2048-token workload (prefill, one decode step, eviction to 512).  Calls only the
oracle (and the seeded input generator).  Run: python -m tests.golden.make_golden"""
import hashlib
import json
import os

import numpy as np

import synth
from oracle import oracle as orc
from tests.helpers import bits_of, class_capacities

D = 128


def _digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()[:32]


def run_tiny():
    w = synth.WORKLOADS["tiny_b1_ctx2k"]
    B, Hkv, Hq, ctx = w["B"], w["Hkv"], w["Hq"], w["ctx"]
    G = Hq // Hkv
    cls = synth.class_ids(0, B, ctx + 1, w["p_r"], w["p_e"])
    cache = orc.OracleCache(B, Hkv, G, cap=class_capacities(cls, w["n_protect"], extra=1),
                            n_protect=w["n_protect"])
    k = synth.normal_bf16(0, 0, synth.TID_K, B, Hkv, 0, ctx + 1, D)
    v = synth.normal_bf16(0, 0, synth.TID_V, B, Hkv, 0, ctx + 1, D)
    kb, vb = bits_of(k), bits_of(v)
    pos = synth.positions(B, 0, ctx + 1).numpy()
    c = cls.numpy()
    assert cache.append(kb[:, :, :ctx], vb[:, :, :ctx], c[:, :ctx], pos[:, :ctx]) == 0
    assert cache.append(kb[:, :, ctx:], vb[:, :, ctx:], c[:, ctx:], pos[:, ctx:]) == 0
    q = synth.normal_bf16(0, 0, synth.TID_Q, B, Hq, ctx, 1, D)[:, :, 0]
    out = cache.attend(bits_of(q), 1 / np.sqrt(D))
    assert cache.evict(w["budget"]) == 0
    res = {"out": _digest(out), "out_sum": float(np.float64(out).sum()),
           "n": cache.state["n"].tolist(), "ft": cache.state["ft"].tolist(),
           "hw": cache.state["hw"].tolist()}
    for cc in range(4):
        n = cache.state["n"]
        res[f"table{cc}"] = _digest(np.concatenate(
            [np.stack([cache.state[f"handle{cc}"][s, :n[s, cc]], cache.state[f"pos{cc}"][s, :n[s, cc]],
                       cache.state[f"score{cc}"][s, :n[s, cc]].view(np.int32)]).ravel()
             for s in range(cache.S)]))
        res[f"pool{cc}"] = _digest(cache.state[f"pool{cc}"])
    return res


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(__file__), "tiny_b1_ctx2k.json")
    json.dump(run_tiny(), open(path, "w"), indent=1)
    print("wrote", path)
