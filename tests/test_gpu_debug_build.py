"""The bounds-checking build (libtkv_debug.so, TKV_DEBUG): the same results as the
release build, and a corrupted state is reported instead of indexed with.

It runs in a child process (the library is chosen per process through TKV_LIBRARY).
The child decodes one step of the 2k workload in every cache mode against the oracle,
then imports a state whose class-1 entry count of stream 0 exceeds its capacity and
runs append, attention and eviction on it: the debug checks must clamp or skip every
access that count would take out of range and report TKV_ERR_INVALID."""
import json
import os
import subprocess
import sys
from pathlib import Path

import pytest

from tests.conftest import gpu_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

ROOT = Path(__file__).resolve().parents[1]

CHILD = r'''
import json, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import synth
from reasoning_model_kv_b200 import tkv
from tests.gpu_harness import MODES, build_pair, np_bits
res = {"lib": str(tkv.LIB_PATH)}
for mode in MODES:
    w, gpu, o, rows = build_pair("tiny_b1_ctx2k", **MODES[mode])
    k, v, cls, pos, q = synth.decode_inputs(w, 0)
    o.load_state(gpu.export_state())
    gpu.quantize_append(k.cuda(), v.cuda(), cls.cuda(), pos.cuda())
    o.append(np_bits(k), np_bits(v), cls.numpy(), pos.numpy())
    out = gpu.decode_attention(q.cuda(), 128 ** -0.5).cpu().numpy()
    err = float(np.max(np.abs(out - o.attend(np_bits(q), 128 ** -0.5))))
    ok_status = gpu.poll_error()
    st = gpu.export_state()
    st["n"][0, 1] = gpu.cap[1] + 7                 # corrupt: more entries than slots
    gpu.import_state({"n": st["n"]})
    k, v, cls, pos, q = synth.decode_inputs(dict(w, cls=synth.class_ids(0, 1, w["ctx"] + 2, 0.4, 0.4)), 1)
    cls[:] = 1
    gpu.quantize_append(k.cuda(), v.cuda(), cls.cuda(), pos.cuda())
    gpu.decode_attention(q.cuda(), 128 ** -0.5)
    gpu.evict_compact(w["budget"])
    torch.cuda.synchronize()
    res[mode] = {"err": err, "status_clean": int(ok_status), "status_corrupt": int(gpu.poll_error())}
print("RESULT " + json.dumps(res))
'''


def test_debug_build_matches_and_reports_out_of_range_counts():
    from reasoning_model_kv_b200 import build as b
    lib = b.build(debug=True)
    env = dict(os.environ, TKV_LIBRARY=str(lib))
    r = subprocess.run([sys.executable, "-c", CHILD, str(ROOT)], env=env, cwd=str(ROOT),
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert res["lib"].endswith("libtkv_debug.so")
    for mode, m in res.items():
        if mode == "lib":
            continue
        assert m["err"] <= 2e-3, (mode, m)
        assert m["status_clean"] == 0, (mode, m)
        assert m["status_corrupt"] == 1, (mode, m)     # TKV_ERR_INVALID
