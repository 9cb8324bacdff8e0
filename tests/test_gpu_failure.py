"""Failure reporting on the GPU without any fault: a bounded device wait that must
give up (the barrier it waits on never completes) latches TKV_ERR_TIMEOUT, which
tkv_poll_error reports once; the context and the cache stay usable afterwards."""
import numpy as np
import pytest
import torch

import synth
from reasoning_model_kv_b200 import TkvCache, tkv
from tests.conftest import gpu_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]


def test_bounded_wait_gives_up_and_reports_timeout():
    gpu = TkvCache(1, 2, 4, cap=[4, 4, 4, 4], n_protect=0)
    assert gpu.poll_error() == tkv.TKV_OK
    n0 = gpu.launch_count()
    gpu.selftest_wait_timeout(1 << 20)             # about half a millisecond of waiting
    assert gpu.poll_error() == tkv.TKV_ERR_TIMEOUT
    assert gpu.poll_error() == tkv.TKV_OK          # cleared by the poll
    assert gpu.launch_count() == n0 + 1
    # the context and the cache still work: an append and an attention step
    k = synth.normal_bf16(0, 0, synth.TID_K, 1, 2, 0, 1, 128).cuda()
    q = synth.normal_bf16(0, 0, synth.TID_Q, 1, 8, 0, 1, 128)[:, :, 0].contiguous().cuda()
    gpu.quantize_append(k, k, torch.tensor([[2]], dtype=torch.uint8, device="cuda"),
                        torch.zeros((1, 1), dtype=torch.int32, device="cuda"))
    out = gpu.decode_attention(q, 128 ** -0.5).cpu().numpy()
    assert np.isfinite(out).all() and np.abs(out).max() > 0
    assert gpu.poll_error() == tkv.TKV_OK
