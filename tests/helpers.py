"""Small helpers shared by the tests (input conversion and workload set-up only)."""
from __future__ import annotations

import numpy as np
import torch

import synth


def bf16_bits(x) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even) and return the uint16 bit patterns."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> uint16 numpy array of its bit patterns."""
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def class_capacities(cls: torch.Tensor, n_protect: int, pos0: int = 0, extra: int = 0):
    """Slots needed per class (max over batch rows) for the given class ids."""
    B, T = cls.shape
    pos = torch.arange(pos0, pos0 + T).view(1, T).expand(B, T)
    eff = torch.where(pos < n_protect, torch.zeros_like(cls), cls)
    caps = []
    for c in range(4):
        caps.append(int((eff == c).sum(dim=1).max().item()) + extra)
    return caps


def make_workload(name: str, seed: int = 0, layer: int = 0, **over):
    """Prefill inputs of a named workload (CPU tensors)."""
    w = dict(synth.WORKLOADS[name])
    w.update(over)
    B, Hkv, D, ctx = w["B"], w["Hkv"], w["D"], w["ctx"]
    k = synth.normal_bf16(seed, layer, synth.TID_K, B, Hkv, 0, ctx, D)
    v = synth.normal_bf16(seed, layer, synth.TID_V, B, Hkv, 0, ctx, D)
    if w["outliers"]:
        k = synth.apply_k_outliers(k, seed, layer)
    total = ctx + w["steps"]
    cls = synth.class_ids(seed, B, total, w["p_r"], w["p_e"])
    return w, k, v, cls
