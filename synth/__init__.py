"""Seeded synthetic inputs for the compressed-KV decode path.

This module only *makes inputs*: it holds none of the method's arithmetic
(no quantisation, attention, scoring or eviction).  Both the CPU oracle
tests and the CUDA path draw their inputs from here, so that any tensor can be
regenerated bit for bit on either device, or for any slice of positions.

Generator
---------
Every value is a pure function of a counter, so CPU and GPU agree exactly:

* ``splitmix64`` (Steele, Lea & Flood 2014; the finaliser popularised by
  Vigna) mixes a 64-bit counter.  It is evaluated with wrapping int64 torch
  ops, which behave the same on CPU and CUDA.
* An approximately N(0, 1) value is an Irwin-Hall sum of twelve 16-bit
  uniforms taken from three hashes, minus six.  The integer sum is exact, the
  division by 2**16 is exact in fp32, and the only rounding is the final
  fp32 -> bf16 round-to-nearest-even, so no transcendental function is
  involved.
* The counter of element (b, head, pos, dim) of tensor ``tid`` is
  ``base(seed, layer, tid) ^ ((((b * 2**8 + head) * 2**24 + pos) * 2**8 + dim) * 4 + k)``
  for hash k = 0, 1, 2.  Positions are absolute, so the K/V of a decode step
  at position p equals what a prefill that reached p would have produced.

Thought segments (ThinKV: thought types R/E/T, "Metodologia"): per batch row,
one sequence of segments from position 0; each has a length drawn uniformly
from [32, 256] and a label R/E/T drawn with the given probabilities.  Labels
are returned as class ids 1 (R), 2 (E), 3 (T).

K outlier channels: for configurations with outliers, four distinct channels
per (layer, kv head) are picked by hash and their K values are multiplied by
10 in fp32, then rounded to bf16.
"""
from __future__ import annotations

import numpy as np
import torch

MASK64 = (1 << 64) - 1
TID_K, TID_V, TID_Q, TID_OUTLIER, TID_SEGMENT = 1, 2, 3, 4, 5

CLS_BF16, CLS_R, CLS_E, CLS_T = 0, 1, 2, 3


def _s64(x: int) -> int:
    """Python int in [0, 2**64) -> the int64 with the same bits."""
    x &= MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


_C0 = _s64(0x9E3779B97F4A7C15)
_C1 = _s64(0xBF58476D1CE4E5B9)
_C2 = _s64(0x94D049BB133111EB)


def splitmix64_int(x: int) -> int:
    """splitmix64 finaliser on a Python int (unsigned 64-bit result)."""
    z = (x + 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64_t(x: torch.Tensor) -> torch.Tensor:
    """splitmix64 finaliser on an int64 tensor (wrapping arithmetic)."""
    z = x + _C0
    z = (z ^ _lsr(z, 30)) * _C1
    z = (z ^ _lsr(z, 27)) * _C2
    return z ^ _lsr(z, 31)


def stream_base(seed: int, layer: int, tid: int) -> int:
    h = splitmix64_int(seed & MASK64)
    h = splitmix64_int(h ^ (layer & MASK64))
    h = splitmix64_int(h ^ tid)
    return h


def _normal_from_counters(base: int, ctr: torch.Tensor) -> torch.Tensor:
    """ctr: int64 tensor of element counters (already shifted by 2 bits)."""
    b64 = torch.tensor(_s64(base), dtype=torch.int64, device=ctr.device)
    acc = torch.zeros(ctr.shape, dtype=torch.int64, device=ctr.device)
    for k in range(3):
        h = splitmix64_t((ctr + k) ^ b64)
        for f in range(4):
            acc += _lsr(h, 16 * f) & 0xFFFF
    x = (acc - 6 * 65536).to(torch.float32) / 65536.0
    return x.to(torch.bfloat16)


def normal_bf16(seed: int, layer: int, tid: int, B: int, H: int, pos0: int, T: int,
                D: int, device="cpu", b0: int = 0) -> torch.Tensor:
    """bf16 tensor [B, H, T, D] for batch rows b0..b0+B-1, positions pos0..pos0+T-1."""
    assert D <= 256 and H <= 256 and pos0 + T <= (1 << 24) and b0 + B <= (1 << 10)
    dev = torch.device(device)
    b = torch.arange(b0, b0 + B, dtype=torch.int64, device=dev).view(B, 1, 1, 1)
    h = torch.arange(H, dtype=torch.int64, device=dev).view(1, H, 1, 1)
    p = torch.arange(pos0, pos0 + T, dtype=torch.int64, device=dev).view(1, 1, T, 1)
    d = torch.arange(D, dtype=torch.int64, device=dev).view(1, 1, 1, D)
    ctr = ((((b * 256 + h) * (1 << 24) + p) * 256 + d) * 4)
    return _normal_from_counters(stream_base(seed, layer, tid), ctr)


def normal_bf16_chunked(seed, layer, tid, B, H, pos0, T, D, device="cpu", b0: int = 0,
                        chunk_elems: int = 1 << 26):
    """Same values as ``normal_bf16``; generated in position chunks to bound temporaries."""
    out = torch.empty((B, H, T, D), dtype=torch.bfloat16, device=device)
    chunk_T = max(1, chunk_elems // max(1, B * H * D))
    for t0 in range(0, T, chunk_T):
        tt = min(chunk_T, T - t0)
        out[:, :, t0:t0 + tt] = normal_bf16(seed, layer, tid, B, H, pos0 + t0, tt, D, device, b0)
    return out


def outlier_channels(seed: int, layer: int, kvh: int, D: int, n: int = 4) -> list[int]:
    """n distinct K channels of kv head ``kvh`` that carry x10 outliers."""
    base = stream_base(seed, layer, TID_OUTLIER)
    chans: list[int] = []
    ctr = 0
    while len(chans) < n:
        c = splitmix64_int(base ^ ((kvh << 16) + ctr)) % D
        ctr += 1
        if c not in chans:
            chans.append(c)
    return chans


def apply_k_outliers(k: torch.Tensor, seed: int, layer: int, kvh0: int = 0, n: int = 4,
                     factor: float = 10.0) -> torch.Tensor:
    """k: bf16 [B, H, T, D] whose head axis starts at kv head ``kvh0``; returns a new tensor."""
    k = k.clone()
    D = k.shape[-1]
    for j in range(k.shape[1]):
        for c in outlier_channels(seed, layer, kvh0 + j, D, n):
            k[:, j, :, c] = (k[:, j, :, c].to(torch.float32) * factor).to(torch.bfloat16)
    return k


def segment_labels(seed: int, b: int, T: int, p_r: float, p_e: float,
                   min_len: int = 32, max_len: int = 256) -> tuple[list[int], list[int]]:
    """(labels, lengths) of the thought segments of batch row b covering [0, T)."""
    base = stream_base(seed, 0, TID_SEGMENT)
    thr_r = round(p_r * 65536)
    thr_e = round((p_r + p_e) * 65536)
    span = max_len - min_len + 1
    labels, lengths = [], []
    covered, i = 0, 0
    while covered < T:
        h = splitmix64_int(base ^ ((b << 32) + i))
        ln = min_len + (h & 0xFFFFFFFF) % span
        u = (h >> 48) & 0xFFFF
        lab = CLS_R if u < thr_r else (CLS_E if u < thr_e else CLS_T)
        labels.append(lab)
        lengths.append(ln)
        covered += ln
        i += 1
    return labels, lengths


def class_ids(seed: int, B: int, T: int, p_r: float, p_e: float) -> torch.Tensor:
    """uint8 [B, T]: thought class of every position (1=R, 2=E, 3=T)."""
    out = torch.empty((B, T), dtype=torch.uint8)
    for b in range(B):
        labels, lengths = segment_labels(seed, b, T, p_r, p_e)
        t = 0
        for lab, ln in zip(labels, lengths):
            e = min(T, t + ln)
            out[b, t:e] = lab
            t = e
            if t >= T:
                break
    return out


def segment_table(seed: int, B: int, upto: int, p_r: float, p_e: float, b0: int = 0,
                  max_seg: int | None = None):
    """Thought segments that have started by position `upto` (inclusive) in batch rows
    b0 .. b0 + B - 1: (starts int32 [B, max_seg], labels uint8 [B, max_seg],
    nseg int32 [B]); the last segment of a row is the open one.  Unused slots hold
    starts past every position and label 0."""
    rows = []
    for b in range(b0, b0 + B):
        labels, lengths = segment_labels(seed, b, upto + 1, p_r, p_e)
        starts, t = [], 0
        for ln in lengths:
            starts.append(t)
            t += ln
        rows.append((starts, labels))
    m = max_seg if max_seg is not None else max(len(r[0]) for r in rows)
    st = np.full((B, m), np.iinfo(np.int32).max, dtype=np.int32)
    lb = np.zeros((B, m), dtype=np.uint8)
    ns = np.zeros(B, dtype=np.int32)
    for i, (starts, labels) in enumerate(rows):
        n = min(len(starts), m)
        st[i, :n] = starts[:n]
        lb[i, :n] = labels[:n]
        ns[i] = n
    return st, lb, ns


def positions(B: int, pos0: int, T: int) -> torch.Tensor:
    """int32 [B, T] absolute positions pos0..pos0+T-1 for every batch row."""
    return torch.arange(pos0, pos0 + T, dtype=torch.int32).view(1, T).expand(B, T).contiguous()


# ---------------------------------------------------------------------------
# Workload configurations (shapes and distributions of the decode workloads)
# ---------------------------------------------------------------------------
WORKLOADS = {
    # single layer, 1 x (8 q heads / 2 kv heads), 2048-token cache, 4 bf16 sinks, budget 512
    "tiny_b1_ctx2k": dict(B=1, Hq=8, Hkv=2, D=128, ctx=2048, n_protect=4, p_r=0.4, p_e=0.4,
                          outliers=False, budget=512, steps=1, evict_every=1, layers=1),
    # batch 8, 32/8 heads, 16k context, 256 steps, 10 % budget every 128 steps
    "b8_ctx16k_256steps": dict(B=8, Hq=32, Hkv=8, D=128, ctx=16384, n_protect=4, p_r=0.4,
                               p_e=0.4, outliers=False, budget=1638, steps=256,
                               evict_every=128, layers=1),
    # batch 64, 32/8 heads, 32k context, K outliers, 5 % budget + 128-token bf16 window
    "b64_ctx32k_evict5pct": dict(B=64, Hq=32, Hkv=8, D=128, ctx=32768, n_protect=128,
                                 p_r=0.35, p_e=0.35, outliers=True, budget=1638, steps=1,
                                 evict_every=0, layers=1),
    # batch 1, 64/8 heads, 131k context, transition heavy, budget 4096 every 64 of 512 steps
    "b1_ctx131k_512steps": dict(B=1, Hq=64, Hkv=8, D=128, ctx=131072, n_protect=4, p_r=0.2,
                                p_e=0.3, outliers=False, budget=4096, steps=512,
                                evict_every=64, layers=1),
    # 32 layers, batch 32, 32/8 heads, 32k context, outliers, 5 % budget every 64 of 1024 steps
    "l32_b32_ctx32k_1024steps": dict(B=32, Hq=32, Hkv=8, D=128, ctx=32768, n_protect=128,
                                     p_r=0.4, p_e=0.4, outliers=True, budget=1638, steps=1024,
                                     evict_every=64, layers=32),
}


def class_counts(cls: torch.Tensor, n_protect: int, pos0: int = 0) -> list[int]:
    """Max over batch rows of the number of positions stored in each class
    (positions below n_protect count as class 0).  Used to size pools."""
    B, T = cls.shape
    pos = torch.arange(pos0, pos0 + T).view(1, T).expand(B, T)
    eff = torch.where(pos < n_protect, torch.zeros_like(cls), cls)
    return [int((eff == c).sum(dim=1).max().item()) for c in range(4)]


def prefill_inputs(name: str, seed: int = 0, layer: int = 0, device="cpu", b0: int = 0,
                   B: int | None = None, **over):
    """Inputs of a named workload: dict with the workload parameters plus
    k, v (bf16 [B, Hkv, ctx, D]), cls (uint8 [B, ctx + steps]), pos (int32 [B, ctx]),
    and cap (slots per class sized for the whole run)."""
    w = dict(WORKLOADS[name])
    w.update(over)
    if B is not None:
        w["B"] = B
    Bn, Hkv, D, ctx = w["B"], w["Hkv"], w["D"], w["ctx"]
    k = normal_bf16_chunked(seed, layer, TID_K, Bn, Hkv, 0, ctx, D, device, b0)
    v = normal_bf16_chunked(seed, layer, TID_V, Bn, Hkv, 0, ctx, D, device, b0)
    if w["outliers"]:
        k = apply_k_outliers(k, seed, layer)
    total = ctx + w["steps"]
    cls_all = class_ids(seed, b0 + Bn, total, w["p_r"], w["p_e"])[b0:]
    w.update(k=k, v=v, cls=cls_all, pos=positions(Bn, 0, ctx),
             cap=[c + 1 for c in class_counts(cls_all, w["n_protect"])],
             G=w["Hq"] // Hkv, seed=seed, layer=layer, b0=b0)
    return w


def decode_inputs(w: dict, step: int, device="cpu"):
    """Inputs of decode step `step` (position ctx + step): k, v [B, Hkv, 1, D],
    cls/pos [B, 1], q [B, Hq, D]."""
    B, Hkv, Hq, D, p = w["B"], w["Hkv"], w["Hq"], w["D"], w["ctx"] + step
    seed, layer, b0 = w["seed"], w["layer"], w.get("b0", 0)
    k = normal_bf16(seed, layer, TID_K, B, Hkv, p, 1, D, device, b0)
    if w["outliers"]:
        k = apply_k_outliers(k, seed, layer)
    v = normal_bf16(seed, layer, TID_V, B, Hkv, p, 1, D, device, b0)
    q = normal_bf16(seed, layer, TID_Q, B, Hq, p, 1, D, device, b0)[:, :, 0].contiguous()
    cls = w["cls"][:, p:p + 1].contiguous().to(device)
    pos = torch.full((B, 1), p, dtype=torch.int32, device=device)
    return k, v, cls, pos, q
