"""Benchmark of the compressed-KV decode step on B200.

Workload (default): batch 64 x 32 query / 8 kv heads, head_dim 128, 32k-token
context with x10 K outlier channels, R/E/T = 0.35/0.35/0.30 segments, a 128-token
bf16 question window, eviction to 1638 tokens, then the timed step: quantize-append
of the new token + decode attention with score accumulation.

One timed step = the new token's quantize-append + decode attention on every stream:
one tkv_decode_step call (default), or tkv_quantize_append then tkv_decode_attention
with --step-call separate (the same two launches).  The cache
counters are restored (untimed) before each step so every step sees the same
post-eviction cache, and the L2 is flushed (untimed) before each step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tkv|reference]

N > 1 runs under torchrun: every rank runs an independent replica (weak scaling,
no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

WORKLOAD = "b64_ctx32k_evict5pct"
METRIC = "decode-attn tokens/s & effective HBM GB/s on packed KV (fraction of 8 TB/s)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
SCALE = 128 ** -0.5
REC_BYTES = (512, 288, 160, 96)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["tkv", "reference"], default="tkv")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--placement", choices=["dense", "reuse"], default="dense",
                    help="record placement: dense (eviction moves kept records together, appends "
                         "go after them) or reuse (records stay put, evicted slots are reused)")
    ap.add_argument("--attn-kernel", choices=["warp", "tc", "ws"], default="warp",
                    help="decode-attention kernel: warp-tile mma.sync (default), the tcgen05 "
                         "tensor-memory kernel, or the warp-tile math on a persistent TMA pipeline "
                         "(the last two: dense placement only)")
    ap.add_argument("--evict-reps", type=int, default=5,
                    help="timed repetitions of the eviction that precedes the timed step")
    ap.add_argument("--evict", choices=["topk", "tbe", "tam"], default="topk",
                    help="eviction before the timed step: topk (each stream keeps its budget of "
                         "highest-scoring tokens), tbe (segment-level: the annealing schedule "
                         "over the rows' thought segments, r0 64, t_keep 16) or tam (the budget "
                         "split over segments in proportion to sqrt(mean score) x length, "
                         "tokens above 3x the mean score kept)")
    ap.add_argument("--codec", choices=["int", "fp"], default="int",
                    help="class record formats: int (8/4/2-bit integer codes) or fp (FP8 E4M3 / NVFP4 / "
                         "ternary; warp-tile kernel)")
    ap.add_argument("--full-reps", type=int, default=3,
                    help="timed attention calls on the full prefill context before the eviction "
                         "(the full-context phase; 0 skips it)")
    ap.add_argument("--step-call", choices=["step", "separate"], default="step",
                    help="the calls a step makes: step (tkv_decode_step, one call) or separate "
                         "(tkv_quantize_append, then tkv_decode_attention)")
    ap.add_argument("--decode-loop", action="store_true",
                    help="time the workload's whole decode loop instead of one step: every layer, "
                         "every step (append + attention), the periodic eviction, CUDA events "
                         "around each 64-step chunk (inputs are generated outside the timed chunks)")
    ap.add_argument("--loop-steps", type=int, default=None, help="decode steps of --decode-loop (default: the workload's)")
    ap.add_argument("--ctx", type=int, default=None,
                    help="prefill context before the eviction (default: the workload's); the "
                         "timed step is the same post-eviction step, with smaller pools")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (MEASURED_PEAKS.json absent)"


def stored_traffic(placement: str, attn_kernel: str):
    """DRAM bytes per attention launch from the committed ncu summary of this kernel,
    if it was taken on the current kernel sources (null otherwise)."""
    p = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"placement={placement},attn_kernel={attn_kernel}")
    if not d:
        return None
    m = hashlib.sha256()
    for f in d["sources"]:
        fp = os.path.join(ROOT, "reasoning_model_kv_b200", "csrc", f)
        if not os.path.exists(fp):
            return None
        m.update(open(fp, "rb").read())
    if d.get("sources_sha256_16") != m.hexdigest()[:16]:
        return None
    return d


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed loop runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


def gpu_smi_id(dev) -> str:
    """PCI bus id of the device, as nvidia-smi -i accepts it."""
    pr = torch.cuda.get_device_properties(dev)
    try:
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except AttributeError:
        return str(torch.cuda.current_device())


def reduce_max(vals, world: int, device) -> list:
    """Max over ranks of per-rank timings (every rank makes the same call)."""
    if world <= 1:
        return list(vals)
    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def packed_bytes(n: np.ndarray, rec=REC_BYTES) -> int:
    return int(sum(int(n[:, c].sum()) * rec[c] for c in range(4)))


# ----------------------------------------------------------------------------
def segment_inputs(w, dev, upto):
    """The rows' thought segments up to position `upto` and their retention under
    the library's TBE schedule, as device tensors for tkv_evict_segments."""
    from reasoning_model_kv_b200 import tkv
    st, lb, ns = synth.segment_table(w["seed"], w["B"], upto, w["p_r"], w["p_e"], b0=w.get("b0", 0))
    keep = torch.full(st.shape, -1, dtype=torch.int32)
    for b in range(w["B"]):
        n = int(ns[b])
        keep[b, :n] = torch.tensor(tkv.tkv_tbe_schedule(lb[b, :n].tolist(), 64, 16), dtype=torch.int32)
    return (torch.from_numpy(st).to(dev), torch.from_numpy(lb).to(dev), keep.to(dev),
            torch.from_numpy(ns).to(dev))


def setup_cache(w, dev, dense, evict_reps, flush, attn_kernel=0, evict="topk", full_reps=0, codec=0):
    """Prefill, one scoring step, then the eviction (to the budget, or the TBE
    schedule at the scoring step's position).  The eviction is timed (CUDA events,
    L2 flushed) over `evict_reps` repetitions, each from a copy of the pre-eviction
    workspace; it is not part of the timed decode step."""
    from reasoning_model_kv_b200 import TkvCache
    gpu = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"], dense=dense,
                   attn_kernel=attn_kernel, codec=codec)
    cls = w["cls"][:, :w["ctx"]].contiguous().to(dev)
    gpu.quantize_append(w["k"], w["v"], cls, w["pos"].to(dev))
    k, v, c, p, q = synth.decode_inputs(w, 0, device=dev)        # untimed scoring step
    gpu.quantize_append(k, v, c, p)
    gpu.decode_attention(q, SCALE)
    full = None
    if full_reps > 0:
        # the full-context phase (before any eviction): the attention call alone, L2
        # flushed, on the whole prefill; it adds to the scores, which the eviction reads
        # anyway (a second scoring step)
        out = torch.empty((w["B"], w["Hq"], 128), dtype=torch.float32, device=dev)
        n_full = gpu.state_views()["n"].cpu().numpy()
        ms = []
        st0 = torch.cuda.current_stream()
        for i in range(full_reps + 1):
            flush.zero_()
            a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st0)
            gpu.decode_attention(q, SCALE, out)
            b2.record(st0)
            b2.synchronize()
            if i > 0:
                ms.append(a.elapsed_time(b2))
        t = sum(ms) / len(ms)
        pkf = packed_bytes(n_full, list(gpu.layout.rec_bytes))
        full = {"live_kv_tokens": int(n_full.sum()), "packed_kv_bytes": pkf, "attention_ms": t,
                "hbm_gbs_packed": pkf / (t * 1e-3) / 1e9, "kv_tokens_per_s": int(n_full.sum()) / (t * 1e-3),
                "reps": full_reps}
    segs = segment_inputs(w, dev, w["ctx"]) if evict in ("tbe", "tam") else None
    evict_ms = []
    snap = gpu.workspace.clone() if evict_reps > 0 else None
    st = torch.cuda.current_stream()
    for i in range(evict_reps + 1 if evict_reps > 0 else 1):
        if snap is not None:
            gpu.workspace.copy_(snap)
        flush.zero_()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        if segs is None:
            gpu.evict_compact(w["budget"])
        elif evict == "tbe":
            gpu.evict_segments(*segs)
        else:
            gpu.evict_tam(segs[0], segs[1], segs[3], w["budget"], 3.0)
        b2.record(st)
        b2.synchronize()
        if i > 0:
            evict_ms.append(a.elapsed_time(b2))
    del snap
    torch.cuda.synchronize()
    assert gpu.poll_error() == 0
    return gpu, (statistics.median(evict_ms) if evict_ms else None), full


def run_tkv(args, rank, world, dev):
    over = {"ctx": args.ctx} if args.ctx else {}
    w = synth.prefill_inputs(args.workload, seed=rank, device=dev, steps=2, **over)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    gpu, evict_ms, full = setup_cache(w, dev, args.placement == "dense", args.evict_reps, flush,
                                      attn_kernel={"warp": 0, "tc": 1, "ws": 2}[args.attn_kernel], evict=args.evict,
                                      full_reps=args.full_reps, codec=1 if args.codec == "fp" else 0)
    del w["k"], w["v"]
    torch.cuda.empty_cache()
    views = gpu.state_views()
    saved = {k: views[k].clone() for k in ("n", "ft", "hw")}
    k, v, c, p, q = synth.decode_inputs(w, 1, device=dev)
    out = torch.empty((w["B"], w["Hq"], 128), dtype=torch.float32, device=dev)

    def restore():
        for key in ("n", "ft", "hw"):
            views[key].copy_(saved[key])

    def call_step(kk, vv, cc, pp, qq):
        if args.step_call == "step":
            gpu.decode_step(kk[:, :, 0], vv[:, :, 0], cc[:, 0], pp[:, 0], qq, SCALE, out)
        else:
            gpu.quantize_append(kk, vv, cc, pp)
            gpu.decode_attention(qq, SCALE, out)

    def step():
        call_step(k, v, c, p, q)

    # packed bytes read by the timed attention: every live entry after the append
    restore()
    step()
    torch.cuda.synchronize()
    n_after = views["n"].cpu().numpy()
    pk = packed_bytes(n_after, list(gpu.layout.rec_bytes))
    kv_tokens = int(n_after.sum())
    saved_post = {key: views[key].clone() for key in ("n", "ft", "hw")}

    def restore_post():
        for key in ("n", "ft", "hw"):
            views[key].copy_(saved_post[key])

    for _ in range(args.warmup):
        restore()
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    st = torch.cuda.current_stream()
    # (1) the step: append + attention back to back, through tkv_decode_step or the two
    #     calls (no event between them: the attention launch overlaps the append as it
    #     does in a decode loop)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    # (2) the attention call alone, on the post-append cache: the kernel the roofline
    #     reports (same live entries and packed bytes as in the step)
    n_attn = max(10, args.steps // 2)
    ea = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n_attn)]
    launches0 = gpu.launch_count()
    torch.cuda.synchronize()
    with ClockSampler(gpu_smi_id(dev)) as cs:
        for i in range(args.steps):
            restore()
            flush.zero_()
            ev[i][0].record(st)
            call_step(k, v, c, p, q)
            ev[i][1].record(st)
        torch.cuda.synchronize()
        launches = gpu.launch_count() - launches0
        for i in range(n_attn):
            restore_post()
            flush.zero_()
            ea[i][0].record(st)
            gpu.decode_attention(q, SCALE, out)
            ea[i][1].record(st)
        torch.cuda.synchronize()
        # (3) the same call with the attention-sparsity statistic (its cost over (2); the
        #     persistent warp-tile pipeline does not form it)
        es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_attn if args.attn_kernel != "ws" else 0)]
        for i in range(len(es)):
            restore_post()
            flush.zero_()
            es[i][0].record(st)
            gpu.decode_attention_sparsity(q, SCALE, 0.5, 0.7, out=out)
            es[i][1].record(st)
        torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b2) for a, b2 in ev]
    attn_ms = [a.elapsed_time(b2) for a, b2 in ea]
    sp_ms = [a.elapsed_time(b2) for a, b2 in es]
    t_step = sum(step_ms) / len(step_ms)
    t_attn = sum(attn_ms) / len(attn_ms)
    t_step, t_attn = reduce_max([t_step, t_attn], world, dev)
    assert gpu.poll_error() == 0

    # ---- end to end through the public API with host buffers
    e2e_steps = args.e2e_steps or max(20, min(500, args.steps // 4))
    # the step's inputs (k, v, q, positions, classes) packed into one pinned host buffer
    # and one device buffer (256-byte aligned pieces), so each step is one H2D copy
    inputs = (k, v, q, p, c)
    sizes = [x.numel() * x.element_size() for x in inputs]
    offs, total = [], 0
    for nb in sizes:
        offs.append(total)
        total += (nb + 255) // 256 * 256
    hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
    dviews = []
    for x, o, nb in zip(inputs, offs, sizes):
        hbuf[o:o + nb].copy_(x.contiguous().view(-1).view(torch.uint8).cpu())
        dviews.append(dbuf[o:o + nb].view(x.dtype).view(x.shape))
    dk, dv, dq, dp, dc = dviews
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_ms = []
    for i in range(args.warmup + e2e_steps):
        restore()
        flush.zero_()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        dbuf.copy_(hbuf, non_blocking=True)
        call_step(dk, dv, dc, dp, dq)
        hout.copy_(out, non_blocking=True)
        b2.record(st)
        b2.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b2))
    t_e2e = sum(e2e_ms) / len(e2e_ms)
    t_e2e, = reduce_max([t_e2e], world, dev)
    h2d = total   # bytes copied per step (the pieces plus their alignment padding)
    d2h = hout.numel() * hout.element_size()

    peak, peak_src = measured_peaks()
    gbs = pk / (t_attn * 1e-3) / 1e9
    B = w["B"]
    res = {
        "metric": METRIC,
        "value": world * B / (t_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8/int4/int2 codes + bf16 -> fp32",
        "data": "synthetic (seeded counter-hash N(0,1) bf16, K x10 outlier channels)",
        "config": {"workload": args.workload + (f" (prefill ctx {args.ctx})" if args.ctx else ""),
                   "batch": B, "q_heads": w["Hq"], "kv_heads": w["Hkv"],
                   "head_dim": 128, "context": w["ctx"], "budget": w["budget"],
                   "bf16_window": w["n_protect"], "p_RET": [w["p_r"], w["p_e"], 1 - w["p_r"] - w["p_e"]],
                   "live_kv_tokens": kv_tokens, "packed_kv_bytes": pk,
                   # besides the packed records, the attention call reads and writes each
                   # live entry's score (8 B), reads q (bf16) and writes out (fp32); reuse
                   # placement also reads each entry's slot handle (4 B)
                   "total_bytes_per_step": pk + kv_tokens * (8 + (0 if args.placement == "dense" else 4))
                   + q.numel() * q.element_size() + out.numel() * out.element_size(),
                   "placement": args.placement, "attn_kernel": args.attn_kernel, "codec": args.codec,
                   "step_call": {"step": "tkv_decode_step",
                                 "separate": "tkv_quantize_append + tkv_decode_attention"}[args.step_call],
                   "eviction": {"topk": f"topk, budget {w['budget']} per stream",
                                "tbe": "tbe segment schedule at the scoring step (r0 64, t_keep 16)",
                                "tam": f"tam segment budgets, {w['budget']} per stream, pivotal above 3x "
                                       "the mean score"}[args.evict],
                   "l2": "flushed (write of %d MB) before every timed step" % (flush.numel() >> 20),
                   "parallelism": f"{world} independent replicas" if world > 1 else "single GPU"},
        "hbm_gbs_packed": gbs,
        "frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
        "attention_ms": t_attn,
        "attention_ms_median": statistics.median(attn_ms),
        "attention_ms_min": min(attn_ms),
        "attention_timing": "attention call alone on the post-append cache (L2 flushed), CUDA events",
        "sparsity_call_ms": statistics.median(sp_ms) if sp_ms else None,
        "sparsity_overhead": statistics.median(sp_ms) / statistics.median(attn_ms) - 1.0 if sp_ms else None,
        "append_exposed_ms": t_step - t_attn,   # step minus the attention call timed alone
        "evict_ms_untimed_step": evict_ms,
        "full_context_phase": full,
        "kv_tokens_per_s": world * kv_tokens / (t_attn * 1e-3),
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "traffic": None, "peak_source": peak_src,
                     "kernel": "tkv_decode_attention (all its launches, CUDA events)"},
        "e2e": {"value": world * B / (t_e2e * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": t_e2e},
        "gpu_launches": int(launches),
        "clocks": cs.summary(),
    }
    tr = stored_traffic(args.placement, args.attn_kernel)
    if tr is not None:
        # DRAM bytes of one launch, from the committed capture, scaled to this launch's packed bytes
        res["roofline"]["traffic"] = int(tr["traffic_per_packed_byte"] * pk)
        res["roofline"]["traffic_source"] = tr["capture"] + " (scaled by packed bytes)"
    return res, gpu, w


# Both oracle legs (the tkv arm's cpu_baseline and the reference arm) time the same
# thing: the oracle's append + attention of the timed step on SAMPLE_ROWS batch rows
# (SAMPLE_ROWS * Hkv streams, which the oracle's OpenMP loop spreads over the host
# cores), and report the sample's own throughput: rows / time per step (decode
# tokens/s).  No time is scaled to the full batch.
SAMPLE_ROWS = 2


def _oracle_step_times(o, state, inputs, warmup, reps, budget_s=None):
    kb, vb, cb, pb, qb = inputs
    times = []
    t_all = time.perf_counter()
    for i in range(warmup + reps):
        o.load_state(state)
        t0 = time.perf_counter()
        o.append(kb, vb, cb, pb)
        o.attend(qb, SCALE)
        dt = time.perf_counter() - t0
        if i >= warmup:
            times.append(dt)
        if budget_s is not None and time.perf_counter() - t_all > budget_s and len(times) >= 3:
            break
    return times


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def cpu_baseline(gpu, w, rows, reps_budget_s=12.0):
    """The oracle (as it stands) on a bounded sample: the same timed step for batch
    rows `rows`, starting from the GPU's post-eviction state of those rows."""
    from oracle import oracle as orc
    sub = [b * w["Hkv"] + h for b in rows for h in range(w["Hkv"])]
    st = gpu.export_state(sub)
    o = orc.OracleCache(len(rows), w["Hkv"], w["G"], cap=w["cap"], n_protect=w["n_protect"],
                        dense=gpu.dense)
    k, v, c, p, q = synth.decode_inputs(w, 1)
    inputs = (_bits(k[rows]), _bits(v[rows]), c[rows].numpy(), p[rows].numpy(), _bits(q[rows]))
    times = _oracle_step_times(o, st, inputs, warmup=1, reps=50, budget_s=reps_budget_s)
    t = statistics.median(times)
    return {"value": len(rows) / t, "unit": "tokens/s", "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{len(rows)} of {w['B']} batch rows ({len(sub)} streams) of the timed step "
                      f"(append + attention), median of {len(times)} reps; value = sampled rows / time",
            "ms_per_step_sample": t * 1e3}


def run_reference(args, rank, world):
    """The oracle as the reference arm: CPU only, on rank 0."""
    if rank != 0:
        return None
    from oracle import oracle as orc
    w = synth.prefill_inputs(args.workload, seed=0, steps=2, B=SAMPLE_ROWS)
    # SAMPLE_ROWS batch rows per step: prefill, scoring step, eviction, then the timed step
    o = orc.OracleCache(w["B"], w["Hkv"], w["G"], cap=w["cap"], n_protect=w["n_protect"])
    o.append(_bits(w["k"]), _bits(w["v"]), w["cls"][:, :w["ctx"]].numpy(), w["pos"].numpy())
    k, v, c, p, q = synth.decode_inputs(w, 0)
    o.append(_bits(k), _bits(v), c.numpy(), p.numpy())
    o.attend(_bits(q), SCALE)
    o.evict(w["budget"])
    st = o.copy_state()
    k, v, c, p, q = synth.decode_inputs(w, 1)
    inputs = (_bits(k), _bits(v), c.numpy(), p.numpy(), _bits(q))
    times = _oracle_step_times(o, st, inputs, warmup=args.warmup, reps=args.steps)
    t_step = sum(times) / len(times)
    val = SAMPLE_ROWS / t_step
    full_B = synth.WORKLOADS[args.workload]["B"]
    sample = (f"{SAMPLE_ROWS} of {full_B} batch rows ({SAMPLE_ROWS * w['Hkv']} streams) per step, append + "
              f"attention of the timed step; value = sampled rows / time per step, ms_per_step = the sample's step")
    return {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded counter-hash N(0,1) bf16, K x10 outlier channels)",
            "config": {"workload": args.workload, "batch": full_B, "q_heads": w["Hq"],
                       "kv_heads": w["Hkv"], "head_dim": 128, "context": w["ctx"],
                       "budget": w["budget"], "bf16_window": w["n_protect"],
                       "sampled_rows": SAMPLE_ROWS},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": orc.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_loop(args, dev):
    """The workload's decode loop on one GPU: prefill every layer's cache, then `steps`
    decode steps of append + attention on every layer with the eviction to the budget
    every `evict_every` steps (ThinKV / TAM periodic compaction).  Per 64-step chunk the
    inputs are generated first (untimed), then the chunk runs between two CUDA events."""
    from reasoning_model_kv_b200 import TkvCache
    spec = synth.WORKLOADS[args.workload]
    L, E = spec.get("layers", 1), spec["evict_every"]
    steps = args.loop_steps or spec["steps"]
    B, Hkv, Hq, D, ctx = spec["B"], spec["Hkv"], spec["Hq"], spec["D"], spec["ctx"]
    kern = {"warp": 0, "tc": 1, "ws": 2}[args.attn_kernel]
    caches, ws = [], []
    t0 = time.time()
    for layer in range(L):
        w = synth.prefill_inputs(args.workload, layer=layer, device=dev, steps=steps)
        g = TkvCache(w["B"], w["Hkv"], w["G"], w["cap"], w["n_protect"], max_append=w["ctx"],
                     dense=args.placement == "dense", attn_kernel=kern, codec=1 if args.codec == "fp" else 0)
        g.quantize_append(w["k"], w["v"], w["cls"][:, :w["ctx"]].contiguous().to(dev), w["pos"].to(dev))
        del w["k"], w["v"]
        caches.append(g)
        ws.append(w)
    # every kernel of the loop launched once before timing (module loading, launch
    # attributes), on a small cache of the same shape class
    wu = synth.prefill_inputs("tiny_b1_ctx2k", device=dev, B=1, Hq=Hq // Hkv, Hkv=1, ctx=512,
                              n_protect=spec["n_protect"], steps=2)
    gw = TkvCache(1, 1, wu["G"], wu["cap"], wu["n_protect"], max_append=wu["ctx"], dense=args.placement == "dense",
                  attn_kernel=kern, codec=1 if args.codec == "fp" else 0)
    gw.quantize_append(wu["k"], wu["v"], wu["cls"][:, :wu["ctx"]].contiguous().to(dev), wu["pos"].to(dev))
    kw, vw, cw, pw, qw = synth.decode_inputs(wu, 0, device=dev)
    gw.quantize_append(kw, vw, cw, pw)
    gw.decode_attention(qw, SCALE)
    gw.decode_step(kw[:, :, 0], vw[:, :, 0], cw[:, 0], pw[:, 0], qw, SCALE)
    gw.evict_compact(128)
    torch.cuda.synchronize()
    del gw
    prefill_s = time.time() - t0
    cls_dev = ws[0]["cls"][:, ctx:ctx + steps].contiguous().to(dev)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()
    chunk_ms, n_evict = [], 0
    for c0 in range(0, steps, 64):
        n = min(64, steps - c0)
        chunk = []
        for layer in range(L):
            seed = ws[layer]["seed"]
            k = synth.normal_bf16(seed, layer, synth.TID_K, B, Hkv, ctx + c0, n, D, dev)
            if spec["outliers"]:
                k = synth.apply_k_outliers(k, seed, layer)
            v = synth.normal_bf16(seed, layer, synth.TID_V, B, Hkv, ctx + c0, n, D, dev)
            q = synth.normal_bf16(seed, layer, synth.TID_Q, B, Hq, ctx + c0, n, D, dev)
            chunk.append(([k[:, :, j:j + 1].contiguous() for j in range(n)], [v[:, :, j:j + 1].contiguous() for j in range(n)],
                          [q[:, :, j].contiguous() for j in range(n)]))
        pos = [torch.full((B, 1), ctx + c0 + j, dtype=torch.int32, device=dev) for j in range(n)]
        cls = [cls_dev[:, c0 + j:c0 + j + 1].contiguous() for j in range(n)]
        torch.cuda.synchronize()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for j in range(n):
            for layer in range(L):
                kk, vv, qq = chunk[layer]
                if args.step_call == "step":
                    caches[layer].decode_step(kk[j][:, :, 0], vv[j][:, :, 0], cls[j][:, 0], pos[j][:, 0], qq[j],
                                              SCALE, out)
                else:
                    caches[layer].quantize_append(kk[j], vv[j], cls[j], pos[j])
                    caches[layer].decode_attention(qq[j], SCALE, out)
            if E and (c0 + j + 1) % E == 0:
                for layer in range(L):
                    caches[layer].evict_compact(spec["budget"])
                n_evict += 1
        b2.record(st)
        b2.synchronize()
        chunk_ms.append(a.elapsed_time(b2))
        del chunk
    for g in caches:
        assert g.poll_error() == 0
    total_ms = sum(chunk_ms)
    return {
        "metric": "decode loop wall time (all layers, append + attention + periodic eviction)",
        "value": total_ms, "unit": "ms", "higher_is_better": False,
        "n_gpus": 1, "steps": steps, "layers": L,
        "decode_tokens_per_s": B * steps / (total_ms * 1e-3),
        "us_per_step_all_layers": total_ms * 1e3 / steps,
        "chunk_ms_64_steps": chunk_ms,
        "first_chunk_note": "steps 0-63 run on the full prefill context (no eviction before step 63)",
        "evictions": n_evict, "prefill_s_untimed": prefill_s,
        "config": {"workload": args.workload, "batch": B, "q_heads": Hq, "kv_heads": Hkv, "context": ctx,
                   "budget": spec["budget"], "evict_every": E, "placement": args.placement,
                   "attn_kernel": args.attn_kernel, "codec": args.codec, "step_call": args.step_call},
        "data": "synthetic (seeded counter-hash N(0,1) bf16)",
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device(dev))
    from reasoning_model_kv_b200 import build as b
    b.build()
    if args.decode_loop:
        if rank == 0:
            print(json.dumps(run_loop(args, dev)), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    res, gpu, w = run_tkv(args, rank, world, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(gpu, w, rows=list(range(SAMPLE_ROWS)))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
