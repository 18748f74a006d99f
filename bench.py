#!/usr/bin/env python
"""TurboQuant hot-path benchmark on B200.

One step = one pass of the whole hot path over one batch of the long-context
decode workload at d = 128, b = 3 (2-bit Lloyd-Max + 1-bit QJL, m = 128):
batch 8 x 8 KV heads x 131072 tokens of bf16 K and V (per-channel log-uniform
scales), 32 query heads (GQA 4):

    tq_quantize(K)  tq_quantize(V)  tq_logits(Q, packed K)  tq_dequant(packed V)

`value` is compressed-key logits per second of the whole step (all ranks);
per-kernel times, the quantize rows/s and the bf16 unquantized-key baseline
kernel on the same shapes are reported beside it.  Inputs (2.1 GB per K/V
tensor) are larger than L2, so no flush is needed between steps.

Secondary workloads (`--workload NAME`, each with its own metric line): the
prefill write path (prefill-b2/b3/b4), decode-time append (append-b3), vector
search (vsearch: quantize a 10^6 x 1024 database, then tq_search's fused
top-10; vsearch-128k for profiler captures) and the long-context decode step
at fractional bit widths (decode-128k-2.5bit / 3.5bit: 64 + 64 channel split).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_vector_15_b200 import dist as dist_util  # noqa: E402
from kv_cache_vector_15_b200 import inputs  # noqa: E402

WORKLOADS = {
    # long-context decode at the headline bit width (the metric's d = 128, b = 3)
    "decode-128k-b3": dict(batch=8, ctx=131072, b=3, m=128, kv_heads=8, q_heads=32, d=128),
    "decode-128k-b4": dict(batch=8, ctx=131072, b=4, m=128, kv_heads=8, q_heads=32, d=128),
    "decode-8k-b3": dict(batch=1, ctx=8192, b=3, m=128, kv_heads=8, q_heads=32, d=128),
    # a 1M-row case (268 MB per tensor, above L2) for profiler captures
    "decode-2x64k-b3": dict(batch=2, ctx=65536, b=3, m=128, kv_heads=8, q_heads=32, d=128),
}
# secondary workloads, each with its own metric (not the headline line)
AUX_WORKLOADS = {
    # prefill write path: quantize K and V of 32 layers x 8 heads x 32768 tokens
    "prefill-b2": dict(kind="prefill", b=2, m=128, d=128),
    "prefill-b3": dict(kind="prefill", b=3, m=128, d=128),
    "prefill-b4": dict(kind="prefill", b=4, m=128, d=128),
    # vector search: 1e6 x 1024 fp32 database, 1024 queries, b = 4, m = 1024, top-10
    "vsearch": dict(kind="vsearch", b=4, m=1024, d=1024),
    # the same on a 131072-row database (0.5 GB, above L2) for profiler captures
    "vsearch-128k": dict(kind="vsearch", b=4, m=1024, d=1024, n=131072),
    # fractional bit widths: the long-context decode step with each row's 128
    # channels split 64 / 64 between two instances (2.5 bits: b = 3 / 2;
    # 3.5 bits: b = 4 / 3)
    "decode-128k-2.5bit": dict(kind="split", d=128, d_hi=64, b_hi=3, b_lo=2, b=2.5, m=64),
    "decode-128k-3.5bit": dict(kind="split", d=128, d_hi=64, b_hi=4, b_lo=3, b=3.5, m=64),
    # decode-time append: one new token of a 32-layer x 8-KV-head model (256 K rows
    # and 256 V rows) scattered into a paged packed cache, latency per token
    "append-b3": dict(kind="append", b=3, m=128, d=128),
}
METRIC = "compressed-key logits/s and % HBM roofline (d=128,b=3); quantize rows/s"
UNIT = "logits/s"


KERNEL_OF = {"quantize": "k_quantize_d128_ws", "logits": "k_logits_d128_ws", "dequant": "k_dequant_d128_ovl"}


def captured_traffic(kernel: str, b: int, units: int):
    """DRAM bytes per launch of `kernel` at bit width `b` from the committed ncu
    capture summary (profiles/traffic.json: one entry per kernel and bit
    width, DRAM bytes read + written per unit over one captured launch),
    scaled by the units one launch processes -- or None when there is no
    capture of that kernel at that bit width, or the kernel's source changed
    since it was taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    name = KERNEL_OF.get(kernel, "")
    for entry in json.load(open(p)).get("entries", []):
        if entry.get("kernel") != name or int(entry.get("b", -1)) != b:
            continue
        src = os.path.join(ROOT, entry["source"])
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != entry["source_sha256"]:
            return None
        return entry["dram_bytes_per_unit"] * units
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Dense fp16/bf16 tensor peak (TFLOP/s) for a kernel timed inside a long
    step: the sustained measurement, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        if "bf16_tflops_sustained" in j:
            return float(j["bf16_tflops_sustained"]), "measured (sustained)"
    return 1400.0, "fallback (sustained)"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        # wait for the first sample: nvidia-smi's start-up (driver queries) must
        # not overlap the timed region, where it can delay kernel launches
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup():
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    dist_util.barrier(ws)


def max_over_ranks(ws, v: float) -> float:
    import torch
    return dist_util.max_over_ranks(ws, v, device=torch.device("cuda", torch.cuda.current_device()))


# ---------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline): a bounded sample of the workload
# ---------------------------------------------------------------------------
def oracle_sample_step(cfg, n_sets: int, n_keys: int):
    """One step of the hot path on the oracle for the first n_sets (batch, kv
    head) sets, n_keys tokens each: quantize their K and V rows, logits for
    each set's g queries, PROD dequant of V.  Returns (logits computed, seconds)."""
    from oracle import params as op
    from oracle import turboquant as ot
    K, V, Q = inputs.decode(cfg["batch"], cfg["ctx"], kv_heads=cfg["kv_heads"], q_heads=cfg["q_heads"])
    g = cfg["q_heads"] // cfg["kv_heads"]
    rows = np.concatenate([np.arange(s * cfg["ctx"], s * cfg["ctx"] + n_keys) for s in range(n_sets)])
    k = K.as_f32(K.take(rows)).astype(np.float64)
    v = V.as_f32(V.take(rows)).astype(np.float64)
    # query rows of set s = (batch b, kv head h) are b * q_heads + h * g + j
    qrows = np.concatenate([np.arange((s // cfg["kv_heads"]) * cfg["q_heads"] + (s % cfg["kv_heads"]) * g,
                                      (s // cfg["kv_heads"]) * cfg["q_heads"] + (s % cfg["kv_heads"]) * g + g)
                            for s in range(n_sets)])
    q = Q.as_f32(Q.take(qrows)).astype(np.float64)
    P = op.Params(cfg["d"], cfg["b"], cfg["m"], seed=0)
    t0 = time.perf_counter()
    pk = ot.quantize(k, P)
    pv = ot.quantize(v, P)
    ot.logits(q, pk, P, n_sets, g, n_keys)
    ot.dequant(pv, P, ot.DEQUANT_PROD)
    return n_sets * g * n_keys, time.perf_counter() - t0


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, cfg, ws, rank):
    if rank != 0:
        return
    n_keys = 8192
    for _ in range(args.warmup):
        oracle_sample_step(cfg, 1, n_keys)
    total_units, total_t = 0, 0.0
    for _ in range(args.steps):
        u, t = oracle_sample_step(cfg, 1, n_keys)
        total_units += u
        total_t += t
    value = total_units / total_t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, **cfg},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"1 (batch, kv head) set x {n_keys} tokens per step: quantize K and V, "
                                   f"logits for its 4 query heads, PROD dequant of V"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# CUDA path
# ---------------------------------------------------------------------------
def run_ours(args, cfg, ws, rank, local):
    import torch
    from kv_cache_vector_15_b200 import tq

    d, b, m = cfg["d"], cfg["b"], cfg["m"]
    # this rank's sequences of a global batch of ws * batch (weak scaling)
    sh = dist_util.decode_shard(cfg["batch"], ws, rank, cfg["kv_heads"], cfg["q_heads"], cfg["ctx"])
    n_sets = sh.n_sets
    g = cfg["q_heads"] // cfg["kv_heads"]
    n_keys = cfg["ctx"]
    N = n_sets * n_keys
    dev = torch.device("cuda", local)
    T = tq.TurboQuant(d, b, m, seed=0)

    # seeded inputs, drawn on the host into pinned buffers (also the e2e source)
    K, V, Q = inputs.decode(sh.global_batch, cfg["ctx"], kv_heads=cfg["kv_heads"], q_heads=cfg["q_heads"])
    hK = torch.empty((N, d), dtype=torch.bfloat16, pin_memory=True)
    hV = torch.empty((N, d), dtype=torch.bfloat16, pin_memory=True)
    hQ = torch.empty((n_sets * g, d), dtype=torch.bfloat16, pin_memory=True)
    K.fill(hK.view(torch.int16).numpy().view(np.uint16), start=sh.kv_rows[0])
    V.fill(hV.view(torch.int16).numpy().view(np.uint16), start=sh.kv_rows[0])
    Q.fill(hQ.view(torch.int16).numpy().view(np.uint16), start=sh.q_rows[0])
    dK, dV, dQ = hK.to(dev), hV.to(dev), hQ.to(dev)
    pK, pV = T.empty_packed(N, dev), T.empty_packed(N, dev)
    logits = torch.empty((n_sets, g, n_keys), dtype=torch.float32, device=dev)
    vhat = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    wbytes = T.workspace_bytes(n_sets, g, n_keys)
    work = torch.empty(max(wbytes, 16), dtype=torch.uint8, device=dev)
    qwork = torch.empty(max(T.quantize_workspace_bytes(N), 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        T.quantize(dK, pK, workspace=qwork, stream=stream)
        if ev:
            ev[1].record(stream)
        T.quantize(dV, pV, workspace=qwork, stream=stream)
        if ev:
            ev[2].record(stream)
        T.logits(dQ, pK, n_sets, g, n_keys, out=logits, workspace=work, stream=stream)
        if ev:
            ev[3].record(stream)
        T.dequant(pV, N, out=vhat, stream=stream)
        if ev:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(ws)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    launches0 = tq.launch_count()
    with ClockSampler(local) as clk:
        torch.cuda.synchronize(dev)
        barrier(ws)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(ws)
    launches = tq.launch_count() - launches0
    elapsed_ms = max_over_ranks(ws, start.elapsed_time(end))
    ms_step = elapsed_ms / args.steps
    per = {"quantize_K": [], "quantize_V": [], "logits": [], "dequant": []}
    for e in evs:
        per["quantize_K"].append(e[0].elapsed_time(e[1]))
        per["quantize_V"].append(e[1].elapsed_time(e[2]))
        per["logits"].append(e[2].elapsed_time(e[3]))
        per["dequant"].append(e[3].elapsed_time(e[4]))
    avg = {k: sum(v) / len(v) for k, v in per.items()}
    n_logits = n_sets * g * n_keys
    total_logits = dist_util.sum_over_ranks(ws, n_logits, device=dev)
    total_rows = dist_util.sum_over_ranks(ws, N, device=dev)
    value = total_logits / (ms_step * 1e-3)

    hbm, hbm_kind = peaks()
    P = T.row_bytes
    alg = {  # algorithmic bytes per launch
        "quantize": N * (2 * d + P),
        "logits": N * (P + 4 * g),
        "dequant": N * (P + 2 * d),
    }
    q_ms = (avg["quantize_K"] + avg["quantize_V"]) / 2
    kern = {
        "quantize": {"ms": q_ms, "launches_per_step": 2, "bytes": alg["quantize"]},
        "logits": {"ms": avg["logits"], "launches_per_step": 2, "bytes": alg["logits"]},
        "dequant": {"ms": avg["dequant"], "launches_per_step": 1, "bytes": alg["dequant"]},
    }
    for k, v in kern.items():
        v["gbs"] = v["bytes"] / (v["ms"] * 1e-3) / 1e9
        v["frac_hbm"] = v["gbs"] / hbm
    dominant = max(kern, key=lambda k: kern[k]["ms"] * (2 if k == "quantize" else 1))
    dk = kern[dominant]

    # bf16 unquantized-key logits on the same shapes (comparison point)
    bf16_out = torch.empty_like(logits)
    for _ in range(3):
        tq.logits_bf16(dQ, dK, n_sets, g, n_keys, out=bf16_out, stream=stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    e0.record(stream)
    for _ in range(reps):
        tq.logits_bf16(dQ, dK, n_sets, g, n_keys, out=bf16_out, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    bf16_ms = e0.elapsed_time(e1) / reps
    bf16_bytes = N * (2 * d + 4 * g)

    # decode attention from the compressed cache (softmax over the estimated
    # logits, value sum in the rotated domain) and torch's bf16 SDPA on the same
    # shapes as a reference point (a library kernel, not part of the path)
    attn_out = torch.empty((n_sets * g, d), dtype=torch.float32, device=dev)
    attn_ws = torch.empty(max(T.attention_workspace_bytes(n_sets, g, n_keys), 16), dtype=torch.uint8, device=dev)
    for _ in range(3):
        T.attention(dQ, pK, pV, n_sets, g, n_keys, out=attn_out, workspace=attn_ws, stream=stream)
    e0.record(stream)
    for _ in range(reps):
        T.attention(dQ, pK, pV, n_sets, g, n_keys, out=attn_out, workspace=attn_ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    attn_ms = e0.elapsed_time(e1) / reps
    sdpa_ms = None
    try:
        import torch.nn.functional as F
        qh = dQ.view(sh.batch, cfg["q_heads"], 1, d)
        kh = dK.view(sh.batch, cfg["kv_heads"], n_keys, d)
        vh = dV.view(sh.batch, cfg["kv_heads"], n_keys, d)
        for _ in range(3):
            F.scaled_dot_product_attention(qh, kh, vh, enable_gqa=True)
        e0.record(stream)
        for _ in range(reps):
            F.scaled_dot_product_attention(qh, kh, vh, enable_gqa=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        sdpa_ms = e0.elapsed_time(e1) / reps
    except Exception:                     # the reference point is optional
        sdpa_ms = None

    # end to end through the public API with host buffers: every step uploads K,
    # V and q from pinned host memory and downloads the logits and V-hat,
    # pipelined over this rank's sequences -- sequence i+1 uploads on one copy
    # stream and sequence i-1's results download on another while sequence i
    # is computed (PCIe is full duplex)
    hL = torch.empty((n_sets, g, n_keys), dtype=torch.float32, pin_memory=True)
    hVh = torch.empty((N, d), dtype=torch.bfloat16, pin_memory=True)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nseq = sh.batch
    kv_per, q_per, sets_per = cfg["kv_heads"] * n_keys, cfg["q_heads"], cfg["kv_heads"]
    computed = [None] * nseq          # per sequence: its compute finished (inputs free)
    downloaded = [None] * nseq        # per sequence: its results are on the host (outputs free)

    def e2e_step():
        for i in range(nseq):
            r0, r1 = i * kv_per, (i + 1) * kv_per
            q0, q1 = i * q_per, (i + 1) * q_per
            s0, s1 = i * sets_per, (i + 1) * sets_per
            if computed[i] is not None:
                s_in.wait_event(computed[i])
            with torch.cuda.stream(s_in):
                dK[r0:r1].copy_(hK[r0:r1], non_blocking=True)
                dV[r0:r1].copy_(hV[r0:r1], non_blocking=True)
                dQ[q0:q1].copy_(hQ[q0:q1], non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_in)
            stream.wait_event(up)
            if downloaded[i] is not None:
                stream.wait_event(downloaded[i])
            pk, pv = pK.rows(r0, r1), pV.rows(r0, r1)
            T.quantize(dK[r0:r1], pk, workspace=qwork, stream=stream)
            T.quantize(dV[r0:r1], pv, workspace=qwork, stream=stream)
            T.logits(dQ[q0:q1], pk, sets_per, g, n_keys, out=logits[s0:s1], workspace=work, stream=stream)
            T.dequant(pv, kv_per, out=vhat[r0:r1], stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            computed[i] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                hL[s0:s1].copy_(logits[s0:s1], non_blocking=True)
                hVh[r0:r1].copy_(vhat[r0:r1], non_blocking=True)
            dn = torch.cuda.Event()
            dn.record(s_out)
            downloaded[i] = dn
        stream.wait_stream(s_out)

    e2e_steps = max(1, min(args.steps, 5))
    e2e_step()
    torch.cuda.synchronize(dev)
    barrier(ws)
    e0.record(stream)
    s_in.wait_stream(stream)          # no upload starts before the timed region
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(ws, e0.elapsed_time(e1)) / e2e_steps
    h2d = (hK.numel() + hV.numel() + hQ.numel()) * 2
    d2h = hL.numel() * 4 + hVh.numel() * 2

    line = None
    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            sets_cpu = 2                 # two whole (batch, kv head) sets: about 10 s of the oracle
            units, secs = oracle_sample_step(cfg, sets_cpu, n_keys)
            cpu = {"value": units / secs, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                   "sample": f"{sets_cpu} (batch, kv head) sets x {n_keys} tokens: quantize K and V, logits for "
                             f"their {g} query heads each, PROD dequant of V ({secs:.1f} s)"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": args.workload, "batch": cfg["batch"], "global_batch": sh.global_batch,
                       "kv_heads": cfg["kv_heads"],
                       "q_heads": cfg["q_heads"], "ctx": cfg["ctx"], "d": d, "b": b, "m": m,
                       "parallelism": f"dp{ws} (each rank owns {cfg['batch']} sequences of the global batch; "
                                      "no data-path collective)",
                       "l2": "inputs larger than L2 (K, V 2.1 GB each); no flush"},
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": dk["gbs"], "peak": hbm,
                         "unit": "GB/s", "frac": dk["frac_hbm"], "traffic": captured_traffic(dominant, cfg["b"], N),
                         "algorithmic_bytes": dk["bytes"], "peak_kind": hbm_kind},
            "quantize_rows_per_s": total_rows / (q_ms * 1e-3),
            "kernels": {k: {"ms_per_launch": v["ms"], "algorithmic_GBps": v["gbs"], "frac_hbm": v["frac_hbm"],
                            "bytes_per_launch": v["bytes"]} for k, v in kern.items()},
            "bf16_key_logits_baseline": {"ms": bf16_ms, "algorithmic_GBps": bf16_bytes / (bf16_ms * 1e-3) / 1e9,
                                         "tq_logits_speedup": bf16_ms / avg["logits"]},
            "attention": {"ms": attn_ms, "packed_GBps": N * 2 * P / (attn_ms * 1e-3) / 1e9,
                          "torch_sdpa_bf16_ms": sdpa_ms},
            "cpu_baseline": cpu,
            "e2e": {"value": total_logits / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    T.close()
    return line


# ---------------------------------------------------------------------------
# Secondary workloads (prefill write path, vector search): CUDA path only
# ---------------------------------------------------------------------------
def append_graph_ms(torch, T, dev, stream, dk, dv, slots, cK, cV, steps):
    """The append step replayed from a CUDA graph (no per-launch host cost);
    None if the capture is not possible here."""
    try:
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            T.quantize_scatter(dk, slots, cK, stream=gs)
            T.quantize_scatter(dv, slots, cV, stream=gs)
        stream.wait_stream(gs)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / steps
        del g
        return ms
    except Exception:
        return None


def run_aux(args, cfg, ws, rank, local):
    import torch
    from kv_cache_vector_15_b200 import tq

    d, b, m = cfg["d"], cfg["b"], cfg["m"]
    dev = torch.device("cuda", local)
    if cfg["kind"] == "split":
        T = tq.TurboQuantSplit(d, cfg["d_hi"], cfg["b_hi"], cfg["b_lo"], seed=0)
        P = T.row_bytes
    else:
        T = tq.TurboQuant(d, b, m, seed=0)
        P = T.row_bytes
    stream = torch.cuda.current_stream(dev)
    hbm, hbm_kind = peaks()
    if cfg["kind"] == "split":
        # the long-context decode step (8 x 8 x 131072 keys and values, GQA 4)
        # on the split format; each rank takes its slice of the batch
        batch, ctx, kvh, qh = 8, 131072, 8, 32
        g = qh // kvh
        b0, b1 = dist_util.shard(batch, ws, rank)
        n_sets, n_keys = (b1 - b0) * kvh, ctx
        N = n_sets * n_keys
        K, V, Q = inputs.decode(batch, ctx, kv_heads=kvh, q_heads=qh)
        hK = torch.empty((N, d), dtype=torch.bfloat16)
        hV = torch.empty((N, d), dtype=torch.bfloat16)
        hQ = torch.empty((n_sets * g, d), dtype=torch.bfloat16)
        K.fill(hK.view(torch.int16).numpy().view(np.uint16), start=b0 * kvh * ctx)
        V.fill(hV.view(torch.int16).numpy().view(np.uint16), start=b0 * kvh * ctx)
        Q.fill(hQ.view(torch.int16).numpy().view(np.uint16), start=b0 * qh)
        dK, dV, dQ = hK.to(dev), hV.to(dev), hQ.to(dev)
        del hK, hV
        pK, pV = T.empty_packed(N, dev), T.empty_packed(N, dev)
        lg = torch.empty((n_sets, g, n_keys), dtype=torch.float32, device=dev)
        vhat = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
        work = torch.empty(max(T.logits_workspace_bytes(n_sets, g, n_keys), 16), dtype=torch.uint8, device=dev)
        qwork = torch.empty(max(T.quantize_workspace_bytes(N), 16), dtype=torch.uint8, device=dev)

        def step():
            T.quantize(dK, pK, workspace=qwork, stream=stream)
            T.quantize(dV, pV, workspace=qwork, stream=stream)
            T.logits(dQ, pK, n_sets, g, n_keys, out=lg, workspace=work, stream=stream)
            T.dequant(pV, N, out=vhat, stream=stream)
        units, unit = n_sets * g * n_keys, "logits/s"
        metric = f"compressed-key logits/s, long-context decode step at {b} bits (64 + 64 channel split)"
        alg = 2 * N * (2 * d + P) + N * (P + 4 * g) + N * (P + 2 * d)
        kern = "step"
    elif cfg["kind"] == "prefill":
        K, V = inputs.prefill()
        N = K.n_rows
        lo, hi = dist_util.shard(N, ws, rank)          # each rank quantizes its slice of the rows
        n = hi - lo
        hK = torch.empty((n, d), dtype=torch.bfloat16)
        hV = torch.empty((n, d), dtype=torch.bfloat16)
        K.fill(hK.view(torch.int16).numpy().view(np.uint16), start=lo)
        V.fill(hV.view(torch.int16).numpy().view(np.uint16), start=lo)
        dK, dV = hK.to(dev), hV.to(dev)
        del hK, hV
        pK, pV = T.empty_packed(n, dev), T.empty_packed(n, dev)
        qwork = torch.empty(max(T.quantize_workspace_bytes(n), 16), dtype=torch.uint8, device=dev)

        def step():
            T.quantize(dK, pK, workspace=qwork, stream=stream)
            T.quantize(dV, pV, workspace=qwork, stream=stream)
        units, unit, metric = 2 * n, "rows/s", f"tq_quantize rows/s, prefill write path (b={b})"
        alg = 2 * n * (2 * d + P)
        kern = "quantize"
    elif cfg["kind"] == "append":
        n_tok_rows, cache_rows = 256, 256 * 8192
        K, V = inputs.prefill(layers=32, heads=8, ctx=1)            # one token: 256 rows each
        hk = torch.empty((n_tok_rows, d), dtype=torch.bfloat16)
        hv = torch.empty((n_tok_rows, d), dtype=torch.bfloat16)
        K.fill(hk.view(torch.int16).numpy().view(np.uint16))
        V.fill(hv.view(torch.int16).numpy().view(np.uint16))
        dk, dv = hk.to(dev), hv.to(dev)
        cK, cV = T.empty_packed(cache_rows, dev), T.empty_packed(cache_rows, dev)
        # token position 4000 of every (layer, head) page of 8192 slots
        slots = torch.arange(n_tok_rows, dtype=torch.int64, device=dev) * 8192 + 4000

        def step():
            T.quantize_scatter(dk, slots, cK, stream=stream)
            T.quantize_scatter(dv, slots, cV, stream=stream)
        units, unit, metric = 1, "tokens/s", "decode-time append: one token's K and V rows (32 layers x 8 heads) into a paged packed cache"
        alg = 2 * n_tok_rows * (2 * d + P)
        kern = "step"
    else:
        db, qs = inputs.vector_search(n=cfg.get("n", 1_000_000))
        nq, ndb = qs.n_rows, db.n_rows
        hdb = torch.empty((ndb, d), dtype=torch.float32)
        db.fill(hdb.numpy())
        ddb = hdb.to(dev)
        del hdb
        dq = torch.from_numpy(qs.all()).to(dev)
        pk = T.empty_packed(ndb, dev)
        kq = 10
        idx = torch.empty((nq, kq), dtype=torch.int32, device=dev)
        val = torch.empty((nq, kq), dtype=torch.float32, device=dev)
        work = torch.empty(max(T.search_workspace_bytes(nq, ndb, kq), 16), dtype=torch.uint8, device=dev)
        qwork = torch.empty(max(T.quantize_workspace_bytes(ndb), 16), dtype=torch.uint8, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        split = {"quantize": 0.0, "search": 0.0}

        def step(timed=False):
            # quantize the database, then every query's top-10 by estimated
            # inner product (estimates on the tensor cores, top-k fused into
            # their epilogue)
            if timed: ev[0].record(stream)
            T.quantize(ddb, pk, workspace=qwork, stream=stream)
            if timed: ev[1].record(stream)
            T.search(dq, pk, ndb, kq, idx=idx, val=val, workspace=work, stream=stream)
            if timed:
                ev[2].record(stream)
                ev[2].synchronize()
                for i, k in enumerate(split):
                    split[k] += ev[i].elapsed_time(ev[i + 1])
        units, unit, metric = nq * ndb, "IP estimates/s", "vector search: quantize DB, all-pairs IP estimates, top-10"
        alg = ndb * (4 * d + P) + ndb * P + nq * kq * 8
        kern = "step"
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(ws)
    launches0 = tq.launch_count()
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(ws)
    ms = max_over_ranks(ws, e0.elapsed_time(e1)) / args.steps
    total = dist_util.sum_over_ranks(ws, units, device=dev)
    launches = tq.launch_count() - launches0
    graph_ms = None
    if cfg["kind"] == "append":
        graph_ms = append_graph_ms(torch, T, dev, stream, dk, dv, slots, cK, cV, args.steps)
    gbs = alg / (ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": kern, "achieved": gbs, "peak": hbm, "unit": "GB/s",
            "frac": gbs / hbm, "traffic": None, "algorithmic_bytes": alg, "peak_kind": hbm_kind}
    phases = None
    if cfg["kind"] == "vsearch":
        # per-phase device times in separate steps (events between the calls),
        # outside the timed region; the estimates are a dense contraction:
        # 2 nq ndb (d + m) algorithmic flops (the fp16 hi/lo form executes
        # 2 nq ndb (3 d + 2 m)), against the sustained tensor peak
        for _ in range(args.steps):
            step(timed=True)
        phases = {k: v / args.steps for k, v in split.items()}
        tf, tf_kind = tensor_peak()
        flops = 2.0 * nq * ndb * (d + m)
        ach = flops / (phases["search"] * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "search (estimates incl. key / query operands, fused top-10)", "achieved": ach,
                "peak": tf, "unit": "TFLOP/s", "frac": ach / tf, "traffic": None, "algorithmic_flops": flops,
                "executed_flops": 2.0 * nq * ndb * (3 * d + 2 * m), "peak_kind": tf_kind}
        recall = exact_recall(torch, ddb, dq, idx, kq)
    if rank == 0:
        print(json.dumps({
            "metric": metric, "value": total / (ms * 1e-3), "unit": unit, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": args.workload, "d": d, "b": b, "m": m, "l2": "inputs larger than L2; no flush"},
            "roofline": roof, "phases_ms": phases,
            "recall_at_10": recall if cfg["kind"] == "vsearch" else None,
            "cuda_graph_ms_per_step": graph_ms,
            "gpu_launches": launches, "clocks": clk.summary()}), flush=True)
    T.close()



def exact_recall(torch, ddb, dq, idx, k):
    """Recall@k of the search's answers against the exact top-k by fp32 inner
    product (the synthetic stand-in for the pages' Recall@k study; 0h-n0
    "ICLR 2026論文解説: TurboQuant", "実験結果 — ベクトル検索（Recall評価）").
    Reporting only, outside the timed region: a plain fp32 product (TF32
    off) per block of database rows, and torch's top-k."""
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        best_v = torch.full((dq.shape[0], k), -float("inf"), device=dq.device)
        best_i = torch.zeros((dq.shape[0], k), dtype=torch.int64, device=dq.device)
        blk = 131072
        for r0 in range(0, ddb.shape[0], blk):
            s = dq @ ddb[r0:r0 + blk].T
            v, i = torch.topk(s, k, dim=1)
            cat_v, cat_i = torch.cat([best_v, v], 1), torch.cat([best_i, i + r0], 1)
            top = torch.topk(cat_v, k, dim=1)
            best_v, best_i = top.values, torch.gather(cat_i, 1, top.indices)
        got = idx.to(torch.int64)
        hits = (got[:, :, None] == best_i[:, None, :]).any(dim=2).sum().item()
        return hits / float(got.numel())
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="decode-128k-b3", choices=sorted(WORKLOADS) + sorted(AUX_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in AUX_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the headline workload only"}))
            return
        ws, rank, local = dist_setup()
        try:
            run_aux(args, AUX_WORKLOADS[args.workload], ws, rank, local)
        finally:
            if ws > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    cfg = WORKLOADS[args.workload]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, cfg, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    ws, rank, local = dist_setup()
    try:
        run_ours(args, cfg, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
