#!/usr/bin/env python3
"""Throughput of the CSA / HCA hot path on B200 -- prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: for the default workload (CSA
decode at 1M context, Pro shape: B=4 requests, 262,144 compressed entries, MXFP4 indexer
keys, top-1024, 128 heads x 512) that is index scores -> top-k -> sparse MQA through
csa_forward. Inputs are resident in HBM; L2 reuse across steps is defeated by rotating
through input replicas whose total is several times the 126 MB L2. With N > 1 (torchrun)
every rank runs its own batch (requests are independent: weak scaling, no collective on
the data path) and the time is the max over ranks.

--impl reference times the float64 CPU oracle on the host cores on a bounded sample of
the same workload (one query per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA decode queries/s at 1M ctx (Flash/Pro shape); % of B200 HBM roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
NOMINAL_HBM_GBS = 8000.0  # a B200's nominal HBM3e bandwidth, reported beside the measured one
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--streams", type=int, default=1,
                    help="CUDA streams the steps alternate over (independent batches in flight; "
                         "1: one step after another)")
    ap.add_argument("--concurrent", type=int, default=3,
                    help="also time the steps over this many streams and report it as an extra "
                         "key (0: skip); `value` stays that of --streams")
    ap.add_argument("--rounds", type=int, default=5,
                    help="timed rounds of K steps each; the median round gives the value")
    ap.add_argument("--workload", default="pro_decode_1m")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--replicas", type=int, default=0,
                    help="input replicas rotated across steps (0: enough to defeat the L2)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end measurement")
    ap.add_argument("--part", default=None, choices=sorted(PARTS),
                    help="time one extension kernel family on the workload's shape instead of "
                         "the hot path (its own JSON line; see run_part)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move; score spill and scratch excluded)
# ---------------------------------------------------------------------------

def indexer_key_bytes(s) -> int:
    d = s.d_idx
    return {"bf16": 2 * d, "fp8": d + 4, "mxfp4": d // 2 + d // 32, "f32": 4 * d}[s.idx]


def indexer_query_bytes(s) -> int:
    d, h = s.d_idx, s.n_idx_heads
    q = {"bf16": 2 * d * h, "fp8": 2 * d * h, "mxfp4": (d // 2 + d // 32) * h,
         "f32": 4 * d * h}[s.idx]
    return q + 4 * h  # + head weights


def algorithmic_bytes_per_query(s, n_vis: int) -> dict:
    """Per query: indexer-key scan + q^I + w (indexer), selected + window KV rows, q, out."""
    io = 2 if s.io == "bf16" else 4
    row = s.c * io
    qo = 2 * s.n_heads * s.c * io
    if s.kind == "hca_decode":
        return {"index": 0, "total": (n_vis + s.n_win) * row + qo}
    idx = n_vis * indexer_key_bytes(s) + indexer_query_bytes(s)
    att = (min(s.topk, n_vis) + s.n_win) * row + qo
    return {"index": idx, "total": idx + att}


def workload_config(s, l2: str, parallelism: str) -> dict:
    """The `config` object of a bench line: the workload and its sizes (both arms)."""
    n_vis = min(s.ctx // s.m, s.n_cap) if s.kind != "csa_prefill" else s.n_cap
    return {"workload": s.name, "B_per_gpu": s.B, "T": s.T, "ctx": s.ctx, "entries": n_vis,
            "heads": s.n_heads, "c": s.c, "topk": s.topk, "indexer_keys": s.idx,
            "n_win": s.n_win, "l2": l2, "parallelism": parallelism}


def prefill_flops(s) -> dict:
    """Indexer: 2 * H_I * d_I per visible (t, s) pair; attention: 4 * c flops per head per
    attended row (q.k and p.v), rows = min(k, visible) + window."""
    vis = [min((s.ctx + i) // s.m, s.n_cap) for i in range(s.T)]
    pairs = sum(vis)
    rows = sum(min(s.topk, v) + min(s.n_win, s.ctx + i + 1) for i, v in enumerate(vis))
    idx = 2 * s.n_idx_heads * s.d_idx * pairs * s.B
    att = 4 * s.c * s.n_heads * rows * s.B
    return {"index": idx, "attention": att, "total": idx + att}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def traffic_from_profile(kernel_src: str, kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary of this kernel and
    workload, or None when there is none or the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_per_launch_bytes:\s*([0-9]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not h:
        return None
    cur = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    return int(m.group(1)) if cur == h.group(1) else None


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index: int):
        self.proc = None
        self.dev = dev_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={dev_index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample of the workload
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [d.get("num_threads", 1) for d in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_queries_per_s(s, inp, budget_s: float, max_queries: int = 64):
    from oracle import pipeline as P

    qs = [(b, t) for t in range(s.T) for b in range(s.B)]
    done, t0 = 0, time.perf_counter()
    while done < min(len(qs), max_queries) and (time.perf_counter() - t0) < budget_s:
        P.run(s, inp, [qs[done]])
        done += 1
    el = time.perf_counter() - t0
    return done / el, done, el


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_ours(args, W, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import long_context_sparse_08_b200 as csa
    from long_context_sparse_08_b200 import runner as R

    torch.cuda.set_device(local_rank)
    s = W.SHAPES[args.workload]
    inp = W.make_inputs(s)
    dev0 = R.upload(inp, s)
    one_set = sum(t.numel() * t.element_size() for t in dev0.values())
    # replicas: device copies, enough that a cycle touches well over the L2
    touched = s.B * s.T * algorithmic_bytes_per_query(
        s, min(s.ctx // s.m if s.kind != "csa_prefill" else s.n_cap, s.n_cap))["total"]
    R_rep = max(2, min(16, int(np.ceil(3 * L2_BYTES / max(touched, 1)))))
    free = torch.cuda.mem_get_info()[0]
    while R_rep > 2 and R_rep * one_set > 0.6 * free:
        R_rep -= 1
    if args.replicas > 0:
        R_rep = args.replicas
    S_str = max(1, args.streams)
    S_all = max(S_str, args.concurrent if args.concurrent > 1 else 1)
    R_rep = -(-R_rep // S_all) * S_all  # a multiple of the streams: a replica stays on one stream
    devs = [dev0] + [{k: v.clone() for k, v in dev0.items()} for _ in range(R_rep - 1)]
    for d in devs:  # per-query inputs side by side, so one copy uploads a step's inputs
        pack_query_inputs(d)
    steps = [R.Step(s, d) for d in devs]
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        steps[i % R_rep]()
    torch.cuda.synchronize()

    K = args.steps
    has_index = s.kind != "hca_decode"
    clocks = Clocks(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # `rounds` timed rounds of K steps each (every round bracketed by events on the launching
    # stream); the median round gives the value
    rounds = max(1, args.rounds)
    t0 = [torch.cuda.Event(enable_timing=True) for _ in range(rounds)]
    t1 = [torch.cuda.Event(enable_timing=True) for _ in range(rounds)]
    side_all = [torch.cuda.Stream() for _ in range(S_all - 1)]

    def timed_rounds(n_streams):
        """ms of each round of K steps, the steps alternating over n_streams streams."""
        side = side_all[:n_streams - 1]
        strs = [stream] + side
        for r in range(rounds):
            t0[r].record(stream)
            for sd in side:  # every stream starts after the round's start event
                sd.wait_event(t0[r])
            for i in range(K):
                j = r * K + i
                steps[j % R_rep](strs[j % n_streams])
            for sd in side:  # and the round ends when every stream has drained
                ev = torch.cuda.Event()
                ev.record(sd)
                stream.wait_event(ev)
            t1[r].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in zip(t0, t1)]

    launches0 = csa.kernel_launches()
    ms_rounds = timed_rounds(S_str)
    launches = (csa.kernel_launches() - launches0) // rounds
    if world > 1:
        dist.barrier()
    conc = None
    if S_all > S_str:  # the same steps with more independent batches in flight
        conc_rounds = timed_rounds(S_all)
        conc = float(np.median(conc_rounds))
    clk = clocks.stop()
    ms = float(np.median(ms_rounds))
    # The dominant kernel (the indexer) is timed by events around each of its launches over
    # a second pass of the same K steps: events between the kernels of a step would stop
    # the next kernel from being launched before its predecessor ends, so they stay out of
    # the pass that gives `value`.
    idx_ms = None
    if has_index:
        ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for e in ev_b + ev_a:  # torch creates the CUDA event on first record
            e.record(stream)
        torch.cuda.synchronize()
        csa.set_index_timing_events(ev_b, ev_a)
        for i in range(K):
            steps[i % R_rep]()
        torch.cuda.synchronize()
        idx_ms = sum(b.elapsed_time(a) for b, a in zip(ev_b, ev_a)) / K
        csa.set_index_timing_events([], [])
    att_ms = None
    if not has_index:
        # HCA: the step is the dense attention call (attention kernel + split merge); events
        # around each call, in a second pass of the same K steps
        ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        for i in range(K):
            ev_b[i].record(stream)
            steps[i % R_rep]()
            ev_a[i].record(stream)
        torch.cuda.synchronize()
        att_ms = sum(b.elapsed_time(a) for b, a in zip(ev_b, ev_a)) / K
    ms = max_over_ranks(ms, world, "cuda")

    # end to end through the public API: per-step query-side inputs from pinned host
    # memory, the call, and the result back to pinned host memory
    e2e = None if args.no_e2e else run_e2e(args, s, devs, steps, R_rep, world)

    n_vis = min(s.ctx // s.m, s.n_cap) if s.kind != "csa_prefill" else s.n_cap
    per_q = algorithmic_bytes_per_query(s, n_vis)
    queries = s.B * s.T
    value = whole_job_rate(world, queries, K, ms)
    peaks, peak_src = load_peaks()
    roof = None
    if has_index and idx_ms and s.kind == "csa_prefill":
        # prefill: the indexer is a dense contraction over the visible (t, s) pairs; its
        # algorithmic flops against the dense bf16 tensor peak (sustained: it runs inside a
        # step of milliseconds)
        fl = prefill_flops(s)["index"]
        tf = fl / (idx_ms / 1e3) / 1e12
        pk = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        src = os.path.join(ROOT, "long_context_sparse_08_b200", "csrc", "indexer_bf16.cu")
        roof = {"kernel": "k_index_bf16_tc", "bound": "tensor", "achieved": round(tf, 1),
                "peak": pk, "unit": "TFLOP/s", "frac": round(tf / pk, 4),
                "frac_of_burst": round(tf / peaks["bf16_tflops"], 4),
                "traffic": traffic_from_profile(src, "k_index_bf16_tc", s.name),
                "alg_flops_per_step": fl, "avg_ms_per_step": round(idx_ms, 5),
                "peak_source": f"{peak_src} bf16_tflops_sustained (cuBLAS, seconds-long loop)"}
    elif att_ms:
        alg = queries * per_q["total"]
        achieved = alg / (att_ms / 1e3) / 1e9
        src = os.path.join(ROOT, "long_context_sparse_08_b200", "csrc", "mqa_tc.cu")
        roof = {"kernel": "k_mqa_tc (dense) + k_mqa_combine", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                "nominal_peak": NOMINAL_HBM_GBS,
                "traffic": traffic_from_profile(src, "k_mqa_tc", s.name),
                "alg_bytes_per_launch": alg, "avg_launch_ms": round(att_ms, 5),
                "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)"}
    elif has_index and idx_ms:
        alg = queries * per_q["index"]
        achieved = alg / (idx_ms / 1e3) / 1e9
        if s.idx == "mxfp4":
            # the MXFP4 indexer also selects the top k of every decode query (fused): the
            # time covers both, the bytes are the key stream's
            kname, kfile = "k_index_mxf4_tc", "indexer_mxf4.cu"
        elif s.idx in ("fp8", "bf16") and s.n_cap % 128 == 0 and s.n_idx_heads == 64 \
                and s.d_idx == 128:
            kname, kfile = "k_index_bf16_tc", "indexer_bf16.cu"
        else:
            kname, kfile = "k_index_scores_cc", "indexer.cu"
        src = os.path.join(ROOT, "long_context_sparse_08_b200", "csrc", kfile)
        roof = {"kernel": kname, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                "nominal_peak": NOMINAL_HBM_GBS,
                "traffic": traffic_from_profile(src, kname, s.name),
                "alg_bytes_per_launch": alg, "avg_launch_ms": round(idx_ms, 5),
                "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)"}
    step_bytes = queries * per_q["total"]
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "queries/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
        "rounds": {"n": rounds, "ms_per_step": [round(x / K, 5) for x in ms_rounds],
                   "value_from": "median round", "streams": S_str},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"mxfp4": "mxfp4+bf16", "fp8": "e4m3+bf16", "bf16": "bf16",
                  "none": "bf16", "f32": "f32"}[s.idx],
        "data": "synthetic (seeded N(0,1); shapes of the Pro/Flash configs)",
        "config": workload_config(
            s, l2=f"{R_rep} rotating input replicas ({R_rep * one_set / 1e9:.2f} GB); "
                  f"bytes touched per cycle {R_rep * step_bytes / 1e6:.0f} MB > L2",
            parallelism=f"replicas x{world} (independent requests)"),
        # decode steps are bounded by HBM; a prefill chunk is compared with the tensor peak
        # instead (`tflops` below)
        "step_hbm_roofline": None if s.kind == "csa_prefill" else {
            "alg_bytes_per_step": step_bytes,
            "frac_of_peak": round(step_bytes / (ms / K / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
            "frac_of_nominal": round(step_bytes / (ms / K / 1e3) / 1e9 / NOMINAL_HBM_GBS, 4)},
        "roofline": roof,
        "concurrent_batches": None if conc is None else {
            "streams": S_all, "batches_in_flight": S_all,
            "value": round(whole_job_rate(world, queries, K, max_over_ranks(conc, world, "cuda")), 2),
            "unit": "queries/s", "ms_per_step": round(conc / K, 5),
            "note": "the same steps, each a whole csa_forward over its own batch, alternating "
                    "over streams so that several independent batches are in flight; `value` "
                    "is the one-batch-at-a-time figure"},
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches,
    }
    if s.kind == "csa_prefill":
        # a compute-bound step: algorithmic flops (indexer over the visible (t, s) pairs,
        # attention over the selected and window rows) against the dense bf16 tensor peak
        fl = prefill_flops(s)
        tf = fl["total"] / (ms / K / 1e3) / 1e12
        res["tflops"] = {"value": round(tf, 1), "flops_per_step": fl,
                         "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
                         "frac_of_bf16_sustained": round(
                             tf / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4),
                         "peak": peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16_tflops (cuBLAS burst)"}
    return res, inp, s


def max_over_ranks(ms: float, world: int, device: str) -> float:
    """The timed region's length as the slowest rank saw it (all ranks get the max)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist

    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def whole_job_rate(world: int, queries_per_rank: int, steps: int, ms: float) -> float:
    """Queries per second of the whole job: every rank ran `steps` steps of its own batch
    (weak scaling) and the job took `ms`, the max over ranks."""
    return world * queries_per_rank * steps / (ms / 1e3)


QUERY_INPUTS = ("q", "qI", "qI_scale", "w", "q_pos")


def pack_query_inputs(d):
    """Move the per-query inputs of one replica into one device buffer (256-byte aligned
    views), so a serving step uploads them with a single copy."""
    import torch

    names = [k for k in QUERY_INPUTS if k in d]
    offs, total = [], 0
    for k in names:
        offs.append(total)
        total += (d[k].numel() * d[k].element_size() + 255) // 256 * 256
    buf = torch.empty((total,), dtype=torch.uint8, device=d[names[0]].device)
    for k, o in zip(names, offs):
        n = d[k].numel() * d[k].element_size()
        view = buf[o:o + n].view(d[k].dtype).view(d[k].shape)
        view.copy_(d[k])
        d[k] = view
    d["_query_pack"] = buf


def run_e2e(args, s, devs, steps, R_rep, world):
    import torch

    host = [d["_query_pack"].cpu().pin_memory() for d in devs]  # one upload per step
    outs = [torch.empty_like(st.out, device="cpu").pin_memory() for st in steps]
    idxs = [torch.empty_like(st.out_idx, device="cpu").pin_memory()
            if st.out_idx is not None else None for st in steps]
    bi = host[0].numel()  # bytes of the packed per-query inputs copied each step
    bo = outs[0].numel() * outs[0].element_size() + \
        (idxs[0].numel() * idxs[0].element_size() if idxs[0] is not None else 0)
    # A serving loop: inputs go up on one copy stream and results come back on another, so
    # step i+1's upload and step i-1's read-back overlap step i's kernels. Every step's
    # copies are inside the timed region; replica buffers are reused only after the step
    # that last used them has finished reading them (events).
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(R_rep)]
    ev_comp = [torch.cuda.Event() for _ in range(R_rep)]
    ev_down = [torch.cuda.Event() for _ in range(R_rep)]
    for e in ev_comp + ev_down:
        e.record(comp)

    def one(i):
        j = i % R_rep
        up.wait_event(ev_comp[j])  # the previous step on these buffers has read its inputs
        with torch.cuda.stream(up):
            devs[j]["_query_pack"].copy_(host[j], non_blocking=True)
        ev_up[j].record(up)
        comp.wait_event(ev_up[j])
        comp.wait_event(ev_down[j])  # the previous result of these buffers is back
        steps[j](comp)
        ev_comp[j].record(comp)
        down.wait_event(ev_comp[j])
        with torch.cuda.stream(down):
            outs[j].copy_(steps[j].out, non_blocking=True)
            if idxs[j] is not None:
                idxs[j].copy_(steps[j].out_idx, non_blocking=True)
        ev_down[j].record(down)

    for i in range(args.warmup):
        one(i)
    torch.cuda.synchronize()
    K = args.steps
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(comp)
    up.wait_event(a)  # the first upload starts inside the timed region
    for i in range(K):
        one(i)
    for j in range(R_rep):  # the last results are back on the host side
        comp.wait_event(ev_down[j])
    b.record(comp)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    return {"value": round(world * s.B * s.T * K / (ms / 1e3), 2), "unit": "queries/s",
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "state_resident": "compressed KV, indexer keys and window rows stay in HBM"}


# ---------------------------------------------------------------------------
# --part: the extension kernels timed alone on the workload's shapes
# ---------------------------------------------------------------------------

# grouped output projection (Q, H, c, g, d_g, d) per decode workload: the model table's
# g / d_g / d with the workload's batch as the queries
OUT_PROJ_SHAPES = {"pro_decode_1m": (4, 128, 512, 16, 1024, 7168),
                   "flash_decode_131k": (8, 64, 512, 8, 1024, 4096),
                   "hca_decode_1m": (16, 64, 512, 8, 1024, 4096)}


def out_proj_bytes(Q, H, c, g, d_g, d) -> int:
    """Algorithmic bytes of one grouped output projection: both weight matrices (bf16), the
    attention outputs read and the projection written (fp32 partials are scratch)."""
    k1 = c * H // g
    return 2 * (g * k1 * d_g + g * d_g * d) + 2 * Q * H * c + 2 * Q * d


def state_append_bytes(c, m, overlap, key_c=128, key_fmt_bytes=68) -> dict:
    """Algorithmic bytes of appending one token to one request, averaged over a block: the
    raw rows read and stored in the state, the window row read and stored (KV only), and,
    every m-th token, the block's rows read back and the finished row written. KV entries
    are bf16 rows of c values; indexer keys are c = 128 values stored as MXFP4 (68 B)."""
    rows = 4 if overlap else 2
    kv = 2 * c * (rows * 2 + 2) + (2 * m * rows * c + 2 * c) // m
    keys = 2 * key_c * rows * 2 + (2 * m * rows * key_c + key_fmt_bytes) // m
    return {"kv": kv, "keys": keys, "total": kv + keys}


def _time_calls(fn, n_rep, warmup, steps):
    """Mean ms per call of fn(i) over `steps` calls (rotating i over n_rep replicas),
    timed with CUDA events on the current stream after `warmup` calls."""
    import torch

    for i in range(warmup):
        fn(i % n_rep)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(steps):
        fn(i % n_rep)
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def check_part_workload(part, s):
    """Exit with a message when a part cannot run on the workload's caches (before any GPU
    work): the paged indexer and the BF16-score path take the tensor-core indexers' keys
    (MXFP4, FP8 or bf16), the paged layer and the layout comparison a decode step."""
    want = None
    if part == "forward_paged" and s.kind == "hca_decode":
        want = None  # the HCA layer: no indexer
    elif part in ("bf16_scores", "forward_paged") and s.idx not in ("mxfp4", "fp8", "bf16"):
        want = "MXFP4, FP8 or bf16 indexer keys"
    elif part == "forward_paged" and s.kind != "csa_decode":
        want = "a CSA or HCA decode step"
    elif part == "kv_layouts" and s.kind not in ("csa_decode", "hca_decode"):
        want = "a CSA or HCA decode step"
    elif part == "stream" and s.kind != "csa_decode":
        want = "a CSA decode step (its indexer's key stream)"
    if want:
        raise SystemExit(f"--part {part} wants a workload with {want} "
                         f"(e.g. --workload pro_decode_1m); {s.name} has "
                         f"{s.kind} / {s.idx} keys")


def run_part(args, W):
    """One JSON line for an extension kernel family on the workload's shape:
    out_proj          grouped output projection of the batch's queries (HBM roofline);
    out_proj_prefill  its tensor-core form on a prefill chunk's queries (tensor roofline);
    state_append      one decode token per request into the KV and indexer-key state caches;
    kv_layouts        the attention alone over bf16, mixed-precision and paged caches (CSA
                      or, on an HCA workload, the dense form);
    bf16_scores       index + top-k with fp32 and with BF16 scores;
    forward_paged     the CSA (or HCA) layer over page pools and a window ring vs the
                      contiguous one;
    stream            the device's own rate for one read of the indexer's key bytes (a torch
                      reduction and a torch copy of that many bytes, no library kernel): the
                      short-stream ceiling the indexer is compared with."""
    s = W.SHAPES[args.workload]
    check_part_workload(args.part, s)
    import torch
    import long_context_sparse_08_b200 as csa
    from long_context_sparse_08_b200 import runner as R

    torch.cuda.set_device(0)
    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
    before = csa.kernel_launches()
    clocks = Clocks(0)
    line = {"part": args.part, "workload": args.workload, "steps": args.steps,
            "warmup": args.warmup, "data": "synthetic (seeded)"}
    if args.part == "out_proj":
        Q, H, c, g, d_g, d = OUT_PROJ_SHAPES[args.workload]
        inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=11)
        nbytes = out_proj_bytes(Q, H, c, g, d_g, d)
        n_rep = max(1, min(4, int(np.ceil(3 * L2_BYTES / nbytes))))
        p = csa.make_params(c=c, n_heads=H)
        reps = []
        for _ in range(n_rep):
            dv = {k: torch.from_numpy(v.view(np.int16)).cuda() for k, v in inp.items()}
            need = csa.grouped_out_proj_workspace_size(p, Q, g, d_g, d)
            dv["ws"] = torch.empty((need,), dtype=torch.uint8, device="cuda")
            dv["out"] = torch.empty((Q, d), dtype=torch.int16, device="cuda")
            reps.append((dv, need))

        def call(i):
            dv, need = reps[i]
            csa.csa_grouped_out_proj(p, Q, g, d_g, d, dv["o"], dv["w_grp"], dv["w_out"],
                                     dv["out"], dv["ws"], need)

        ms = _time_calls(call, n_rep, args.warmup, args.steps)
        ach = nbytes / (ms / 1e3) / 1e9
        line.update(metric="grouped output projection calls/s", value=round(1e3 / ms, 2),
                    unit="calls/s", ms_per_call=round(ms, 5),
                    config={"Q": Q, "H": H, "c": c, "g": g, "d_g": d_g, "d": d,
                            "replicas": n_rep},
                    roofline={"bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
                              "peak_source": peak_src, "unit": "GB/s",
                              "frac": round(ach / hbm, 4), "bytes_per_call": nbytes})
    elif args.part == "state_append":
        B, c = s.B, s.c
        p_kv = csa.make_params(m=4, overlap=1, c=c, rope_dims=s.rope_dims, n_win=s.n_win)
        p_k = csa.make_params(m=4, overlap=1, c=128, rope_dims=64, n_win=s.n_win)
        g = torch.Generator(device="cuda").manual_seed(5)
        rnd = lambda *sh: torch.randn(*sh, generator=g, device="cuda").to(torch.bfloat16)  # noqa
        n_steps = args.warmup + args.steps
        t0 = 4 * 128  # every request past its first page
        kv_rows = {k: rnd(n_steps, B, c) for k in ("Ca", "Cb", "Za", "Zb", "win")}
        key_rows = {k: rnd(n_steps, B, 128) for k in ("Ca", "Cb", "Za", "Zb")}
        bias_kv, bias_k = rnd(8, c), rnd(8, 128)
        max_pages = (t0 + n_steps) // 128 + 2
        table32 = torch.arange(B * max_pages, dtype=torch.int32, device="cuda").view(B, -1)
        table128 = table32.clone()
        st_kv = torch.zeros((B, 8, 4, c), dtype=torch.bfloat16, device="cuda")
        st_k = torch.zeros((B, 8, 4, 128), dtype=torch.bfloat16, device="cuda")
        ring = torch.zeros((B, s.n_win, c), dtype=torch.bfloat16, device="cuda")
        pages_kv = torch.zeros((B * max_pages, 32, c), dtype=torch.bfloat16, device="cuda")
        pages_k = torch.zeros((B * max_pages, 128, 64), dtype=torch.uint8, device="cuda")
        exps_k = torch.zeros((B * max_pages, 128, 4), dtype=torch.uint8, device="cuda")
        pos_all = t0 + torch.arange(n_steps, device="cuda", dtype=torch.int64)[:, None].repeat(1, B)

        def call(i):
            pos = pos_all[i]
            csa.csa_state_append(p_kv, csa.CSA_BF16, B, pos, kv_rows["Ca"][i], kv_rows["Cb"][i],
                                 kv_rows["Za"][i], kv_rows["Zb"][i], kv_rows["win"][i], bias_kv,
                                 None, 1, st_kv, ring, csa.CSA_BF16, pages_kv, None,
                                 B * max_pages, 32, table32, max_pages)
            csa.csa_state_append(p_k, csa.CSA_BF16, B, pos, key_rows["Ca"][i], key_rows["Cb"][i],
                                 key_rows["Za"][i], key_rows["Zb"][i], None, bias_k, None, 0,
                                 st_k, None, csa.CSA_MXFP4, pages_k, exps_k, B * max_pages, 128,
                                 table128, max_pages)

        for i in range(args.warmup):
            call(i)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(args.warmup, n_steps):
            call(i)
        b.record()
        torch.cuda.synchronize()
        eager_ms = a.elapsed_time(b) / args.steps
        # The two launches of a step take microseconds on the device, less than the host
        # needs to issue them: the same timed steps captured once in a CUDA graph and
        # replayed give the device's rate (every replay repeats the same appends).
        ms, how = eager_ms, "eager launches (host-bound)"
        try:
            gs = torch.cuda.Stream()
            gs.wait_stream(torch.cuda.current_stream())
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=gs, capture_error_mode="thread_local"):
                for i in range(args.warmup, n_steps):
                    call(i)
            graph.replay()
            torch.cuda.synchronize()
            reps = 5
            a.record()
            for _ in range(reps):
                graph.replay()
            b.record()
            torch.cuda.synchronize()
            ms, how = a.elapsed_time(b) / (reps * args.steps), "CUDA graph replay"
            del graph
        except Exception as e:  # capture not possible here: keep the eager number
            how = f"eager launches (graph capture failed: {type(e).__name__})"
        per = state_append_bytes(c, 4, 1)
        ach = B * per["total"] / (ms / 1e3) / 1e9
        line.update(metric="decode appends/s (KV + indexer keys, one token per request)",
                    value=round(B / (ms / 1e3), 1), unit="appends/s", ms_per_step=round(ms, 5),
                    timing=how, eager_ms_per_step=round(eager_ms, 5),
                    config={"requests": B, "c": c, "kv": "bf16 pages of 32 entries",
                            "keys": "MXFP4 pages of 128 keys"},
                    roofline={"bound": "latency (a few KB per request)", "achieved": round(ach, 2),
                              "peak": hbm, "peak_source": peak_src, "unit": "GB/s",
                              "frac": round(ach / hbm, 6), "bytes_per_append": per})
    elif args.part == "kv_layouts":
        # the attention alone over the bf16 cache, mixed-precision rows and a shuffled page
        # pool: CSA (the selected rows; pages of 32 entries) or HCA (every visible entry;
        # pages of one entry)
        inp = W.make_inputs(s)
        dev = R.upload(inp, s)
        p = R.params_for(s)
        B, T, k = s.B, s.T, s.topk
        hca = s.kind == "hca_decode"
        g = torch.Generator(device="cpu").manual_seed(9)
        n_vis = min(s.ctx // s.m, s.n_cap)
        if not hca:
            idx = torch.stack([torch.randperm(n_vis, generator=g)[:k] for _ in range(B * T)])
            idx = idx.view(B, T, k).to(torch.int32).cuda()
        kv = W.bf16_bits_to_f32(inp["kv_cache"])
        codes, scale, rope = W.quant_mixed_kv(kv, s.rope_dims)
        del kv
        mixed = torch.from_numpy(np.concatenate([codes, rope.view(np.uint8)], axis=-1)).cuda()
        mscale = torch.from_numpy(scale).cuda()
        del codes, rope
        pr = 1 if hca else 32
        max_pages = s.n_cap // pr
        perm = torch.randperm(B * max_pages, generator=g).to(torch.int32)
        table = perm.view(B, max_pages).cuda()
        pool = torch.empty((B * max_pages, pr, s.c), dtype=dev["kv_cache"].dtype, device="cuda")
        pool[table.view(-1).long()] = dev["kv_cache"].view(B * max_pages, pr, s.c)
        out = torch.empty((B, T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
        entry = csa.CSA_WS_HCA_MQA if hca else csa.CSA_WS_SPARSE_MQA
        ws_bytes = csa.workspace_size(p, entry, 0, B, T, s.n_cap)
        ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
        pkv = csa.paged_kv(csa.CSA_BF16, pool, None, table, B * max_pages, pr, max_pages)
        L = dev["win_kv"].shape[1]
        q, qp, win, w0, sink = dev["q"], dev["q_pos"], dev["win_kv"], dev["win_pos0"], dev["sink"]
        if hca:
            calls = {
                "bf16": lambda i: csa.hca_dense_mqa(p, csa.CSA_BF16, B, T, q, qp, dev["kv_cache"],
                                                    s.n_cap, win, L, w0, sink, None, out, ws,
                                                    ws_bytes),
                "mixed": lambda i: csa.hca_dense_mqa_mixed_kv(p, B, T, q, qp, mixed, mscale,
                                                              s.n_cap, win, L, w0, sink, None,
                                                              out, ws, ws_bytes),
                "paged_bf16": lambda i: csa.hca_dense_mqa_paged(p, B, T, q, qp, pkv, win, L, w0,
                                                                sink, None, out, ws, ws_bytes)}
        else:
            calls = {
                "bf16": lambda i: csa.csa_sparse_mqa(p, csa.CSA_BF16, B, T, q, qp,
                                                     dev["kv_cache"], s.n_cap, idx, win, L, w0,
                                                     sink, None, out, ws, ws_bytes),
                "mixed": lambda i: csa.csa_sparse_mqa_mixed_kv(p, B, T, q, qp, mixed, mscale,
                                                               s.n_cap, idx, win, L, w0, sink,
                                                               None, out, ws, ws_bytes),
                "paged_bf16": lambda i: csa.csa_sparse_mqa_paged(p, B, T, q, qp, pkv, idx, win,
                                                                 L, w0, sink, None, out, ws,
                                                                 ws_bytes)}
        rows = n_vis if hca else k  # cache rows each query reads
        res = {}
        for name, fn in calls.items():
            ms = _time_calls(fn, 1, args.warmup, args.steps)
            row = 1024 if name != "mixed" else s.c + s.rope_dims + 4
            nbytes = B * T * ((rows * row) + s.n_win * 2 * s.c + 2 * 2 * s.n_heads * s.c)
            res[name] = {"ms_per_call": round(ms, 5), "bytes_per_call": nbytes,
                         "achieved_gbs": round(nbytes / (ms / 1e3) / 1e9, 1)}
        line.update(metric=f"{'dense' if hca else 'sparse'} MQA calls/s by cache layout",
                    value=round(1e3 / res["mixed"]["ms_per_call"], 2), unit="calls/s (mixed)",
                    layouts=res, config={"B": B, "T": T, "rows_per_query": rows,
                                         "n_cap": s.n_cap, "page_rows": pr},
                    roofline={"bound": "hbm (dense rows)" if hca else
                              "latency (one CTA per query and head group)", "peak": hbm,
                              "peak_source": peak_src, "unit": "GB/s"})
    elif args.part == "bf16_scores":
        # index + top-k with fp32 scores (csa_index_topk) and with BF16 scores
        # (csa_index_topk_bf16) on the workload's keys (MXFP4 / FP8 / bf16 tensor-core indexers)
        inp = W.make_inputs(s)
        dev = R.upload(inp, s)
        p = R.params_for(s)
        kdt = csa.DTYPES[s.idx]
        B, T, N = s.B, s.T, s.n_cap
        out_idx = torch.empty((B, T, s.topk), dtype=torch.int32, device="cuda")
        res = {}
        for name, entry in (("fp32", csa.CSA_WS_INDEX_TOPK), ("bf16", csa.CSA_WS_INDEX_TOPK_BF16)):
            need = csa.workspace_size(p, entry, kdt, B, T, N)
            ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
            if name == "fp32":
                fn = lambda i, ws=ws, need=need: csa.csa_index_topk(  # noqa: E731
                    p, kdt, B, T, N, dev["qI"], dev.get("qI_scale"), dev["w"], dev["KI"],
                    dev.get("KI_scale"), dev["q_pos"], out_idx, None, ws, need)
            else:
                fn = lambda i, ws=ws, need=need: csa.csa_index_topk_bf16(  # noqa: E731
                    p, kdt, B, T, N, dev["qI"], dev.get("qI_scale"), dev["w"], dev["KI"],
                    dev.get("KI_scale"), dev["q_pos"], out_idx, None, ws, need)
            ms = _time_calls(fn, 1, args.warmup, args.steps)
            res[name] = {"ms_per_call": round(ms, 5),
                         "score_bytes_per_call": B * T * N * (4 if name == "fp32" else 2)}
        line.update(metric="index + top-k calls/s by score precision",
                    value=round(1e3 / res["bf16"]["ms_per_call"], 2), unit="calls/s (bf16)",
                    precisions=res, config={"B": B, "T": T, "n_cap": N, "k": s.topk,
                                            "keys": s.idx},
                    roofline={"bound": "hbm (key stream)", "peak": hbm, "peak_source": peak_src,
                              "unit": "GB/s"})
    elif args.part == "out_proj_prefill":
        # the tensor-core form on a prefill chunk: Flash shapes, the workload's queries
        Q, (H, c, g, d_g, d) = max(s.B * s.T, 128), (64, 512, 8, 1024, 4096)
        inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=12)
        p = csa.make_params(c=c, n_heads=H)
        dv = {k: torch.from_numpy(v.view(np.int16)).cuda() for k, v in inp.items()}
        need = csa.grouped_out_proj_workspace_size(p, Q, g, d_g, d)
        ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
        out = torch.empty((Q, d), dtype=torch.int16, device="cuda")
        fn = lambda i: csa.csa_grouped_out_proj(p, Q, g, d_g, d, dv["o"], dv["w_grp"],  # noqa
                                                dv["w_out"], out, ws, need)
        ms = _time_calls(fn, 1, args.warmup, args.steps)
        flops = 2.0 * Q * (c * H * d_g + g * d_g * d)
        tf = flops / (ms / 1e3) / 1e12
        peak_tf = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
        line.update(metric="grouped output projection TFLOP/s (prefill)", value=round(tf, 1),
                    unit="TFLOP/s", ms_per_call=round(ms, 5),
                    config={"Q": Q, "H": H, "c": c, "g": g, "d_g": d_g, "d": d},
                    roofline={"bound": "tensor", "achieved": round(tf, 1), "peak": peak_tf,
                              "peak_source": peak_src, "unit": "TFLOP/s",
                              "frac": round(tf / peak_tf, 4), "flops_per_call": flops})
    elif args.part == "forward_paged" and s.kind == "hca_decode":
        # the HCA layer over a shuffled pool of one-entry pages with the window as a ring,
        # against hca_dense_mqa on the contiguous cache and the linear window
        inp = W.make_inputs(s)
        dev = R.upload(inp, s)
        p = R.params_for(s)
        B, T, N = s.B, s.T, s.n_cap
        g = torch.Generator(device="cpu").manual_seed(10)
        perm = torch.randperm(B * N, generator=g).to(torch.int32).cuda()
        table = perm.view(B, N)
        pool = torch.empty((B * N, 1, s.c), dtype=dev["kv_cache"].dtype, device="cuda")
        pool[perm.long()] = dev["kv_cache"].view(B * N, 1, s.c)
        kv = csa.paged_kv(csa.CSA_BF16, pool, None, table, B * N, 1, N)
        ring = torch.empty((B, s.n_win, s.c), dtype=dev["win_kv"].dtype, device="cuda")
        for b in range(B):
            t, p0 = int(inp["q_pos"][b, 0]), int(inp["win_pos0"][b])
            for q0 in range(max(t - s.n_win + 1, 0), t + 1):
                ring[b, q0 % s.n_win] = dev["win_kv"][b, q0 - p0]
        need = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, B, T, N)
        ws = torch.empty((max(need, 1),), dtype=torch.uint8, device="cuda")
        out = torch.empty((B, T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
        L = dev["win_kv"].shape[1]
        calls = {
            "contiguous": lambda i: csa.hca_dense_mqa(
                p, csa.CSA_BF16, B, T, dev["q"], dev["q_pos"], dev["kv_cache"], N, dev["win_kv"],
                L, dev["win_pos0"], dev["sink"], None, out, ws, need),
            "paged": lambda i: csa.hca_dense_mqa_paged(
                p, B, T, dev["q"], dev["q_pos"], kv, ring, s.n_win, None, dev["sink"], None, out,
                ws, need)}
        res = {name: round(_time_calls(fn, 1, args.warmup, args.steps), 5)
               for name, fn in calls.items()}
        line.update(metric="HCA layer calls/s over the state cache's page pool",
                    value=round(1e3 / res["paged"], 2), unit="calls/s (paged)",
                    ms_per_call=res, config={"B": B, "T": T, "n_cap": N, "page_rows": 1,
                                             "window": "ring"},
                    roofline={"bound": "hbm (dense rows)", "peak": hbm, "peak_source": peak_src,
                              "unit": "GB/s"})
    elif args.part == "forward_paged":
        # the CSA layer over page pools (KV pages of 32 entries, key pages of 128 keys, both
        # shuffled; the window as a ring) against csa_forward on the contiguous caches
        inp = W.make_inputs(s)
        dev = R.upload(inp, s)
        p = R.params_for(s)
        B, T, N = s.B, s.T, s.n_cap
        contiguous = R.Step(s, dev)
        g = torch.Generator(device="cpu").manual_seed(10)

        def pool_of(t, rows, perm=None):
            # t [B, n, ...] -> a pool of B * n / rows pages in shuffled order and its table
            pages = t.shape[1] // rows
            if perm is None:
                perm = torch.randperm(t.shape[0] * pages, generator=g).to(torch.int32).cuda()
            pool = torch.empty((t.shape[0] * pages, rows) + tuple(t.shape[2:]), dtype=t.dtype,
                               device="cuda")
            pool[perm.long()] = t.reshape((t.shape[0] * pages, rows) + tuple(t.shape[2:]))
            return pool, perm.view(t.shape[0], pages)

        kv_pool, kv_table = pool_of(dev["kv_cache"], 32)
        k_pool, k_table = pool_of(dev["KI"], 128)
        k_scales = None
        if "KI_scale" in dev:  # the key scales in the keys' page order
            k_scales, _ = pool_of(dev["KI_scale"], 128, k_table.view(-1))
        kv = csa.paged_kv(csa.CSA_BF16, kv_pool, None, kv_table, kv_pool.shape[0], 32,
                          kv_table.shape[1])
        keys = csa.paged_kv(csa.DTYPES[s.idx], k_pool, k_scales, k_table, k_pool.shape[0], 128,
                            k_table.shape[1])
        # the window ring: position p in row p mod n_win
        ring = torch.empty((B, s.n_win, s.c), dtype=dev["win_kv"].dtype, device="cuda")
        for b in range(B):
            t, p0 = int(inp["q_pos"][b, 0]), int(inp["win_pos0"][b])
            for q0 in range(max(t - s.n_win + 1, 0), t + 1):
                ring[b, q0 % s.n_win] = dev["win_kv"][b, q0 - p0]
        need = csa.workspace_size(p, csa.CSA_WS_FORWARD, csa.DTYPES[s.idx], B, T, N)
        ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
        out = torch.empty((B, T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
        idx = torch.empty((B, T, s.topk), dtype=torch.int32, device="cuda")
        res = {"contiguous": round(_time_calls(lambda i: contiguous(), 1, args.warmup,
                                               args.steps), 5)}
        for name, b16 in (("paged", 0), ("paged_bf16_scores", 1)):
            fn = lambda i, b16=b16: csa.csa_forward_paged(  # noqa: E731
                p, B, T, kv, keys, b16, dev["qI"], dev.get("qI_scale"), dev["w"], dev["q"], None,
                dev["q_pos"], ring, s.n_win, None, dev["sink"], idx, None, out, ws, need)
            res[name] = round(_time_calls(fn, 1, args.warmup, args.steps), 5)
        line.update(metric="CSA layer calls/s over the state cache's page pools",
                    value=round(1e3 / res["paged"], 2), unit="calls/s (paged, fp32 scores)",
                    ms_per_call=res, config={"B": B, "T": T, "n_cap": N, "keys": s.idx,
                                             "kv_page_rows": 32, "key_page_rows": 128,
                                             "window": "ring"},
                    roofline={"bound": "hbm (key stream)", "peak": hbm, "peak_source": peak_src,
                              "unit": "GB/s"})
    elif args.part == "stream":
        n_vis = min(s.ctx // s.m, s.n_cap)
        nbytes = s.B * s.T * n_vis * indexer_key_bytes(s)
        n = nbytes // 4
        n_rep = max(2, int(np.ceil(3 * L2_BYTES / nbytes)))
        src = [torch.rand(n, device="cuda") for _ in range(n_rep)]
        dst = [torch.empty(n, device="cuda") for _ in range(n_rep)]
        sink = torch.empty(n_rep, device="cuda")

        def read(i):
            torch.sum(src[i], dim=0, out=sink[i])

        def copy(i):
            dst[i].copy_(src[i])

        ms_read = _time_calls(read, n_rep, args.warmup, args.steps)
        ms_copy = _time_calls(copy, n_rep, args.warmup, args.steps)
        rd, cp = nbytes / (ms_read / 1e3) / 1e9, 2 * nbytes / (ms_copy / 1e3) / 1e9
        line.update(metric="HBM rate of one stream of the indexer's key bytes",
                    value=round(rd, 1), unit="GB/s (read)",
                    bytes_per_stream=nbytes, replicas=n_rep,
                    ms_per_stream={"read": round(ms_read, 5), "copy": round(ms_copy, 5)},
                    copy_gbs=round(cp, 1),
                    roofline={"bound": "hbm", "peak": hbm, "peak_source": peak_src,
                              "unit": "GB/s", "read_frac": round(rd / hbm, 4),
                              "copy_frac": round(cp / hbm, 4)},
                    note="torch kernels (a sum and a copy), each call a whole stream; the "
                         "indexer reads the same bytes in one launch")
    line["gpu_launches"] = int(csa.kernel_launches() - before)
    line["clocks"] = clocks.stop()
    line["device_error"] = csa.device_error()
    print(json.dumps(line))
    return 0


PARTS = {"out_proj", "state_append", "kv_layouts", "bf16_scores", "out_proj_prefill",
         "forward_paged", "stream"}


def main():
    args = parse()
    if args.part is not None:
        from long_context_sparse_08_b200 import workloads as W

        return run_part(args, W)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from long_context_sparse_08_b200 import workloads as W

    if args.impl == "reference":
        if rank != 0:
            return 0
        s = W.SHAPES[args.workload]
        inp = W.make_inputs(s)
        from oracle import pipeline as P

        qs = [(b, t) for t in range(s.T) for b in range(s.B)]
        for i in range(args.warmup):
            P.run(s, inp, [qs[i % len(qs)]])
        t0 = time.perf_counter()
        for i in range(args.steps):
            P.run(s, inp, [qs[i % len(qs)]])
        el = time.perf_counter() - t0
        v = args.steps / el
        cores = blas_threads()
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "queries/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1); shapes of the Pro/Flash configs)",
            "config": workload_config(s, l2="host memory (float64 oracle)",
                                      parallelism="oracle on the host cores; "
                                                  "one query of the batch per step"),
            "cpu_baseline": {"value": round(v, 4), "unit": "queries/s", "cores": cores,
                             "kind": "oracle", "sample": "one query per step"},
            "e2e": {"value": round(v, 4), "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res, inp, s = run_ours(args, W, rank, world, local_rank)
    if rank == 0 and not args.no_cpu_baseline:
        v, n, el = oracle_queries_per_s(s, inp, args.cpu_seconds)
        res["cpu_baseline"] = {"value": round(v, 4), "unit": "queries/s",
                               "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{n} queries of the batch ({el:.1f} s)"}
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
