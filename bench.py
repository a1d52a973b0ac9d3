#!/usr/bin/env python
"""Bench: fused hybrid-batch (prefill + decode) attention on B200.

Metric: hybrid-batch attention time in microseconds per batch (lower is
better) and its fraction of the fused roofline
max(prefill FLOPs / tensor peak, (KV + Q + O bytes) / HBM peak).

One step = one ``pod_attn_run`` of the whole hybrid batch (counter reset, the
persistent fused kernel, the LSE merge) on the Llama-3-8B-shaped workload
(32 q / 8 kv heads, d = 128, prefill chunk 512 over 4096 prior tokens, 64
decode requests with lengths uniform in [1024, 4096], 16-token pages), inputs
resident in HBM.  The KV streamed per step (~0.67 GB) is larger than the 126 MB
L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the batch (the path has no exchange step); the reported time is the
max over ranks.  ``--impl reference`` times the CPU float64 oracle instead (on
rank 0 only): each step is one oracle pass over the whole batch.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "hybrid-batch attention µs and % of fused max(tensor,HBM) roofline on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["prefill_decode_b200/csrc/pod_attn.cu", "prefill_decode_b200/csrc/pod_ptx.cuh",
                  "prefill_decode_b200/csrc/pod_plan.h"]


HOST_SIDE_MARKER = b"// =========================================================== host side (ABI)"


def _code_only(data: bytes) -> bytes:
    """C++ source without comments and with whitespace runs collapsed, so that an
    edit to a comment does not count as a change of the device code."""
    import re
    text = data.decode("utf-8", "replace")
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return re.sub(r"\s+", " ", text).strip().encode()


def kernel_source_sha(root: str = ROOT) -> str:
    """Hash of the device code: the kernel sources without comments, with the
    host-side ABI part of the .cu file (launch plumbing, tensor-map encoding)
    left out."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(root, f), "rb") as fh:
            data = fh.read()
        i = data.find(HOST_SIDE_MARKER)
        h.update(_code_only(data if i < 0 else data[:i]))
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch of the fused kernel from a committed ncu summary,
    valid only while the kernel sources are unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 5:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        inside = [p for (t, p) in self.samples if t0 <= t <= t1]
        window = "timed region"
        if not inside:
            inside = [p for (t, p) in self.samples if t0 - 0.3 <= t <= t1 + 0.3]
            window = "within 0.3 s of the timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(p[1]) for p in inside if num(p[1]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in inside:
            for n, v in zip(names, p[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(inside[0][2]),
                "reasons": sorted(reasons), "samples": len(inside), "window": window,
                "power_w_max": max((num(p[3]) or 0.0) for p in inside)}


# ------------------------------------------------------------ multi-rank
def reduce_max(x: float, dist, device) -> float:
    """Max of a per-rank scalar over all ranks (timings are reported as the
    slowest replica); identity without a process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def plan_digest(plan) -> str:
    """Hash of a plan's work tables: every replica must plan its batch alike."""
    pre, dec, mer = plan.tables()
    h = hashlib.sha256()
    for a in (pre, dec, mer):
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- CPU oracle
def cpu_oracle_time(b, decode_reqs, prefill_rows):
    """Time the float64 oracle on a subset; return (seconds, decode part, prefill part, outputs)."""
    from oracle import attention as A
    w = b.workload
    t0 = time.perf_counter()
    od = A.attend_decode(b.q_decode, b.k_pool, b.v_pool, b.block_table, b.kv_lens, b.scale, w.num_kv_heads,
                         requests=decode_reqs, first_row=b.num_prefill) if len(decode_reqs) else None
    t1 = time.perf_counter()
    op = A.attend_prefill_batched(b.q_prefill, b.k_pool, b.v_pool, b.block_table, b.prefill_qo_lens,
                                  b.prefill_kv_lens, b.scale, w.num_kv_heads,
                                  rows=prefill_rows) if len(prefill_rows) else None
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, od, op


def cpu_oracle_single_thread_us(b, decode_reqs, prefill_rows):
    """The same sampled oracle run with BLAS held to one thread, scaled to the whole batch (µs)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1, user_api="blas"):
        td, tp, _, _ = cpu_oracle_time(b, decode_reqs, prefill_rows)
    return extrapolate(b, decode_reqs, prefill_rows, td, tp) * 1e6


def extrapolate(b, decode_reqs, prefill_rows, t_dec, t_pre):
    """Scale sampled oracle time to the whole batch by keys visited."""
    L = b.decode_lens.astype(np.int64)
    dec_scale = float(L.sum()) / max(1.0, float(L[list(decode_reqs)].sum())) if len(decode_reqs) else 0.0
    keys = prefill_row_keys(b)
    keys_all = int(keys.sum())
    keys_s = int(keys[list(prefill_rows)].sum()) if len(prefill_rows) else 0
    pre_scale = keys_all / keys_s if keys_s else 0.0
    return t_dec * dec_scale + t_pre * pre_scale


def prefill_row_keys(b) -> np.ndarray:
    """Keys each prefill row sees (C_i + i + 1 for row i of request i), over all requests in order."""
    out = [np.arange(P, dtype=np.int64) + (K - P) + 1 for P, K in zip(b.prefill_qo_lens, b.prefill_kv_lens)]
    return np.concatenate(out) if out else np.zeros(0, dtype=np.int64)


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return 1


def sample_sets(b, frac_den: int):
    B, P = b.workload.num_decode, b.workload.prefill_rows
    reqs = list(range(0, B, frac_den)) if B else []
    rows = list(range(0, P, frac_den)) if P else []
    return reqs, rows


def single_launch(kw, info) -> bool:
    """True when one step of a plan made with these keywords is one fused-kernel launch and nothing
    else (no counter memset, no second kernel): its back-to-back step time is the kernel's time."""
    import prefill_decode_b200 as pod
    flags = kw.get("flags", 0)
    if flags & (pod.POD_FLAG_SEQUENTIAL | pod.POD_FLAG_TRACE | pod.POD_FLAG_MERGE_KERNEL):
        return False
    two = flags & pod.POD_FLAG_TWO_STREAMS
    return not (two and info.num_prefill_items > 0 and info.num_decode_items > 0)


def fp8_alg_bytes(info, w) -> int:
    """Algorithmic bytes of a run whose decodes read e4m3 K/V (1 byte per element) and whose
    prefill requests read bf16 K/V: decode K/V + prefill K/V + Q + O."""
    dec_tokens = info.decode_flops // (4 * w.head_dim * w.num_q_heads)
    dec_kv16 = 4 * w.head_dim * w.num_kv_heads * dec_tokens
    return int(info.kv_bytes - dec_kv16 // 2 + info.qo_bytes)


# ------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The reference arm: the float64 oracle over the WHOLE batch per step (every decode
    request and every prefill row, all heads), on the host cores, rank 0 only."""
    if rank != 0:
        return 0
    w = synth.NAMED[args.workload]()
    b = synth.make_batch(w)
    reqs, rows = list(range(w.num_decode)), list(range(w.prefill_rows))
    times = []
    for i in range(args.warmup + args.steps):
        td, tp, _, _ = cpu_oracle_time(b, reqs, rows)
        if i >= args.warmup:
            times.append((td + tp) * 1e6)
    v = float(np.mean(times))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "us", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, b, "oracle"),
            "cpu_baseline": {"value": v, "unit": "us", "cores": blas_threads(), "kind": "oracle",
                             "host_cpus": os.cpu_count(),
                             "sample": f"the whole batch every step: all {len(reqs)} decode requests and all "
                                       f"{len(rows)} prefill rows, every head; no extrapolation"},
            "e2e": {"value": v, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, b, mode):
    L = b.decode_lens
    return {"workload": w.name, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "prefill_len": w.prefill_len, "prefill_ctx": w.prefill_ctx,
            "num_decode": w.num_decode, "decode_lens": f"{w.lens_kind}{list(w.lens_args)}, seed {w.seed}",
            **({"prefill_requests": [list(r) for r in w.prefill_requests]} if w.prefill_reqs is not None else {}),
            "sum_decode_len": int(L.sum()) if len(L) else 0, "page_size": 16, "mode": mode,
            "l2": "no flush: inputs larger than L2 (the KV streamed per step exceeds 126 MB)"}


# ---------------------------------------------------------------- sweep mode
def run_sweep(args):
    """Every named workload and every mix-sweep point (fused, sequential, two streams),
    one JSON object per line; for the committed result tables, not the bench
    line the contract reads."""
    import torch
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as pod
    from prefill_decode_b200.device_batch import DeviceBatch
    peaks, peak_src = load_peaks()
    names = args.sweep.split(",") if args.sweep not in ("1", "all") else None
    wls = [synth.NAMED[n]() for n in sorted(synth.NAMED)] + synth.sweep_points()
    if names:
        wls = [w for w in wls if w.name in names]
    stream = torch.cuda.current_stream()
    gpu_id = "0"
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(0).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    for w in wls:
        db = DeviceBatch.generated_on_device(torch, w)
        res = {"workload": w.name, "values": "torch.Generator(cuda, seed) normals; layout from synth"}
        arms = (("fused", {}), ("sequential", dict(flags=pod.POD_FLAG_SEQUENTIAL)),
                ("two_streams", dict(flags=pod.POD_FLAG_TWO_STREAMS)))
        if args.sweep_ratios:
            arms += (("fused_1_1", dict(ratio=(1, 1))), ("fused_1_0", dict(ratio=(1, 0))),
                     ("sm_partition", dict(flags=pod.POD_FLAG_SM_PARTITION)),
                     ("four_decode_warps", dict(flags=pod.POD_FLAG_DECODE_FOUR_WARPS)))
        if args.sweep_splits:
            arms += (("split_unlimited", dict(flags=pod.POD_FLAG_PREFILL_SPLIT_UNLIMITED)),
                     ("split_never", dict(max_prefill_splits=1)),
                     ("sequential_split_unlimited",
                      dict(flags=pod.POD_FLAG_SEQUENTIAL | pod.POD_FLAG_PREFILL_SPLIT_UNLIMITED)))
        if args.sweep_fp8 and w.num_decode:
            db.fp8_on_device()
            arms += (("fused_fp8_kv", dict(_fp8=True)),)
        for mode, kw in arms:
            kw = dict(kw)
            use8 = kw.pop("_fp8", False)
            pl = db.plan(pod, **kw)
            ws = db.workspace(pl)
            pl.upload(ws, stream)
            run = (lambda: db.run_fp8(pod, pl, ws, stream=stream)) if use8 else (lambda: db.run(pod, pl, ws, stream=stream))
            for _ in range(args.warmup):
                run()
            torch.cuda.synchronize()
            # enough steps for the timed window to span a few clock samples (>= 0.4 s), at most 4000
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(5):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
            est_s = e0.elapsed_time(e1) / 5e3
            steps = int(min(4000, max(args.steps, 0.4 / max(est_s, 1e-6))))
            t_w0 = time.time()
            e0.record(stream)
            for i in range(steps):
                run()
            e1.record(stream)
            torch.cuda.synchronize()
            t_w1 = time.time()
            step_us = e0.elapsed_time(e1) * 1e3 / steps
            # then the same steps with events around each launch (kernel time with its launch latency)
            ev = [(pod.Event(), pod.Event()) for _ in range(steps)]
            for i in range(steps):
                pl.set_events(ev[i][0].handle, ev[i][1].handle)
                run()
            torch.cuda.synchronize()
            pl.set_events(None, None)
            info = pl.info
            kern_iso_us = float(np.mean([a.elapsed_ms(c) for a, c in ev])) * 1e3
            kern_us = step_us if single_launch(kw, info) else kern_iso_us
            alg_bytes = fp8_alg_bytes(info, w) if use8 else info.kv_bytes + info.qo_bytes
            t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9) * 1e6
            t_tc = info.prefill_flops / (peaks["bf16_tflops"] * 1e12) * 1e6
            ck = sampler.summary(t_w0, t_w1)
            res[mode] = {"steps": steps, "step_us": step_us, "kernel_us": kern_us, "kernel_us_isolated": kern_iso_us,
                         "roofline_us": max(t_hbm, t_tc),
                         "frac_step": max(t_hbm, t_tc) / step_us, "frac_kernel": max(t_hbm, t_tc) / kern_us,
                         "bound": "hbm" if t_hbm >= t_tc else "tensor", "algorithmic_bytes": int(alg_bytes),
                         "hbm_GBps": alg_bytes / (kern_us * 1e-6) / 1e9,
                         "prefill_TFLOPs": info.prefill_flops / (kern_us * 1e-6) / 1e12,
                         "prefill_items": info.num_prefill_items, "prefill_partials": info.num_prefill_partials,
                         "error_word": db.error_word(pl, ws),
                         "clocks": {"sm_mhz": ck["sm_mhz"], "sm_max_mhz": ck["sm_max_mhz"],
                                    "reasons": ck["reasons"], "samples": ck["samples"]}}
        res["speedup_vs_sequential"] = res["sequential"]["step_us"] / res["fused"]["step_us"]
        res["speedup_vs_two_streams"] = res["two_streams"]["step_us"] / res["fused"]["step_us"]
        res["peaks"] = peak_src
        print(json.dumps(res), flush=True)
        del db
        torch.cuda.empty_cache()
    sampler.stop()
    return 0


# --------------------------------------------------------------------- ours
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama3_8b_mix", choices=sorted(synth.NAMED))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 KV-cache arm")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--sweep-ratios", action="store_true",
                    help="sweep mode: also time the fused kernel at forced role ratios 1:1 and 1:0")
    ap.add_argument("--sweep-splits", action="store_true",
                    help="sweep mode: also time the prefill KV split without its co-located limit and without any split")
    ap.add_argument("--sweep-fp8", action="store_true",
                    help="sweep mode: also time the fused kernel with the decode requests on an e4m3 KV cache")
    ap.add_argument("--sweep", default=None,
                    help="'all' or comma-separated workload names: per-workload table lines instead of the bench line")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.sweep:
        args.steps = min(args.steps, 200)   # a floor: each arm runs for at least 0.4 s of steps
        return run_sweep(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from prefill_decode_b200 import build
    build.build()
    import prefill_decode_b200 as pod
    from prefill_decode_b200.device_batch import DeviceBatch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = synth.NAMED[args.workload]()
    b = synth.make_batch(w)
    db = DeviceBatch(torch, b, device=dev)
    stream = torch.cuda.current_stream(dev)
    fused = db.plan(pod)
    seq = db.plan(pod, flags=pod.POD_FLAG_SEQUENTIAL)
    ws = db.workspace(fused)
    ws_seq = db.workspace(seq)
    fused.upload(ws, stream)
    seq.upload(ws_seq, stream)
    info = fused.info
    launches_per_step = 1          # the fused kernel merges split-KV rows itself

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed_loop(plan, wsp, K, per_step_events):
        # K steps back to back, events only at the two ends (an event between two launches would
        # keep the fused kernel's CTAs from being scheduled while the previous one finishes);
        # then, with per_step_events, K more steps with events around each launch for the
        # kernel-only time
        for _ in range(args.warmup):
            db.run(pod, plan, wsp, stream=stream)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        t_wall0 = time.time()
        e0.record(stream)
        for i in range(K):
            db.run(pod, plan, wsp, stream=stream)
        e1.record(stream)
        barrier()
        t_wall1 = time.time()
        total_ms = e0.elapsed_time(e1)
        kern = []
        if per_step_events:
            evs = [(pod.Event(), pod.Event()) for _ in range(K)]
            for i in range(K):
                plan.set_events(evs[i][0].handle, evs[i][1].handle)
                db.run(pod, plan, wsp, stream=stream)
            plan.set_events(None, None)
            torch.cuda.synchronize()
            kern = [a.elapsed_ms(c) for a, c in evs]
        return total_ms, kern, (t_wall0, t_wall1)

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dist if world > 1 else None, dev)

    gpu_id = str(local)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    total_ms, kern_ms, (tw0, tw1) = timed_loop(fused, ws, args.steps, True)
    clocks = sampler.summary(tw0, tw1)
    seq_ms, seq_kern, _ = timed_loop(seq, ws_seq, max(50, args.steps // 4), True)
    # ablations through the same API: the two kernels of the sequential path on two concurrent streams,
    # roles by SM id, four decode warps per CTA, and every CTA starting on one role (the proportional
    # rule gives 1:1 with two CTAs per SM)
    k_abl = max(50, args.steps // 4)
    ablations = {}
    for name, kw in (("two_streams", dict(flags=pod.POD_FLAG_TWO_STREAMS)),
                     ("sm_partition", dict(flags=pod.POD_FLAG_SM_PARTITION)),
                     ("decode_four_warps", dict(flags=pod.POD_FLAG_DECODE_FOUR_WARPS)),
                     ("prefill_first_1_0", dict(ratio=(1, 0))), ("decode_first_0_1", dict(ratio=(0, 1))),
                     ("prefill_split_unlimited", dict(flags=pod.POD_FLAG_PREFILL_SPLIT_UNLIMITED)),
                     ("prefill_split_never", dict(max_prefill_splits=1))):
        pl_a = db.plan(pod, **kw)
        ws_a = db.workspace(pl_a)
        pl_a.upload(ws_a, stream)
        # timed exactly like the fused arm (the same per-step events), so the step times compare directly
        a_ms, a_kern, _ = timed_loop(pl_a, ws_a, k_abl, True)
        a_iso = float(np.mean(a_kern)) * 1e3
        ablations[name] = {"step_us": max_over_ranks(a_ms * 1e3 / k_abl),
                           "kernels_us": max_over_ranks(a_ms * 1e3 / k_abl if single_launch(kw, pl_a.info) else a_iso),
                           "kernels_us_isolated": max_over_ranks(a_iso),
                           "error_word": db.error_word(pl_a, ws_a)}
        del ws_a
    # the decode requests on an e4m3 copy of the cache (pod_attn_run_fp8kv), same plan and timing
    fp8_arm = None
    if w.num_decode and not args.no_fp8:
        db.fp8_on_device()
        ws8 = db.workspace(fused)
        fused.upload(ws8, stream)
        ev8 = [(pod.Event(), pod.Event()) for _ in range(k_abl)]
        for _ in range(args.warmup):
            db.run_fp8(pod, fused, ws8, stream=stream)
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(k_abl):
            fused.set_events(ev8[i][0].handle, ev8[i][1].handle)
            db.run_fp8(pod, fused, ws8, stream=stream)
        f1.record(stream)
        barrier()
        fused.set_events(None, None)
        k8_us = max_over_ranks(float(np.mean([a.elapsed_ms(c) for a, c in ev8])) * 1e3)
        b8 = fp8_alg_bytes(fused.info, w)
        fp8_arm = {"step_us": max_over_ranks(f0.elapsed_time(f1) * 1e3 / k_abl), "kernel_us": k8_us,
                   "algorithmic_bytes": b8, "hbm_GBps": b8 / (k8_us * 1e-6) / 1e9,
                   "error_word": db.error_word(fused, ws8),
                   "note": "decode K/V as e4m3 codes with one fp32 scale per kv head (made on the GPU from the "
                           "bf16 pools), prefill K/V bf16; bytes = decode K/V at 1 byte + prefill K/V at 2 + Q + O"}
        # parity spot check of the e4m3 run against the float64 oracle on the same codes
        from oracle import attention as A8, fp8 as F8
        reqs8 = [0, w.num_decode // 2, w.num_decode - 1]
        # only the sampled requests' blocks are copied back and decoded (block table remapped onto them)
        rows8 = [b.num_prefill + r for r in reqs8]
        npg = [-(-int(b.kv_lens[r]) // 16) for r in rows8]
        blocks = np.unique(np.concatenate([b.block_table[r, :n] for r, n in zip(rows8, npg)]))
        remap = {int(x): i for i, x in enumerate(blocks)}
        bt8 = np.zeros((len(rows8), max(npg)), dtype=np.int32)
        for i, (r, n) in enumerate(zip(rows8, npg)):
            bt8[i, :n] = [remap[int(x)] for x in b.block_table[r, :n]]
        idx = torch.from_numpy(blocks.astype(np.int64)).to(db.k8.device)
        K8 = F8.dequant_pool(db.k8[idx].cpu().numpy(), db.k_scale.cpu().numpy())
        V8 = F8.dequant_pool(db.v8[idx].cpu().numpy(), db.v_scale.cpu().numpy())
        ref8 = A8.attend_decode(b.q_decode[reqs8], K8, V8, bt8, np.asarray([int(b.kv_lens[r]) for r in rows8]),
                                b.scale, w.num_kv_heads, first_row=0)
        got8 = db.o_dec.float().cpu().numpy()[reqs8]
        fp8_arm["parity_sample"] = {"requests": reqs8, "max_abs": float(np.abs(got8 - ref8).max()),
                                    "mean_abs": float(np.abs(got8 - ref8).mean())}
        del K8, V8, ws8
        db.run(pod, fused, ws, stream=stream)   # leave the bf16 outputs for the parity sample below
        torch.cuda.synchronize()
    sampler.stop()
    err_word = db.error_word(fused, ws)

    us = max_over_ranks(total_ms * 1e3 / args.steps)
    # a step is one launch of the fused kernel and nothing else on the stream, so the timed region's
    # average per step is the kernel's average launch duration (back to back, the gaps between
    # launches included); the events around each launch give the time of one launch in isolation
    kern_us = us
    kern_iso_us = max_over_ranks(float(np.mean(kern_ms)) * 1e3)
    seq_us = max_over_ranks(seq_ms * 1e3 / max(50, args.steps // 4))
    seq_kern_us = max_over_ranks(float(np.mean(seq_kern)) * 1e3)

    # ------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        host = {}
        for name in ("q_pre", "q_dec", "k", "v", "bt", "lens"):
            t = getattr(db, name)
            if t is not None:
                host[name] = t.cpu().pin_memory()
        outs_host = {n: torch.empty(getattr(db, n).shape, dtype=getattr(db, n).dtype, pin_memory=True)
                     for n in ("o_pre", "o_dec") if getattr(db, n) is not None}
        h2d = sum(t.numel() * t.element_size() for t in host.values()) + info.table_bytes
        d2h = sum(t.numel() * t.element_size() for t in outs_host.values())

        def e2e_step():
            for n, t in host.items():
                getattr(db, n).copy_(t, non_blocking=True)
            fused.upload(ws, stream)
            db.run(pod, fused, ws, stream=stream)
            for n, t in outs_host.items():
                t.copy_(getattr(db, n), non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        a1.record(stream)
        barrier()
        e2e_us = max_over_ranks(a0.elapsed_time(a1) * 1e3 / args.e2e_steps)
        e2e = {"value": e2e_us, "unit": "us", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": args.e2e_steps,
               "note": "pinned host Q, K/V pools, block table and lengths copied in, plan tables uploaded, "
                       "outputs copied out, every step"}

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    # ------------------------------------------------------------ roofline
    peaks, peak_src = load_peaks()
    alg_bytes = info.kv_bytes + info.qo_bytes
    t_hbm_us = alg_bytes / (peaks["hbm_gbs"] * 1e9) * 1e6
    t_tc_us = info.prefill_flops / (peaks["bf16_tflops"] * 1e12) * 1e6
    bound = "hbm" if t_hbm_us >= t_tc_us else "tensor"
    if bound == "hbm":
        achieved = alg_bytes / (kern_us * 1e-6) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
    else:
        achieved = info.prefill_flops / (kern_us * 1e-6) / 1e12
        peak, unit = peaks["bf16_tflops"], "TFLOP/s"
    traffic = load_traffic(w.name)

    # ---------------------------------------------------------- CPU oracle
    cpu = None
    parity = None
    if not args.no_cpu_baseline:
        # the oracle as it stands over the whole batch (all cores), and a single-thread figure from every
        # 8th request and row scaled by keys visited; the full-batch outputs double as a parity check
        reqs, rows = list(range(w.num_decode)), list(range(w.prefill_rows))
        td, tp, od, op = cpu_oracle_time(b, reqs, rows)
        s_reqs, s_rows = sample_sets(b, 8)
        cpu = {"value": (td + tp) * 1e6, "unit": "us", "cores": blas_threads(), "kind": "oracle",
               "sample": f"the whole batch: all {len(reqs)} decode requests and all {len(rows)} prefill rows, "
                         f"every head, one pass ({td + tp:.2f} s)",
               "host_cpus": os.cpu_count(),
               "single_thread_value": cpu_oracle_single_thread_us(b, s_reqs, s_rows),
               "single_thread_sample": f"every 8th decode request ({len(s_reqs)}) and prefill row "
                                       f"({len(s_rows)}) with BLAS on one thread, scaled by keys visited"}
        gp, gd = db.outputs()
        e_dec = np.abs(gd - od) if od is not None else np.zeros(1)
        e_pre = np.abs(gp - op) if op is not None else np.zeros(1)
        parity = {"max_abs": float(max(e_dec.max(), e_pre.max())),
                  "mean_abs": float(np.concatenate([e_dec.ravel(), e_pre.ravel()]).mean()),
                  "elements": int(e_dec.size + e_pre.size),
                  "tolerance": {"max_abs": 2e-2, "mean_abs": 2e-3}}

    line = {
        "metric": METRIC, "value": us, "unit": "us", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(w, b, "fused"),
        "fused_roofline": {"t_tensor_us": t_tc_us, "t_hbm_us": t_hbm_us, "t_roofline_us": max(t_tc_us, t_hbm_us),
                           "frac_step": max(t_tc_us, t_hbm_us) / us, "frac_kernel": max(t_tc_us, t_hbm_us) / kern_us,
                           "peaks": f"{peak_src}: HBM {peaks['hbm_gbs']} GB/s, bf16 {peaks['bf16_tflops']} TFLOP/s"},
        "roofline": {"kernel": f"pod::pod_attn_kernel<{w.head_dim}> (fused persistent)", "bound": bound,
                     "achieved": achieved,
                     "peak": peak, "unit": unit, "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": traffic, "algorithmic_bytes": int(alg_bytes),
                     "algorithmic_flops_prefill": int(info.prefill_flops), "kernel_us": kern_us,
                     "kernel_us_isolated": kern_iso_us,
                     "kernel_us_note": "kernel_us = the timed region's events / steps (one launch per step, "
                                       "back to back); kernel_us_isolated = mean of events recorded around "
                                       "each launch in a second loop (launch latency exposed)"},
        "sequential_us": seq_us, "sequential_kernels_us": seq_kern_us, "speedup_vs_sequential": seq_us / us,
        "ablations": dict(ablations, fused_step_us=us,
                          note="two_streams = prefill-only and decode-only kernels on concurrent streams; "
                               "sm_partition = roles by SM id instead of per-SM tickets; "
                               "decode_four_warps = only 4 of a decoding CTA's 6 warps run decode items (deeper page rings); "
                               "x_first = ratio p:d forced so every CTA starts on that role; "
                               "prefill_split_unlimited = the prefill KV split fills every CTA slot (the "
                               "co-located-decode limit for <= 1536 prefill tokens off); prefill_split_never = "
                               "no prefill KV split"),
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": launches_per_step * args.steps,
        "launches_note": "per step: one pod_attn_kernel launch (split-KV rows merged inside it; its last CTA "
                         "returns the workspace counters to zero, so no memset between steps)",
        "plan": {"prefill_items": info.num_prefill_items, "decode_items": info.num_decode_items,
                 "merge_items": info.num_merge_items, "chunk_pages": info.chunk_pages,
                 "ctas_per_sm": info.ctas_per_sm, "ratio": [info.ratio_prefill, info.ratio_decode],
                 "grid": info.grid, "prefill_partials": info.num_prefill_partials},
        "device_error_word": err_word, "parity_sample": parity,
        "fp8_kv": dict(fp8_arm, frac_of_hbm_peak=fp8_arm["hbm_GBps"] / peaks["hbm_gbs"],
                       t_roofline_us=max(fp8_arm["algorithmic_bytes"] / (peaks["hbm_gbs"] * 1e3), t_tc_us))
        if fp8_arm else None,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
