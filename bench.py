"""Benchmark: radial sparse attention at the Wan2.1-1.3B shape on B200.

One step = the whole hot path on one batch: the radial selector
(sta_build_blocks) and the block-sparse attention (sta_sparse_attn_fwd) over
12 heads x 32760 tokens x d=128, bf16.  Reported:

  value      effective TFLOP/s on retained blocks (4*d FLOPs per kept query-key
             pair, true block lengths) per step, inputs resident in HBM
  e2e        the same metric through the C ABI with host buffers: pinned H2D
             copies of q, k, v and the D2H copy of o inside the timed region
  speedup_vs_dense   dense attention (sta_dense_attn_fwd, same kernel, all
             keys) time / sparse attention time at the same shape
  roofline   the attention kernel against the measured bf16 tensor peak
  cpu_baseline  the fp64 oracle on a bounded sample, host cores

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no
data-path collective); the time is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective TFLOP/s on retained blocks; speedup vs dense at same shape (1×B200)"
WORKLOAD = "wan_radial"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of one attention launch from an ncu capture, valid only for
# the kernel source it was taken on (sha256 of attn_fwd.cu, first 16 hex).
NCU_TRAFFIC = {"source_sha": "61bd247adb317a0a", "bytes_per_launch": 303713280 + 87362304}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def source_sha():
    path = os.path.join(ROOT, "sparse_spatiotemporal_attention_video_b200", "csrc", "attn_fwd.cu")
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, device_index=0):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            n = pynvml.nvmlDeviceGetCount()
            for i in range(n):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self._h = h
            if self._h is None and n == 1:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(0)
            if self._h is not None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception:
            self._h = None

    _NAMES = [(0x8, "hw_slowdown"), (0x40, "hw_thermal_slowdown"), (0x20, "sw_thermal_slowdown"),
              (0x4, "sw_power_cap"), (0x80, "hw_power_brake_slowdown")]

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = fn(self._h)
                for bit, name in self._NAMES:
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(s)}


def dist_setup(n_gpus):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, ws, local


def max_over_ranks(x, ws):
    import torch
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    import torch
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def cpu_baseline(w, budget_s=15.0):
    """Oracle (fp64, numpy) on a bounded sample of the workload: the full radial
    list build, then attention for query blocks of head 0 until the budget is
    spent.  Returns the oracle's effective TFLOP/s over the sampled work."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import radial
    from oracle.pipeline import block_sparse_rows
    from synthetic import make_qkv

    q, k, v = make_qkv(dict(w, heads=1))
    t0 = time.perf_counter()
    lists = radial.block_lists(w["F"], w["H"], w["W"], w["block_q"], w["radial"])
    t_sel = time.perf_counter() - t0
    N, B, d = w["N"], w["block_q"], w["d"]
    qh, kh, vh = (x[0].float().numpy().astype(np.float64) for x in (q, k, v))
    rng = np.random.default_rng(0)
    order = rng.permutation(len(lists))
    flops = 0.0
    done = 0
    t0 = time.perf_counter()
    for qb in order:
        block_sparse_rows(qh, kh, vh, int(qb), lists[qb], B, B)
        qlen = min(B, N - qb * B)
        keys = sum(min(B, N - u * B) for u in lists[qb])
        flops += 4.0 * d * qlen * keys
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    t_att = time.perf_counter() - t0
    frac = done / (len(lists) * w["heads"])
    t = t_att + t_sel * frac
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": int(threads),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle: full radial list build ({t_sel:.2f} s, charged "
                      f"pro rata) + attention of {done} of {len(lists) * w['heads']} "
                      f"(head, query-block) items of head 0, {flops / 1e12:.3f} TFLOP retained",
            "host_cpus": os.cpu_count()}


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded sample."""
    from synthetic import workload
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(WORKLOAD)
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=budget)
    vals = [cpu_baseline(w, budget_s=budget) for _ in range(args.steps)]
    val = sum(v["value"] for v in vals) / len(vals)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "heads": w["heads"], "F": w["F"], "H": w["H"],
                       "W": w["W"], "d": w["d"], "block_q": w["block_q"]},
            "cpu_baseline": dict(vals[-1], value=val),
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch

    import sparse_spatiotemporal_attention_video_b200 as sta
    from sparse_spatiotemporal_attention_video_b200 import session
    from synthetic import make_qkv, workload

    rank, ws, local = dist_setup(args.gpus)
    w = workload(WORKLOAD)
    q, k, v = make_qkv(w)
    prob = session.problem(w)
    sel = session.selector(w)
    prm = session.attn_params(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    od = torch.empty_like(qd)
    L = session.Lists(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    l2_flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")

    def step(qq, kk, vv, oo, ev=None):
        if ev is not None:
            ev[0].record(stream)
        sta.sta_build_blocks(prob, sel, None, None, L.struct, dev_status=st, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        sta.sta_sparse_attn_fwd(prob, prm, qq, kk, vv, L.struct, oo, dev_status=st,
                                stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step(qd, kd, vd, od)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError("device status " + sta.sta_dev_status_string(int(st.item())))
    pairs = session.retained_pairs(w, L)
    flops = 4.0 * w["d"] * pairs
    dense_flops = 4.0 * w["d"] * float(w["N"]) ** 2 * w["heads"]

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(ws)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            l2_flush.zero_()
            step(qd, kd, vd, od, evs[i])
        torch.cuda.synchronize()
    barrier(ws)
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    ms = sum(step_ms) / len(step_ms)
    ms = max_over_ranks(ms, ws)
    attn_avg = sum(attn_ms) / len(attn_ms)

    # dense at the same shape (the speedup denominator)
    for _ in range(3):
        sta.sta_dense_attn_fwd(prob, qd, kd, vd, 0.0, od, dev_status=st, stream=stream)
    dense_ms = []
    for _ in range(max(3, args.steps // 2)):
        l2_flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sta.sta_dense_attn_fwd(prob, qd, kd, vd, 0.0, od, dev_status=st, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        dense_ms.append(a.elapsed_time(b))
    dense_avg = sum(dense_ms) / len(dense_ms)

    # end to end through the C ABI with host buffers
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    h2d = 3 * qh.numel() * qh.element_size()
    d2h = oh.numel() * oh.element_size()
    e2e_ms = []
    for i in range(args.warmup + max(3, args.steps // 2)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        step(qd, kd, vd, od)
        oh.copy_(od, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_avg = max_over_ranks(sum(e2e_ms) / len(e2e_ms), ws)
    if int(st.item()) != 0:
        raise RuntimeError("device status " + sta.sta_dev_status_string(int(st.item())))

    pk, pk_kind = peaks()
    peak = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (attn_avg * 1e-3) / 1e12
    traffic = None
    if NCU_TRAFFIC["source_sha"] and NCU_TRAFFIC["source_sha"] == source_sha():
        traffic = NCU_TRAFFIC["bytes_per_launch"]
    line = {
        "metric": METRIC, "value": flops * ws / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "heads": w["heads"], "F": w["F"], "H": w["H"],
                   "W": w["W"], "N": w["N"], "d": w["d"], "block_q": w["block_q"],
                   "kv_unit": w["kv_unit"], "selector": "radial",
                   "l2": "inputs 302 MB > 126 MB L2; 256 MB flush write between steps"},
        "retained_pairs": pairs, "retained_fraction": pairs / (w["N"] ** 2 * w["heads"]),
        "attn_ms": attn_avg, "dense_ms": dense_avg,
        "dense_tflops": dense_flops / (dense_avg * 1e-3) / 1e12,
        "speedup_vs_dense": dense_avg / attn_avg,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{pk_kind} bf16 (burst)"},
        "e2e": {"value": flops * ws / (e2e_avg * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_avg, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
