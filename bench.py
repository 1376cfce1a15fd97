"""Benchmark: one step of the sparse-attention hot path on B200.

Default workload: importance-sampled block attention at the HunyuanVideo
latent grid (24 heads x 33x45x80 = 118,800 tokens x d=128, bf16, 128-query
blocks, 16-key sub-blocks, ~10% sampled), the largest workload that fits one
GPU.  One step = the selector (sta_build_blocks: sub-block means, k-means,
importance, Philox sampling) plus the weighted block-sparse attention
(sta_sparse_attn_fwd) on one batch.  --workload picks the other workloads
(wan_radial, tra_entropy, heta_routed, tra_token, dynrad_static,
dynrad_dynamic); a step is then that workload's selector plus attention.

Timing: the step, selector-only and attention-only CUDA graphs are replayed
in one interleaved loop, each after the same L2 flush, so the three device
times come from the same clock state; every figure is a mean over the K
timed iterations.

Reported (one JSON line on rank 0):
  value      effective TFLOP/s on retained blocks (4*d FLOPs per kept
             query-key pair, true block lengths) per step, inputs resident in
             HBM, summed over ranks
  e2e        the same metric through the C ABI with pinned host buffers: H2D
             copies of the step's inputs and the D2H copy of o are inside the
             timed region
  speedup_vs_dense   dense attention (sta_dense_attn_fwd, same kernel, all
             keys) time / sparse attention time at the same shape
  roofline   the attention kernel against the measured bf16 tensor peak
  selector   the selector's own time and, where it is bandwidth-bound, its
             algorithmic bytes against the measured HBM bandwidth
  cpu_baseline  the fp64 oracle on a bounded sample, host cores

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                [--impl reference]
Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no
data-path collective); the time is the max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective TFLOP/s on retained blocks; speedup vs dense at same shape (1×B200)"
DEFAULT_WORKLOAD = "ab_sampled"
WORKLOADS = ("wan_radial", "tra_entropy", "heta_routed", "ab_sampled", "tra_token",
             "tra_token_tiled", "dynrad_static", "dynrad_dynamic")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 * 1024 * 1024

# DRAM traffic of one attention launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from an ncu capture, valid only for the kernel
# source it was taken on (sha256 of attn_fwd.cu, first 16 hex).  Captured on
# 2 of the 24 heads (one launch, inputs larger than L2) and scaled by 12:
# every head carries the same work.
NCU_TRAFFIC = {"ab_sampled": {"source_sha": "90414ec2ef9bfaba",
                              "bytes_per_launch": 12 * (422881536 + 62861056)}}


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOADS)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-budget-s", type=float, default=15.0,
                   help="seconds of oracle work in the cpu_baseline sample")
    p.add_argument("--heads", type=int, default=None,
                   help="override the workload's head count (smaller cases for profiling)")
    return p.parse_args(argv)


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

    _NAMES = [(0x8, "hw_slowdown"), (0x40, "hw_thermal_slowdown"), (0x20, "sw_thermal_slowdown"),
              (0x4, "sw_power_cap"), (0x80, "hw_power_brake_slowdown")]

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

    def _run(self):
        nv = self._nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
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


# ------------------------------------------------------------------ ranks
def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup(backend="nccl", timeout_s=120):
    """One process per GPU; returns (rank, world_size, local_rank)."""
    rank, ws, local = rank_env()
    if backend == "nccl":
        import torch
        torch.cuda.set_device(local if ws > 1 else 0)
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, ws, local


def max_over_ranks(x, ws):
    """Max of a host float over ranks (NCCL on the device, gloo on the host)."""
    if ws == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, ws):
    if ws == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(ws, cuda=True):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        import torch
        torch.cuda.synchronize()


# ------------------------------------------------------------ CPU baseline
def _threads():
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] or [1]))
    except Exception:
        return 1


def cpu_baseline(w, budget_s=15.0, seed=0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload.

    Per workload: the oracle selector on (a sample of) the rows it needs,
    then oracle attention for query blocks of head 0 in a seeded order until
    the budget is spent.  Selector time is charged pro rata to the sampled
    fraction.  Returns effective TFLOP/s over the sampled retained pairs."""
    import numpy as np

    from oracle import dynrad, entropy, ibcs_sip, radial, routed, tra_token
    from oracle.grid import n_blocks
    from oracle.pipeline import block_sparse_rows, routed_rows
    from synthetic import make_difficulty, make_qkv

    N, d, heads = w["N"], w["d"], w["heads"]
    B, U = w["block_q"], w["kv_unit"]
    q, k, v = make_qkv(dict(w, heads=1))
    qh, kh, vh = (x[0].float().numpy().astype(np.float64) for x in (q, k, v))
    rng = np.random.default_rng(seed)
    nqb = n_blocks(N, B)
    order = rng.permutation(nqb)
    flops = 0.0
    done = 0
    t_sel_per_item = 0.0
    sel = w["selector"]
    t0 = time.perf_counter()
    if sel == "radial":
        lists = radial.block_lists(w["F"], w["H"], w["W"], B, w["radial"])
        t_sel_per_item = (time.perf_counter() - t0) / (nqb * heads)
        logw = None
    elif sel == "entropy":
        e = w["entropy"]
        lists, _, _, _ = entropy.select(qh, kh, w["F"], w["H"], w["W"], B, e["alpha"], e["beta"],
                                        e["r_lo"], e["r_hi"], e["tile_h"], e["tile_w"])
        t_sel_per_item = (time.perf_counter() - t0) / nqb  # one head's selector
        logw = None
    elif sel == "routed":
        c = w["routed"]
        dif = make_difficulty(w)
        ids = routed.route(dif, c["dense_frac"])
        flag = np.zeros(N, bool)
        flag[ids] = True
        t_sel_per_item = (time.perf_counter() - t0) / (nqb * heads)
    elif sel == "ibcs_sip":
        c = w["ibcs"]
        kbar, n_j = ibcs_sip.subblock_means(kh, U)
        t_sel_per_item = (time.perf_counter() - t0) / nqb  # one head's sub-block means
    elif sel == "tra_token":
        c = w["tra_token"]
        Hq = np.zeros(N)
        t_lists = 0.0
        perm = None
        if w.get("layout"):
            # tile-major order: blocks are runs of positions of the permuted
            # sequence; attention runs on the permuted rows
            from oracle import tile_major
            perm = tile_major.order(w["F"], w["H"], w["W"], *w["layout"])
            qp, kp, vp = (tile_major.to_layout(x, perm) for x in (qh, kh, vh))
    elif sel == "dynrad":
        c = w["dynrad"]
        got = dynrad.select(qh, kh, w["F"], w["H"], w["W"], B, w["radial"], c["mode"],
                            c.get("ratio"), c.get("threshold"))
        lists = {b: ids for b, (ids, _) in got.items()}
        t_sel_per_item = (time.perf_counter() - t0) / nqb  # one head's selector
        logw = None
    budget_end = time.perf_counter() + budget_s
    t_att = 0.0
    for qb in order:
        qb = int(qb)
        ts = time.perf_counter()
        if sel == "tra_token":
            # the entropies are the warm-up's (not charged to the step); the
            # block lists and the attention are
            lo, hi = qb * B, min(N, qb * B + B)
            toks = np.arange(lo, hi) if perm is None else perm[lo:hi]
            Hq[toks] = tra_token.query_entropy(qh[toks], kh, 1.0 / np.sqrt(d))
            ts = time.perf_counter()
            ids, _ = tra_token.block_lists(Hq, w["F"], w["H"], w["W"], B, c["tau"], c["gamma"],
                                           c["vote"], [qb], perm=perm)[qb]
            t_lists += time.perf_counter() - ts
            ts = time.perf_counter()
            if perm is None:
                block_sparse_rows(qh, kh, vh, qb, ids, B, U)
            else:
                block_sparse_rows(qp, kp, vp, qb, ids, B, U)
            t_att += time.perf_counter() - ts
            keys = sum(min(U, N - u * U) for u in ids)
            flops += 4.0 * d * (hi - lo) * keys
            t_sel_per_item = t_lists / (done + 1)
        elif sel == "ibcs_sip":
            lo, hi = qb * B, min(N, qb * B + B)
            row = ibcs_sip.select_row(qh[lo:hi], kbar, n_j, c["seed"], qb, c["k"], c["iters"],
                                      c["sample_frac"])
            block_sparse_rows(qh, kh, vh, qb, row["ids"], B, U, row["logw"])
            t_att += time.perf_counter() - ts
            keys = sum(min((u + 1) * U, N) - u * U for u in row["ids"])
            flops += 4.0 * d * (hi - lo) * keys
        elif sel == "routed":
            c = w["routed"]
            toks = np.arange(qb * B, min(N, qb * B + B))
            routed_rows(qh, kh, vh, toks, flag, w["F"], w["H"], w["W"], c["win_f"], c["win_h"],
                        c["win_w"])
            t_att += time.perf_counter() - ts
            for t in toks:
                if flag[t]:
                    flops += 4.0 * d * N
                else:
                    flops += 4.0 * d * len(routed.window_keys(int(t), w["F"], w["H"], w["W"],
                                                              c["win_f"], c["win_h"],
                                                              c["win_w"]))
        else:
            block_sparse_rows(qh, kh, vh, qb, lists[qb], B, U, logw)
            t_att += time.perf_counter() - ts
            qlen = min(B, N - qb * B)
            keys = sum(min(U, N - u * U) for u in lists[qb])
            flops += 4.0 * d * qlen * keys
        done += 1
        if time.perf_counter() > budget_end:
            break
    t = t_att + t_sel_per_item * done
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle on {w['name']}: selector charged pro rata "
                      f"({t_sel_per_item * 1e3:.2f} ms per (head, query-block) item) + "
                      f"attention of {done} of {nqb * heads} (head, query-block) items of "
                      f"head 0, {flops / 1e12:.4f} TFLOP retained, {t:.1f} s",
            "host_cpus": os.cpu_count()}


def run_reference(args):
    """The oracle as the reference arm: each step is a bounded sample of the
    workload on the host cores.  Under torchrun rank 0 alone runs it."""
    from synthetic import workload
    rank, ws, _ = rank_env()
    if rank != 0:
        return 0
    w = workload(args.workload, **({"heads": args.heads} if args.heads else {}))
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup):
        cpu_baseline(w, budget_s=budget, seed=i)
    vals = [cpu_baseline(w, budget_s=budget, seed=100 + i) for i in range(args.steps)]
    val = sum(v["value"] for v in vals) / len(vals)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": dict(vals[-1], value=val),
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def config_of(w):
    c = {"workload": w["name"], "heads": w["heads"], "F": w["F"], "H": w["H"], "W": w["W"],
         "N": w["N"], "d": w["d"], "block_q": w["block_q"], "kv_unit": w["kv_unit"],
         "selector": w["selector"],
         "l2": f"inputs {3 * w['heads'] * w['N'] * w['d'] * 2 / 1e6:.0f} MB > 126 MB L2; "
               f"{L2_FLUSH_BYTES >> 20} MB flush write between steps"}
    return c


# ------------------------------------------------------------------- GPU arm
SELECTOR_LAUNCHES = {"radial": 1, "entropy": 3, "routed": 2, "ibcs_sip": 4, "tra_token": 1,
                     "dynrad": 3}


def selector_bytes(w, lists_entries):
    """Algorithmic bytes of the selector: each input read once plus the list
    entries written (4 B per id, 4 more per log-weight), and the bound."""
    h, N, d = w["heads"], w["N"], w["d"]
    sel = w["selector"]
    if sel in ("entropy", "dynrad"):
        return 2 * h * N * d * 2 + 4 * lists_entries, "hbm"
    if sel == "ibcs_sip":
        return 2 * h * N * d * 2 + 8 * lists_entries, "hbm (Q and K read once, lists written)"
    if sel == "routed":
        return 4 * N + 5 * N + 4 * lists_entries, "latency"
    if sel == "tra_token":
        return 4 * h * N + 4 * lists_entries, "alu (disk counting per query and key block)"
    return 4 * lists_entries, "launch"


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        return run_reference(args)
    import torch

    import sparse_spatiotemporal_attention_video_b200 as sta
    from sparse_spatiotemporal_attention_video_b200 import session
    from synthetic import make_difficulty, make_qkv, workload

    rank, ws, local = dist_setup("nccl")
    w = workload(args.workload, **({"heads": args.heads} if args.heads else {}))
    q, k, v = make_qkv(w)
    routed = w["selector"] == "routed"
    dif = torch.from_numpy(make_difficulty(w)) if routed else None
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    difd = dif.cuda() if routed else None
    od = torch.empty_like(qd)
    prob = session.problem(w)
    # token-level TRA: the per-query entropies come from a dense warm-up pass
    # (dense attention that also writes each query's entropy), run once and
    # reused by every step, as the pipeline reuses them across denoising steps
    # tile-major token order (layout workloads): the attention runs on
    # permuted copies of q, k, v and its output is permuted back; both
    # permutations are part of the step
    layout = w.get("layout")
    if layout:
        qt, kt, vt, ot = (torch.empty_like(qd) for _ in range(4))

        def permute_in():
            for x, y in ((qd, qt), (kd, kt), (vd, vt)):
                sta.sta_permute_tokens(prob, layout[0], layout[1], 0, x, y)

        def permute_out():
            sta.sta_permute_tokens(prob, layout[0], layout[1], 1, ot, od)

        permute_in()
    else:
        qt, kt, vt, ot = qd, kd, vd, od
    ent = None
    warm = None

    def warmup_entropy(qq, kk, vv):
        e = torch.empty(w["heads"], w["N"], dtype=torch.float32, device="cuda")
        ow = torch.empty_like(qd)
        stw = torch.zeros(1, dtype=torch.int32, device="cuda")
        ms = None
        for i in range(4):
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record()
            sta.sta_dense_attn_entropy_fwd(session.problem(w), qq, kk, vv, 0.0, ow, e,
                                           dev_status=stw)
            b_.record()
            torch.cuda.synchronize()
            ms = a_.elapsed_time(b_)
        if int(stw.item()) != 0:
            raise RuntimeError("device status " + sta.sta_dev_status_string(int(stw.item())))
        return e, ms

    if w["selector"] == "tra_token":
        ent, warm = warmup_entropy(qt, kt, vt)  # entropies by position of the sequence
    sel = session.selector(w, difd, entropy=ent)
    prm = session.attn_params(w)
    L = session.Lists(w)
    sws = session.selector_workspace(w)
    needs_qk = w["selector"] in ("entropy", "ibcs_sip", "dynrad")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()  # the stream every library call below uses
    l2_flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def select():
        sta.sta_build_blocks(prob, sel, qt if needs_qk else None, kt if needs_qk else None,
                             L.struct, workspace=sws, dev_status=st)

    def attend(qq=qt, kk=kt, vv=vt, oo=ot):
        sta.sta_sparse_attn_fwd(prob, prm, qq, kk, vv, L.struct, oo, dev_status=st)

    def step():
        if layout:
            permute_in()
        select()
        attend()
        if layout:
            permute_out()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError("device status " + sta.sta_dev_status_string(int(st.item())))
    if routed:
        pairs = session.retained_pairs_routed(w, L.routed_flag)
    else:
        pairs = session.retained_pairs(w, L)
    flops = 4.0 * w["d"] * pairs
    dense_flops = 4.0 * w["d"] * float(w["N"]) ** 2 * w["heads"]
    entries = int(L.cnt.sum().item())

    # One CUDA graph per step (selector + attention) so that the timed region
    # holds device work only; selector-only and attention-only graphs give
    # the per-stage device times.
    graphs = {}
    try:
        stages = [("step", step), ("select", select), ("attend", attend)]
        if layout:
            stages.append(("permute", lambda: (permute_in(), permute_out())))
        for name, fn in stages:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs[name] = g
        torch.cuda.synchronize()
        run_step = graphs["step"].replay
    except Exception as exc:  # capture not possible: time direct calls
        print(f"bench: CUDA graph capture failed ({exc}); timing direct calls", file=sys.stderr)
        graphs = {}
        run_step = step
    run_step()
    torch.cuda.synchronize()

    def timed(fn, n):
        ts = []
        for _ in range(n):
            l2_flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ts]

    # K iterations of (step, selector alone, attention alone), interleaved,
    # each replay after the same L2 flush and timed with its own events on
    # the launching stream
    run_sel = graphs["select"].replay if graphs else select
    run_att = graphs["attend"].replay if graphs else attend
    barrier(ws)
    with ClockSampler(local) as clk:
        ev = []
        for _ in range(args.steps):
            trip = []
            for fn in (run_step, run_sel, run_att):
                l2_flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                trip.append((a, b))
            ev.append(trip)
        torch.cuda.synchronize()
    barrier(ws)
    step_ms = [t[0][0].elapsed_time(t[0][1]) for t in ev]
    sel_ms = [t[1][0].elapsed_time(t[1][1]) for t in ev]
    attn_ms = [t[2][0].elapsed_time(t[2][1]) for t in ev]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), ws)
    sel_avg = sum(sel_ms) / len(sel_ms)
    attn_avg = sum(attn_ms) / len(attn_ms)

    layout_info = None
    if layout:
        run_perm = graphs["permute"].replay if graphs else (lambda: (permute_in(), permute_out()))
        perm_ms = timed(run_perm, max(5, min(20, args.steps)))
        perm_avg = sum(perm_ms) / len(perm_ms)
        # q, k, v in and o out: each element read once and written once
        pbytes = 4 * 2 * w["heads"] * w["N"] * w["d"] * 2
        layout_info = {"tile": list(layout), "permute_ms": perm_avg, "permute_bytes": pbytes,
                       "permute_gbs": pbytes / (perm_avg * 1e-3) / 1e9}
        # the same pipeline in raster order on the same grid, for comparison
        w_r = dict(w, layout=None)
        ent_r, _ = warmup_entropy(qd, kd, vd)
        sel_r = session.selector(w_r, None, entropy=ent_r)
        L_r = session.Lists(w_r)
        sta.sta_build_blocks(prob, sel_r, None, None, L_r.struct, dev_status=st)
        torch.cuda.synchronize()
        pairs_r = session.retained_pairs(w_r, L_r)
        att_r = timed(lambda: sta.sta_sparse_attn_fwd(prob, prm, qd, kd, vd, L_r.struct, od,
                                                      dev_status=st), max(5, min(20, args.steps)))
        layout_info["raster_comparison"] = {
            "retained_fraction": pairs_r / (w["N"] ** 2 * w["heads"]),
            "attn_ms": sum(att_r) / len(att_r)}
        del L_r, ent_r

    # dense at the same shape (the speedup denominator)
    def dense():
        sta.sta_dense_attn_fwd(prob, qd, kd, vd, 0.0, od, dev_status=st)

    for _ in range(2):
        dense()
    dense_ms = timed(dense, max(3, min(10, args.steps // 3)))
    dense_avg = sum(dense_ms) / len(dense_ms)

    # end to end through the C ABI with host buffers
    host_in = [x.pin_memory() for x in (q, k, v)] + ([dif.pin_memory()] if routed else [])
    dev_in = [qd, kd, vd] + ([difd] if routed else [])
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = oh.numel() * oh.element_size()
    e2e_ms = []
    for i in range(args.warmup + max(3, args.steps // 3)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for hsrc, ddst in zip(host_in, dev_in):
            ddst.copy_(hsrc, non_blocking=True)
        step()  # direct C-ABI calls, as a user makes them
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
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = flops / (attn_avg * 1e-3) / 1e12
    traffic = None
    rec = NCU_TRAFFIC.get(w["name"])
    if rec and rec["source_sha"] == source_sha() and not args.heads:
        traffic = rec["bytes_per_launch"]
    sbytes, sbound = selector_bytes(w, entries)
    sel_gbs = sbytes / (sel_avg * 1e-3) / 1e9
    total_flops = sum_over_ranks(flops, ws)
    line = {
        "metric": METRIC, "value": total_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_of(w), "cuda_graph": bool(graphs),
        "retained_pairs": pairs, "retained_fraction": pairs / (w["N"] ** 2 * w["heads"]),
        "attn_ms": attn_avg, "selector_ms": sel_avg,
        "stage_medians_ms": {"step": sorted(step_ms)[len(step_ms) // 2],
                             "selector": sorted(sel_ms)[len(sel_ms) // 2],
                             "attention": sorted(attn_ms)[len(attn_ms) // 2]},
        "dense_ms": dense_avg,
        "dense_tflops": dense_flops / (dense_avg * 1e-3) / 1e12,
        "speedup_vs_dense": dense_avg / attn_avg,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{pk_kind} bf16 (burst)"},
        "selector": {"ms": sel_avg, "bytes": sbytes, "bound": sbound, "achieved_gbs": sel_gbs,
                     "hbm_peak_gbs": hbm, "frac_of_hbm": sel_gbs / hbm,
                     "list_entries": entries},
        "e2e": {"value": total_flops / (e2e_avg * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_avg, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (SELECTOR_LAUNCHES[w["selector"]] + 1 + (4 if layout else 0))
                        * args.steps,
        "clocks": clk.summary(),
    }
    # Lists (and, for tra_token, entropies) reused across steps: a step is the
    # attention alone, timed by its own CUDA graph above.
    line["list_reuse"] = {"ms_per_step": attn_avg,
                          "value": total_flops / (max_over_ranks(attn_avg, ws) * 1e-3) / 1e12,
                          "unit": "TFLOP/s",
                          "note": "selector run once, its lists reused by every step"}
    if layout_info is not None:
        hbm_pk = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        layout_info["permute_frac_of_hbm"] = layout_info["permute_gbs"] / hbm_pk
        line["layout"] = layout_info
    if warm is not None:
        dflops = 4.0 * w["d"] * float(w["N"]) ** 2 * w["heads"]
        line["tra_warmup"] = {"ms": warm, "tflops": dflops / (warm * 1e-3) / 1e12,
                              "note": "dense attention + per-query entropy, run once and "
                                      "reused by the steps (not in the timed step)"}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget_s)
    if rank == 0:
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
