#!/usr/bin/env python
"""Fused classifier matmul + cross-entropy, forward+backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--parallel dp|vocab] [--impl ours|reference]

One step = the whole hot path on one batch of synthetic input, inputs already
resident in HBM: cce_fwd (loss, lse, and the colmax statistic when the
vocabulary sort is on) -> cce_vocab_sort (when on) -> cce_bwd (dH, dE).
Prints ONE JSON line (rank 0).  With N > 1 (torchrun, one process per GPU):
  --parallel dp     every rank runs its own batch (weak scaling, no collective
                    on the data path);
  --parallel vocab  the classifier is split by vocabulary over the ranks and
                    all ranks run the same batch (strong scaling): shard
                    forward, an all-gather of the [2, N] per-row parts and the
                    combine kernel, shard backward, an all-reduce of dH.
The time is the max over ranks.

`--impl reference` times the fp64 CPU oracle on a bounded row sample of the
same workload on the host cores (the only other place this file runs the
oracle is the cpu_baseline leg of the default arm).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_cross_entropy_cce_b200 import synthetic as syn  # noqa: E402

METRIC = "fused CE fwd+bwd tokens/s and % of B200 bf16 tensor peak; peak MB"
UNIT = "tokens/s"
EPS_BF16 = 2.0 ** -12
# per workload: (gradient filter on, vocabulary sort on)
MODES = {
    "tiny": (False, False),
    "gemma2_2b_head": (True, True),
    "llama3_8b_head": (False, False),
    "llama3_8b_head_8k": (False, False),
    "phi35_mini_head": (True, False),
    "composite_two_segment": (True, False),
}
L2_BYTES = 126 * 2 ** 20


# The peaks measured on this machine's B200s by the benchmark driver (cuBLAS bf16
# 8192^3 burst and 4 s sustained under the power cap; STREAM-style copy),
# used when the driver's MEASURED_PEAKS.json is not in the tree.
RECORDED_PEAKS = {"bf16_tflops": 1665.4, "bf16_tflops_sustained": 1339.0, "hbm_gbs": 6547.0}


def peaks():
    """(peaks, source): MEASURED_PEAKS.json when present, else the recorded
    measurement of this machine."""
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "MEASURED_PEAKS.json"
    except Exception:
        return dict(RECORDED_PEAKS), "recorded measurement of this pool (MEASURED_PEAKS.json absent)"


def tensor_roofline(kernel: str, flops_per_step: float, steps: int, ms_total: float, n_launches: int,
                    P: dict, src: str) -> dict:
    """Roofline entry of a tensor-core kernel class: achieved = its
    algorithmic FLOPs over the summed CUDA-event durations of its launches;
    frac against the measured burst bf16 peak (the kernels are timed as
    millisecond launches), the sustained figure beside it."""
    achieved = flops_per_step * steps / (ms_total / 1e3) / 1e12 if ms_total > 0 else None
    burst = float(P["bf16_tflops"])
    sus = float(P.get("bf16_tflops_sustained", burst))
    return {"bound": "tensor", "kernel": kernel,
            "achieved": round(achieved, 1) if achieved else None, "peak": burst,
            "unit": "TFLOP/s", "frac": round(achieved / burst, 4) if achieved else None,
            "peak_kind": "burst bf16 (measured, cuBLAS), of measured",
            "peak_source": src,
            "frac_of_sustained": round(achieved / sus, 4) if achieved else None,
            "sustained_peak": sus,
            "launches_per_step": n_launches // max(1, steps),
            "avg_launch_ms": round(ms_total / max(1, n_launches), 4)}


def src_hash16():
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "linear_cross_entropy_cce_b200", "csrc", "*.cu*")))
    for f in files + [os.path.join(ROOT, "include", "cce.h")]:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None
    when the CUDA sources changed since it was captured."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "roofline_traffic.json")))
    except Exception:
        return None
    if rec.get("csrc_sha256_16") != src_hash16():
        return None
    return rec.get("per_launch_dram_bytes", {}).get(kernel)


def host_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ oracle
def grow_sample(run, n_max: int, seconds: float, r0: int, quantum: int):
    """Size a CPU sample: time run(R) on growing R until one run takes at
    least half of `seconds` (or R reaches n_max).  The oracle's fixed costs
    per call (allocating and touching its full-vocabulary buffers) would make
    a single small calibration run overstate the time per row.  Returns the
    (R, seconds) of the last run."""
    n_max = max(1, n_max)
    R = min(r0, n_max)
    while True:
        t = run(R)
        if t >= 0.5 * seconds or R >= n_max:
            return R, t
        nxt = int(min(n_max, max(2 * R, 0.9 * seconds / max(t, 1e-6) * R)))
        if nxt < n_max:  # a multiple of the quantum, and always larger
            nxt = max(R + 1, (nxt // quantum) * quantum)
        R = nxt


def oracle_runner(x):
    """run(R): seconds of the fp64 oracle's forward + backward over R valid
    rows of x spread evenly over the batch."""
    import oracle
    segs64 = [(b, e, oracle.widen_bf16(E)) for b, e, E in x.segments]
    valid = np.nonzero(x.valid)[0]
    dl = x.dloss_mean()

    def run(R):
        rows = valid[np.linspace(0, len(valid) - 1, R).astype(np.int64)]
        Hs, ys, ds = x.H[rows], x.y[rows], dl[rows]
        t = time.perf_counter()
        oracle.forward(Hs, segs64, ys, x.wl.V, x.ignore_index)
        oracle.backward(Hs, segs64, ys, x.wl.V, ds, x.ignore_index,
                        filter_eps=EPS_BF16 if MODES.get(x.wl.name, (False,))[0] else 0.0)
        return time.perf_counter() - t

    return run, len(valid)


def oracle_desc(x, R):
    return (f"fp64 numpy oracle, forward+backward over {R} valid rows of {x.wl.name} "
            f"(N={x.wl.N}, D={x.wl.D}, V={x.wl.V}); full vocabulary and full dE per slice")


def oracle_sample(x, seconds: float, max_rows: int = 2048):
    """Time the fp64 oracle (forward + backward) on a row sample of about
    `seconds`; returns (rows/s, rows, seconds, description)."""
    run, n_valid = oracle_runner(x)
    R, t = grow_sample(run, min(max_rows, n_valid), seconds, 8, 8)
    return R / t, R, t, oracle_desc(x, R)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.out = self.p.communicate(timeout=10)[0]
            except Exception:
                self.p.kill()
                self.out = ""

    def summary(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "out", "").splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9 or (self.uuid and f[0] != self.uuid):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- multi-rank
class Prefetcher:
    """Double-buffered host -> device upload of every step's inputs, as a
    data loader does it: step k's copies run on a copy stream into buffer
    k % 2 and overlap step k-1's kernels; the compute stream waits for them
    before step k's kernels, and the copy stream waits for step k-2's kernels
    (the last readers of the buffer it overwrites)."""

    def __init__(self, host, dev_like, device):
        import torch
        self.host = host  # pinned host tensors, same dtypes as the views below
        self.bufs = [[torch.empty_like(d) for d in dev_like] for _ in range(2)]
        self.cs = torch.cuda.Stream(device)
        self.copied = [torch.cuda.Event() for _ in range(2)]
        self.used = [None, None]
        self.k = 0

    def start(self, event):
        """Orders the next copy after `event` (the start of a timed region)."""
        self.cs.wait_event(event)

    def next(self, compute):
        import torch
        b = self.k & 1
        self.k += 1
        with torch.cuda.stream(self.cs):
            if self.used[b] is not None:
                self.cs.wait_event(self.used[b])
            for d, h in zip(self.bufs[b], self.host):
                (d.view(h.dtype) if d.dtype != h.dtype else d).copy_(h, non_blocking=True)
            self.copied[b].record(self.cs)
        compute.wait_event(self.copied[b])
        return b, self.bufs[b]

    def release(self, b, compute):
        import torch
        ev = torch.cuda.Event()
        ev.record(compute)
        self.used[b] = ev


def timed_pipelined(fn, k, pf, world, dev):
    """Device time per step of k calls of fn (max over ranks), the copy
    stream ordered after the region's start event."""
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    pf.start(e0)
    for _ in range(k):
        fn()
    e1.record(s)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1) / k, world, dev)


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest `value` over all ranks (one all-reduce of one float); the
    value itself when there is a single rank."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tokens_per_s(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms / 1e3)


def vocab_shard_plan(segments, V: int, world: int, rank: int):
    """This rank's part of the head for --parallel vocab: the segments
    [(begin, end, E_rows)] of the head cut to the rank's 256-aligned vocabulary
    range (rows sliced, no copy; empty for a rank whose range holds no ids)."""
    from linear_cross_entropy_cce_b200 import vocab_parallel as vp
    v0, v1 = vp.shard_ranges(V, world)[rank]
    return [(lo, hi, E[lo - b:hi - b]) for b, e, E in segments
            for lo, hi in [(max(b, v0), min(e, v1))] if lo < hi]


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="gemma2_2b_head", choices=sorted(syn.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parallel", default="dp", choices=["dp", "vocab"],
                    help="dp: one batch per rank; vocab: the classifier split by vocabulary "
                         "over the ranks, one shared batch")
    ap.add_argument("--filter", choices=["on", "off", "default"], default="default")
    ap.add_argument("--sort", choices=["on", "off", "default"], default="default")
    ap.add_argument("--loss", choices=["ce", "kl"], default="ce",
                    help="ce: the cross-entropy hot path; kl: the soft-target KL between a "
                         "student and a teacher softmax")
    ap.add_argument("--kl-workload", default="soft_kl_24k_248k", choices=sorted(syn.KL_WORKLOADS))
    ap.add_argument("--kahan", action="store_true",
                    help="accumulate dE across steps with the Kahan-compensated bf16 path")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph replay timing of the step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if a.loss == "kl":
        return kl_main(a, world, rank, local)
    wl = syn.WORKLOADS[a.workload]
    filt, sort = MODES[wl.name]
    if a.filter != "default":
        filt = a.filter == "on"
    if a.sort != "default":
        sort = a.sort == "on"
    eps = EPS_BF16 if filt else 0.0

    if a.impl == "reference":
        return reference_arm(a, wl, world, rank, filt)

    import torch
    import torch.distributed as dist
    from linear_cross_entropy_cce_b200 import cce
    from linear_cross_entropy_cce_b200 import vocab_parallel as vp

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    vocab = a.parallel == "vocab"
    if world > 1:
        from datetime import timedelta
        # the bound on ranks waiting for one another; generous because every
        # rank first draws its inputs on the shared host cores
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)
    elif vocab:
        # the vocabulary-parallel step runs its exchanges over a process
        # group; a single GPU gets a group of one
        import socket
        from datetime import timedelta
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=timedelta(seconds=120), device_id=dev)
    # vocabulary parallel: one batch shared by all ranks, each holding the E
    # rows of its vocabulary range; data parallel: one batch per rank
    x = syn.make_inputs(wl, seed=0 if vocab else rank)
    N, D, V = wl.N, wl.D, wl.V
    n_valid = x.n_valid
    if vocab:
        host_segs = vocab_shard_plan(x.segments, V, world, rank)
    else:
        host_segs = list(x.segments)
    head_ranges = list(wl.segs())
    H = cce.bf16_from_bits(x.H, dev)
    segs = [(b, e, cce.bf16_from_bits(E, dev)) for b, e, E in host_segs]
    single = (not vocab) and len(segs) == 1 and segs[0][0] == 0 and segs[0][1] == V
    y = torch.from_numpy(x.y).to(dev)
    dloss = torch.from_numpy(x.dloss_mean()).to(dev)
    nseg = 0 if single else max(1, len(segs))
    v_live_rank = sum(e - b for b, e, _ in segs)
    v_live = wl.v_live
    # one caller-owned workspace serves the three calls of a step in turn (no
    # call's scratch outlives it: loss, lse, colmax and the permutation are
    # separate outputs)
    ws_all = torch.empty(max(cce.fwd_workspace_size(N, D, V, nseg),
                             cce.bwd_workspace_size(N, D, V, nseg),
                             cce.vocab_sort_workspace_size(N, V, nseg)), dtype=torch.uint8, device=dev)
    ws_f = ws_b = ws_s = ws_all
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    input_bytes = H.numel() * 2 + sum(s[2].numel() * 2 for s in segs) + y.numel() * 4
    kahan_kw = {}
    if a.kahan:  # running bf16 sum and compensation, kept across steps
        if vocab:
            ap.error("--kahan runs with --parallel dp")
        S = [torch.zeros_like(t) for _, _, t in segs]
        C = [torch.zeros_like(t) for _, _, t in segs]
        kahan_kw = dict(kahan=True, dE_out=S[0] if single else S, dE_comp=C[0] if single else C)

    def dp_step(Hd=H, segd=segs, yd=y):
        kw = dict(workspace=ws_f, status=status)
        if single:
            out = cce.fwd(Hd, segd[0][2], yd, x.ignore_index, want_colmax=sort, **kw)
        else:
            out = cce.fwd(Hd, None, yd, x.ignore_index, segments=segd, V=V, want_colmax=sort, **kw)
        loss, lse = out[0], out[1]
        perm = None
        if sort:
            perm = cce.vocab_sort(out[2], yd, V, x.ignore_index,
                                  segments=None if single else segd, workspace=ws_s)
        kw = dict(filter_eps=eps, vocab_perm=perm, colmax=out[2] if sort else None,
                  workspace=ws_b, status=status, **kahan_kw)
        if single:
            dH, dE, _ = cce.bwd(Hd, segd[0][2], yd, lse, dloss, x.ignore_index, **kw)
        else:
            dH, dE, _ = cce.bwd(Hd, None, yd, lse, dloss, x.ignore_index, segments=segd, V=V, **kw)
        return loss, dH, dE

    def vocab_step(Hd=H, segd=segs, yd=y):
        # shard forward + all-gather + combine kernel; shard backward + all-reduce
        out = vp.vp_forward(Hd, yd, segd, V, x.ignore_index, want_colmax=sort,
                            head_ranges=head_ranges)
        loss, lse = out[0], out[1]
        perm = None
        if sort and segd:
            perm = cce.vocab_sort(out[2], yd, V, x.ignore_index, segments=segd, workspace=ws_s)
        dH, dE = vp.vp_backward(Hd, yd, lse, dloss, segd, V, x.ignore_index, filter_eps=eps,
                                vocab_perm=perm, colmax=out[2] if (sort and segd) else None)
        return loss, dH, dE

    step = vocab_step if vocab else dp_step

    def fwd_only():
        if vocab:
            return vp.vp_forward(H, y, segs, V, x.ignore_index, head_ranges=head_ranges)
        if single:
            return cce.fwd(H, segs[0][2], y, x.ignore_index, workspace=ws_f, status=status)
        return cce.fwd(H, None, y, x.ignore_index, segments=segs, V=V, workspace=ws_f,
                       status=status)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, k):
        barrier()
        torch.cuda.synchronize(dev)
        s = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(k):
            fn()
        e1.record(s)
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1) / k, world, dev)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} during warm-up")

    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", ""))
    uuid = uuid if uuid.startswith("GPU-") or not uuid else "GPU-" + uuid
    l0 = cce.launch_count()
    with ClockSampler(uuid) as clk:
        ms_step = timed(step, a.steps)
    launches = cce.launch_count() - l0
    clocks = clk.summary()

    # the same step captured once into a CUDA graph and replayed (no host
    # launch work per step; supplementary to the eager value above)
    graph = None
    if not vocab and not a.no_graph:
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        ms_graph = timed(g.replay, a.steps)
        graph = {"ms_per_step": round(ms_graph, 3),
                 "value": round(tokens_per_s(N, world, ms_graph), 1), "unit": UNIT,
                 "note": "the same step captured once into a CUDA graph, replayed K times"}
        del g
        torch.cuda.synchronize(dev)

    # forward alone (context), then a per-kernel-class timing pass
    for _ in range(3):
        fwd_only()
    ms_fwd = timed(fwd_only, a.steps)
    cce.timing_enable(0b111111)
    ms_prof = timed(step, a.steps)
    per_class = cce.timing_read()
    cce.timing_enable(0)

    # peak memory of one step beyond the resident inputs and workspaces
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    step()
    torch.cuda.synchronize(dev)
    peak_extra = torch.cuda.max_memory_allocated(dev) - base
    ws_bytes = ws_all.numel()

    # end to end through the public API from pinned host buffers: every
    # step's inputs are copied host -> device (double-buffered on a copy
    # stream, overlapping the previous step's kernels) and its loss read back
    e2e = None
    if not a.no_e2e:
        hH = torch.from_numpy(x.H.view(np.int16)).pin_memory()
        hE = [torch.from_numpy(E.view(np.int16)).pin_memory() for _, _, E in host_segs]
        hy = torch.from_numpy(x.y).pin_memory()
        hloss = torch.empty(N, dtype=torch.float32).pin_memory()
        pf = Prefetcher([hH, hy] + hE, [H, y] + [s_[2] for s_ in segs], dev)

        def e2e_step():
            cs = torch.cuda.current_stream(dev)
            b, (Hb, yb, *Eb) = pf.next(cs)
            segd = [(b0, e0, d) for (b0, e0, _), d in zip(segs, Eb)]
            loss, _, _ = step(Hb, segd, yb)
            hloss.copy_(loss, non_blocking=True)
            pf.release(b, cs)

        for _ in range(3):
            e2e_step()
        ms_e2e = timed_pipelined(e2e_step, a.steps, pf, world, dev)
        h2d = hH.numel() * 2 + sum(h.numel() * 2 for h in hE) + hy.numel() * 4
        tok_e2e = N / (ms_e2e / 1e3) if vocab else tokens_per_s(N, world, ms_e2e)
        e2e = {"value": round(tok_e2e, 1), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(N * 4),
               "ms_per_step": round(ms_e2e, 3),
               "copies": "pinned host -> device every step on a copy stream, double-buffered "
                         "(step k+1's copies overlap step k's kernels); loss read back every step"}

    P, psrc = peaks()
    flops_fwd = 2.0 * n_valid * D * v_live_rank  # per rank (its vocabulary shard in vocab mode)
    flops_step_job = 8.0 * n_valid * D * v_live * (1 if vocab else world)
    class_flops = {"fwd_tile_stream": flops_fwd, "bwd_g_producer": flops_fwd,
                   "bwd_dE_contraction": flops_fwd, "bwd_dH_contraction": flops_fwd}
    dom = max(class_flops, key=lambda k: per_class[k][0])
    dom_ms, dom_n = per_class[dom]
    roofline = tensor_roofline(dom, class_flops[dom], a.steps, dom_ms, dom_n, P, psrc)
    roofline.update({
        "traffic": recorded_traffic(dom) if (wl.name == "gemma2_2b_head" and not vocab) else None,
        "traffic_note": "DRAM bytes of one working launch of this kernel (one vocabulary chunk "
                        "for the G producer) from the committed ncu capture "
                        "(profiles/roofline_traffic.json, cold cache); null if the sources changed",
        "achieved_note": "algorithmic FLOPs of the class per step (2 N_v D V_live of this rank) "
                         "over the summed CUDA-event durations of all its launches in the step",
        "launches_note": "the G producer launches twice per vocabulary chunk when filtering; the "
                         "second (repair) launch exits at once unless the chunk overflowed its "
                         "sparse list"})
    step_tflops = flops_step_job / (ms_step / 1e3) / 1e12
    burst = float(P["bf16_tflops"])
    sustained = float(P.get("bf16_tflops_sustained", burst))

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rps, R, t, desc = oracle_sample(x, a.cpu_seconds)
        cpu = {"value": round(rps, 3), "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": desc, "seconds": round(t, 2)}

    value = N / (ms_step / 1e3) if vocab else tokens_per_s(N, world, ms_step)
    parallelism = (f"vocab{world} (E split by vocabulary, one shared batch)" if vocab
                   else f"dp{world} (independent batches)")
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "strong" if vocab else "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and value recipe of the workload; no dataset or trained weights)",
        "config": {"workload": wl.name, "N": N, "N_valid": n_valid, "D": D, "V": V,
                   "V_live": v_live, "V_live_per_rank": v_live_rank,
                   "segments": [list(s) for s in wl.segs()],
                   "logit_std": wl.logit_std, "filter_eps": eps, "vocab_sort": sort,
                   "kahan_dE": bool(a.kahan),
                   "global_batch_tokens": N if vocab else N * world, "parallelism": parallelism,
                   "l2": f"inputs larger than L2 (E = {sum(s[2].numel() for s in segs) * 2 / 2**20:.0f} MiB per rank > 126 MiB)",
                   "tokens_per_s_valid_rows": round(value * n_valid / N, 1)},
        "tensor_peak_frac": {"of_measured_burst": round(step_tflops / burst, 4),
                             "of_measured_sustained": round(step_tflops / sustained, 4),
                             "of_spec_2250": round(step_tflops / 2250.0, 4),
                             "tflops_unfiltered_8NDV": round(step_tflops, 1),
                             "peak_source": psrc},
        "fwd_ms": round(ms_fwd, 3), "fwd_bwd_ms": round(ms_step, 3),
        "peak_mb": round((peak_extra + ws_bytes) / 2 ** 20, 1),
        "peak_mb_detail": {"workspaces_mb": round(ws_bytes / 2 ** 20, 1),
                           "step_allocations_mb": round(peak_extra / 2 ** 20, 1),
                           "inputs_mb": round(input_bytes / 2 ** 20, 1),
                           "materialised_logits_bf16_mb": round(N * V * 2 / 2 ** 20, 1)},
        "roofline": roofline,
        "per_kernel_ms_per_step": {k: round(v[0] / a.steps, 3) for k, v in per_class.items()},
        "untimed_ms_per_step": round(ms_prof - sum(v[0] for v in per_class.values()) / a.steps, 3),
        "profiled_ms_per_step": round(ms_prof, 3),
        "gpu_launches": int(launches),
        "gpu_launches_per_step": int(launches // max(1, a.steps)),
        "clocks": clocks,
        "e2e": e2e,
        "graph": graph,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
    if dist.is_initialized():
        dist.destroy_process_group()


KL_METRIC = "soft-target KL fwd+bwd positions/s (and % of B200 bf16 tensor peak)"


def kl_oracle_runner(wl, Hs, Ht, E, eps: float):
    """run(R): seconds of the fp64 oracle's KL forward + backward over R rows
    spread evenly over the batch."""
    import oracle
    E64 = oracle.widen_bf16(E)
    dl = np.full(wl.N, 1.0 / wl.N)

    def run(R):
        rows = np.linspace(0, wl.N - 1, R).astype(np.int64)
        t = time.perf_counter()
        oracle.kl_forward(Hs[rows], E64, Ht[rows], E64)
        oracle.kl_backward(Hs[rows], E64, Ht[rows], E64, dl[rows], filter_eps=eps)
        return time.perf_counter() - t

    return run


def kl_oracle_desc(wl, R):
    return (f"fp64 numpy oracle, KL forward+backward over {R} rows of {wl.name} "
            f"(N={wl.N}, D={wl.D}, V={wl.V}); full vocabulary and full dE per slice")


def kl_oracle_sample(wl, Hs, Ht, E, seconds: float, eps: float):
    """Time the fp64 oracle's KL forward + backward on a row sample of about
    `seconds`; returns (rows/s, rows, seconds, description)."""
    run = kl_oracle_runner(wl, Hs, Ht, E, eps)
    R, t = grow_sample(run, min(1024, wl.N), seconds, 4, 4)
    return R / t, R, t, kl_oracle_desc(wl, R)


def kl_main(a, world, rank, local):
    """The soft-target KL path: cce_kl_fwd + cce_kl_bwd per step."""
    wl = syn.KL_WORKLOADS[a.kl_workload]
    eps = 0.0 if a.filter == "off" else EPS_BF16
    Hs, Ht, E = syn.make_kl_inputs(wl, seed=rank)
    if a.impl == "reference":
        if rank != 0:
            return
        # one sizing pass, then every step runs the same R rows
        run = kl_oracle_runner(wl, Hs, Ht, E, eps)
        R, _ = grow_sample(run, min(1024, wl.N), max(2.0, 120.0 / (a.steps + a.warmup)), 4, 4)
        desc = kl_oracle_desc(wl, R)
        times = []
        for i in range(a.warmup + a.steps):
            t = run(R)
            if i >= a.warmup:
                times.append(t)
        ms = 1e3 * float(np.mean(times))
        v = R / (ms / 1e3)
        print(json.dumps({"impl": "reference", "metric": KL_METRIC, "value": round(v, 3),
                          "unit": "positions/s", "n_gpus": world, "steps": a.steps,
                          "warmup": a.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": {"workload": wl.name, "rows_per_step": R},
                          "cpu_baseline": {"value": round(v, 3), "unit": "positions/s",
                                           "cores": host_cores(), "kind": "oracle", "sample": desc},
                          "e2e": {"value": round(v, 3), "unit": "positions/s",
                                  "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return
    import torch
    import torch.distributed as dist
    from linear_cross_entropy_cce_b200 import cce
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)
    N, D, V = wl.N, wl.D, wl.V
    Hs_d, Ht_d, E_d = (cce.bf16_from_bits(t, dev) for t in (Hs, Ht, E))
    dl = torch.full((N,), 1.0 / N, dtype=torch.float32, device=dev)
    ws_f = torch.empty(cce.lib().cce_kl_fwd_workspace_size(N, D, V), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(cce.lib().cce_kl_bwd_workspace_size(N, D, V, 0), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(hs=Hs_d, ht=Ht_d, e=E_d):
        kl, ls, lt = cce.kl_fwd(hs, e, ht, e, workspace=ws_f, status=status)
        cce.kl_bwd(hs, e, ht, e, ls, lt, dl, filter_eps=eps, workspace=ws_b, status=status)
        return kl

    def timed(fn, k):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        s = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(k):
            fn()
        e1.record(s)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        return max_over_ranks(e0.elapsed_time(e1) / k, world, dev)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())} during warm-up")
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", ""))
    uuid = uuid if uuid.startswith("GPU-") or not uuid else "GPU-" + uuid
    l0 = cce.launch_count()
    with ClockSampler(uuid) as clk:
        ms_step = timed(step, a.steps)
    launches = cce.launch_count() - l0
    ms_fwd = timed(lambda: cce.kl_fwd(Hs_d, E_d, Ht_d, E_d, workspace=ws_f, status=status), a.steps)
    cce.timing_enable(0b111111)
    timed(step, a.steps)
    per_class = cce.timing_read()
    cce.timing_enable(0)

    P, psrc = peaks()
    ndv = float(N) * D * V
    class_flops = {"fwd_tile_stream": 4 * ndv, "bwd_g_producer": 4 * ndv,
                   "bwd_dE_contraction": 2 * ndv, "bwd_dH_contraction": 2 * ndv}
    dom = max(class_flops, key=lambda k: per_class[k][0])
    dom_ms, dom_n = per_class[dom]
    roofline = tensor_roofline(dom, class_flops[dom], a.steps, dom_ms, dom_n, P, psrc)
    roofline["traffic"] = None
    peak_sus = float(P.get("bf16_tflops_sustained", P["bf16_tflops"]))
    step_tflops = 12 * ndv / (ms_step / 1e3) / 1e12

    e2e = None
    if not a.no_e2e:
        hHs = torch.from_numpy(Hs.view(np.int16)).pin_memory()
        hHt = torch.from_numpy(Ht.view(np.int16)).pin_memory()
        hE = torch.from_numpy(E.view(np.int16)).pin_memory()
        hkl = torch.empty(N, dtype=torch.float32).pin_memory()
        pf = Prefetcher([hHs, hHt, hE], [Hs_d, Ht_d, E_d], dev)

        def e2e_step():
            cs = torch.cuda.current_stream(dev)
            b, (bs, bt, be) = pf.next(cs)
            hkl.copy_(step(bs, bt, be), non_blocking=True)
            pf.release(b, cs)

        for _ in range(3):
            e2e_step()
        ms_e2e = timed_pipelined(e2e_step, a.steps, pf, world, dev)
        e2e = {"value": round(tokens_per_s(N, world, ms_e2e), 1), "unit": "positions/s",
               "h2d_bytes_per_step": int((Hs.size + Ht.size + E.size) * 2),
               "d2h_bytes_per_step": int(N * 4), "ms_per_step": round(ms_e2e, 3),
               "copies": "pinned host -> device every step on a copy stream, double-buffered "
                         "(step k+1's copies overlap step k's kernels); KL read back every step"}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rps, R, t, desc = kl_oracle_sample(wl, Hs, Ht, E, a.cpu_seconds, eps)
        cpu = {"value": round(rps, 3), "unit": "positions/s", "cores": host_cores(),
               "kind": "oracle", "sample": desc, "seconds": round(t, 2)}
    out = {
        "metric": KL_METRIC, "value": round(tokens_per_s(N, world, ms_step), 1),
        "unit": "positions/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(ms_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded student and teacher rows, one shared head)",
        "config": {"workload": wl.name, "N": N, "D": D, "V": V, "logit_std": wl.logit_std,
                   "filter_eps": eps, "parallelism": f"dp{world} (independent batches)",
                   "l2": f"inputs larger than L2 (E = {E.size * 2 / 2**20:.0f} MiB > 126 MiB)"},
        "tensor_peak_frac": {"of_measured_burst": round(step_tflops / float(P["bf16_tflops"]), 4),
                             "of_measured_sustained": round(step_tflops / peak_sus, 4),
                             "tflops_unfiltered_12NDV": round(step_tflops, 1)},
        "fwd_ms": round(ms_fwd, 3), "fwd_bwd_ms": round(ms_step, 3),
        "roofline": roofline,
        "per_kernel_ms_per_step": {k: round(v[0] / a.steps, 3) for k, v in per_class.items()},
        "gpu_launches": int(launches), "gpu_launches_per_step": int(launches // max(1, a.steps)),
        "clocks": clk.summary(), "e2e": e2e, "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def reference_arm(a, wl, world, rank, filt):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    x = syn.make_inputs(wl, seed=0)
    per_step = max(2.0, 120.0 / max(1, a.steps + a.warmup))
    # one sizing pass, then every step runs the same R rows
    run, n_valid = oracle_runner(x)
    R, _ = grow_sample(run, min(2048, n_valid), per_step, 8, 8)
    desc = oracle_desc(x, R)
    times = []
    for i in range(a.warmup + a.steps):
        t = run(R)
        if i >= a.warmup:
            times.append(t)
    ms = 1e3 * float(np.mean(times))
    v = R / (ms / 1e3)
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": UNIT,
           "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": wl.name, "N": wl.N, "D": wl.D, "V": wl.V,
                                            "rows_per_step": R},
           "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": host_cores(),
                            "kind": "oracle", "sample": desc},
           "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
