"""Benchmark: masked attention forward TFLOP/s on attended pairs (bf16), B200.

One step = the whole hot path on one batch: plan the dense causal (N, N) mask
(bfa_plan_dense: classify + lists + order) and run the fused forward (bfa_fwd)
for B=4, H=Hkv=32, N=8192, D=128.  FLOPs are counted on attended pairs only:
4 * D * nnz per (batch, head), nnz = N (N + 1) / 2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bfa|reference]
    python bench.py --sweep      # forward and backward on every workload, one JSON line each

Multi-GPU (torchrun): every rank runs its own full workload (weak scaling, no
collective on the data path); value = all ranks' FLOPs / max-over-ranks time.
``--impl reference`` times the CPU float64 oracle on the host cores instead (rank
0 only), on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# kernels of one step: k_dense_classify, k_rows (the plan) and bfa_fwd_kernel<128>
# (the forward)
LAUNCHES_PER_STEP = 3
METRIC = "masked attn fwd TFLOP/s on attended pairs (bf16), % of B200 tensor peak"
WORKLOAD = dict(workload="causal_8192", B=4, H=32, Hkv=32, N=8192, D=128, mask="dense causal (N,N) bool",
                plan="bfa_plan_dense per step", layout="BSHD")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _fwd_traffic():
    """DRAM bytes per launch of the forward from the committed ncu record, or None
    when the kernel sources have changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "bfa_fwd_kernel_causal_8192.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for name in rec["source_files"]:
            with open(os.path.join(ROOT, name), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return rec["dram_bytes_read"] + rec["dram_bytes_write"]
    except Exception:
        return None


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank timings (the job time is the slowest rank's)."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tflops(flops_per_rank, world, ms_per_step):
    """Weak scaling: every rank processes its own batch; value = all ranks' FLOPs / max time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def _attended_flops(N, D, BH):
    nnz = N * (N + 1) // 2
    return 4.0 * D * nnz * BH, nnz


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        srt = sorted(sm)
        loaded = [x for x in srt if x > 0.5 * max(srt)] or srt
        return {"sm_mhz": loaded[len(loaded) // 2], "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _threads_used():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _host_cores():
    """The host's core count and torch's intra-op thread count, reported beside
    the threads the oracle's BLAS actually used."""
    import torch
    return {"os_cpu_count": os.cpu_count(), "torch_threads": torch.get_num_threads()}


def _median(xs):
    xs = sorted(xs)
    n = len(xs)
    return xs[n // 2] if n % 2 else 0.5 * (xs[n // 2 - 1] + xs[n // 2])


# Public datasheet dense bf16 tensor throughput of one B200 (context beside the
# measured denominators).
DATASHEET_BF16_TFLOPS = 2250.0


def planner_leg(bfa, masks, dev, reps=10):
    """bfa_plan_dense alone, L2 flushed before every timed call (a 256 MB write),
    CUDA events around the call: median ms and GB/s on the algorithmic bytes
    (mask read once + plan written: class grid, 2 KB of packed bits per partial
    tile, 8 B per listed tile, 8 B per row)."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    out = {}
    for name, mask in masks:
        Sq, Sk = mask.shape
        plan = bfa.plan_dense(mask)
        n_full, n_part, n_empty = plan.stats()
        plan.destroy()
        nqt = -(-Sq // 128)
        algo = Sq * Sk + (n_full + n_part + n_empty) + 2048 * n_part + 8 * (n_full + n_part) + 8 * nqt
        times = []
        for i in range(reps + 2):
            flush.fill_(i & 255)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            plan = bfa.plan_dense(mask)
            e1.record(stream)
            torch.cuda.synchronize()
            plan.destroy()
            if i >= 2:
                times.append(e0.elapsed_time(e1))
        ms = _median(times)
        out[name] = {"ms_median": ms, "algorithmic_bytes": algo, "gbs": algo / (ms * 1e-3) / 1e9,
                     "tiles": {"full": n_full, "partial": n_part, "empty": n_empty}}
    del flush
    return out


def cpu_oracle_sample(w, n_heads=4, rows=None):
    """Time the float64 oracle on a bounded sample: ``n_heads`` (b, h) pairs, all rows."""
    from oracle import attention as oa
    M = w["mask"].numpy()
    N, D = w["N"], w["D"]
    pairs = [(b, h) for b in range(w["B"]) for h in range(w["H"])][:n_heads]
    t0 = time.perf_counter()
    for (b, h) in pairs:
        q = w["q"][b, :, h]
        MM = M
        if rows is not None:
            q, MM = q[:rows], M[:rows]
        oa.masked_attention(q, w["k"][b, :, h], w["v"][b, :, h], MM)
    dt = time.perf_counter() - t0
    nnz = int(M.sum()) if rows is None else int(M[:rows].sum())
    flops = 4.0 * D * nnz * len(pairs)
    return flops / dt / 1e12, dt, len(pairs)


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import workloads
    w = workloads.causal_8192()
    times, vals = [], []
    per_step_heads = 2
    for i in range(args.warmup + args.steps):
        v, dt, n = cpu_oracle_sample(w, n_heads=per_step_heads)
        if i >= args.warmup:
            times.append(dt)
            vals.append(v)
    value = _median(vals)
    cores = _threads_used()
    sample = f"{per_step_heads} of 128 (batch, head) pairs per step, all 8192 rows, float64 NumPy oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * _median(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(WORKLOAD, parallelism=f"dp{args.gpus}"),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample,
                         **_host_cores()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_bfa(args, rank, world, local_rank):
    import numpy as np
    import torch

    import mask_skipping_flashattention_b200 as bfa
    import workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = workloads.causal_8192()
    B, H, N, D = w["B"], w["H"], w["N"], w["D"]
    q, k, v = w["q"].to(dev), w["k"].to(dev), w["v"].to(dev)
    mask = w["mask"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flops, nnz = _attended_flops(N, D, B * H)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        plan = bfa.plan_dense(mask)
        if ev is not None:
            ev[1].record(stream)
        bfa.fwd(plan, q, k, v, out=out, lse=lse)
        if ev is not None:
            ev[2].record(stream)
        plan.destroy()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    # per-step forward and plan times: the median of the K event pairs
    fwd_ms = _median([e[1].elapsed_time(e[2]) for e in evs])
    plan_ms = _median([e[0].elapsed_time(e[1]) for e in evs])
    ms, fwd_ms, plan_ms = max_over_ranks([ms, fwd_ms, plan_ms], dist, dev)
    ms_per_step = ms / args.steps
    value = whole_job_tflops(flops, world, ms_per_step)

    # end to end through the public API with host buffers: every step copies its
    # q, k, v and mask in from pinned memory, plans, runs the forward and reads out
    # and lse back.  Copies in, compute and copies out go on three streams over two
    # device buffer sets, so step i's inputs stream in while step i - 1 computes and
    # its results stream out (PCIe moves both directions at once).
    hq, hk, hv = w["q"].pin_memory(), w["k"].pin_memory(), w["v"].pin_memory()
    hm = w["mask"].pin_memory()
    ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hm))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    bufs = [dict(q=q, k=k, v=v, mask=mask, out=out, lse=lse),
            dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), mask=torch.empty_like(mask),
                 out=torch.empty_like(out), lse=torch.empty_like(lse))]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run_e2e(n):
        ev = [[torch.cuda.Event(enable_timing=(i == 0 and r == 0) or (i == n - 1 and r == 2)) for r in range(3)]
              for i in range(n)]
        start = torch.cuda.Event(enable_timing=True)
        start.record(s_in)
        for i in range(n):
            b = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev[i - 2][1])  # step i - 2 has finished reading this buffer set
                b["q"].copy_(hq, non_blocking=True)
                b["k"].copy_(hk, non_blocking=True)
                b["v"].copy_(hv, non_blocking=True)
                b["mask"].copy_(hm, non_blocking=True)
                ev[i][0].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev[i][0])
                if i >= 2:
                    s_cmp.wait_event(ev[i - 2][2])  # step i - 2's results have been read back
                plan = bfa.plan_dense(b["mask"])
                bfa.fwd(plan, b["q"], b["k"], b["v"], out=b["out"], lse=b["lse"])
                ev[i][1].record(s_cmp)
                plan.destroy()
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[i][1])
                ho.copy_(b["out"], non_blocking=True)
                hl.copy_(b["lse"], non_blocking=True)
                ev[i][2].record(s_out)
        return start, ev[n - 1][2]

    e2e_steps = max(2, min(args.steps, 6))
    run_e2e(2)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = run_e2e(e2e_steps)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], dist, dev)[0]
    e2e_value = whole_job_tflops(flops, world, e2e_ms)

    # backward (f1) on the same workload, timed on its own after the forward
    # metric: dq, dk, dv for a seeded upstream gradient, plan and LSE reused
    g = torch.Generator(device="cpu")
    g.manual_seed(4242)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
    plan = bfa.plan_dense(mask)
    bfa.fwd(plan, q, k, v, out=out, lse=lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for _ in range(2):
        bfa.bwd(plan, q, k, v, out, dout, lse, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bwd_steps = max(1, min(args.steps, 5))
    b0.record(stream)
    for _ in range(bwd_steps):
        bfa.bwd(plan, q, k, v, out, dout, lse, dq=dq, dk=dk, dv=dv)
    b1.record(stream)
    torch.cuda.synchronize()
    plan.device_status()
    plan.destroy()
    bwd_ms = max_over_ranks([b0.elapsed_time(b1) / bwd_steps], dist, dev)[0]

    # the planner on its own (L2 flushed before each call), on the bench's 67 MB
    # causal mask and the 268 MB union mask of the 16384 workload
    plan_masks = [("causal_8192", mask)]
    if rank == 0 and not args.no_union_planner:
        plan_masks.append(("union_16384", workloads.union_16384(with_qkv=False)["mask"].to(dev)))
    planner = planner_leg(bfa, plan_masks, dev)
    del plan_masks

    peaks, src = _peaks()
    fwd_tflops = flops / (fwd_ms * 1e-3) / 1e12
    # bytes the forward must move at least: read q, k, v once, write out and lse
    algo_bytes = 3 * q.numel() * q.element_size() + out.numel() * out.element_size() + lse.numel() * 4
    peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(WORKLOAD, global_batch=B * world, seq_len=N, parallelism=f"dp{world}",
                       attended_pairs_per_head=nnz, gflop_per_step=flops / 1e9,
                       l2="inputs larger than L2 (q, k, v 268 MB each, mask 67 MB); no flush"),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "kernel": "bfa_fwd_kernel<128>", "achieved": fwd_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": fwd_tflops / peak, "peak_source": f"{src} bf16_tflops (burst)",
                     "frac_of_sustained": fwd_tflops / peaks.get("bf16_tflops_sustained", peak),
                     "frac_of_datasheet": fwd_tflops / DATASHEET_BF16_TFLOPS,
                     "timing": f"median of {args.steps} per-step CUDA-event pairs around the forward",
                     "traffic": _fwd_traffic(), "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "algorithmic_bytes": algo_bytes},
        "fwd_ms": fwd_ms, "plan_ms": plan_ms,
        "planner": {"call": "bfa_plan_dense (k_dense_classify, k_rows)", "bound": "hbm",
                    "peak_gbs": peaks["hbm_gbs"], "peak_source": f"{src} hbm_gbs",
                    "l2": "256 MB written before every timed call", **{
                        k: dict(v, frac=v["gbs"] / peaks["hbm_gbs"]) for k, v in planner.items()}},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "overlap": "copies in, plan + forward and copies out on three streams over two device buffer sets"},
        "bwd": {"ms_per_step": bwd_ms, "tflops": 2.5 * flops / (bwd_ms * 1e-3) / 1e12,
                "frac": 2.5 * flops / (bwd_ms * 1e-3) / 1e12 / peak,
                "flops_counted": "2.5 x the forward's attended-pair flops (dV, dP, dQ, dK and the recomputed S)",
                "kernels": "k_bwd_prep, k_bwd_fused, k_bwd_dq_store (fused pass, D = 128)", "steps": bwd_steps},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
    }
    if rank == 0 and not args.no_cpu_baseline:
        v_cpu, dt, n = cpu_oracle_sample(w, n_heads=16)  # about 10 s of float64 work
        line["cpu_baseline"] = {"value": v_cpu, "unit": "TFLOP/s", "cores": _threads_used(), "kind": "oracle",
                                "sample": f"{n} of 128 (batch, head) pairs, all 8192 rows, {dt:.1f} s float64",
                                **_host_cores()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _time_ms(fn, reps):
    import torch
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def run_sweep(args):
    """Forward and backward throughput (attended-pair TFLOP/s) on every workload
    configuration, one JSON line each (information; not the driver's metric line)."""
    import numpy as np
    import torch

    import mask_skipping_flashattention_b200 as bfa
    import workloads
    from oracle import masks as om

    torch.cuda.set_device(0)
    reps = max(3, args.steps)
    only = args.workload  # None: every workload

    def cuda(x):
        return torch.as_tensor(np.ascontiguousarray(x)).cuda()

    def measure(name, P, q, k, v, pairs, D, plan_desc, bwd=True):
        if only is not None and name != only:
            return
        out, lse = bfa.fwd(P, q, k, v)
        if args.fwd_only:  # a few forward calls only (an ncu capture of the forward)
            for _ in range(reps):
                bfa.fwd(P, q, k, v, out=out, lse=lse)
            torch.cuda.synchronize()
            P.device_status()
            print(json.dumps({"workload": name, "fwd_calls": reps + 1}), flush=True)
            return
        g = torch.Generator(device="cuda")
        g.manual_seed(7)
        dout = torch.randn(q.shape, device="cuda", generator=g).to(torch.bfloat16)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fms = _time_ms(lambda: bfa.fwd(P, q, k, v, out=out, lse=lse), reps)
        bms = _time_ms(lambda: bfa.bwd(P, q, k, v, out, dout, lse, dq=dq, dk=dk, dv=dv), reps) if bwd else None
        P.device_status()
        flops = 4.0 * D * pairs
        print(json.dumps({"workload": name, "plan": plan_desc, "attended_pairs": pairs, "fwd_ms": fms,
                          "fwd_tflops": flops / (fms * 1e-3) / 1e12, "bwd_ms": bms,
                          "bwd_tflops": 2.5 * flops / (bms * 1e-3) / 1e12 if bwd else None, "reps": reps}),
              flush=True)

    w = workloads.causal_8192()
    measure("causal_8192", bfa.plan_dense(w["mask"].cuda()), w["q"].cuda(), w["k"].cuda(), w["v"].cuda(),
            float(w["mask"].sum()) * w["B"] * w["H"], w["D"], "dense")
    del w
    w = workloads.blockcausal_gqa()
    ids = bfa.make_att_block_ids(cuda(w["pad_masks"]), cuda(w["att_masks"]), w["n_cross"], cuda(w["cross_pad_masks"]))
    dense = om.blockid_dense(*om.make_att_block_ids(w["pad_masks"], w["att_masks"], w["n_cross"],
                                                    w["cross_pad_masks"]))
    measure("blockcausal_gqa", bfa.plan_blockids(*ids), w["q"].cuda(), w["k"].cuda(), w["v"].cuda(),
            float(dense.sum()) * w["H"], w["D"], "block ids")
    w = workloads.varlen_16()
    cu = cuda(w["cu_seqlens"])
    lens = np.diff(w["cu_seqlens"]).astype(np.int64)
    for W in (-1, w["window"]):
        P = bfa.plan_blockids(cu_seqlens_q=cu, cu_seqlens_k=cu, max_q=w["max_len"], max_k=w["max_len"],
                              window_left=W)
        per_head = float((lens * (lens + 1) // 2).sum()) if W < 0 else \
            float(sum(int(np.minimum(np.arange(1, L + 1), W).sum()) for L in lens))
        measure(f"varlen_16 window={W}", P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), per_head * 32, w["D"],
                "varlen positions")
    del w
    w = workloads.bsr_16384()
    ip, ix = w["block_indptr"], w["block_indices"]
    nb = -(-w["S"] // w["block"])
    per_group = 0.0
    for b in range(ip.shape[0]):
        for h in range(ip.shape[1]):
            for r in range(nb):
                sel = ix[ip[b, h, r]:ip[b, h, r + 1]]
                per_group += float((sel < r).sum()) * 128 * 128 + float((sel == r).sum()) * 128 * 129 / 2
    P = bfa.plan_bsr(cuda(ip), cuda(ix), w["S"], w["S"], w["block"], w["block"], causal=True)
    measure("bsr_16384", P, w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), per_group * (w["H"] // w["Hkv"]), w["D"],
            "BSR, causal inside blocks")
    # the union workload's q, k, v are the BSR workload's (the same configuration,
    # shapes and seeds: workloads.qkv(5, ...)), so the tensors above are reused
    u = workloads.union_16384(with_qkv=False)
    measure("union_16384", bfa.plan_dense(u["mask"].cuda()), w["q"].cuda(), w["k"].cuda(), w["v"].cuda(),
            float(u["mask"].sum()) * w["B"] * w["H"], w["D"], "dense")
    del w, u
    # 16-token BSR rows with 8 query heads per kv head: GQA-packed tiles (one BSR
    # row of all 8 heads per tile) against 128-token tiles (the union of 8 rows'
    # lists)
    w = workloads.bsr_16384_q16_gqa8()
    ip, ix, S, qb, kb = w["block_indptr"], w["block_indices"], w["S"], w["q_block"], w["kv_block"]
    G = w["H"] // w["Hkv"]
    per_group = 0.0
    for b in range(ip.shape[0]):
        for h in range(ip.shape[1]):
            for r in range(ip.shape[2] - 1):
                sel = ix[ip[b, h, r]:ip[b, h, r + 1]]
                d = (r * qb) // kb
                t = np.arange(r * qb, min(S, (r + 1) * qb))
                per_group += float((sel < d).sum()) * t.size * kb + float((t - d * kb + 1).sum())
    q, k, v = w["q"].cuda(), w["k"].cuda(), w["v"].cuda()
    for name, plan in (("bsr_16384_q16_gqa8 packed", bfa.plan_bsr_packed(cuda(ip), cuda(ix), S, S, G, qb, kb,
                                                                         causal=True)),
                       ("bsr_16384_q16_gqa8 unpacked", bfa.plan_bsr(cuda(ip), cuda(ix), S, S, qb, kb, causal=True))):
        measure(name, plan, q, k, v, per_group * G, w["D"], "BSR, 16-token rows, causal inside blocks")
        del plan
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["bfa", "reference"], default="bfa")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-union-planner", action="store_true", help="skip the planner leg on the 268 MB union mask")
    ap.add_argument("--sweep", action="store_true", help="forward/backward on every workload (information)")
    ap.add_argument("--workload", default=None,
                    help="with --sweep: only this workload (causal_8192, blockcausal_gqa, 'varlen_16 window=-1', "
                         "'varlen_16 window=1024', bsr_16384, union_16384, 'bsr_16384_q16_gqa8 packed', "
                         "'bsr_16384_q16_gqa8 unpacked')")
    ap.add_argument("--fwd-only", action="store_true", help="with --sweep: forward calls only, no timing line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.sweep:
        return run_sweep(args)
    return run_bfa(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
