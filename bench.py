"""Benchmark of the frame-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path over one batch of the LVSA workload at a
Wan-2.1-1.3B-like shape (T=41 latent frames, P=1560 tokens/frame, H=12, d=128,
budget C=21, window W=9, anchor period T_per=4, denoising step s=0): the attended
frame sets are built on the GPU (sfa_build_sets), then frame-sparse attention runs
over them (sfa_forward), all through the C ABI of libsfa.so.

Metric: effective attended TFLOP/s = 4 d sum_{b,h,t} P * P |A(h,t)| / time, i.e. only
the QK^T and PV flops of attended, unpadded (query, key) pairs count.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch of the
same workload (weak scaling; heads and batches are independent, so there is no
data-path collective); timing is the max over ranks.

--impl reference times the CPU oracle (float64, the repository's plain reference
implementation of the same computation) on the host cores, on a bounded sample of
query rows of the same workload per step, sized so that the warm-up and timed steps
take about --reference-seconds (120 s by default) of oracle time; rank 0 alone runs it.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sfa_workloads import WORKLOADS, workload_qkv  # noqa: E402

METRIC = "effective attended TFLOP/s (and % of BF16 tensor peak); ms per sparse-attn call"
WORKLOAD = WORKLOADS["lvsa41"]
STEP_S = 0
WORKLOAD_DESC = ("LVSA frame-sparse attention, Wan-2.1-1.3B-like shape: T=41 frames, P=1560 "
                 "tokens/frame, H=12, d=128, B=1, C=21, W=9, T_per=4, step s=0")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["source"] = "fallback"
    return p


# DRAM bytes (read + write) of one forward launch on this workload, from one ncu capture
# of the same kernel on the 4-head version of the workload scaled by 3 to 12 heads (the
# traffic is per (head, frame, query tile) unit): 3 x (196.842496 + 51.089408) MB.  Set
# back to None whenever the forward kernel changes, until it is re-measured.
NCU_TRAFFIC_BYTES = 743_795_712
# DRAM bytes read + written by the gated-delta kernels of one call on the gdn workload,
# from an ncu capture: prep 231.952896 + 3.159552 MB, recurrence 143.392256 + 67.441664 MB.
# None once the kernels change, until they are re-measured.
GDN_NCU_TRAFFIC_BYTES = 445_946_368


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job rate: every rank does flops_per_rank per step; time is the slowest rank's."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def attended_flops(counts: np.ndarray, w) -> float:
    """4 d sum_{b,h,t} P * P |A(h,t)| (QK^T + PV, attended pairs only)."""
    return 4.0 * w.d * w.B * float(counts.sum()) * w.P * w.P


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import frame_sparse_attention_b200 as sfa
    sfa.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOAD
    if args.heads:
        from dataclasses import replace
        w = replace(w, H=args.heads, heads=w.heads[:1] * args.heads)
    kinds = [hs.kind for hs in w.heads]
    params = sfa.set_params(T_kv=w.Tkv, Tq=w.Tq, q_off=w.q_off, C=w.C, W=w.W, T_per=w.T_per,
                            step=STEP_S, n_sink=w.n_sink, n_prev=w.n_prev, chunk_len=w.chunk_len)
    Amax = sfa.set_max_count(params, kinds)

    q_h, k_h, v_h = workload_qkv(w, seed=rank)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    frames = torch.empty((w.H, w.Tq, Amax), dtype=torch.int32, device=dev)
    counts = torch.empty((w.H, w.Tq), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Lq), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # 256 MB > L2
    stream = torch.cuda.current_stream(dev)

    def step():
        sfa.build_sets(params, kinds, None, Amax, frames, counts, stream=stream)
        sfa.forward(q, k, v, frames, counts, w.P, out=out, lse=lse, dev_status=status, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise RuntimeError(f"device status {sfa.error_string(status.item())}")
    flops = attended_flops(counts.cpu().numpy(), w)

    # timed region: K steps, per-step events (the L2 flush between steps is outside them)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()
        e0, e1, e2 = ev[i]
        e0.record(stream)
        sfa.build_sets(params, kinds, None, Amax, frames, counts, stream=stream)
        e1.record(stream)
        sfa.forward(q, k, v, frames, counts, w.P, out=out, lse=lse, dev_status=status, stream=stream)
        e2.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [e0.elapsed_time(e2) for e0, _, e2 in ev]
    fwd_ms = [e1.elapsed_time(e2) for _, e1, e2 in ev]
    sets_ms = [e0.elapsed_time(e1) for e0, e1, _ in ev]
    if status.item() != 0:
        raise RuntimeError(f"device status {sfa.error_string(status.item())}")
    total_ms = max_over_ranks(float(sum(step_ms)), dev)

    if args.skip_extras:
        return None if rank != 0 else {
            "metric": METRIC, "value": round(job_rate_tflops(flops, world, total_ms / args.steps), 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4), "heads": w.H,
            "forward_ms": round(float(np.mean(fwd_ms)), 4), "note": "device step only (--skip-extras)"}

    # end to end through the C ABI with host buffers: H2D of Q, K, V from pinned memory,
    # sets + attention, D2H of O and LSE into pinned memory, every step (sfa_forward_host
    # pipelines the copies of one head group with the attention of another in the library)
    q_p, k_p, v_p = (x.pin_memory() for x in (q_h, k_h, v_h))
    o_p = torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory()
    lse_p = torch.empty((w.B, w.H, w.Lq), dtype=torch.float32).pin_memory()
    host_ws = torch.empty(sfa.host_workspace_bytes(q_p, k_p, w.P, Amax), dtype=torch.uint8, device=dev)

    def e2e_step():
        # sets on the device, then the host-to-host forward: per (batch, head-group) chunk,
        # the copy in, the attention and the copy out run on their own streams as a pipeline
        sfa.build_sets(params, kinds, None, Amax, frames, counts, stream=stream)
        sfa.forward_host(q_p, k_p, v_p, frames, counts, w.P, out_host=o_p, lse_host=lse_p, workspace=host_ws,
                         dev_status=status, stream=stream)

    e2e_step()
    torch.cuda.synchronize(dev)
    n_e2e = max(3, min(args.steps, 10))
    if world > 1:
        torch.distributed.barrier()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / n_e2e, dev)
    h2d = sum(x.numel() * x.element_size() for x in (q_h, k_h, v_h))
    d2h = o_p.numel() * o_p.element_size() + lse_p.numel() * lse_p.element_size()

    merge = bench_merge(sfa, dev, stream, flush) if rank == 0 else None
    workloads = None
    if rank == 0 and world == 1 and not args.no_workloads:
        workloads = bench_workloads(sfa, dev, stream, flush, with_cpu=not args.no_cpu_baseline)

    if rank != 0:
        return None
    peaks = measured_peaks()
    ms_per_step = total_ms / args.steps
    value = job_rate_tflops(flops, world, ms_per_step)  # whole job
    fwd_avg = float(np.mean(fwd_ms))
    achieved = flops / (fwd_avg * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    rec = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: Q, K, V ~ N(0,1) fp32 rounded to bf16, seeded per rank",
        "config": {"workload": WORKLOAD_DESC, "B": w.B, "H": w.H, "T": w.Tq, "P": w.P, "d": w.d,
                   "C": w.C, "W": w.W, "T_per": w.T_per, "step_s": STEP_S,
                   "attended_tflop_per_step": round(flops / 1e12, 4),
                   "parallelism": f"replica x{world} (independent batch per GPU)",
                   "l2": "flushed (256 MB write) between timed steps, outside the timed events"},
        "roofline": {"bound": "tensor", "kernel": "sfa_forward_kernel<128>",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "frac_of_sustained": round(achieved / float(peaks["bf16_tflops_sustained"]), 4),
                     "traffic": NCU_TRAFFIC_BYTES if w.H == 12 else None,
                     "traffic_note": "DRAM read+write bytes per launch, ncu capture of the 4-head case x 3",
                     "forward_ms": round(fwd_avg, 4), "set_build_ms": round(float(np.mean(sets_ms)), 4)},
        "e2e": {"value": round(job_rate_tflops(flops, world, e2e_ms), 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "sfa_build_sets + sfa_forward_host (C ABI, host buffers)"},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
        "merge": merge,
        "workloads": workloads,
    }
    if world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    return rec


def bench_merge(sfa, dev, stream, flush, reps=20, rows=None):
    """LSE merge of the ISPA dual-stream shape (1560 rows x 12 heads, d=128), or of `rows`
    rows of d=128 (a size large enough to show the kernel's own HBM rate)."""
    w = WORKLOADS["lsemerge_local"]
    ispa = rows is None
    rows = w.B * w.H * w.Lq if ispa else rows
    g = torch.Generator(dev).manual_seed(7)
    o1 = torch.randn(rows, w.d, generator=g, device=dev).to(torch.bfloat16)
    o2 = torch.randn(rows, w.d, generator=g, device=dev).to(torch.bfloat16)
    l1 = torch.randn(rows, generator=g, device=dev)
    l2 = torch.randn(rows, generator=g, device=dev)
    o = torch.empty_like(o1)
    lse = torch.empty_like(l1)
    for _ in range(3):
        sfa.lse_merge(o1, l1, o2, l2, out=o, lse=lse, stream=stream)
    times = []
    for _ in range(reps):
        flush.zero_()
        gpu_lead(stream)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sfa.lse_merge(o1, l1, o2, l2, out=o, lse=lse, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        times.append(a.elapsed_time(b))
    ms = float(np.median(times))
    nbytes = rows * (3 * 2 * w.d + 3 * 4)
    peaks = measured_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "lse_merge_kernel<128>", "rows": rows, "bytes": nbytes, "us": round(ms * 1e3, 2),
            "workload": "ISPA shape: 1560 rows x 12 heads, d=128" if ispa else f"{rows} rows, d=128",
            "achieved_gbs": round(gbs, 1), "peak_gbs": float(peaks["hbm_gbs"]), "bound": "hbm",
            "frac": round(gbs / float(peaks["hbm_gbs"]), 4),
            "note": "launch-latency bound at this size" if ispa else "inputs 1.6 GB, larger than L2"}


def bench_sets(sfa, dev, stream, flush, reps=20):
    """sfa_build_sets of the LVSA (41 and 121 frames) and streaming workloads: device time
    and bytes written (4 (Amax + 1) per (head, query frame)); launch-bound at these sizes."""
    out = {}
    for name in ("lvsa41", "long121", "stream"):
        w = WORKLOADS[name]
        kinds = [hs.kind for hs in w.heads]
        n_extra = max((len(hs.extra) for hs in w.heads), default=0)
        extra = None
        if n_extra:
            ex = torch.full((w.H, n_extra), -1, dtype=torch.int32)
            for h, hs in enumerate(w.heads):
                ex[h, :len(hs.extra)] = torch.tensor(hs.extra, dtype=torch.int32)
            extra = ex.to(dev)
        params = sfa.set_params(T_kv=w.Tkv, Tq=w.Tq, q_off=w.q_off, C=max(w.C, 1), W=max(w.W, 1), T_per=w.T_per,
                                step=0, n_sink=w.n_sink, n_prev=w.n_prev, chunk_len=w.chunk_len)
        Amax = sfa.set_max_count(params, kinds, n_extra)
        fr = torch.empty((w.H, w.Tq, Amax), dtype=torch.int32, device=dev)
        cn = torch.empty((w.H, w.Tq), dtype=torch.int32, device=dev)
        ms = time_device(lambda: sfa.build_sets(params, kinds, extra, Amax, fr, cn, stream=stream), flush, stream,
                         dev, reps, 3)
        nbytes = 4 * (Amax + 1) * w.H * w.Tq
        out[name] = {"us": round(ms * 1e3, 2), "bytes": nbytes, "achieved_gbs": round(nbytes / (ms * 1e-3) / 1e9, 2),
                     "bound": "launch latency"}
    return out


def block_list_flops(blocks: np.ndarray, counts: np.ndarray, P: int, d: int) -> float:
    """4*d * sum over query blocks of (query rows) x (tokens of the listed key blocks)."""
    nb = (P + 127) // 128
    size = np.array([min(b * 128 + 128, P) - b * 128 for b in range(nb)], dtype=np.int64)
    rows = np.array([min(256, P - 256 * i) for i in range((P + 255) // 256)], dtype=np.int64)
    keys = np.zeros(counts.shape, dtype=np.int64)
    for idx in np.ndindex(counts.shape):
        ids = blocks[idx][:counts[idx]]
        keys[idx] = int(size[ids % nb].sum())
    return 4.0 * d * float((keys * rows).sum())


def bench_hsa(sfa, dev, stream, flush, reps=20):
    """Light Forcing HSA on the hsa workload: selection, then attention over the lists."""
    w = WORKLOADS["hsa"]
    q_h, k_h, v_h = workload_qkv(w, seed=0)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    params = sfa.set_params(T_kv=w.Tkv, Tq=w.Tq, q_off=w.q_off, n_sink=w.n_sink, n_prev=w.n_prev,
                            chunk_len=w.chunk_len)
    blocks, counts = sfa.hsa_select(q, k, params, w.k_frames, w.k_blocks, stream=stream)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Lq), dtype=torch.float32, device=dev)
    desc = sfa.attn_desc(q, k, k, q, w.P, blocks.shape[-1])
    import ctypes
    nbytes = ctypes.c_size_t(0)
    sfa.load().sfa_hsa_workspace(ctypes.byref(desc), ctypes.byref(nbytes))
    wsp = torch.empty(max(nbytes.value, 1), dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            gpu_lead(stream)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    sel_ms = timed(lambda: sfa.hsa_select(q, k, params, w.k_frames, w.k_blocks, workspace=wsp, stream=stream))
    # steady state of an autoregressive cache: the history keys' means pooled once, then
    # every call pools the queries and selects (sfa_hsa_select_pooled)
    sfa.hsa_pool_keys(k, q, w.P, wsp, blocks.shape[-1], stream=stream)
    selp_ms = timed(lambda: sfa.hsa_select_pooled(q, k, params, w.k_frames, w.k_blocks, wsp, Amax=blocks.shape[-1],
                                                  stream=stream))
    fwd_ms = timed(lambda: sfa.forward_blocks(q, k, v, blocks, counts, w.P, out=o, lse=lse, stream=stream))
    # 252 CTAs are 1.7 waves of 148 SMs: the split form balances them
    split_ws = torch.empty(max(sfa.split_workspace_bytes(desc, 2), 1), dtype=torch.uint8, device=dev)
    fwd2_ms = timed(lambda: sfa.forward_blocks(q, k, v, blocks, counts, w.P, out=o, lse=lse, stream=stream,
                                               n_split=2, workspace=split_ws))
    nb0 = ctypes.c_size_t(0)
    sfa.load().sfa_forward_blocks_split_workspace(ctypes.byref(desc), 0, ctypes.byref(nb0))
    sched_ws = torch.empty(max(nb0.value, 1), dtype=torch.uint8, device=dev)
    fwd0_ms = timed(lambda: sfa.forward_blocks(q, k, v, blocks, counts, w.P, out=o, lse=lse, stream=stream,
                                               n_split=0, workspace=sched_ws))
    flops = block_list_flops(blocks.cpu().numpy(), counts.cpu().numpy(), w.P, w.d)
    peak = float(measured_peaks()["bf16_tflops"])
    tf = flops / (fwd_ms * 1e-3) / 1e12
    pool_bytes = (k.numel() + q.numel()) * 2
    hbm = float(measured_peaks()["hbm_gbs"])
    # the oracle on a bounded sample: one query block per (head, frame), its selection and
    # its rows' attention (float64 numpy), about a few seconds of host work
    import time
    from oracle import hsa as ohsa
    qf, kf_, vf = q_h.float().numpy(), k_h.float().numpy(), v_h.float().numpy()
    t0 = time.perf_counter()
    kw = dict(P=w.P, T_kv=w.Tkv, q_off=w.q_off, chunk_len=w.chunk_len, n_prev=w.n_prev, n_sink=w.n_sink,
              k_frames=w.k_frames, k_blocks=w.k_blocks)
    o_lists, o_counts = ohsa.build_block_lists(qf, kf_, Bmax=blocks.shape[-1], **kw)
    rows = np.asarray([(h * w.Lq) + t * w.P + r for h in range(w.H) for t in range(w.Tq) for r in range(0, 256, 8)])
    ohsa.attention_blocks(qf, kf_, vf, o_lists, o_counts, w.P, 1 / math.sqrt(w.d), rows=rows)
    dt = time.perf_counter() - t0
    keys_per_row = float(np.mean([o_counts[0, h, t, 0] for h in range(w.H) for t in range(w.Tq)])) * 128
    return {"workload": "hsa: 3 query frames after 21 history frames, P=1560, H=12, d=128; sink 1 + "
                        "local 6 frames always, 24 blocks of the 4 best history frames per 256-row query block",
            "select_ms": round(sel_ms, 4), "select_pool_bytes": pool_bytes,
            "select_pooled_keys_ms": round(selp_ms, 4),
            "select_share_of_attention": round(sel_ms / fwd_ms, 4),
            "select_pooled_keys_share_of_attention": round(selp_ms / fwd_ms, 4),
            "forward_blocks_ms": round(fwd_ms, 4), "attended_tflop": round(flops / 1e12, 4),
            "forward_tflops": round(tf, 1), "forward_frac": round(tf / peak, 4),
            "forward_blocks_split2_ms": round(fwd2_ms, 4),
            "forward_blocks_scheduled_ms": round(fwd0_ms, 4),
            "forward_scheduled_tflops": round(flops / (fwd0_ms * 1e-3) / 1e12, 1),
            "forward_split2_tflops": round(flops / (fwd2_ms * 1e-3) / 1e12, 1),
            "step_tflops": round(flops / ((sel_ms + fwd_ms) * 1e-3) / 1e12, 1),
            "mean_blocks_per_list": round(float(counts.float().mean().item()), 2),
            "roofline": {"forward_blocks": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak,
                                            "unit": "TFLOP/s", "frac": round(tf / peak, 4)},
                         "select": {"bound": "hbm", "achieved": round(pool_bytes / (sel_ms * 1e-3) / 1e9, 1),
                                    "peak": hbm, "unit": "GB/s",
                                    "frac": round(pool_bytes / (sel_ms * 1e-3) / 1e9 / hbm, 4),
                                    "note": "bytes = K and Q read once by the pooling"}},
            "cpu_baseline": {"value": round(4.0 * w.d * keys_per_row * len(rows) / dt / 1e12, 8), "unit": "TFLOP/s",
                             "cores": os.cpu_count() or 1, "kind": "oracle",
                             "sample": f"selection of every list + attention of {len(rows)} query rows "
                                       f"(float64 numpy, {dt:.1f} s; value counts the attention rows only)"}}


def bench_gdn(sfa, dev, stream, flush, reps=20):
    """ARL2 inter-frame branch on the gdn workload (24 frames, 12 heads, P=1560, d=128)."""
    from sfa_workloads import gdn_inputs
    w = WORKLOADS["gdn"]
    q, k, v, a, b = (x.to(dev) for x in gdn_inputs(w.B, w.H, w.Tq, w.P, w.d, seed=0))
    o = torch.empty_like(q)
    s = torch.empty((w.B, w.H, w.d, w.d), dtype=torch.float32, device=dev)
    desc = sfa.GdnDesc()
    desc.B, desc.H, desc.T, desc.P, desc.d = w.B, w.H, w.Tq, w.P, w.d
    nbytes = ctypes.c_size_t(0)
    sfa.load().sfa_gdn_workspace(ctypes.byref(desc), ctypes.byref(nbytes))
    ws = torch.empty(nbytes.value, dtype=torch.uint8, device=dev)

    def run():
        sfa.gdn_forward(q, k, v, a, b, w.P, out=o, state_out=s, workspace=ws, stream=stream)

    for _ in range(3):
        run()
    ts = []
    for _ in range(reps):
        flush.zero_()
        gpu_lead(stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1))
    ms = float(np.median(ts))
    flop = 3 * 2.0 * w.P * w.d * w.d * w.Tq * w.H * w.B
    peak = float(measured_peaks()["bf16_tflops"])
    # the oracle on a bounded sample: one head, all 24 frames (float64 numpy)
    import time
    from oracle import gdn as ogdn
    qh, kh, vh, ah, bh = gdn_inputs(w.B, w.H, w.Tq, w.P, w.d, seed=0)
    t0 = time.perf_counter()
    ogdn.gdn_frames(qh[:, :1].float().numpy(), kh[:, :1].float().numpy(), vh[:, :1].float().numpy(),
                    ah[:, :1].numpy(), bh[:, :1].numpy(), w.P)
    dt = time.perf_counter() - t0
    hbm = float(measured_peaks()["hbm_gbs"])
    # compulsory bytes: Q', K', V' read and O written (bf16), beta and alpha read, the state written
    nbytes = 4 * w.B * w.H * w.Tq * w.P * w.d * 2 + w.B * w.H * w.Tq * (w.P + 1) * 4 + w.B * w.H * w.d * w.d * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    tf = flop / (ms * 1e-3) / 1e12
    return {"workload": "gdn: ARL2 inter-frame gated delta rule, 24 frames x 1560 tokens, H=12, d=128",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "bytes": nbytes,
                         "traffic": GDN_NCU_TRAFFIC_BYTES,
                         "traffic_note": "DRAM read+write bytes of the call's two kernels, ncu capture",
                         "tensor": {"achieved": round(tf, 2), "peak": peak, "unit": "TFLOP/s",
                                    "frac": round(tf / peak, 4)}},
            "cpu_baseline": {"value": round(flop / w.H / dt / 1e12, 8), "unit": "TFLOP/s",
                             "cores": os.cpu_count() or 1, "kind": "oracle",
                             "sample": f"one head of the workload, all 24 frames (float64 numpy, {dt:.2f} s)"},
            "ms": round(ms, 4), "gflop": round(flop / 1e9, 3), "tflops": round(tf, 2),
            "frac": round(tf / peak, 4),
            "note": "M_N = K^T diag(beta) K and B_N = K^T diag(beta) V of every frame at once, then the "
                    "recurrence and O = Q S_{N-1} in several CTAs per head (sfa_gdn_forward: two kernels)"}


# ----------------------------------------------------------------------------- oracle timing
def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(seconds: float = 15.0, inputs=None):
    """Time the float64 oracle on host cores for about `seconds` on sampled query rows."""
    import oracle
    from oracle import sets as S
    from sfa_workloads import sample_rows
    w = WORKLOAD
    q, k, v = inputs if inputs is not None else workload_qkv(w, seed=0)
    frames, counts = S.workload_sets(w, step=STEP_S)
    cores = os.cpu_count() or 1
    scale = 1.0 / math.sqrt(w.d)

    def run(n_per_head, seed):
        rows = sample_rows(w, n_per_head, seed=seed)
        t0 = time.perf_counter()
        oracle.attention(q, k, v, frames, counts, w.P, scale, rows=rows, n_threads=cores)
        dt = time.perf_counter() - t0
        h = (rows // w.Lq) % w.H
        t = (rows % w.Lq) // w.P
        fl = 4.0 * w.d * w.P * counts[h, t].astype(np.float64).sum()
        return rows.size, fl, dt

    n, fl, dt = run(max(1, cores // w.H + 1), seed=100)    # calibration
    per_row = dt / max(n, 1)
    n_per_head = max(1, int(seconds / per_row / w.H))
    n, fl, dt = run(n_per_head, seed=101)
    call_flop = 4.0 * w.d * w.P * w.P * w.B * counts.astype(np.float64).sum()
    return {"value": round(fl / dt / 1e12, 8), "unit": "TFLOP/s", "cores": cores, "cpu_model": cpu_model(),
            "kind": "oracle", "sample": f"{n} sampled query rows of the LVSA workload (float64 C oracle, "
                                        f"{cores} threads, {dt:.1f} s)", "seconds": round(dt, 2),
            "rows_per_s": round(n / dt, 1),
            "extrapolated_ms_per_call": round(call_flop / (fl / dt) * 1e3, 1)}


def run_reference(args, rank):
    """Reference arm: the oracle on host cores, a bounded sample of rows per step."""
    if rank != 0:
        return None
    import oracle
    from oracle import sets as S
    from sfa_workloads import sample_rows
    w = WORKLOAD
    q, k, v = workload_qkv(w, seed=0)
    frames, counts = S.workload_sets(w, step=STEP_S)
    cores = os.cpu_count() or 1
    scale = 1.0 / math.sqrt(w.d)
    # rows per step sized so that warmup + steps end within a few minutes
    probe = sample_rows(w, max(1, cores // w.H + 1), seed=999)
    t0 = time.perf_counter()
    oracle.attention(q, k, v, frames, counts, w.P, scale, rows=probe, n_threads=cores)
    per_row = (time.perf_counter() - t0) / probe.size
    budget_s = args.reference_seconds / max(1, args.steps + args.warmup)
    n_per_head = max(1, int(budget_s / per_row / w.H))
    step_times, step_flops = [], []
    for i in range(args.warmup + args.steps):
        rows = sample_rows(w, n_per_head, seed=i)
        h = (rows // w.Lq) % w.H
        t = (rows % w.Lq) // w.P
        fl = 4.0 * w.d * w.P * counts[h, t].astype(np.float64).sum()
        t0 = time.perf_counter()
        oracle.attention(q, k, v, frames, counts, w.P, scale, rows=rows, n_threads=cores)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            step_times.append(dt)
            step_flops.append(fl)
    total = sum(step_times)
    value = sum(step_flops) / total / 1e12
    sample = (f"{rows.size} sampled query rows per step of the LVSA workload, float64 C oracle "
              f"on {cores} host threads")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 8), "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "B": w.B, "H": w.H, "T": w.Tq, "P": w.P, "d": w.d,
                   "C": w.C, "W": w.W, "T_per": w.T_per, "step_s": STEP_S},
        "cpu_baseline": {"value": round(value, 8), "unit": "TFLOP/s", "cores": cores, "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 8), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def setup_workload(sfa, dev, stream, name, split=1, dual=False):
    """Device buffers and one step (set build + forward per branch; the LSE-decomposed
    workload adds the merge of its local and history branches) of another workload.
    Returns (step, flops, branches) with flops counted after one step has run."""
    names = {"long121": ["long121"], "stream": ["stream"], "tiny_dense": ["tiny_dense"],
             "tiny_sinkwin": ["tiny_sinkwin"], "lsemerge": ["lsemerge_local", "lsemerge_hist"]}[name]
    ws = [WORKLOADS[n] for n in names]
    q_h, k_h, v_h = workload_qkv(ws[0], seed=0)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    branches = []
    for w in ws:
        kinds = [hs.kind for hs in w.heads]
        n_extra = max((len(hs.extra) for hs in w.heads), default=0)
        extra = None
        if n_extra:
            ex = torch.full((w.H, n_extra), -1, dtype=torch.int32)
            for h, hs in enumerate(w.heads):
                ex[h, :len(hs.extra)] = torch.tensor(hs.extra, dtype=torch.int32)
            extra = ex.to(dev)
        params = sfa.set_params(T_kv=w.Tkv, Tq=w.Tq, q_off=w.q_off, C=max(w.C, 1), W=max(w.W, 1),
                                T_per=w.T_per, step=0, n_sink=w.n_sink, n_prev=w.n_prev,
                                chunk_len=w.chunk_len)
        Amax = max(1, sfa.set_max_count(params, kinds, n_extra))
        fr = torch.empty((w.H, w.Tq, Amax), dtype=torch.int32, device=dev)
        cn = torch.empty((w.H, w.Tq), dtype=torch.int32, device=dev)
        o_b = torch.empty_like(q)
        desc = sfa.attn_desc(q, k, v, o_b, w.P, Amax)
        ws_bytes = sfa.split_workspace_bytes(desc, split)
        wsp = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
        branches.append([w, params, kinds, extra, Amax, fr, cn, o_b,
                         torch.empty((w.B, w.H, w.Lq), dtype=torch.float32, device=dev), wsp])
    merged = (torch.empty_like(q), torch.empty((ws[0].B, ws[0].H, ws[0].Lq), dtype=torch.float32, device=dev))
    dual = dual and len(branches) == 2
    dual_ws = None
    if dual:  # both branches in one launch, local result + their merge (sfa_forward_dual)
        Amax = max(b[4] for b in branches)
        for b in branches:
            b[4] = Amax
            b[5] = torch.empty((b[0].H, b[0].Tq, Amax), dtype=torch.int32, device=dev)
        nbytes = ctypes.c_size_t(0)
        ddesc = sfa.attn_desc(q, k, v, merged[0], branches[0][0].P, Amax)
        if sfa.load().sfa_forward_dual_workspace(ctypes.byref(ddesc), split, ctypes.byref(nbytes)) != 0:
            raise SystemExit("dual launch: bad split for this head dimension")
        dual_ws = torch.empty(max(1, nbytes.value), dtype=torch.uint8, device=dev)

    def step():
        if dual:
            (w0, p0, k0, e0, A0, f0, c0, o0, l0, _), (w1, p1, k1, e1, A1, f1, c1, o1, l1, _) = branches
            sfa.build_sets(p0, k0, e0, A0, f0, c0, stream=stream)
            sfa.build_sets(p1, k1, e1, A1, f1, c1, stream=stream)
            sfa.forward_dual(q, k, v, f0, c0, f1, c1, w0.P, split, out_local=o0, lse_local=l0,
                             out_full=merged[0], lse_full=merged[1], workspace=dual_ws, stream=stream)
            return
        for (w, params, kinds, extra, Amax, fr, cn, o, lse, wsp) in branches:
            sfa.build_sets(params, kinds, extra, Amax, fr, cn, stream=stream)
            if split != 1:  # 0: scheduled (the library's ranges, longest first)
                sfa.forward_split(q, k, v, fr, cn, w.P, split, out=o, lse=lse, workspace=wsp, stream=stream)
            else:
                sfa.forward(q, k, v, fr, cn, w.P, out=o, lse=lse, stream=stream)
        if len(branches) == 2:
            sfa.lse_merge(branches[0][7], branches[0][8], branches[1][7], branches[1][8],
                          out=merged[0], lse=merged[1], stream=stream)

    step()
    torch.cuda.synchronize(dev)
    flops = sum(attended_flops(b[6].cpu().numpy(), b[0]) for b in branches)
    return step, flops, branches


def gpu_lead(stream):
    """Keep the GPU busy for about 50 us (a spin of 10^5 cycles) right before a start
    event: the host then enqueues the timed launches before the GPU reaches the event, so
    that the events bracket device work only, not the host's launch overhead (which the
    e2e figure includes).  Matters for calls of a few microseconds."""
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is not None:  # without it, the events may also time some host launch overhead
        with torch.cuda.stream(stream):
            sleep(100_000)


def time_device(step, flush, stream, dev, steps=20, warmup=5):
    """Median device time (ms) of `step` over `steps` runs after `warmup`, L2 flushed
    before every run (outside the events)."""
    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(steps):
        flush.zero_()
        gpu_lead(stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        times.append(e0.elapsed_time(e1))
    return float(np.median(times))


def run_other_workload(args):
    """Device time of one step of another workload (one JSON line, not the bench line)."""
    import frame_sparse_attention_b200 as sfa
    sfa.load()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    step, flops, branches = setup_workload(sfa, dev, stream, args.workload, args.split, getattr(args, "dual", False))
    ms = time_device(step, flush, stream, dev, args.steps, args.warmup)
    return {"workload": args.workload, "branches": [b[0].name for b in branches], "split": args.split,
            "dual_launch": bool(getattr(args, "dual", False)), "attended_tflop_per_step": round(flops / 1e12, 4),
            "ms_per_step": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
            "steps": args.steps, "warmup": args.warmup, "note": "device time, median, L2 flushed between steps"}


def oracle_full(name, rows_per_head=None, seed=0):
    """The float64 oracle on host cores over every query row of a workload (or over
    rows_per_head sampled rows per head): (seconds, flops done, rows, extra info).
    The LSE-decomposed workload runs both branches and their merge."""
    import oracle
    from oracle import merge as M
    from oracle import sets as S
    from sfa_workloads import sample_rows
    names = {"lsemerge": ["lsemerge_local", "lsemerge_hist"]}.get(name, [name])
    ws = [WORKLOADS[n] for n in names]
    q, k, v = workload_qkv(ws[0], seed=seed)
    cores = os.cpu_count() or 1
    rows = None
    if rows_per_head:
        rows = sample_rows(ws[0], rows_per_head, seed=1)
    t0 = time.perf_counter()
    outs, fl = [], 0.0
    for w in ws:
        frames, counts = S.workload_sets(w, step=0)
        outs.append(oracle.attention(q, k, v, frames, counts, w.P, 1.0 / math.sqrt(w.d), rows=rows, n_threads=cores))
        if rows is None:
            fl += attended_flops(counts, w)
        else:
            h = (rows // w.Lq) % w.H
            t = (rows % w.Lq) // w.P
            fl += 4.0 * w.d * w.P * counts[h, t].astype(np.float64).sum()
    if len(outs) == 2:
        M.lse_merge(outs[0][0], outs[0][1], outs[1][0], outs[1][1])
    dt = time.perf_counter() - t0
    n_rows = ws[0].B * ws[0].H * ws[0].Lq if rows is None else rows.size
    return dt, fl, n_rows, cores


def _cpu_record(name, sample, rows_per_head=None):
    dt, fl, n_rows, cores = oracle_full(name, rows_per_head)
    return {"value": round(fl / dt / 1e12, 8), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": sample.format(rows=n_rows, s=dt), "seconds": round(dt, 2)}


def bench_workloads(sfa, dev, stream, flush, steps=20, warmup=5, with_cpu=True):
    """Every other workload's device time, roofline and oracle baseline (rank 0, N = 1)."""
    peaks = measured_peaks()
    peak = float(peaks["bf16_tflops"])
    out = {}

    def entry(name, variants, workload_desc):
        rec = {"workload": workload_desc, "launches": {}}
        best = None
        for label, split, dual in variants:
            step, flops, _ = setup_workload(sfa, dev, stream, name, split, dual)
            ms = time_device(step, flush, stream, dev, steps, warmup)
            tf = flops / (ms * 1e-3) / 1e12
            rec["launches"][label] = {"ms_per_call": round(ms, 4), "tflops": round(tf, 1),
                                      "frac": round(tf / peak, 4)}
            rec["attended_tflop_per_call"] = round(flops / 1e12, 4)
            if best is None or ms < best[1]:
                best = (label, ms, tf)
        rec["ms_per_call"] = round(best[1], 4)
        rec["tflops"] = round(best[2], 1)
        rec["best_launch"] = best[0]
        rec["roofline"] = {"bound": "tensor", "achieved": round(best[2], 1), "peak": peak, "unit": "TFLOP/s",
                           "frac": round(best[2] / peak, 4), "peak_source": f"{peaks['source']} bf16_tflops (burst)"}
        return rec

    out["tiny"] = {"workload": "tiny: T=4, P=64, H=2, d=64; dense and sink+window {0, t-1, t}",
                   "launches": {}}
    for nm in ("tiny_dense", "tiny_sinkwin"):
        step, flops, _ = setup_workload(sfa, dev, stream, nm)
        ms = time_device(step, flush, stream, dev, steps, warmup)
        out["tiny"]["launches"][nm] = {"ms_per_call": round(ms, 4), "attended_gflop": round(flops / 1e9, 5),
                                       "note": "launch-latency bound (correctness case)"}
    out["stream"] = entry("stream", [("sfa_forward", 1, False), ("sfa_forward_split n_split=2", 2, False),
                                     ("sfa_forward_split n_split=4", 4, False),
                                     ("sfa_forward_split scheduled (n_split=0)", 0, False)],
                          "stream: 3 query frames x 1560 after 21 history frames, H=12, d=128; heads 4 local (6 "
                          "frames), 4 anchor (7), 4 memory (13)")
    out["long121"] = entry("long121", [("sfa_forward", 1, False), ("sfa_forward_split scheduled (n_split=0)", 0, False)],
                           "long121: T=121, P=1560, H=12, d=128, LVSA C=21, W=13, T_per=6, s=0 (|A| = 30-32)")
    out["lsemerge"] = entry("lsemerge", [("local + history + merge (3 calls)", 1, False),
                                         ("3 calls, n_split=2", 2, False), ("3 calls, n_split=4", 4, False),
                                         ("3 calls, scheduled (n_split=0)", 0, False),
                                         ("sfa_forward_dual n_split=1", 1, True),
                                         ("sfa_forward_dual n_split=2", 2, True),
                                         ("sfa_forward_dual scheduled (n_split=0)", 0, True)],
                            "lsemerge: query frame 13 (1560 rows), H=12, d=128; local {0, 13} + history {1..12}, "
                            "LSE-merged")
    if with_cpu:
        out["tiny"]["cpu_baseline"] = _cpu_record("tiny_dense", "every row of tiny_dense ({rows} rows, float64 C "
                                                                "oracle, {s:.2f} s)")
        out["stream"]["cpu_baseline"] = _cpu_record("stream", "every row of the workload ({rows} rows, float64 C "
                                                              "oracle, {s:.1f} s)")
        out["lsemerge"]["cpu_baseline"] = _cpu_record("lsemerge", "every row of both branches and their merge "
                                                                  "({rows} rows, float64, {s:.1f} s)")
        out["long121"]["cpu_baseline"] = _cpu_record("long121", "the checked rows: 256 seeded rows per head "
                                                                "({rows} rows, float64 C oracle, {s:.1f} s)",
                                                     rows_per_head=256)
    out["merge_2M"] = bench_merge(sfa, dev, stream, flush, rows=2 * 1024 * 1024)
    out["hsa"] = bench_hsa(sfa, dev, stream, flush, reps=steps)
    out["gdn"] = bench_gdn(sfa, dev, stream, flush, reps=steps)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="oracle time of the reference arm's warm-up and timed steps together")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads instead of 12 (smaller profiling case)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="leave out the other workloads (stream, long121, lsemerge, tiny, hsa, gdn, large merge)")
    ap.add_argument("--skip-extras", action="store_true",
                    help="time the device step only: no end-to-end, merge or CPU-baseline legs")
    ap.add_argument("--workload", choices=["lvsa41", "long121", "stream", "lsemerge", "hsa", "gdn", "merge",
                                           "tiny_dense", "tiny_sinkwin"],
                    default="lvsa41",
                    help="other workloads are timed on the device only (one JSON line, not the bench line)")
    ap.add_argument("--dual", action="store_true",
                    help="--workload lsemerge: both branches in one launch (sfa_forward_dual)")
    ap.add_argument("--split", type=int, default=1,
                    help="split-KV ranges per unit for --workload other than lvsa41 (sfa_forward_split)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.workload != "lvsa41":
        if rank == 0:
            if args.workload in ("hsa", "gdn", "merge"):
                import frame_sparse_attention_b200 as sfa
                sfa.load()
                dev = torch.device("cuda", 0)
                flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
                st = torch.cuda.current_stream(dev)
                if args.workload == "merge":  # the ISPA shape, 2M rows, and the set builds
                    rec = {"merge": bench_merge(sfa, dev, st, flush, reps=args.steps),
                           "merge_2M": bench_merge(sfa, dev, st, flush, reps=args.steps, rows=2 * 1024 * 1024),
                           "sets": bench_sets(sfa, dev, st, flush, reps=args.steps)}
                else:
                    fn = bench_hsa if args.workload == "hsa" else bench_gdn
                    rec = fn(sfa, dev, st, flush, reps=args.steps)
            else:
                rec = run_other_workload(args)
            print(json.dumps(rec), flush=True)
        return

    if args.impl == "reference":
        rec = run_reference(args, rank)
        if rec is not None:
            print(json.dumps(rec), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        rec = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rec is not None:
        print(json.dumps(rec), flush=True)


if __name__ == "__main__":
    main()
