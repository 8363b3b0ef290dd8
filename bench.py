"""Benchmark: causal attention fwd+bwd TFLOP/s at 32 heads x 128, bf16, on B200.

    python bench.py [--gpus N --steps K --warmup W] [--workload long_128k]
    python bench.py --impl reference ...     (the float64 CPU oracle, timed)

One step = lwm_attn_fwd + lwm_attn_bwd over one batch of the workload (all of
the hot path: segment prepass, RoPE, forward, dot(dO, O), backward).  The
default workload is 128K tokens, one segment, theta 1e7, B1 H32 D128 bf16.
Work is counted algorithmically: forward 4*D*H*Pi flops, backward 2.5x that,
Pi = allowed (i, j) pairs (causal within segments; skipped tiles and masked
elements are not counted).

With --gpus N > 1 the bench launches N ranks itself (torch.distributed.run,
one process per GPU) unless it already runs under torchrun with WORLD_SIZE =
N.  Default --parallel heads: the heads of one problem are split over the
ranks (the pages' tensor-parallel axis; each rank runs the single-GPU
kernels on H/N heads, no collective on the data path), strong scaling.
--parallel replicas: each rank runs an independent problem of the same size
(different seed), weak scaling.  Timing is on the device (CUDA events) with a
barrier and a synchronize on both sides; rank 0 prints one JSON line with
the max time over ranks and the whole job's throughput.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, segment_ids  # noqa: E402

METRIC = "causal attn fwd+bwd TFLOP/s (32x128 heads, bf16) and % of B200 BF16 peak"
LOSS_METRIC = "packed re-weighted cross-entropy HBM GB/s (bf16 logits and gradient)"
DECODE_METRIC = "decode attention HBM GB/s (new tokens against a rotated KV cache, 32x128 heads, bf16)"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
L2_BYTES = 126 * 2 ** 20

# DRAM traffic of one attn_bwd_dkdv_kernel launch (dram__bytes_read.sum +
# dram__bytes_write.sum, one-pass ncu capture of the full-size workload, see
# profiles/attn_bwd_dkdv_traffic_long_128k.md); valid only for the kernel
# source it was taken on (sha256 of the kernel file and the device headers).
DKDV_TRAFFIC = {"bytes": {"long_128k": 6.24e9 + 2.12e9},
                "source_sha256": "88f50d7a60fb86e4bcb66285ffc1fdbb9b8dc0be947c6e46ceac951a3c116497"}


def kept_pairs(seg: np.ndarray, causal: bool = True) -> int:
    total = 0
    for row in seg:
        _, counts = np.unique(row[row >= 0], return_counts=True)
        c = counts.astype(np.int64)
        total += int((c * (c + 1) // 2).sum()) if causal else int((c * c).sum())
    return total


# The same for the one-pass backward kernel (attn_bwd_fused_kernel), from a
# one-pass capture of the full-size 128K launch (profiles/
# attn_bwd_fused_traffic_long_128k.md).
FUSED_TRAFFIC = {"bytes": {"long_128k": 14.88e9 + 8.94e9},
                 "source_sha256": "ee25513c06328c0c673b4628fb38bd0933778954cefc51950b25ab4bafbe1d33"}


def split_backward() -> bool:
    """The library runs the two-kernel backward (LWM_ATTN_SPLIT_BWD=1)."""
    return os.environ.get("LWM_ATTN_SPLIT_BWD") == "1"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws an independent problem of the same shape."""
    return seed + rank


def max_over_ranks(values, ws: int, device):
    """Element-wise max of a list of floats over all ranks (identity at ws=1)."""
    if ws == 1:
        return [float(x) for x in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(flops_per_rank_step: float, ws: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return flops_per_rank_step * ws / (ms_per_step * 1e-3) / 1e12


def tile_pairs(seg: np.ndarray, heads: int, causal: bool = True, tile: int = 128) -> int:
    """(query tile, key tile) pairs that share a segment id range, over all
    rows and heads: the units the dK/dV kernel streams."""
    total = 0
    for row in seg:
        n = (len(row) + tile - 1) // tile
        lo = np.full(n, np.iinfo(np.int64).max)
        hi = np.full(n, np.iinfo(np.int64).min)
        for t in range(n):
            r = row[t * tile:(t + 1) * tile]
            r = r[r >= 0]
            if len(r):
                lo[t], hi[t] = r.min(), r.max()
        valid = hi >= lo
        for qt in np.nonzero(valid)[0]:
            kt = slice(0, qt + 1) if causal else slice(0, n)
            total += int(np.count_nonzero(valid[kt] & (lo[kt] <= hi[qt]) & (hi[kt] >= lo[qt])))
    return total * heads


def kernel_source_sha256(name: str) -> str:
    import hashlib
    d = os.path.join(ROOT, "long_context_causal_attention_b200", "csrc")
    h = hashlib.sha256()
    for f in (name, "sm100.cuh", "common.cuh"):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def time_oracle_sample(w, seg, rows: int, seed: int):
    """Oracle fwd+bwd on the last `rows` query rows of head 0 of batch row 0.

    Returns (seconds, algorithmic flops of the sample, threads used)."""
    import torch
    import oracle
    from workloads import make_tensors
    small = w.with_(batch=1, heads=1)
    t = make_tensors(small, seed=seed, device="cpu", with_grad_out=True)
    f = lambda x: x.double().numpy()
    rows = min(rows, w.seqlen)
    r0 = w.seqlen - rows
    t0 = time.perf_counter()
    oracle.attention_backward(f(t["q"]), f(t["k"]), f(t["v"]), f(t["do"]), seg[:1],
                              causal=w.causal, theta=w.theta, row_start=r0)
    dt = time.perf_counter() - t0
    row = seg[0]
    pairs = 0
    for i in range(r0, w.seqlen):
        if row[i] >= 0:
            keys = row[: i + 1] if w.causal else row
            pairs += int(np.count_nonzero(keys == row[i]))
    flops = 3.5 * 4.0 * w.head_dim * pairs
    try:
        from threadpoolctl import threadpool_info
        threads = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    except Exception:
        threads = len(os.sched_getaffinity(0))
    return dt, flops, threads


def reference_arm(args):
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    seg = segment_ids(w, seed=args.seed)
    rows = min(args.oracle_rows, w.seqlen)
    for _ in range(args.warmup):
        time_oracle_sample(w, seg, rows, args.seed)
    times, flops, threads = [], 0.0, 1
    for _ in range(args.steps):
        dt, flops, threads = time_oracle_sample(w, seg, rows, args.seed)
        times.append(dt)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = (f"float64 numpy oracle, fwd+bwd of the last {rows} query rows of one head "
              f"(b=0, h=0) of {w.name}; {flops / 1e9:.2f} GFLOP algorithmic per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen, "heads": w.heads,
                   "head_dim": w.head_dim, "theta": w.theta},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def ours(args):
    import torch
    import torch.distributed as dist

    import long_context_causal_attention_b200 as lwm
    from workloads import make_tensors

    ws, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if ws > 1:
            dist.barrier()

    w = WORKLOADS[args.workload]
    heads_split = ws > 1 and args.parallel == "heads"
    # head split: every rank draws the same whole problem and keeps its heads
    # (the scatter); replicas: each rank draws its own problem
    seed = args.seed if heads_split else rank_seed(args.seed, rank)
    seg = segment_ids(w, seed=seed)
    single = w.segments == "single"
    seg_d = None if single else torch.as_tensor(seg, dtype=torch.int32, device=dev)
    t = make_tensors(w, seed=seed, device=dev, with_grad_out=True)
    if heads_split:
        from long_context_causal_attention_b200.heads import scatter_heads
        t = {name: scatter_heads(x, rank, ws) for name, x in t.items()}
        torch.cuda.empty_cache()
        w = w.with_(heads=w.heads // ws)
    q, k, v, do = t["q"], t["k"], t["v"], t["do"]
    desc = lwm.make_desc(q, seg_d, w.causal, w.theta, w.scale)
    ws_f = lwm.alloc_workspace(desc, False, dev)
    ws_b = lwm.alloc_workspace(desc, True, dev)
    o = torch.empty_like(q)
    lse = torch.empty(w.batch, w.heads, w.seqlen, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def step():
        lwm.lwm_attn_fwd(q, k, v, seg_d, w.causal, w.theta, w.scale, o=o, lse=lse,
                         workspace=ws_f, stream=stream)
        lwm.lwm_attn_bwd(q, k, v, o, lse, do, seg_d, w.causal, w.theta, w.scale, dq=dq, dk=dk,
                         dv=dv, workspace=ws_b, stream=stream)

    pairs = kept_pairs(seg, w.causal)
    fwd_flops = 4.0 * w.head_dim * w.heads * pairs
    step_flops = 3.5 * fwd_flops

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # per-step events around the main kernels (recorded by the library)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    for evs in kev:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    launches0 = lwm.lwm_attn_kernel_launches()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for s in range(args.steps):
        lwm.lwm_attn_set_timing_events(*kev[s])
        step()
    stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    lwm.lwm_attn_set_timing_events()
    launches = lwm.lwm_attn_kernel_launches() - launches0
    clk = clocks.stop()
    ms = start.elapsed_time(stop)
    fwd_k = sum(e[0].elapsed_time(e[1]) for e in kev) / args.steps
    bwd_k = sum(e[2].elapsed_time(e[3]) for e in kev) / args.steps
    dkdv_k = sum(e[2].elapsed_time(e[4]) for e in kev) / args.steps
    ms, fwd_k, bwd_k, dkdv_k = max_over_ranks([ms, fwd_k, bwd_k, dkdv_k], ws, dev)
    ms_step = ms / args.steps
    value = job_tflops(step_flops, ws, ms_step)

    # end to end through the public API: every step copies its inputs in from
    # pinned host memory and its gradients out to pinned host memory.  Two
    # device buffer sets alternate, so the copies of step s+1's inputs (copy-in
    # stream) and of step s-1's gradients (copy-out stream) run while step s
    # computes, as a training loop streaming its batches would.
    e2e = None
    if not args.no_e2e:
        n_e2e = max(2, args.steps)
        host_in = [x.cpu().pin_memory() for x in (q, k, v, do)]
        host_out = [[torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(3)]
                    for _ in range(2)]
        sets = [(q, k, v, do, o, lse, dq, dk, dv)]
        sets.append(tuple(torch.empty_like(x) for x in sets[0]))
        copy_in = torch.cuda.Stream(device=dev)
        copy_out = torch.cuda.Stream(device=dev)

        def run_step(bufs):
            q_, k_, v_, do_, o_, lse_, dq_, dk_, dv_ = bufs
            lwm.lwm_attn_fwd(q_, k_, v_, seg_d, w.causal, w.theta, w.scale, o=o_, lse=lse_,
                             workspace=ws_f, stream=stream)
            lwm.lwm_attn_bwd(q_, k_, v_, o_, lse_, do_, seg_d, w.causal, w.theta, w.scale,
                             dq=dq_, dk=dk_, dv=dv_, workspace=ws_b, stream=stream)

        def e2e_run(n):
            ev = lambda: torch.cuda.Event(enable_timing=False)
            start_ev = torch.cuda.Event(enable_timing=True)
            stop_ev = torch.cuda.Event(enable_timing=True)
            start_ev.record(stream)
            copy_in.wait_event(start_ev)
            in_done, comp_done, out_done = [], [], []
            for s_ in range(n):
                bufs = sets[s_ % 2]
                with torch.cuda.stream(copy_in):
                    if s_ >= 2:
                        copy_in.wait_event(comp_done[s_ - 2])  # step s-2 is done with the set
                    for hsrc, dst in zip(host_in, bufs[:4]):
                        dst.copy_(hsrc, non_blocking=True)
                    in_done.append(ev())
                    in_done[-1].record(copy_in)
                stream.wait_event(in_done[s_])
                if s_ >= 2:
                    stream.wait_event(out_done[s_ - 2])   # its gradients have left the set
                run_step(bufs)
                comp_done.append(ev())
                comp_done[-1].record(stream)
                with torch.cuda.stream(copy_out):
                    copy_out.wait_event(comp_done[s_])
                    for src, hdst in zip(bufs[6:], host_out[s_ % 2]):
                        hdst.copy_(src, non_blocking=True)
                    out_done.append(ev())
                    out_done[-1].record(copy_out)
            stream.wait_event(out_done[-1])
            stop_ev.record(stream)
            torch.cuda.synchronize()
            return start_ev.elapsed_time(stop_ev)

        e2e_run(2)
        barrier()
        ems = e2e_run(n_e2e)
        barrier()
        ems, = max_over_ranks([ems], ws, dev)
        nb = q.numel() * q.element_size()
        e2e = {"value": job_tflops(step_flops, ws, ems / n_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": 4 * nb, "d2h_bytes_per_step": 3 * nb, "steps": n_e2e,
               "overlap": "double-buffered: copies of neighbouring steps run during compute"}

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    units = tile_pairs(seg, w.heads, w.causal)
    bwd_flops = 2.5 * fwd_flops
    dq_k = bwd_k - dkdv_k
    traffic = None
    tensor_cores = w.dtype == "bf16" and w.head_dim == 128
    split_fp32 = (w.dtype == "fp32" and w.head_dim in (64, 128)
                  and os.environ.get("LWM_ATTN_FP32_SIMT") != "1")
    if split_fp32:
        # fp32 on the tensor cores: every product is three bf16 products, so
        # the roofline is the dense bf16 peak / 3; the dominant part is the
        # backward (dK/dV then dQ kernels, timed together): 10*D*H flops per
        # kept pair of algorithmic work
        main_flops = bwd_flops
        kernel, algorithmic = "attn_bwd_dkdv_x3_kernel + attn_bwd_dq_x3_kernel", \
            "10*D*H flops per kept (query, key) pair (fp32 products as three bf16 products)"
    elif split_backward() or not tensor_cores:
        # dominant kernel: dK/dV, whose four GEMMs per kept pair (S^T, dP^T,
        # dV, dK) are all algorithmic work: 8*D flops per pair and head
        main_flops = 8.0 * w.head_dim * w.heads * pairs
        kernel, algorithmic = "attn_bwd_dkdv_kernel", \
            "8*D*H flops per kept (query, key) pair: S^T, dP^T, dV, dK"
        if (w.name in DKDV_TRAFFIC["bytes"] and
                DKDV_TRAFFIC["source_sha256"] == kernel_source_sha256("attn_bwd_sm100.cu")):
            traffic = DKDV_TRAFFIC["bytes"][w.name]
    else:
        # dominant kernel: the one-pass backward, all five GEMMs per kept pair
        # (S^T, dP^T, dV, dK, dQ): the whole backward's algorithmic work
        main_flops = bwd_flops
        kernel, algorithmic = "attn_bwd_fused_kernel", \
            "10*D*H flops per kept (query, key) pair: S^T, dP^T, dV, dK, dQ"
        if (w.name in FUSED_TRAFFIC["bytes"] and
                FUSED_TRAFFIC["source_sha256"] == kernel_source_sha256("attn_bwd_fused_sm100.cu")):
            traffic = FUSED_TRAFFIC["bytes"][w.name]
    achieved = main_flops / (dkdv_k * 1e-3) / 1e12 if dkdv_k > 0.0 else None
    bound, rpeak, peak_note = "tensor", peak, \
        f"{peak_src} bf16 sustained (kernel timed inside a long step)"
    if split_fp32:
        rpeak = peak / 3.0
        peak_note = f"{peak_src} bf16 sustained / 3 (three bf16 products per fp32 product)"
    elif not tensor_cores:
        # the CUDA-core kernels (fp32 arithmetic): bound by the FFMA pipes,
        # 128 fp32 lanes per SM, one fused multiply-add (2 flops) per lane
        # per clock, at the maximum SM clock the device reports
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        sm_max = float((clk or {}).get("sm_max_mhz") or 1965.0)
        rpeak = sms * 128 * 2 * sm_max * 1e6 / 1e12
        kernel, bound, traffic = "simt_bwd_dkdv_kernel", "alu", None
        peak_note = (f"fp32 FFMA peak derived: {sms} SMs x 128 lanes x 2 flops x "
                     f"{sm_max:.0f} MHz (maximum SM clock)")
    roofline = {"bound": bound, "achieved": achieved, "peak": rpeak, "unit": "TFLOP/s",
                "frac": achieved / rpeak if achieved else None, "traffic": traffic,
                "kernel": kernel, "algorithmic": algorithmic,
                "tile_pairs": units,
                "peak_source": peak_note,
                "bwd_main_kernel_ms": dkdv_k, "bwd_tail_ms": dq_k, "fwd_kernel_ms": fwd_k,
                "fwd_kernel_tflops": fwd_flops / (fwd_k * 1e-3) / 1e12,
                "bwd_kernels_tflops": bwd_flops / (bwd_k * 1e-3) / 1e12}
    if tensor_cores and clk and clk.get("sm_mhz") and achieved:
        # clock-normalised: the dense bf16 rate of one SM is 8192 flops per
        # clock (a 128x128x16 MMA every 64 clocks), at the SM clock measured
        # during the timed region
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        roofline["frac_of_clock_peak"] = achieved * 1e12 / (sms * 8192.0 * clk["sm_mhz"] * 1e6)

    # the HBM-bound pre-pass on its own (step A2): lwm_rope_apply over q,
    # reading and writing every element once, against the copy bandwidth
    rope_out = torch.empty_like(q)
    lwm.lwm_rope_apply(q, w.theta, out=rope_out, stream=stream)
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    n_rope = 5
    for _ in range(n_rope):
        lwm.lwm_rope_apply(q, w.theta, out=rope_out, stream=stream)
    r1.record(stream)
    torch.cuda.synchronize()
    rope_ms = r0.elapsed_time(r1) / n_rope
    rope_bytes = 2 * q.numel() * q.element_size()
    del rope_out
    hbm_kernels = {"rope_apply": {"bytes": rope_bytes, "ms": rope_ms,
                                  "GB/s": rope_bytes / (rope_ms * 1e-3) / 1e9,
                                  "frac_of_hbm": rope_bytes / (rope_ms * 1e-3) / 1e9
                                  / float(peaks["hbm_gbs"])}}
    if tensor_cores and not split_fp32 and not split_backward() and dq_k > 0.0:
        # step B3 of the one-pass backward, timed in the step above: the fp32
        # dQ~ accumulator read once, dq written once
        n_tiles = -(-w.seqlen // 128)
        fin_bytes = (w.batch * w.heads * n_tiles * 128 * w.head_dim * 4
                     + w.batch * w.seqlen * w.heads * w.head_dim * q.element_size())
        hbm_kernels["dq_finish"] = {"bytes": fin_bytes, "ms": dq_k,
                                    "GB/s": fin_bytes / (dq_k * 1e-3) / 1e9,
                                    "frac_of_hbm": fin_bytes / (dq_k * 1e-3) / 1e9
                                    / float(peaks["hbm_gbs"])}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rows = min(args.oracle_rows, w.seqlen)
        dt, fl, threads = time_oracle_sample(w, seg, rows, seed)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"float64 numpy oracle, fwd+bwd of the last {rows} query rows "
                         f"of one head of {w.name} ({fl / 1e9:.2f} GFLOP in {dt:.1f} s)"}

    if rank == 0:
        if heads_split:
            parallelism = f"tp{ws}: the heads of one problem split, {w.heads} per GPU"
            tokens = w.batch * w.seqlen
        else:
            parallelism = f"independent problem per GPU x{ws}"
            tokens = w.batch * w.seqlen * ws
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if heads_split else "weak",
            "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen,
                       "heads": w.heads * ws if heads_split else w.heads,
                       "head_dim": w.head_dim, "theta": w.theta,
                       "causal": w.causal, "segments": w.segments,
                       "parallelism": parallelism,
                       "l2": "inputs larger than L2 (1 GiB per tensor vs 126 MB), no flush",
                       "algorithmic_fwd_bwd_tflop_per_gpu": step_flops / 1e12,
                       "tokens_per_s": tokens / (ms_step * 1e-3),
                       "pct_of_bf16_peak": 100.0 * value / ws / peak},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "hbm_kernels": hbm_kernels,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def decode_bytes(w, seg, n_new: int) -> int:
    """Algorithmic HBM bytes of one decode step: every cache row (key and
    value, all heads) some new token may attend to, read once, plus the new
    queries, the outputs and the segment ids of the cache."""
    row = w.heads * w.head_dim * 2
    S = w.seqlen
    total = 0
    for b in range(w.batch):
        r = seg[b]
        sq = r[S - n_new:]
        need = np.isin(r, sq[sq >= 0]) & (r >= 0)
        total += 2 * row * int(np.count_nonzero(need))
    total += 2 * w.batch * n_new * row                  # q in, o out
    if w.segments != "single":
        total += 4 * w.batch * S
    return total


def time_oracle_decode(w, seg, seed: int, heads: int = 1):
    """Oracle decode on the first ``heads`` heads of the workload."""
    import torch
    import oracle
    n_new = w.extra["n_new"]
    g = torch.Generator()
    g.manual_seed(seed)
    shape = (1, w.seqlen, heads, w.head_dim)
    q = (torch.randn((1, n_new, heads, w.head_dim), generator=g) * w.sigma).to(torch.bfloat16)
    k = (torch.randn(shape, generator=g) * w.sigma).to(torch.bfloat16)
    v = (torch.randn(shape, generator=g) * w.sigma).to(torch.bfloat16)
    f = lambda x: x.double().numpy()
    t0 = time.perf_counter()
    oracle.attention_decode(f(q), f(k), f(v), seg[:1], causal=w.causal, theta=w.theta)
    dt = time.perf_counter() - t0
    sub = w.with_(batch=1, heads=heads)
    try:
        from threadpoolctl import threadpool_info
        threads = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    except Exception:
        threads = len(os.sched_getaffinity(0))
    return dt, decode_bytes(sub, seg[:1], n_new), threads


def decode_line(w, value, ms, args, ws, extra):
    line = {"metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "cache_len": w.seqlen,
                       "n_new": w.extra["n_new"], "heads": w.heads, "head_dim": w.head_dim,
                       "theta": w.theta, "segments": w.segments,
                       "parallelism": f"independent problem per GPU x{ws}",
                       "l2": "cache larger than L2 (16 GiB vs 126 MB), no flush"}}
    line.update(extra)
    return line


def reference_decode(args):
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    seg = segment_ids(w, seed=args.seed)
    for _ in range(args.warmup):
        time_oracle_decode(w, seg, args.seed)
    tot, nbytes, threads = 0.0, 0, 1
    for _ in range(args.steps):
        dt, nbytes, threads = time_oracle_decode(w, seg, args.seed)
        tot += dt
    value = nbytes * args.steps / tot / 1e9
    sample = f"float64 numpy oracle decode, head 0 of {w.name} ({nbytes / 1e9:.2f} GB of cache)"
    line = decode_line(w, value, 1e3 * tot / args.steps, args, ws, {
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
    print(json.dumps(line), flush=True)
    return 0


def ours_decode(args):
    import torch
    import torch.distributed as dist

    import long_context_causal_attention_b200 as lwm

    ws, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = WORKLOADS[args.workload]
    n_new = w.extra["n_new"]
    seed = rank_seed(args.seed, rank)
    seg = segment_ids(w, seed=seed)
    seg_d = None if w.segments == "single" else torch.as_tensor(seg, dtype=torch.int32,
                                                                device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    shape = (w.batch, w.seqlen, w.heads, w.head_dim)
    q = (torch.randn((w.batch, n_new, w.heads, w.head_dim), generator=g, device=dev)
         * w.sigma).to(torch.bfloat16)
    k = (torch.randn(shape, generator=g, device=dev) * w.sigma).to(torch.bfloat16)
    v = (torch.randn(shape, generator=g, device=dev) * w.sigma).to(torch.bfloat16)
    k_cache = lwm.lwm_rope_apply(k, w.theta, out=k)  # the cache holds rotated keys
    desc = lwm.make_desc(k_cache, seg_d, w.causal, w.theta, w.scale)
    wsp = torch.empty(lwm.lwm_attn_decode_workspace_size(desc, n_new), dtype=torch.uint8,
                      device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.batch, w.heads, n_new), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        lwm.lwm_attn_decode(q, k_cache, v, seg_d, w.causal, w.theta, w.scale, o=o, lse=lse,
                            workspace=wsp, stream=stream)

    nbytes = decode_bytes(w, seg, n_new)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    launches0 = lwm.lwm_attn_kernel_launches()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for s_ in range(args.steps):
        lwm.lwm_attn_set_timing_events(kev[s_][0], kev[s_][1])
        step()
    stop.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    lwm.lwm_attn_set_timing_events()
    launches = lwm.lwm_attn_kernel_launches() - launches0
    clk = clocks.stop()
    ms = start.elapsed_time(stop) / args.steps
    kern = sum(e[0].elapsed_time(e[1]) for e in kev) / args.steps
    ms, kern = max_over_ranks([ms, kern], ws, dev)
    value = nbytes * ws / (ms * 1e-3) / 1e9
    # end to end: the new queries come from the host, outputs go back; the
    # cache stays resident on the device as it does while generating
    hq = q.cpu().pin_memory()
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    ems, = max_over_ranks([e0.elapsed_time(e1) / args.steps], ws, dev)
    peaks, src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = nbytes / (kern * 1e-3) / 1e9
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, nb, threads = time_oracle_decode(w, seg, seed)
        cpu = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"float64 numpy oracle decode, head 0 of {w.name} "
                         f"({nb / 1e9:.2f} GB of cache in {dt:.1f} s)"}
    if rank == 0:
        line = decode_line(w, value, ms, args, ws, {
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None,
                         "kernel": "decode_partial_kernel + decode_merge_kernel",
                         "algorithmic": "key and value rows the new tokens may attend to, "
                                        "all heads, once; q in, o out",
                         "bytes_per_step": nbytes, "kernels_ms": kern,
                         "peak_source": f"{src} HBM copy bandwidth"},
            "cpu_baseline": cpu,
            "e2e": {"value": nbytes * ws / (ems * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": hq.numel() * hq.element_size(),
                    "d2h_bytes_per_step": ho.numel() * ho.element_size()
                    + hl.numel() * hl.element_size()},
            "gpu_launches": launches,
            "clocks": clk})
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def loss_inputs(w, seed, device):
    """Seeded bf16 logits [B, S, V] ~ N(0, 4) and int32 targets (one in five
    tokens without loss, as prompt tokens of chat samples)."""
    import torch
    V = w.extra["vocab"]
    rng = np.random.default_rng(seed + 17)
    targets = rng.integers(0, V, size=(w.batch, w.seqlen)).astype(np.int32)
    targets[rng.random((w.batch, w.seqlen)) < 0.2] = -1
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    logits = (torch.randn((w.batch, w.seqlen, V), generator=g, device=device) * 2.0)
    return logits.to(torch.bfloat16), targets


def loss_bytes(V, elt, targets, seg):
    """Algorithmic bytes of one packed-loss step: the logits of the tokens
    that carry a loss are read once (the kernel never reads the others), the
    gradient of every token is written once (zero rows included), targets
    and segment ids are read once."""
    has_loss = (targets >= 0) & (targets < V) & (np.asarray(seg) >= 0)
    return V * elt * (int(has_loss.sum()) + targets.size) + 4 * 2 * targets.size


def loss_line(w, value, ms, args, ws, extra):
    line = {"metric": LOSS_METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen,
                       "vocab": w.extra["vocab"], "segments": w.segments,
                       "parallelism": f"independent problem per GPU x{ws}",
                       "l2": "logits larger than L2 (2.1 GB vs 126 MB), no flush"}}
    line.update(extra)
    return line


def time_oracle_loss(w, seg, seed, rows=64):
    """Oracle loss and gradient on the first `rows` tokens of row 0 (their
    weights from the whole batch's samples)."""
    import oracle
    V = w.extra["vocab"]
    rng = np.random.default_rng(seed + 17)
    targets = rng.integers(0, V, size=(w.batch, w.seqlen)).astype(np.int32)
    targets[rng.random((w.batch, w.seqlen)) < 0.2] = -1
    z = np.random.default_rng(seed).standard_normal((1, rows, V)) * 2.0
    t0 = time.perf_counter()
    oracle.packed_cross_entropy(z, targets[:1, :rows], seg[:1, :rows])
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    except Exception:
        threads = len(os.sched_getaffinity(0))
    return dt, 2 * rows * V * 2, threads


def reference_loss(args):
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    seg = segment_ids(w, seed=args.seed)
    for _ in range(args.warmup):
        time_oracle_loss(w, seg, args.seed)
    tot, nbytes, threads = 0.0, 0, 1
    for _ in range(args.steps):
        dt, nbytes, threads = time_oracle_loss(w, seg, args.seed)
        tot += dt
    value = nbytes * args.steps / tot / 1e9
    sample = f"float64 numpy oracle, loss and gradient of 64 tokens of {w.name}"
    print(json.dumps(loss_line(w, value, 1e3 * tot / args.steps, args, ws, {
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}})), flush=True)
    return 0


def ours_loss(args):
    import torch
    import torch.distributed as dist

    import long_context_causal_attention_b200 as lwm

    ws, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = WORKLOADS[args.workload]
    seed = rank_seed(args.seed, rank)
    seg = segment_ids(w, seed=seed)
    logits, targets = loss_inputs(w, seed, dev)
    t_d = torch.as_tensor(targets, device=dev)
    s_d = torch.as_tensor(seg, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    nbytes = loss_bytes(logits.shape[-1], logits.element_size(), targets, seg)
    for _ in range(args.warmup):
        lwm.lwm_packed_cross_entropy(logits, t_d, s_d, stream=stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    launches0 = lwm.lwm_attn_kernel_launches()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(args.steps):
        loss, d = lwm.lwm_packed_cross_entropy(logits, t_d, s_d, stream=stream)
    stop.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    launches = lwm.lwm_attn_kernel_launches() - launches0
    clk = clocks.stop()
    ms, = max_over_ranks([start.elapsed_time(stop) / args.steps], ws, dev)
    value = nbytes * ws / (ms * 1e-3) / 1e9
    # end to end: logits in from pinned host memory, loss and gradient out
    hz = logits.cpu().pin_memory()
    hd = torch.empty(logits.shape, dtype=logits.dtype, pin_memory=True)
    hl = torch.empty(1, dtype=torch.float32, pin_memory=True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        logits.copy_(hz, non_blocking=True)
        loss, d = lwm.lwm_packed_cross_entropy(logits, t_d, s_d, stream=stream)
        hd.copy_(d, non_blocking=True)
        hl.copy_(loss, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    ems, = max_over_ranks([e0.elapsed_time(e1) / args.steps], ws, dev)
    peaks, src = load_peaks()
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, nb, threads = time_oracle_loss(w, seg, seed)
        cpu = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"float64 numpy oracle, loss and gradient of 64 tokens of {w.name} "
                         f"({dt:.2f} s)"}
    if rank == 0:
        print(json.dumps(loss_line(w, value, ms, args, ws, {
            "roofline": {"bound": "hbm", "achieved": value / ws, "peak": float(peaks["hbm_gbs"]),
                         "unit": "GB/s", "frac": value / ws / float(peaks["hbm_gbs"]),
                         "traffic": None, "kernel": "run_count + ce + loss_sum kernels",
                         "algorithmic": "logits of the tokens with a loss read once, the "
                                        "gradient of every token written once, targets and "
                                        "segment ids",
                         "bytes_per_step": nbytes, "peak_source": f"{src} HBM copy bandwidth"},
            "cpu_baseline": cpu,
            "e2e": {"value": nbytes * ws / (ems * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": hz.numel() * hz.element_size(),
                    "d2h_bytes_per_step": hd.numel() * hd.element_size() + 4},
            "gpu_launches": launches, "clocks": clk})), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def launch_ranks(n: int) -> int:
    """Run this command as n ranks on this node (one process per GPU),
    rendezvous on 127.0.0.1; returns the launcher's exit status."""
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_128k", choices=sorted(WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--oracle-rows", type=int, default=1024)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", choices=["heads", "replicas"], default="heads",
                    help="N > 1: split the heads of one problem (strong scaling) or run "
                         "one independent problem per GPU (weak scaling)")
    args = ap.parse_args()
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return launch_ranks(args.gpus)
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={ws}: launch one rank per GPU")
    extra = WORKLOADS[args.workload].extra
    if args.impl == "reference":
        if "n_new" in extra:
            return reference_decode(args)
        return reference_loss(args) if "vocab" in extra else reference_arm(args)
    if "n_new" in extra:
        return ours_decode(args)
    return ours_loss(args) if "vocab" in extra else ours(args)


if __name__ == "__main__":
    sys.exit(main())
