#!/usr/bin/env python
"""Throughput of the fused attention forward on B200, one JSON line on rank 0.

Default workload (one step = one qbsa_fwd call): quantized block-sparse attention,
B=1, N=40, S=65536, D=128, INT8 Q/K per 128-token block, E4M3 V per channel, 128x128
block mask keeping 10% of the blocks per (head, query block) with the diagonal kept.
Reported beside it under "extra": bf16 block-sparse attention on the same mask, the
on-GPU quantisers, block-mask estimation, dense bf16 attention at S=61440 (the video
workload) and S=65536, the causal (B=2, N=16, S=4096) and GQA varlen TND workloads, an
explicit atten_mask and a pse (B=1, N=16, S=4096), and the sweep over S = 8K..128K at keep 0.1 and 0.5 plus dense at each S (the metric's
"vs S" curve; ``--no-sweep`` skips it).  Lines whose inputs fit in L2 flush it (a
256 MB write) before every timed step and time each step alone.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs the same per-GPU workload
(the heads are independent; no collective on the data path) and ``value`` is the
total work of all ranks divided by the max over ranks of the timed span ("weak").
``--impl reference`` times the CPU oracle on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOPS (B=1,N=40,D=128) and % of B200 tensor peak vs S"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 vs 2.25 PFLOP/s), applied to the measured bf16 peak
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attn_qbsa_kernel launch from
# one ncu capture at S=16384, keep 0.1; it holds only for the kernel sources it was taken on,
# identified by their sha1.
QBSA_NCU_TRAFFIC = {"sources": {"quantized_block_sparse_attn_b200/csrc/attn_qbsa.cuh": "57ac69cc0f60dc779bf1ce860d9f5d522335c4ff",
                                "quantized_block_sparse_attn_b200/csrc/ptx_sm100.cuh": "79c119816b887e6d7279a127e6ec8586f11eaa4e"},
                    "seq": 16384, "keep": 0.1, "bytes": 461676288, "alg_bytes": 420147200}


def qbsa_traffic(seq: int, keep: float, alg_bytes: int):
    """Per-launch DRAM traffic from the recorded ncu capture, scaled to this launch by its
    algorithmic bytes (Q, K, V, O all grow linearly in S), or None when the kernel sources
    changed since the capture or the keep fraction differs."""
    import hashlib
    rec = QBSA_NCU_TRAFFIC
    for rel, sha in rec["sources"].items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha1(f.read()).hexdigest() != sha:
                    return None, "kernel changed since the ncu capture"
        except OSError:
            return None, "kernel sources not found"
    if abs(keep - rec["keep"]) > 1e-9:
        return None, "no capture at this keep fraction"
    return (rec["bytes"] * alg_bytes / rec["alg_bytes"],
            f"ncu at S={rec['seq']} keep {rec['keep']}: {rec['bytes'] / 1e6:.1f} MB, scaled by algorithmic bytes")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--seq", type=int, default=65536)
    p.add_argument("--keep", type=float, default=0.1)
    p.add_argument("--dense-seq", type=int, default=61440)
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--no-dense", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) every 10 ms."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.thread = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            return
        self.stop_flag = threading.Event()

        def loop():
            while not self.stop_flag.is_set():
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
                    get = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                        getattr(self.nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                    rs = get(self.handle)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                self.stop_flag.wait(0.01)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        reasons = sorted({nm for _, rs in self.samples for nm, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(self.samples), "source": "NVML, 10 ms"}


# ----------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------

def qbsa_inputs(S: int, keep: float, device):
    """Device-resident quantized inputs of the block-sparse workload (B=1, N=40, D=128)."""
    import numpy as np
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, block_keep_mask, device_blocky_qk_bf16, device_iid_normal_bf16
    c = CONFIGS["qbsa"]
    N, D, seed = c["Nq"], c["D"], c["seed"]
    q = device_blocky_qk_bf16(seed, "q", 1, N, S, D, device)
    k = device_blocky_qk_bf16(seed, "k", 1, N, S, D, device)
    v = device_iid_normal_bf16(seed, 2, (1, N, S, D), device)
    q8, qs = qb.quantize_qk(q)
    k8, ks = qb.quantize_qk(k)
    v8, vs = qb.quantize_v(v)
    torch.cuda.synchronize(device)
    del q, k, v
    nb = -(-S // 128)
    bm_np = block_keep_mask(seed, 1, N, nb, nb, keep)
    bm = torch.from_numpy(bm_np).to(device)
    kept = int(bm_np.sum())
    return dict(q8=q8, qs=qs, k8=k8, ks=ks, v8=v8, vs=vs, bm=bm, bm_np=bm_np, kept=kept, N=N, D=D, S=S,
                scale=c["scale"], seed=seed)


def qbsa_work(inp):
    """Executed FLOPs (kept blocks), dense-equivalent FLOPs and algorithmic bytes of one call."""
    N, S, D, kept = inp["N"], inp["S"], inp["D"], inp["kept"]
    executed = 4.0 * D * 128 * 128 * kept
    dense_eq = 4.0 * D * S * S * N
    nb = -(-S // 128)
    bytes_ = 3 * N * S * D + 2 * N * S * D + N * nb * nb + 4 * (2 * N * nb + N * D)
    return executed, dense_eq, bytes_


def step_stats(per_ms):
    """Median, extremes and coefficient of variation of per-step device times (ms); the
    stability rule asks for a CV below 0.05."""
    mean_ms = sum(per_ms) / len(per_ms)
    return {"median_ms": statistics.median(per_ms), "min_ms": min(per_ms), "max_ms": max(per_ms),
            "cv": (statistics.pstdev(per_ms) / mean_ms) if len(per_ms) > 1 else 0.0,
            "stable": len(per_ms) < 2 or statistics.pstdev(per_ms) / mean_ms < 0.05,
            "rule": "coefficient of variation of the per-step device times below 0.05"}


def time_steps(fn, steps: int, warmup: int, stream, dist=None, sampler=None, flush=None):
    """Run fn warmup times, then time exactly `steps` calls with CUDA events on `stream`.

    With ``flush`` (a device buffer larger than L2) the buffer is overwritten before every
    step, outside the events, so each step starts with a cold L2; the total is then the sum
    of the per-step times.  Before the first event of a timed interval the stream runs a
    ~100 us device-side sleep, so that the step's kernels are already queued when the GPU
    reaches the event: the events then bracket device work only, not the host's time to
    issue it (the host path is what the e2e figure measures)."""
    import torch
    hold = lambda: torch.cuda._sleep(200_000)  # ~100 us at ~2 GHz
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    if flush is None:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        hold()
        evs[0].record(stream)
        for i in range(steps):
            fn()
            evs[i + 1].record(stream)
    else:
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in pairs:
            flush.zero_()
            hold()
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if flush is None:
        per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
        total = evs[0].elapsed_time(evs[-1])
    else:
        per = [a.elapsed_time(b) for a, b in pairs]
        total = sum(per)
    return total, per, clocks


def l2_flush_buffer(device):
    """A 256 MB device buffer (twice the 126 MB L2) to overwrite between timed steps."""
    import torch
    return torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)


def max_over_ranks(x: float, dist, device="cuda"):
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(local_total_ms: float, flops_per_step: float, steps: int, dist, device="cuda"):
    """(max-over-ranks time of the timed span in ms, whole-job TFLOP/s).

    Every rank runs the same per-GPU workload, so the job's work is world x steps x
    flops_per_step, delivered in the slowest rank's time.
    """
    world = 1 if dist is None else dist.get_world_size()
    span_ms = max_over_ranks(local_total_ms, dist, device)
    return span_ms, world * flops_per_step * steps / (span_ms / 1e3) / 1e12


def cpu_oracle_sample(inp_host, n_qblocks: int):
    """Time the oracle (as it stands) on n_qblocks query blocks of head 0.  Returns (TFLOP/s, s, desc)."""
    import numpy as np
    from oracle import quant
    from workloads import sample_rows
    S, D = inp_host["S"], inp_host["D"]
    qbs = sample_rows(inp_host["seed"], S, n_qblocks)
    bm = inp_host["bm_np"][:, :1]
    t0 = time.perf_counter()
    quant.qbsa_forward(inp_host["q8"], inp_host["k8"], inp_host["qs"], inp_host["ks"], inp_host["v8"],
                       inp_host["vs"], bm, inp_host["scale"], q_blocks=qbs)
    dt = time.perf_counter() - t0
    kept = int(bm[0, 0, qbs].sum())
    flops = 4.0 * D * 128 * 128 * kept
    return flops / dt / 1e12, dt, f"head 0, {len(qbs)} query blocks ({kept} kept 128x128 blocks) of S={S}"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def host_head0(inp):
    """Host copies of head 0's quantized inputs (for the CPU oracle sample)."""
    return dict(q8=inp["q8"][:, :1].cpu().numpy(), k8=inp["k8"][:, :1].cpu().numpy(),
                qs=inp["qs"][:, :1].cpu().numpy(), ks=inp["ks"][:, :1].cpu().numpy(),
                v8=inp["v8"][:, :1].cpu().numpy(), vs=inp["vs"][:, :1].cpu().numpy(), bm_np=inp["bm_np"],
                S=inp["S"], D=inp["D"], scale=inp["scale"], seed=inp["seed"])


# ----------------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------------

def run_reference(args):
    """CPU oracle arm: each step is one query block of head 0 of the same workload."""
    import numpy as np
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import quant
    from workloads import CONFIGS, block_keep_mask, blocky_qk_bf16, iid_normal_bf16, sample_rows
    c = CONFIGS["qbsa"]
    S, D, seed = args.seq, c["D"], c["seed"]
    # head 0 only, generated on the host; quantised by the oracle's own quantiser
    q = blocky_qk_bf16(seed, "q", 1, 1, S, D)
    k = blocky_qk_bf16(seed, "k", 1, 1, S, D)
    v = iid_normal_bf16(seed, 2, 1, 1, S, D)
    q8, qs = quant.quantize_qk_per_block(q)
    k8, ks = quant.quantize_qk_per_block(k)
    v8, vs = quant.quantize_v_per_channel(v)
    nb = S // 128
    bm = block_keep_mask(seed, 1, 1, nb, nb, args.keep)
    qbs = sample_rows(seed, S, args.steps + args.warmup)
    while len(qbs) < args.steps + args.warmup:
        qbs = qbs + qbs
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        qb_ = qbs[i]
        t0 = time.perf_counter()
        quant.qbsa_forward(q8, k8, qs, ks, v8, vs, bm, c["scale"], q_blocks=[qb_])
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            flops.append(4.0 * D * 128 * 128 * int(bm[0, 0, qb_].sum()))
    tot = sum(times)
    value = sum(flops) / tot / 1e12
    cores = blas_threads()
    sample = f"one query block of head 0 per step (S={S}, keep={args.keep}), {args.steps} steps"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8+e4m3 (emulated in f64)",
            "data": "synthetic",
            "config": {"workload": f"qbsa_fwd B=1 N=40 S={S} D=128 keep={args.keep}", "global_batch": 1,
                       "seq_len": S, "parallelism": "cpu oracle, rank 0 only"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def run_ours(args):
    import torch
    import quantized_block_sparse_attn_b200 as qb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peaks, peak_src = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    bf16_peak = peaks["bf16_tflops"]
    hbm_peak = peaks["hbm_gbs"]

    # ---------------------------------------------------------------- main: qbsa_fwd
    inp = qbsa_inputs(args.seq, args.keep, device)
    executed, dense_eq, alg_bytes = qbsa_work(inp)
    out = torch.empty((1, inp["N"], inp["S"], inp["D"]), dtype=torch.bfloat16, device=device)

    def step():
        qb.qbsa_fwd(inp["q8"], inp["k8"], inp["qs"], inp["ks"], inp["v8"], inp["vs"], inp["bm"], inp["scale"],
                    out=out, return_stats=False)

    sampler = ClockSampler(local)
    total_ms, per_ms, clocks = time_steps(step, args.steps, args.warmup, stream, dist, sampler)
    qb.check(device)
    total_ms, value = weak_scaling_value(total_ms, executed, args.steps, dist)
    ms_step = total_ms / args.steps
    launch_ms = sum(per_ms) / len(per_ms)
    achieved = executed / (launch_ms / 1e3) / 1e12

    traffic, traffic_src = qbsa_traffic(args.seq, args.keep, alg_bytes)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8xi8->s32, e4m3xe4m3->f32, bf16 out", "data": "synthetic",
            "config": {"workload": f"qbsa_fwd B=1 N=40 S={args.seq} D=128 keep={args.keep} (per GPU)",
                       "global_batch": world, "seq_len": args.seq, "parallelism": f"dp{world} (heads independent)",
                       "l2": f"inputs {3 * inp['N'] * inp['S'] * inp['D'] / 1e9:.2f} GB > 126 MB L2, no flush",
                       "dense_equivalent_tflops": world * dense_eq * args.steps / (total_ms / 1e3) / 1e12,
                       "pct_of_fp8_int8_peak": 100.0 * achieved / fp8_peak},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp8_peak, "traffic": traffic, "traffic_source": traffic_src,
                         "peak_source": f"{peak_src} bf16 burst {bf16_peak} x {FP8_OVER_BF16} (nominal fp8/int8:bf16)",
                         "kernel": "attn_qbsa_kernel", "algorithmic_bytes": alg_bytes,
                         "hbm_gbs_algorithmic": alg_bytes / (launch_ms / 1e3) / 1e9},
            "gpu_launches": args.steps, "clocks": clocks}
    line["step_stats"] = step_stats(per_ms)

    # ---------------------------------------------------------------- e2e through the public API, host buffers
    if not args.no_e2e:
        host = {k: inp[k].cpu().pin_memory() for k in ("q8", "qs", "k8", "ks", "v8", "vs", "bm")}
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        d2h = host_out.numel() * host_out.element_size()
        e2e_steps = max(2, min(10, args.steps))

        def e2e_step():
            res = qb.qbsa_fwd(host["q8"], host["k8"], host["qs"], host["ks"], host["v8"], host["vs"], host["bm"],
                              inp["scale"], out=host_out, return_stats=False, device=device)
            return res[0]

        e2e_step()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            e2e_step()
        torch.cuda.synchronize()
        e2e_s = max_over_ranks((time.perf_counter() - t0) / e2e_steps, dist)
        line["e2e"] = {"value": world * executed / e2e_s / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": 1e3 * e2e_s,
                       "note": "through the C ABI's qbsa_fwd_host: host pinned int8/e4m3/fp32 inputs copied in, "
                               "bf16 output copied out, every step"}

    # ---------------------------------------------------------------- CPU oracle sample (rank 0, N=1)
    if rank == 0 and world == 1 and not args.no_cpu:
        tf, secs, desc = cpu_oracle_sample(host_head0(inp), n_qblocks=128)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": desc + f", {secs:.1f} s"}

    extra = {}
    flush = l2_flush_buffer(device)
    # ---------------------------------------------------------------- bf16 block-sparse, same mask
    if not args.no_dense:
        extra["bsa_bf16_same_mask"] = bsa_line(device, stream, inp, executed, bf16_peak, ms_step)
    del inp
    torch.cuda.empty_cache()
    # ---------------------------------------------------------------- on-GPU quantisers
    extra["quantize"] = quantize_line(device, stream, args.seq, hbm_peak)
    # ---------------------------------------------------------------- block-mask estimation
    if not args.no_dense:
        extra["mask_estimation"] = estimate_line(device, stream, args.seq, args.keep, hbm_peak)
    # ---------------------------------------------------------------- dense bf16
    if not args.no_dense:
        extra["dense_video"] = dense_line(device, stream, args.dense_seq, max(2, args.warmup), 10, bf16_peak, dist)
        extra["dense_S65536"] = dense_line(device, stream, 65536, 2, 10, bf16_peak, dist)
        extra["causal"] = causal_line(device, stream, bf16_peak, flush)
        extra["gqa_varlen"] = gqa_varlen_line(device, stream, bf16_peak, flush)
        extra["explicit_mask"] = explicit_mask_line(device, stream, bf16_peak, hbm_peak, flush)
    # ---------------------------------------------------------------- the metric's curve over S
    if not args.no_sweep:
        sweep = []
        for S in (8192, 16384, 32768, 65536, 131072):
            for keep in (0.1, 0.5):
                sweep.append(qbsa_line(device, stream, S, keep, fp8_peak, flush if S <= 8192 else None))
            if not args.no_dense:
                sweep.append(dense_line(device, stream, S, 2, 3 if S > 65536 else 5, bf16_peak, None,
                                        flush if S <= 8192 else None))
        extra["sweep"] = sweep
    if extra:
        line["extra"] = extra
    if dist is not None:
        dist.barrier()
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


def qbsa_line(device, stream, S, keep, fp8_peak, flush=None):
    import torch
    import quantized_block_sparse_attn_b200 as qb
    inp = qbsa_inputs(S, keep, device)
    executed, dense_eq, _ = qbsa_work(inp)
    out = torch.empty((1, inp["N"], S, inp["D"]), dtype=torch.bfloat16, device=device)

    def step():
        qb.qbsa_fwd(inp["q8"], inp["k8"], inp["qs"], inp["ks"], inp["v8"], inp["vs"], inp["bm"], inp["scale"],
                    out=out, return_stats=False)

    total, per, _ = time_steps(step, 10, 2, stream, flush=flush)
    qb.check(device)
    ms = total / 10
    del inp
    torch.cuda.empty_cache()
    return {"kernel": "attn_qbsa_kernel", "S": S, "keep": keep, "ms": ms, "executed_tflops": executed / ms / 1e9,
            "dense_equivalent_tflops": dense_eq / ms / 1e9, "pct_of_fp8_peak": 100 * executed / ms / 1e9 / fp8_peak,
            "l2": "flushed before each step" if flush is not None else "inputs > L2"}


def bsa_line(device, stream, inp, executed, bf16_peak, qbsa_ms):
    """bf16 block-sparse attention on the quantized workload's shape and block mask."""
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, device_blocky_qk_bf16, device_iid_normal_bf16
    N, S, D, seed = inp["N"], inp["S"], inp["D"], inp["seed"]
    q = device_blocky_qk_bf16(seed, "q", 1, N, S, D, device)
    k = device_blocky_qk_bf16(seed, "k", 1, N, S, D, device)
    v = device_iid_normal_bf16(seed, 2, (1, N, S, D), device)
    out = torch.empty_like(q)

    def step():
        qb.bsa_fwd(q, k, v, inp["bm"], inp["scale"], out=out, return_stats=False)

    total, per, _ = time_steps(step, 10, 2, stream)
    qb.check(device)
    ms = total / 10
    del q, k, v, out
    torch.cuda.empty_cache()
    return {"workload": f"bsa_fwd bf16 B=1 N=40 S={S} D=128, same block mask", "ms": ms,
            "executed_tflops": executed / ms / 1e9, "pct_of_bf16_peak": 100 * executed / ms / 1e9 / bf16_peak,
            "qbsa_speedup_over_bsa": ms / qbsa_ms, "kernel": "attn_dense_kernel<128> (block-mask list)"}


def estimate_line(device, stream, S, keep, hbm_peak):
    """Block-mask estimation (block mean pooling of Q and K, pooled scores, top-k) on the
    quantized workload's bf16 Q/K recipe at this S."""
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, block_keep_mask, device_blocky_qk_bf16
    c = CONFIGS["qbsa"]
    N, D, seed = c["Nq"], c["D"], c["seed"]
    q = device_blocky_qk_bf16(seed, "q", 1, N, S, D, device)
    k = device_blocky_qk_bf16(seed, "k", 1, N, S, D, device)
    nb = -(-S // 128)
    state = {}

    def pool():
        state["qm"] = qb.block_mean(q)
        state["km"] = qb.block_mean(k)

    def topk():
        state["mask"] = qb.block_topk(state["qm"], state["km"], c["scale"], keep=keep)

    pool_ms, _, _ = time_steps(pool, 5, 2, stream)
    topk_ms, _, _ = time_steps(topk, 5, 2, stream)
    qb.check(device)
    pool_ms, topk_ms = pool_ms / 5, topk_ms / 5
    pool_bytes = 2 * N * S * D * 2 + 2 * N * nb * D * 4  # bf16 Q and K read, fp32 means written
    kept = int(state["mask"].sum().item())
    expected = int(block_keep_mask(seed, 1, 1, nb, nb, keep).sum()) * N  # same count rule, one head's rows
    del q, k, state
    torch.cuda.empty_cache()
    return {"workload": f"block-mask estimation B=1 N=40 S={S} D=128 keep={keep}", "ms": pool_ms + topk_ms,
            "block_mean_ms": pool_ms, "block_mean_gbs": pool_bytes / (pool_ms / 1e3) / 1e9,
            "block_mean_frac_of_hbm": pool_bytes / (pool_ms / 1e3) / 1e9 / hbm_peak,
            "block_topk_ms": topk_ms, "kept_blocks": kept, "expected_kept": expected,
            "kernels": "block_mean_kernel x2 (HBM-bound), block_topk_kernel"}


def dense_line(device, stream, S, warmup, steps, bf16_peak, dist, flush=None):
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, device_blocky_qk_bf16, device_iid_normal_bf16
    c = CONFIGS["video"]
    N, D, seed = c["Nq"], c["D"], c["seed"]
    q = device_blocky_qk_bf16(seed, "q", 1, N, S, D, device)
    k = device_blocky_qk_bf16(seed, "k", 1, N, S, D, device)
    v = device_iid_normal_bf16(seed, 2, (1, N, S, D), device)
    out = torch.empty_like(q)

    def step():
        qb.attn_fwd(q, k, v, N, "BNSD", scale=c["scale"], out=out, return_stats=False)

    total, per, clocks = time_steps(step, steps, warmup, stream, dist, flush=flush)
    qb.check(device)
    ms = max_over_ranks(total / steps, dist)
    flops = 4.0 * D * S * S * N
    del q, k, v, out
    torch.cuda.empty_cache()
    return {"workload": f"attn_fwd bf16 B=1 N=40 S={S} D=128 no mask", "S": S, "ms": ms, "tflops": flops / ms / 1e9,
            "pct_of_bf16_peak": 100 * flops / ms / 1e9 / bf16_peak, "kernel": "attn_pair_kernel",
            "l2": "flushed before each step" if flush is not None else "inputs > L2"}


def _visited_tiles(sq: int, skv: int, mode: int) -> int:
    """K tiles the kernel visits for one head of one sequence (the library's own schedule export)."""
    import quantized_block_sparse_attn_b200 as qb
    kb, ke, _, _ = qb.attn_tile_schedule(sq, skv, mode)
    return int((ke - kb).sum())


def causal_line(device, stream, bf16_peak, flush):
    """The causal training-style workload: B=2, N=16, S=4096, D=128, BNSD, sparse_mode 3, with stats."""
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, device_iid_normal_bf16
    c = CONFIGS["causal"]
    B, N, S, D, seed = c["B"], c["Nq"], c["S"], c["D"], c["seed"]
    q, k, v = (device_iid_normal_bf16(seed, t, (B, N, S, D), device) for t in range(3))
    out = torch.empty_like(q)
    smax = torch.empty((B, N, S), dtype=torch.float32, device=device)
    ssum = torch.empty_like(smax)

    def step():
        qb.attn_fwd(q, k, v, N, "BNSD", scale=c["scale"], sparse_mode=3, out=out, softmax_max=smax,
                    softmax_sum=ssum)

    total, per, _ = time_steps(step, 20, 3, stream, flush=flush)
    qb.check(device)
    ms = total / 20
    executed = 4.0 * D * 128 * 128 * _visited_tiles(S, S, 3) * B * N
    useful = 4.0 * D * (S * (S + 1) // 2) * B * N
    del q, k, v, out, smax, ssum
    torch.cuda.empty_cache()
    return {"workload": f"attn_fwd bf16 causal (sparse_mode 3) B={B} N={N} S={S} D={D} BNSD, stats", "ms": ms,
            "executed_tflops": executed / ms / 1e9, "useful_tflops": useful / ms / 1e9,
            "pct_of_bf16_peak": 100 * executed / ms / 1e9 / bf16_peak, "kernel": "attn_pair_masked_kernel",
            "l2": "flushed before each step"}


def gqa_varlen_line(device, stream, bf16_peak, flush):
    """The GQA varlen workload: TND, Nq=32, Nkv=8, D=128, sequences 1024/5000/10360, causal."""
    import numpy as np
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, device_iid_normal_bf16
    c = CONFIGS["gqa_varlen"]
    Nq, Nkv, D, seed, lens = c["Nq"], c["Nkv"], c["D"], c["seed"], c["seqlens"]
    T = sum(lens)
    cum = np.cumsum(lens).tolist()
    q = device_iid_normal_bf16(seed, 0, (T, Nq, D), device)
    k = device_iid_normal_bf16(seed, 1, (T, Nkv, D), device)
    v = device_iid_normal_bf16(seed, 2, (T, Nkv, D), device)
    out = torch.empty_like(q)

    def step():
        qb.attn_fwd(q, k, v, Nq, "TND", scale=c["scale"], sparse_mode=c["sparse_mode"], actual_seq_qlen=cum,
                    actual_seq_kvlen=cum, out=out, return_stats=False)

    total, per, _ = time_steps(step, 20, 3, stream, flush=flush)
    qb.check(device)
    ms = total / 20
    executed = 4.0 * D * 128 * 128 * sum(_visited_tiles(n, n, 3) for n in lens) * Nq
    useful = 4.0 * D * sum(n * (n + 1) // 2 for n in lens) * Nq
    del q, k, v, out
    torch.cuda.empty_cache()
    return {"workload": f"attn_fwd bf16 TND GQA Nq={Nq} Nkv={Nkv} D={D} lengths {list(lens)} causal", "ms": ms,
            "executed_tflops": executed / ms / 1e9, "useful_tflops": useful / ms / 1e9,
            "pct_of_bf16_peak": 100 * executed / ms / 1e9 / bf16_peak, "kernel": "attn_pair_masked_kernel",
            "l2": "flushed before each step"}


def explicit_mask_line(device, stream, bf16_peak, hbm_peak, flush):
    """attn_fwd with an explicit atten_mask (SS, shared by all heads) or a pse (BNSS), B=1,
    N=16, S=4096, D=128, BNSD, sparse_mode 0, with stats: the one-tile kernel's general path."""
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import device_iid_normal_bf16, random_atten_mask
    B, N, S, D, seed = 1, 16, 4096, 128, 41
    q, k, v = (device_iid_normal_bf16(seed, t, (B, N, S, D), device) for t in range(3))
    mask = torch.from_numpy(random_atten_mask(seed, (S, S), 0.5)).to(device)
    pse = device_iid_normal_bf16(seed, 3, (B, N, S, S), device)
    out = torch.empty_like(q)
    smax = torch.empty((B, N, S), dtype=torch.float32, device=device)
    ssum = torch.empty_like(smax)
    flops = 4.0 * D * S * S * B * N
    res = {}
    for name, kw, extra_bytes in (("atten_mask_SS", dict(atten_mask=mask, mask_shape="SS"), S * S),
                                  ("pse_BNSS", dict(pse=pse), 2 * B * N * S * S)):
        def step(kw=kw):
            qb.attn_fwd(q, k, v, N, "BNSD", scale=D ** -0.5, out=out, softmax_max=smax, softmax_sum=ssum, **kw)

        total, per, _ = time_steps(step, 20, 3, stream, flush=flush)
        qb.check(device)
        ms = total / 20
        res[name] = {"ms": ms, "tflops": flops / ms / 1e9, "pct_of_bf16_peak": 100 * flops / ms / 1e9 / bf16_peak,
                     "extra_input_bytes": extra_bytes,
                     "extra_input_frac_of_hbm": extra_bytes / (ms * 1e-3) / 1e9 / hbm_peak}
    del q, k, v, mask, pse, out, smax, ssum
    torch.cuda.empty_cache()
    res.update({"workload": f"attn_fwd bf16 B={B} N={N} S={S} D={D} BNSD, sparse_mode 0, stats; an SS atten_mask "
                            "(half the keys masked, iid) or a BNSS pse (iid N(0,1))",
                "kernel": "attn_dense_kernel<128, general>", "l2": "flushed before each step"})
    return res


def quantize_line(device, stream, S, hbm_peak):
    """The on-GPU quantisers on the quantized workload's bf16 Q/K/V at this S (HBM-bound)."""
    import torch
    import quantized_block_sparse_attn_b200 as qb
    from workloads import CONFIGS, device_blocky_qk_bf16, device_iid_normal_bf16
    c = CONFIGS["qbsa"]
    N, D, seed = c["Nq"], c["D"], c["seed"]
    q = device_blocky_qk_bf16(seed, "q", 1, N, S, D, device)
    v = device_iid_normal_bf16(seed, 2, (1, N, S, D), device)
    nb = -(-S // 128)
    codes = torch.empty((1, N, S, D), dtype=torch.int8, device=device)
    qsc = torch.empty((1, N, nb), dtype=torch.float32, device=device)
    vcodes = torch.empty((1, N, S, D), dtype=torch.uint8, device=device)
    vsc = torch.empty((1, N, D), dtype=torch.float32, device=device)
    L = qb.lib()
    from quantized_block_sparse_attn_b200._binding import _ptr, _stream

    def qk():
        L.qbsa_quantize_qk(_ptr(q), 1, N, S, D, _ptr(codes), _ptr(qsc), _stream(device))

    def vq():
        L.qbsa_quantize_v(_ptr(v), 1, N, S, D, _ptr(vcodes), _ptr(vsc), _stream(device))

    qk_ms, _, _ = time_steps(qk, 10, 3, stream)
    v_ms, _, _ = time_steps(vq, 10, 3, stream)
    qb.check(device)
    qk_ms, v_ms = qk_ms / 10, v_ms / 10
    qk_bytes = N * S * D * 2 + N * S * D + N * nb * 4
    v_bytes = N * S * D * 2 + N * S * D + N * D * 4
    del q, v, codes, vcodes
    torch.cuda.empty_cache()
    return {"workload": f"quantisers B=1 N=40 S={S} D=128 (one tensor each)",
            "qk_ms": qk_ms, "qk_gbs": qk_bytes / (qk_ms / 1e3) / 1e9,
            "qk_frac_of_hbm": qk_bytes / (qk_ms / 1e3) / 1e9 / hbm_peak,
            "v_ms": v_ms, "v_gbs": v_bytes / (v_ms / 1e3) / 1e9,
            "v_frac_of_hbm": v_bytes / (v_ms / 1e3) / 1e9 / hbm_peak,
            "v_moved_frac_of_hbm": (v_bytes + N * S * D * 2) / (v_ms / 1e3) / 1e9 / hbm_peak,
            "algorithmic_bytes": "bf16 read once + 8-bit codes and fp32 scales written once",
            "v_moved_bytes": "V's column maxima span all of S, so its bf16 is read twice (maxima, then codes)",
            "kernels": "quantize_qk_kernel<128>; v_colmax_kernel<128> then v_quant_kernel<128> (V read twice)"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
