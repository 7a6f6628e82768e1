"""Benchmark of the quantized attention forward on B200.

One step = one pass of the whole hot path over one batch: quantisation of
q, k, v (K mean, INT8 Q/K, FP8 V) followed by the fused attention kernel, on
the video-like workload B=1, H=12, N=32760 (21x30x52 token grid), d=128, bf16,
non-causal, mode I8QK_F8PV.  Inputs are resident in HBM when the timed region
starts; L2 is flushed (a 256 MiB write) between steps, outside the per-step
events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) every rank runs its own
copy of the workload (independent heads: no data exchange), the step time is
the max over ranks and ``value`` counts the operations of all ranks.
``--impl reference`` times the CPU oracle instead (rank 0 only), each step a
bounded sample of the same workload.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

import workloads as W

METRIC = "quantized attention fwd TOPS (4*B*H*N^2*d/s) and % of B200 dense tensor peak"
ROOT = os.path.dirname(os.path.abspath(__file__))
WORKLOAD = W.VIDEO_32760
MODE = "i8f8"
L2_FLUSH_BYTES = 256 << 20


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def max_over_ranks(values, device="cpu"):
    """Element-wise max of a list of floats over all ranks (identity with one rank).

    Device-timed step times are combined this way: the job's time is the slowest
    rank's.  Works with gloo (CPU tensors) and NCCL (CUDA tensors)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(ops_per_rank, world, ms_max):
    """Whole-job TOPS: operations of all ranks over the slowest rank's time."""
    return world * ops_per_rank / (ms_max * 1e-3) / 1e12


def mufu_bound(pairs, attn_ms, sm_count, sm_mhz):
    """The attention kernel's second roofline: one ex2 per (query, key) pair on
    the special-function unit, 16 results per clock per SM (measured on this
    part), at the SM clock seen during the timed region."""
    achieved = pairs / (attn_ms * 1e-3)
    peak = sm_count * 16 * sm_mhz * 1e6
    return {"bound": "mufu", "achieved": achieved, "peak": peak, "unit": "exp2/s", "frac": achieved / peak,
            "peak_source": f"{sm_count} SMs x 16 exp2/clk x {sm_mhz:.0f} MHz"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
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
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        if not sm:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows if len(r) >= 9 for i in range(4) if r[5 + i].strip() == "Active"})
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(sm)}


# ---------------------------------------------------------------------------- oracle arm

def oracle_sample(w, target_s, rows_n=None):
    """Time the CPU oracle on head 0 of the workload; rows sized to ~target_s.

    Returns (ops processed, seconds, rows).  Quantisation of the whole head is
    part of every sample (the oracle always quantises full heads)."""
    from oracle import attention as A
    qf, kf, vf = W.make_heads_f32(w, [(0, 0)])
    if rows_n is not None:
        rows = np.linspace(0, w.N - 1, rows_n).astype(np.int64)
        t0 = time.perf_counter()
        A.attn_quant_emul_i8f8(qf, kf, vf, rows=rows)
        return 4.0 * rows_n * w.N * w.d, time.perf_counter() - t0, rows_n
    A.attn_quant_emul_i8f8(qf, kf, vf, rows=np.arange(1))            # warm caches
    t0 = time.perf_counter()
    A.attn_quant_emul_i8f8(qf, kf, vf, rows=np.arange(65))
    t65 = time.perf_counter() - t0
    # linear through the origin: over-estimates the per-row cost (the time
    # includes the head's quantisation), so the sample stays within target_s
    rows_n = int(max(1, min(w.N, 65 * target_s / t65)))
    rows = np.linspace(0, w.N - 1, rows_n).astype(np.int64)
    t0 = time.perf_counter()
    A.attn_quant_emul_i8f8(qf, kf, vf, rows=rows)
    dt = time.perf_counter() - t0
    return 4.0 * rows_n * w.N * w.d, dt, rows_n


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOAD
    per_step = min(4.0, 150.0 / max(1, args.steps + args.warmup))
    _, _, rows_n = oracle_sample(w, per_step)            # calibration (untimed)
    for _ in range(args.warmup):
        oracle_sample(w, per_step, rows_n)
    ops, secs = 0.0, 0.0
    rows_used = 0
    for _ in range(args.steps):
        o, t, r = oracle_sample(w, per_step, rows_n)
        ops += o
        secs += t
        rows_used = r
    value = ops / secs / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "mode": "I8QK_F8PV", "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": False, "io_dtype": w.dtype},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": f"head 0, {rows_used} query rows x {w.N} keys per step, full-head "
                                   f"quantisation included; numpy float64 BLAS"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------- GPU arm

def run_gpu(args):
    import bit_quantized_attention_smooth_b200 as sattn
    ws_n, rank, local = dist_env()
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    w = WORKLOAD
    q, k, v = W.make_inputs(w, dev)
    B, H, N, d = q.shape
    ops = w.ops()
    mode = args.mode
    workspace = torch.empty(sattn.workspace_bytes(B, H, N, d, mode=mode), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(m=mode, ws=workspace):
        sattn.quantize(q, k, v, mode=m, workspace=ws)
        ev_mid = torch.cuda.Event(enable_timing=True)
        ev_mid.record(stream)
        sattn.fwd_quantized(ws, (B, H, N, d), mode=m, dtype=q.dtype, out=out)
        return ev_mid

    def timed_steps(n, m=mode, ws=workspace):
        """n device-timed steps with an L2 flush before each; returns (step ms list, attention ms list)."""
        evs = []
        for _ in range(n):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e2 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e1 = step(m, ws)
            e2.record(stream)
            evs.append((e0, e1, e2))
        torch.cuda.synchronize()
        return [a.elapsed_time(c) for a, b, c in evs], [b.elapsed_time(c) for a, b, c in evs], \
            [a.elapsed_time(b) for a, b, c in evs]

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if args.profile:
        # Profiling mode (for ncu): the same steps, no e2e leg, no CPU baseline.
        for _ in range(args.steps):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        print(json.dumps({"profile": True, "workload": w.name, "steps": args.steps,
                          "device_error_word": sattn.device_error()}), flush=True)
        return 0

    def barrier():
        if ws_n > 1:
            torch.distributed.barrier()

    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    step_ms, attn_ms, quant_ms = timed_steps(args.steps)
    barrier()
    clocks = sampler.stop()
    # the other mode on the same inputs (reported beside the headline mode)
    other = "nvfp4" if mode == "i8f8" else "i8f8"
    ws_other = torch.empty(sattn.workspace_bytes(B, H, N, d, mode=other), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step(other, ws_other)
    o_step, o_attn, o_quant = timed_steps(args.steps, other, ws_other)
    del ws_other
    ms = sum(step_ms) / len(step_ms)
    attn_avg = sum(attn_ms) / len(attn_ms)
    ms, attn_avg = max_over_ranks([ms, attn_avg], dev)

    # ---- end to end through the C-ABI call on host buffers (pinned): every
    # step copies q, k, v in and the output back, pipelined by the library in
    # chunks of heads (sattn_fwd_host)
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()

    def e2e_step():
        sattn.fwd_host(hq, hk, hv, out=hout, mode=mode)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e_start.elapsed_time(e_end) / args.steps], dev)[0]
    err = sattn.device_error()

    line = None
    if rank == 0:
        peaks, src = measured_peaks()
        ratio = {"i8f8": 2.0, "nvfp4": 4.0}               # dense INT8/FP8 = 2 x bf16, FP4 = 4 x bf16 (nominal)
        datasheet = {"i8f8": 4500.0, "nvfp4": 9000.0}
        peak_i8 = ratio[mode] * peaks["bf16_tflops"]
        achieved = ops / (attn_avg * 1e-3) / 1e12
        o_ms, o_attn_avg = sum(o_step) / len(o_step), sum(o_attn) / len(o_attn)
        o_achieved = ops / (o_attn_avg * 1e-3) / 1e12
        other_line = {"mode": other, "value": ops / (o_ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": o_ms,
                      "attention_kernel": {"ms": o_attn_avg, "tops": o_achieved,
                                           "frac_of_datasheet": o_achieved / datasheet[other],
                                           "frac_of_measured_peak": o_achieved / (ratio[other] * peaks["bf16_tflops"])},
                      "quantize_ms": sum(o_quant) / len(o_quant)}
        traffic = None
        tpath = os.path.join(ROOT, "profiles", "attn_i8f8_traffic.json")
        if os.path.exists(tpath):
            with open(tpath) as f:
                tj = json.load(f)
            if tj.get("kernel_hash") == kernel_hash():
                traffic = tj.get("dram_bytes_per_launch_full")
        cpu = None
        if ws_n == 1 and not args.no_cpu_baseline:
            cpu_ops, cpu_s, rows_n = oracle_sample(w, args.cpu_seconds)
            cpu = {"value": cpu_ops / cpu_s / 1e12, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"head 0 of {w.H}, {rows_n} query rows x {w.N} keys, full-head quantisation "
                             f"included ({cpu_s:.1f} s); numpy float64 BLAS"}
        value = job_throughput(ops, ws_n, ms)
        try:                       # a reported second bound; never lose the bench line over it
            sm_mhz = clocks["sm_mhz"] if clocks and clocks.get("sm_mhz") else 1965.0
            mufu = mufu_bound(float(w.B) * w.H * w.N * w.N, attn_avg,
                              torch.cuda.get_device_properties(dev).multi_processor_count, sm_mhz)
            mufu["binds"] = mufu["frac"] > achieved / peak_i8      # the bound this kernel is closer to
        except Exception as exc:   # noqa: BLE001
            mufu = {"bound": "mufu", "error": repr(exc)}
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws_n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("int8 QK^T / e4m3 PV (fp32 softmax + accumulation)" if mode == "i8f8"
                      else "nvfp4 QK^T / nvfp4 PV (e2m1 + e4m3 block scales; fp32 softmax + accumulation)"),
            "data": "synthetic",
            "config": {"workload": w.name, "mode": "I8QK_F8PV" if mode == "i8f8" else "NVFP4", "B": w.B, "H": w.H,
                       "N": w.N, "d": w.d,
                       "causal": False, "io_dtype": w.dtype, "parallelism": f"replicas x{ws_n} (independent heads)",
                       "l2": "flushed between steps (256 MiB write, outside the step events)"},
            "attention_kernel": {"ms": attn_avg, "tops": achieved,
                                 "frac_of_datasheet": achieved / datasheet[mode]},
            "other_mode": other_line,
            "quantize_ms": sum(quant_ms) / len(quant_ms),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_i8, "unit": "TFLOP/s",
                         "frac": achieved / peak_i8, "traffic": traffic,
                         "peak_source": f"{src}: {ratio[mode]:.0f} x bf16 burst {peaks['bf16_tflops']} "
                                        f"(nominal dense ratio of {mode} to bf16)"},
            "roofline_mufu": mufu,
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(ops, ws_n, e2e_ms), "unit": "TOPS",
                    "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": e2e_ms},
            "gpu_launches": 5 * args.steps,   # per step: stats, quant Q, quant K, quant V, attention
            "clocks": clocks,
            "device_error_word": err,
        }
    if ws_n > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def kernel_hash():
    import hashlib
    h = hashlib.sha256()
    for f in ("attn_i8f8.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "bit_quantized_attention_smooth_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sattn", choices=["sattn", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="i8f8", choices=["i8f8", "nvfp4"])
    ap.add_argument("--profile", action="store_true",
                    help="run warm-up + steps of the GPU path only (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
