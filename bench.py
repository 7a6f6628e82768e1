"""Benchmark of the quantized attention forward on B200.

One step = one pass of the whole hot path over one batch: quantisation of
q, k, v (K mean, INT8 Q/K, FP8 V) followed by the fused attention kernel, on
the video-like workload B=1, H=12, N=32760 (21x30x52 token grid), d=128, bf16,
non-causal, mode I8QK_F8PV.  Inputs are resident in HBM when the timed region
starts; L2 is flushed (a 256 MiB write) between steps, outside the per-step
events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--mode i8f8|nvfp4|mxfp4] [--workload NAME] [--causal] [--q-per-token]
    python bench.py --sweep [--steps K]      # the B=4 H=32 sweep, all three modes

Prints ONE JSON line on rank 0 (the sweep: one per point and mode).  Step and
kernel times are medians over the timed steps.  Under torchrun (N > 1) every rank runs its own
copy of the workload (independent heads: no data exchange), the step time is
the max over ranks and ``value`` counts the operations of all ranks.
``--impl reference`` times the CPU oracle instead (rank 0 only), each step a
bounded sample of the same workload.
"""

import argparse
import json
import math
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
    import functools
    from oracle import attention as A
    from bit_quantized_attention_smooth_b200 import I8F8_LAZY_TAU
    emul = functools.partial(A.attn_quant_emul_i8f8, tau=I8F8_LAZY_TAU)
    qf, kf, vf = W.make_heads_f32(w, [(0, 0)])
    if rows_n is not None:
        rows = np.linspace(0, w.N - 1, rows_n).astype(np.int64)
        t0 = time.perf_counter()
        emul(qf, kf, vf, rows=rows)
        return 4.0 * rows_n * w.N * w.d, time.perf_counter() - t0, rows_n
    emul(qf, kf, vf, rows=np.arange(1))            # warm caches
    t0 = time.perf_counter()
    emul(qf, kf, vf, rows=np.arange(64))
    t64 = time.perf_counter() - t0
    t0 = time.perf_counter()
    emul(qf, kf, vf, rows=np.arange(320))
    t320 = time.perf_counter() - t0
    # fixed cost (the head's quantisation) plus a cost per row, fitted on two sizes
    per_row = max((t320 - t64) / 256, 1e-6)
    fixed = max(t64 - 64 * per_row, 0.0)
    rows_n = int(max(1, min(w.N, (target_s - fixed) / per_row)))
    rows = np.linspace(0, w.N - 1, rows_n).astype(np.int64)
    t0 = time.perf_counter()
    emul(qf, kf, vf, rows=rows)
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

PEAK_RATIO = {"i8f8": 2.0, "nvfp4": 4.0, "mxfp4": 4.0}   # dense INT8/FP8 = 2 x bf16, FP4 = 4 x bf16 (nominal)
DATASHEET = {"i8f8": 4500.0, "nvfp4": 9000.0, "mxfp4": 9000.0}  # dense TOPS


def median(xs):
    return statistics.median(xs) if xs else float("nan")


class ModeRunner:
    """One mode on one set of device inputs: its workspace, device-timed steps
    (quantize + attention, L2 flushed before each) and an accuracy sample."""

    def __init__(self, sattn, q, k, v, causal, mode, q_per_token, flush, p_per_token=False):
        self.sattn, self.q, self.k, self.v = sattn, q, k, v
        self.causal, self.mode, self.qtok, self.flush = causal, mode, q_per_token, flush
        self.ptok = p_per_token
        B, H, N, d = q.shape
        self.shape = (B, H, N, d)
        self.ws = torch.empty(sattn.workspace_bytes(B, H, N, d, mode=mode, dtype=q.dtype, q_per_token=q_per_token),
                              dtype=torch.uint8, device=q.device)
        self.out = torch.empty_like(q)

    def step(self, stream):
        s = self.sattn
        s.quantize(self.q, self.k, self.v, mode=self.mode, workspace=self.ws, q_per_token=self.qtok)
        mid = torch.cuda.Event(enable_timing=True)
        mid.record(stream)
        s.fwd_quantized(self.ws, self.shape, causal=self.causal, mode=self.mode, dtype=self.q.dtype, out=self.out,
                        q_per_token=self.qtok, p_per_token=self.ptok)
        return mid

    def timed(self, n, stream):
        """n steps; returns lists of (step ms, attention ms, quantize ms)."""
        evs = []
        for _ in range(n):
            self.flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e2 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e1 = self.step(stream)
            e2.record(stream)
            evs.append((e0, e1, e2))
        torch.cuda.synchronize()
        return ([a.elapsed_time(c) for a, b, c in evs], [b.elapsed_time(c) for a, b, c in evs],
                [a.elapsed_time(b) for a, b, c in evs])

    def warm(self, n, stream):
        for _ in range(n):
            self.flush.zero_()
            self.step(stream)
        torch.cuda.synchronize()

    def cosine_to_exact(self, heads, rows):
        """Cosine similarity of the output rows to exact float64 attention of the
        same device inputs (plain torch on the GPU), over the sampled heads x rows."""
        got, ref = [], []
        idx = torch.as_tensor(rows, device=self.q.device)
        B, H, N, d = self.shape
        scale = 1.0 / math.sqrt(d)
        for (b, h) in heads:
            qh = self.q[b, h].double()[idx]
            S = (qh @ self.k[b, h].double().T) * scale
            if self.causal:
                S = S.masked_fill(torch.arange(N, device=S.device)[None, :] > idx[:, None], float("-inf"))
            ref.append(torch.softmax(S, dim=1) @ self.v[b, h].double())
            got.append(self.out[b, h].double()[idx])
        a, b_ = torch.cat(got).flatten(), torch.cat(ref).flatten()
        return float(a @ b_ / (a.norm() * b_.norm()))


def accuracy_sample(w, n_rows=64, n_heads=2):
    heads = [(0, 0), (w.B - 1, w.H - 1)][:n_heads]
    rows = np.unique(np.linspace(0, w.N - 1, n_rows).astype(np.int64))
    return heads, rows


def attention_report(w, mode, causal, attn_ms, peaks):
    ops = w.ops()
    tops = ops / (attn_ms * 1e-3) / 1e12
    r = {"ms": attn_ms, "tops": tops, "frac_of_datasheet": tops / DATASHEET[mode],
         "frac_of_measured_peak": tops / (PEAK_RATIO[mode] * peaks["bf16_tflops"])}
    if causal:
        r["tops_causal_half_count"] = tops / 2     # the algorithmic work of a causal pass is half the pairs
    return r


def init_dist():
    ws_n, rank, local = dist_env()
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws_n, rank, local


def run_sweep(args):
    """The B=4, H=32 sweep (d in {64,128}, N in 1024..32768, causal and
    non-causal), in the three modes: one JSON line per point and mode.  Inputs follow
    the workload recipe but are drawn on the device (a different random stream
    from the CPU recipe the parity tests use), so that 1 GB tensors are made
    in milliseconds."""
    import bit_quantized_attention_smooth_b200 as sattn
    ws_n, rank, _ = init_dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, _ = measured_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for (d, N, causal) in W.SWEEP_POINTS:
        w = W.sweep(d, N, causal)
        q, k, v = W.make_inputs_device(w, dev)
        for mode in ("i8f8", "nvfp4", "mxfp4"):
            r = ModeRunner(sattn, q, k, v, causal, mode, False, flush)
            r.warm(args.warmup, stream)
            step_ms, attn_ms, quant_ms = r.timed(args.steps, stream)
            step_med, attn_med = max_over_ranks([median(step_ms), median(attn_ms)], dev)
            heads, rows = accuracy_sample(w, 32, 2)
            cos = r.cosine_to_exact(heads, rows)
            if rank == 0:
                print(json.dumps({"sweep": True, "workload": w.name, "mode": mode, "B": w.B, "H": w.H, "N": N, "d": d,
                                  "causal": causal, "steps": args.steps, "ms_per_step": step_med,
                                  "value": job_throughput(w.ops(), ws_n, step_med), "unit": "TOPS",
                                  "quantize_ms": median(quant_ms),
                                  "attention_kernel": attention_report(w, mode, causal, attn_med, peaks),
                                  "cos_vs_exact": cos, "accuracy_sample": f"{len(heads)} heads x {len(rows)} rows",
                                  "inputs": "device-drawn (same recipe, other random stream)"}), flush=True)
            del r
        del q, k, v
        torch.cuda.empty_cache()
    if ws_n > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def run_gpu(args):
    import bit_quantized_attention_smooth_b200 as sattn
    ws_n, rank, local = init_dist()
    dev = torch.device("cuda", torch.cuda.current_device())
    w = W.WORKLOADS[args.workload]
    causal = bool(args.causal)
    q, k, v = W.make_inputs(w, dev)
    B, H, N, d = q.shape
    ops = w.ops()
    mode = args.mode
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    main = ModeRunner(sattn, q, k, v, causal, mode, args.q_per_token, flush)
    main.warm(args.warmup, stream)
    if args.profile:
        # Profiling mode (for ncu): the same steps, no e2e leg, no CPU baseline.
        for _ in range(args.steps):
            flush.zero_()
            main.step(stream)
        torch.cuda.synchronize()
        print(json.dumps({"profile": True, "workload": w.name, "mode": mode, "steps": args.steps,
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
    sattn.kernel_launches(reset=True)
    step_ms, attn_ms, quant_ms = main.timed(args.steps, stream)
    launches = sattn.kernel_launches()
    barrier()
    clocks = sampler.stop()
    ms, attn_med = max_over_ranks([median(step_ms), median(attn_ms)], dev)
    heads, rows = accuracy_sample(w)
    cos_main = main.cosine_to_exact(heads, rows)

    # the other mode on the same inputs, and per-token Q scales (I8QK_F8PV), beside the headline
    legs = {}
    for name, (m, qtok, ptok) in {"nvfp4": ("nvfp4", False, False), "i8f8": ("i8f8", False, False),
                                  "i8f8_q_per_token": ("i8f8", True, False),
                                  "i8f8_p_per_token": ("i8f8", False, True),
                                  "mxfp4": ("mxfp4", False, False)}.items():
        if m == mode and qtok == args.q_per_token and not ptok:
            continue
        r = ModeRunner(sattn, q, k, v, causal, m, qtok, flush, p_per_token=ptok)
        r.warm(args.warmup, stream)
        o_step, o_attn, o_quant = r.timed(args.steps, stream)
        legs[name] = {"ms_per_step": median(o_step), "quantize_ms": median(o_quant),
                      "value": ops / (median(o_step) * 1e-3) / 1e12,
                      "attention_kernel_ms": median(o_attn), "cos_vs_exact": r.cosine_to_exact(heads, rows)}
        del r

    # ---- end to end through the C-ABI call on host buffers (pinned): every
    # step copies q, k, v in and the output back, pipelined by the library in
    # chunks of heads (sattn_fwd_host)
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()

    def e2e_step():
        sattn.fwd_host(hq, hk, hv, out=hout, causal=causal, mode=mode, q_per_token=args.q_per_token)

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
        peak = PEAK_RATIO[mode] * peaks["bf16_tflops"]
        att = attention_report(w, mode, causal, attn_med, peaks)
        achieved = att["tops"] / (2 if causal else 1)   # algorithmic work: a causal pass does half the pairs
        for name, leg in legs.items():
            m = name if name in ("nvfp4", "mxfp4") else "i8f8"
            leg["attention_kernel"] = attention_report(w, m, causal, leg.pop("attention_kernel_ms"), peaks)
        traffic = None
        tpath = os.path.join(ROOT, "profiles", f"attn_{mode}_traffic.json")
        if os.path.exists(tpath):
            with open(tpath) as f:
                tj = json.load(f)
            # the record is of the dense non-causal kernel on this workload
            if tj.get("kernel_hash") == kernel_hash(mode) and tj.get("workload") == w.name and not causal:
                traffic = tj.get("dram_bytes_per_launch_full")
        quant = quantizer_roofline(sattn, w, q, mode, args.q_per_token, median(quant_ms), peaks, src)
        cpu = None
        if ws_n == 1 and not args.no_cpu_baseline:
            cpu_ops, cpu_s, rows_n = oracle_sample(w, args.cpu_seconds)
            cpu = {"value": cpu_ops / cpu_s / 1e12, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"head 0 of {w.H}, {rows_n} query rows x {w.N} keys, full-head quantisation "
                             f"included ({cpu_s:.1f} s); numpy float64 BLAS"}
        value = job_throughput(ops, ws_n, ms)
        try:                       # a reported second bound; never lose the bench line over it
            sm_mhz = clocks["sm_mhz"] if clocks and clocks.get("sm_mhz") else 1965.0
            pairs = float(w.B) * w.H * w.N * w.N / (2 if causal else 1)
            mufu = mufu_bound(pairs, attn_med, torch.cuda.get_device_properties(dev).multi_processor_count, sm_mhz)
            mufu["binds"] = mufu["frac"] > achieved / peak      # the bound this kernel is closer to
        except Exception as exc:   # noqa: BLE001
            mufu = {"bound": "mufu", "error": repr(exc)}
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": ws_n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"i8f8": "int8 QK^T / e4m3 PV (fp32 softmax + accumulation)",
                      "nvfp4": "nvfp4 QK^T / nvfp4 PV (e2m1 + e4m3 block scales; fp32 softmax + accumulation)",
                      "mxfp4": "mxfp4 QK^T / mxfp4 PV (e2m1 + e8m0 block scales; fp32 softmax + accumulation)"}[mode],
            "data": "synthetic",
            "config": {"workload": w.name, "mode": {"i8f8": "I8QK_F8PV", "nvfp4": "NVFP4", "mxfp4": "MXFP4"}[mode], "B": w.B, "H": w.H,
                       "N": w.N, "d": w.d, "causal": causal, "io_dtype": w.dtype,
                       "q_scales": "per token" if args.q_per_token else "per 128-token block",
                       "lazy_max_tau": sattn.I8F8_LAZY_TAU if mode == "i8f8" else None,
                       "parallelism": f"replicas x{ws_n} (independent heads)",
                       "l2": "flushed between steps (256 MiB write, outside the step events)"},
            "attention_kernel": att,
            "quantize_ms": median(quant_ms),
            "timing": "median of the timed steps (CUDA events on the launching stream); max over ranks",
            "accuracy": {"cos_vs_exact": cos_main, "sample": f"{len(heads)} heads x {len(rows)} rows, "
                                                             "exact float64 attention of the same device inputs"},
            "other_legs": legs,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{src}: {PEAK_RATIO[mode]:.0f} x bf16 burst {peaks['bf16_tflops']} "
                                        f"(nominal dense ratio of {mode} to bf16)"},
            "roofline_mufu": mufu,
            "roofline_quantize": quant,
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(ops, ws_n, e2e_ms), "unit": "TOPS",
                    "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                    "d2h_bytes_per_step": q.numel() * q.element_size(), "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clocks,
            "device_error_word": err,
        }
    if ws_n > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def kernel_hash(mode="i8f8", files=None):
    """Hash of the sources a kernel is built from (the attention kernel of
    `mode` by default): a recorded ncu traffic figure is reported only while
    it matches."""
    import hashlib
    h = hashlib.sha256()
    for f in files or (f"attn_{'i8f8' if mode == 'i8f8' else 'nvfp4'}.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "bit_quantized_attention_smooth_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


QUANT_SOURCES = ("quant_fused.cuh", "quant_i8f8.cuh", "quant_nvfp4.cuh", "ptx.cuh")


def quantizer_roofline(sattn, w, q, mode, q_per_token, quant_ms, peaks, src):
    """HBM roofline of the quantiser (one launch, after one memset): its
    algorithmic bytes are Q, K, V read once and the codes and scales written
    once (the workspace sections before the scratch), over its device time."""
    B, H, N, d = q.shape
    lay = sattn.workspace_layout(B, H, N, d, mode=mode, dtype=q.dtype, q_per_token=q_per_token)
    read = 3 * q.numel() * q.element_size()
    write = lay["ksum"] - lay["q8"]
    achieved = (read + write) / (quant_ms * 1e-3) / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", f"quant_{mode}_traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tj = json.load(f)
        if (tj.get("kernel_hash") == kernel_hash(files=QUANT_SOURCES) and tj.get("workload") == w.name
                and tj.get("q_per_token", False) == bool(q_per_token)):
            traffic = tj.get("dram_bytes_per_launch_full")
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "algorithmic_bytes": read + write,
            "ms": quant_ms, "peak_source": f"{src}: copy bandwidth"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sattn", choices=["sattn", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)   # the two-size fit underestimates large samples
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="i8f8", choices=["i8f8", "nvfp4", "mxfp4"])
    ap.add_argument("--workload", default=WORKLOAD.name, choices=sorted(W.WORKLOADS))
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--q-per-token", action="store_true", help="I8QK_F8PV with one Q scale per token")
    ap.add_argument("--sweep", action="store_true",
                    help="time the B=4 H=32 sweep in the three modes (one JSON line per point and mode)")
    ap.add_argument("--profile", action="store_true",
                    help="run warm-up + steps of the GPU path only (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
