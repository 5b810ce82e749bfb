"""Benchmark: exact-attention forward TFLOP/s on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward pass (the whole hot path: schedule, TMA loads, S = QK^T,
online softmax, O += PV, epilogue) over one batch of the workload, inputs
resident in HBM.  L2 is flushed (a 256 MiB write) before every timed step; the
flush is outside the CUDA-event-timed interval.  FLOPs: 4*B*H*N^2*d, halved for
causal, summed per sequence for varlen.

N > 1 (torchrun): every rank runs an independent replica of the workload on its
own GPU (the forward pass needs no exchange); value = all ranks' FLOPs / the
slowest rank's time (max over ranks).

--impl reference times the fp64 CPU oracle (the correctness reference, not a
tuned program) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import attn_inputs as ai  # noqa: E402

METRIC = "attention fwd TFLOP/s (bf16, d=128, 1 B200) and % of dense-BF16 tensor peak"
METRIC_E4M3 = "attention fwd TFLOP/s (e4m3 inputs, d=128, 1 B200) and % of dense-FP8 tensor peak"


FLUSH_BYTES = 256 << 20
MUFU_EX2_PER_CLK_PER_SM = 16  # 4 SFU lanes per SM sub-partition, 4 sub-partitions


def metric_for(w: ai.Workload) -> str:
    return METRIC_E4M3 if w.e4m3 else METRIC


def visible_pairs(L: int, causal: bool, window=None) -> float:
    """(query, key) pairs a sequence of length L attends to.  Causal without a
    window counts L^2/2 (the convention of the published causal TFLOP/s figures);
    under a sliding window the exact count."""
    if window is None:
        return L * L / 2.0 if causal else float(L * L)
    import numpy as np
    i = np.arange(L, dtype=np.int64)
    wl, wr = window
    lo = np.maximum(i - wl, 0) if wl >= 0 else np.zeros_like(i)
    hi = np.full_like(i, L - 1)
    if wr >= 0:
        hi = np.minimum(hi, i + wr)
    if causal:
        hi = np.minimum(hi, i)
    return float((hi - lo + 1).sum())


def workload_flops(w: ai.Workload) -> float:
    return sum(4.0 * w.H * w.d * visible_pairs(L, w.causal, w.window) for L in w.seq_lengths())


def workload_exps(w: ai.Workload) -> float:
    """Score elements the method exponentiates (visible (query, key) pairs)."""
    return workload_flops(w) / (4.0 * w.d)


def _code_only(text: str) -> str:
    """C/C++ source with comments and blank lines removed (string literals in these
    files hold PTX, which has no comment markers)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def _device_part(text: str) -> str:
    """The kernel file up to its host-side launch functions (which only pick the
    template instantiation to launch)."""
    cut = text.find("\nint fwd_smem_bytes(")
    return text if cut < 0 else text[:cut]


def kernel_source_hash() -> str:
    """sha256 of the forward kernel's device sources without comments (the ncu
    traffic figure applies only to the kernel these hash to)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_103_b200", "csrc")
    for name in ("attn_fwd_sm100.cu", "attn_fwd_sm100.h", "sm100_ptx.cuh", "softmax_math.cuh",
                 "exp2_poly.h"):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        if name.endswith(".cu"):
            text = _device_part(text)
        h.update(_code_only(text).encode())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed machine-readable ncu record of this
    workload (``profiles/fwd_kernel_<workload>.json``), or None when there is none
    or it was taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", f"fwd_kernel_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"),
                "sm_max_mhz": p.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0, "source": "fallback"}


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no samples
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for name, bit in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.002)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()
            if not self.samples:
                try:
                    self._sample()
                except Exception:
                    pass

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_setup(gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's value (NCCL on the GPU; gloo tests pass device="cpu")."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """All ranks' FLOPs (each rank runs one replica) over the slowest rank's time."""
    return world * flops_per_step * steps / (max_total_ms / 1e3) / 1e12


def make_inputs(w: ai.Workload, device):
    """CPU inputs of a workload: (q, k, v, cu_seqlens); E4M3 workloads give the
    8-bit tensors (their per-tensor scales come from e4m3_scales)."""
    if w.e4m3:
        q, k, v, _ = ai.make_qkv_e4m3(w)
    else:
        q, k, v = ai.make_qkv(w)
    cu = None
    if w.varlen:
        cu = torch.tensor(w.cu_seqlens(), dtype=torch.int32)
    return q, k, v, cu


def e4m3_scales(w: ai.Workload):
    return ai.make_qkv_e4m3(w)[3] if w.e4m3 else None


def cpu_oracle_sample(w: ai.Workload, q, k, v, budget_s: float):
    """Times the fp64 oracle on whole (sequence, head) units of the workload until
    about budget_s of CPU time is spent; returns (TFLOP/s, threads, description).
    E4M3 inputs are dequantised (x8 * scale) first, outside the timing.  Returns
    (TFLOP/s, threads, description, seconds spent)."""
    import numpy as np
    import oracle
    lengths = w.seq_lengths()
    cu = np.concatenate([[0], np.cumsum(lengths)])
    if w.e4m3:
        scales = e4m3_scales(w)
        q, k, v = (t.double() * sc for t, sc in zip((q, k, v), scales))
    # fp64 copies made once, outside the timing (the oracle takes fp64 arrays as they are)
    qp, kp, vp = (np.ascontiguousarray(t.reshape(-1, w.H, w.d).double().numpy()) for t in (q, k, v))
    scale = 1.0 / math.sqrt(w.d)
    done_flops, spent, units, threads = 0.0, 0.0, 0, 0
    order = sorted(range(len(lengths)), key=lambda b: lengths[b])  # cheapest sequences first
    for b in order:
        L = lengths[b]
        sl = slice(int(cu[b]), int(cu[b + 1]))
        for h in range(w.H):
            rows = np.arange(cu[b], cu[b + 1])
            heads = np.full(L, h)
            t0 = time.perf_counter()
            oracle.fwd_rows(qp, kp, vp, cu, w.causal, scale, rows, heads, window=w.window)
            spent += time.perf_counter() - t0
            f = 4.0 * w.d * visible_pairs(L, w.causal, w.window)
            done_flops += f
            units += 1
            if spent >= budget_s:
                break
        if spent >= budget_s:
            break
        del sl
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = f"{units} of {len(lengths) * w.H} (sequence, head) units, {done_flops / 1e9:.1f} GFLOP"
    return done_flops / spent / 1e12, threads, desc, spent


def bench_config(w: ai.Workload, world: int) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "window": w.window, "global_batch": w.B * world, "seq_len": w.N, "parallelism": f"replicas{world}",
            "l2": "flushed (256 MiB write) before every timed step"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores.  Each step is a bounded
    sample of the workload (whole (sequence, head) units until about --ref-seconds
    of CPU time); value = the sample's FLOPs over its time, ms_per_step = the
    sample's time (what was actually run), and the time the whole workload would
    take at that rate is reported separately."""
    if rank != 0:
        return
    w = ai.ALL[args.workload]
    q, k, v, _ = make_inputs(w, "cpu")
    flops = workload_flops(w)
    import oracle
    oracle.build()
    vals, step_ms = [], []
    per_step = args.ref_seconds
    desc, threads = "", 0
    for i in range(args.warmup + args.steps):
        tf, threads, desc, spent = cpu_oracle_sample(w, q, k, v, per_step)
        if i >= args.warmup:
            vals.append(tf)
            step_ms.append(spent * 1e3)
    value = statistics.median(vals)
    line = {"metric": metric_for(w), "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(step_ms),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": bench_config(w, world),
            "step": f"a bounded sample of the workload: {desc}",
            "workload_ms_at_this_rate": flops / (value * 1e12) * 1e3,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    import exact_attention_103_b200 as ea
    ea.load_library()
    if args.workload == ai.BWD_NAME:
        return run_bwd(args, rank, world, local)
    w = ai.ALL[args.workload]
    dev = torch.device("cuda", local)
    q_h, k_h, v_h, cu_h = make_inputs(w, "cpu")
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    cu = None if cu_h is None else cu_h.to(dev)
    max_len = w.N if w.varlen else None
    scale = 1.0 / math.sqrt(w.d)
    f8 = e4m3_scales(w)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse_shape = (w.H, w.total_tokens) if w.varlen else (w.B, w.H, w.N)
    lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flops = workload_flops(w)
    peaks = load_peaks()

    def step():
        ea.fwd(q, k, v, causal=w.causal, scale=scale, cu_seqlens=cu, max_seqlen=max_len,
               out=out, lse=lse, window=w.window, exp_poly_per8=args.exp_poly_per8,
               e4m3_scales=f8, cta_pair=args.cta_pair)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    ea.get_device_status()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
    barrier(world)
    ea.get_device_status()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(times), world)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(flops, args.steps, world, total_ms)

    # One untimed launch with the kernel's counters on: how often the conditional
    # rescale fired (the counters are not kept under a sliding window).
    # Also at tau = 0 (rescale whenever a row's maximum grows: the rule the pages'
    # skip-rate figure compares against).
    rescale = None
    if w.window is None:
        rescale = {}
        for tau in (None, 0.0):
            counters = torch.zeros(2, dtype=torch.int64, device=dev)
            ea.fwd(q, k, v, causal=w.causal, scale=scale, cu_seqlens=cu, max_seqlen=max_len,
                   out=out, lse=lse, exp_poly_per8=args.exp_poly_per8, e4m3_scales=f8,
                   stats=counters, cta_pair=args.cta_pair, rescale_threshold=tau)
            ea.get_device_status()
            rescaled, row_tiles = (int(x) for x in counters.cpu())
            key = "default" if tau is None else "tau0"
            rescale[key] = {"tau_log2": (4.0 if w.e4m3 else 8.0) if tau is None else tau,
                            "rows_rescaled": rescaled, "row_tiles_after_first": row_tiles,
                            "skip_rate": (1.0 - rescaled / row_tiles) if row_tiles else None}
    achieved = flops / (statistics.mean(times) / 1e3) / 1e12  # per launch, this rank
    clk = clocks.summary()
    # The denominator: the measured cuBLAS bf16 peak as a burst (each launch is one
    # whole step, timed on its own).  When the power cap was active during the timed
    # region the fraction of the sustained figure (seconds-long, under the cap) is
    # reported beside it, for context only.  An E4M3 contraction's peak: that x the
    # nominal 2x ratio of dense FP8 to BF16 tensor throughput.
    ratio = 2.0 if w.e4m3 else 1.0
    peak = peaks["bf16_tflops"] * ratio
    capped = "sw_power_cap" in clk["reasons"] and peaks.get("bf16_tflops_sustained")
    frac_sustained = achieved / (peaks["bf16_tflops_sustained"] * ratio) if capped else None
    peak_source = (f"bf16_tflops (burst) x 2 (nominal e4m3/bf16), {peaks['source']}" if w.e4m3
                   else f"bf16_tflops (burst), {peaks['source']}")
    mhz = clk["sm_mhz"] or peaks["sm_max_mhz"]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mufu_peak = sms * MUFU_EX2_PER_CLK_PER_SM * mhz * 1e6
    mufu_share = 1.0 - args.exp_poly_per8 / 8.0
    mufu_achieved = mufu_share * workload_exps(w) / (statistics.mean(times) / 1e3)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(args, ea, w, q_h, k_h, v_h, cu_h, out, lse, scale, max_len, f8, dev,
                          world, flops)
    barrier(world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, threads, desc, _ = cpu_oracle_sample(w, q_h, k_h, v_h, args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {"metric": metric_for(w), "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e4m3" if w.e4m3 else "bf16", "data": "synthetic",
                "config": bench_config(w, world),
                "options": {"exp_poly_per8": args.exp_poly_per8, "cta_pair": args.cta_pair},
                "rescale": rescale,
                "pct_of_peak": 100.0 * achieved / peak,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                             "unit": "TFLOP/s", "frac": achieved / peak,
                             "peak_source": peak_source,
                             "frac_of_sustained_peak": frac_sustained,
                             "traffic": profiled_traffic(w.name),
                             "traffic_unit": "bytes per launch (ncu dram read+write)"},
                "mufu": {"achieved_ex2_per_s": mufu_achieved, "peak_ex2_per_s": mufu_peak,
                         "frac": mufu_achieved / mufu_peak,
                         "mufu_share_of_exps": mufu_share,
                         "note": "ex2 executed on MUFU (the rest on the FMA-pipe polynomial); "
                                 "peak = SMs x 16 ex2/clk at the median sampled SM clock"},
                "e2e": e2e,
                "gpu_launches": args.steps,
                "clocks": clk,
                "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)


def measure_e2e(args, ea, w, q_h, k_h, v_h, cu_h, out, lse, scale, max_len, f8, dev, world,
                flops):
    # End to end through the public API from pinned host buffers: every call copies
    # its Q/K/V (and cu_seqlens) to the device, runs the forward and copies O and
    # LSE back; HostPipeline overlaps neighbouring calls' copies with compute.
    q_p, k_p, v_p = (t.pin_memory() for t in (q_h, k_h, v_h))
    cu_p = None if cu_h is None else cu_h.pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    o_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    l_host = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    pipe = ea.HostPipeline(q_h.shape, causal=w.causal, scale=scale, cu_seqlens_host=cu_p,
                           max_seqlen=max_len, device=str(dev), window=w.window,
                           exp_poly_per8=args.exp_poly_per8, e4m3_scales=f8)
    for _ in range(2):
        pipe.submit(q_p, k_p, v_p, o_host, l_host)
    pipe.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.streams[0])
    for _ in range(e2e_steps):
        pipe.submit(q_p, k_p, v_p, o_host, l_host)
    e1.record(pipe.streams[2])
    pipe.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    o_h, l_h = o_host, l_host
    h2d = 3 * q_h.numel() * q_h.element_size() + (0 if cu_h is None else cu_h.numel() * 4)
    d2h = o_h.numel() * 2 + l_h.numel() * 4
    barrier(world)

    return {"value": world * flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "api": "HostPipeline (2 device buffer sets, copy-in / compute / copy-out streams)"}


def run_bwd(args, rank, world, local):
    """Backward of the causal B2-H16-N8192-d128 problem: a step is one attn_bwd call
    (D = rowsum(dO*O), dK/dV kernel, dQ kernel) with O and LSE from an untimed forward.
    FLOPs counted as 2.5x the forward's."""
    import exact_attention_103_b200 as ea
    w = ai.BWD_CAUSAL
    dev = torch.device("cuda", local)
    q, k, v, do = (t.to(dev) for t in ai.make_qkv(w, with_dout=True))
    scale = 1.0 / math.sqrt(w.d)
    o, lse = ea.fwd(q, k, v, causal=True, scale=scale)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flops = 2.5 * workload_flops(w)
    peaks = load_peaks()
    for _ in range(args.warmup):
        flush.fill_(1.0)
        ea.bwd(q, k, v, o, lse, do, causal=True, scale=scale)
    ea.get_device_status()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record()
            ea.bwd(q, k, v, o, lse, do, causal=True, scale=scale)
            ends[i].record()
        torch.cuda.synchronize()
    barrier(world)
    ea.get_device_status()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(times), world)
    value = whole_job_tflops(flops, args.steps, world, total_ms)
    achieved = flops / (statistics.mean(times) / 1e3) / 1e12
    if rank == 0:
        cfg = bench_config(w, world)
        cfg["workload"] = ai.BWD_NAME
        line = {"metric": "attention bwd TFLOP/s (bf16, d=128, 1 B200; 2.5x forward FLOPs)",
                "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic", "config": cfg,
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                             "traffic": None},
                "gpu_launches": 3 * args.steps, "clocks": clocks.summary()}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=ai.VARLEN.name, choices=sorted(ai.ALL) + [ai.BWD_NAME])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU time of the cpu_baseline sample (our arm, rank 0, N=1)")
    ap.add_argument("--ref-seconds", type=float, default=2.0,
                    help="CPU time of each reference-arm step (a bounded sample)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (profiling runs only)")
    ap.add_argument("--cta-pair", action="store_true",
                    help="clusters of two CTAs sharing each item (tcgen05.mma.cta_group::2)")
    ap.add_argument("--exp-poly-per8", type=int, default=0, choices=[0, 2, 8],
                    help="exponential pairs of every 8 computed by the FMA-pipe polynomial")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
