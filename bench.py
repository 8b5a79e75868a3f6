"""Benchmark of the NVFP4 W4A4 linear (quantize + GEMM) on Qwen3-8B-shaped
prefill projections at 8192 tokens: QKV (4096 -> 6144), O (4096 -> 4096),
gate/up (4096 -> 24576), down (12288 -> 4096).

One step = the four projections, each: tensor scale of X, NVFP4 quantization
of X, block-scaled FP4 GEMM against the pre-quantized weight (weights are
quantized once, outside the timed region).  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (plain C + numpy binary64) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_w4a4_quantized_03_b200 import inputs  # noqa: E402

TOKENS = 8192
METRIC = "W4A4 NVFP4 linear TFLOPS (quant+GEMM) & % of B200 FP4 peak; quant GB/s"
WORKLOAD = "qwen3-8b prefill projections (qkv, o, gate_up, down) at 8192 tokens, NVFP4 W4A4"


def _traffic(record: str, key: str):
    """DRAM bytes from a committed ncu capture (profiles/<record>), or None
    once the kernels' sources have changed since the capture (the counters
    would describe other kernels)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != rec["sources_sha256_16"]:
        return None
    return rec[key]


def _gemm_traffic():
    """DRAM bytes per k_gemm launch, mean over the four projections."""
    return _traffic("k_gemm_dram_traffic.json", "mean_per_launch_bytes")


def _quant_traffic():
    """DRAM bytes of the stand-alone quantizer per activation (k_amax +
    k_quantize_ws), mean over the four activations."""
    return _traffic("quant_dram_traffic.json", "mean_per_activation_bytes")


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running (every
    half millisecond, so that even a timed region of ~15 ms gets 20 or more
    samples).  Entering waits until NVML is up and the first sample is taken,
    so the samples cover the region that follows."""

    def __init__(self, index: int, period_s: float = 0.0005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self._ready = threading.Event()
        self._t = None
        self.max_mhz = None

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            flags = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                     "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}
            while not self._stop.is_set():
                self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in flags.items():
                    if r & bit:
                        self.reasons.add(name)
                self._ready.set()
                time.sleep(self.period)
        except Exception as e:  # pragma: no cover - NVML missing
            self.reasons.add(f"nvml-unavailable: {type(e).__name__}")
        finally:
            self._ready.set()

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        self._ready.wait(timeout=10.0)
        del self.samples[:len(self.samples)]     # taken before the region
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join()

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "sm_mhz_min": min(self.samples) if self.samples else None,
                "period_ms": self.period * 1e3}


# Dense FP4 (kind::mxf4nvf4) work of one SM per clock: one M 128 x N 256 x K 64
# block-scaled MMA (4.19 MFLOP) per 128 SM cycles (measured back to back).
FP4_FLOP_PER_SM_CLK = 32768
NOMINAL_FP4_TFLOPS = 9000.0


def _fp4_peaks(peaks, sm_mhz, num_sms):
    """The FP4 roofline figures a tensor-bound kernel is compared with:
    burst and sustained (the measured bf16 peaks of this machine times the
    nominal FP4 : BF16 ratio 9 : 2.25 = 4), the nominal 9.0 PFLOP/s, and the
    clock-derived peak at the SM clock sampled during the timing."""
    out = {"burst": 4.0 * peaks["bf16_tflops"], "sustained": 4.0 * peaks["bf16_tflops_sustained"],
           "nominal": NOMINAL_FP4_TFLOPS}
    if sm_mhz:
        out["at_sampled_clock"] = num_sms * FP4_FLOP_PER_SM_CLK * sm_mhz * 1e6 / 1e12
    return out


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def _max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _projection_inputs(seed_base: int, device):
    projs = []
    for i, p in enumerate(inputs.QWEN3_8B_PROJECTIONS):
        x = inputs.activation_bf16(TOKENS, p.K, seed=seed_base + i, outlier_channels=inputs.outlier_count(p.K),
                                   outlier_scale=50.0, device=device)
        w = inputs.weight_bf16(p.N, p.K, seed=seed_base + 100 + i, device=device)
        projs.append((p, x, w))
    return projs


def _flops_per_step():
    return sum(2.0 * TOKENS * p.N * p.K for p in inputs.QWEN3_8B_PROJECTIONS)


# ----------------------------------------------------------------- CPU oracle

def oracle_sample_step(projs_cpu, rows_per_proj: int, rng):
    """One oracle pass over a sample: alpha of the whole X, then quantize,
    dequantize and binary64-multiply `rows_per_proj` sampled rows against the
    pre-dequantized weight.  Returns the sampled FLOPs."""
    import oracle
    flops = 0.0
    for p, xb, w_hat in projs_cpu:
        ax = oracle.tensor_scale(xb)
        rows = np.sort(rng.choice(xb.shape[0], rows_per_proj, replace=False))
        xc, xs = oracle.quantize(np.ascontiguousarray(xb[rows]), ax)
        y = oracle.bf16_rne_array(oracle.gemm_f64(oracle.dequantize(xc, xs, ax), w_hat))
        assert y.shape == (rows_per_proj, p.N)
        flops += 2.0 * rows_per_proj * p.N * p.K
    return flops


def _oracle_projections():
    import oracle
    out = []
    for p, x, w in _projection_inputs(0, "cpu"):
        xb, wb = inputs.bf16_bits(x), inputs.bf16_bits(w)
        aw = oracle.tensor_scale(wb)
        wc, ws = oracle.quantize(wb, aw)
        out.append((p, xb, oracle.dequantize(wc, ws, aw)))
    return out


def cpu_baseline(target_s: float = 12.0):
    import oracle
    projs = _oracle_projections()
    rng = np.random.default_rng(0)
    rows = 32
    oracle_sample_step(projs, 8, rng)                      # warm-up
    t0 = time.perf_counter()
    flops, steps = 0.0, 0
    while time.perf_counter() - t0 < target_s or steps < 2:
        flops += oracle_sample_step(projs, rows, rng)
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{steps} oracle steps, each {rows} of {TOKENS} rows per projection (alpha over all rows), "
                      f"weights dequantized once beforehand; {dt:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    projs = _oracle_projections()
    rng = np.random.default_rng(0)
    rows = 8
    for _ in range(args.warmup):
        oracle_sample_step(projs, rows, rng)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += oracle_sample_step(projs, rows, rng)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "tokens": TOKENS},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"each step: {rows} of {TOKENS} rows per projection"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- GPU path

def run_ours(args, world, rank, local):
    from nvfp4_w4a4_quantized_03_b200 import mq
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()

    projs = _projection_inputs(rank * 1000, device)
    work = []
    for p, x, w in projs:
        qw = mq.quantize(w)                       # offline weight quantization (not timed)
        lws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(TOKENS, p.K), device)
        y = torch.empty(TOKENS, p.N, dtype=torch.bfloat16, device=device)
        work.append(dict(p=p, x=x, qw=qw, lws=lws, y=y))
        del w
    torch.cuda.synchronize()

    def step(ev=None):
        # the product call: alpha_x pass, then the GEMM with X quantized inside
        for i, t in enumerate(work):
            if ev is not None:
                ev[i][0].record(stream)
            mq.mq_linear_w4a4(t["x"], t["qw"].codes, t["qw"].scales, t["qw"].alpha, t["p"].N, t["y"], t["lws"],
                              stream)
            if ev is not None:
                ev[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for t in work:
        assert mq.mq_read_status(t["lws"]) == mq.MQ_OK

    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in work] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        end.record(stream)
        torch.cuda.synchronize()
    _barrier(world)
    elapsed_ms = _max_over_ranks(start.elapsed_time(end), world, device)
    lin_ms = sum(e[0].elapsed_time(e[1]) for ev in evs for e in ev) / args.steps
    by_proj = {}
    for i, t in enumerate(work):
        ms_i = sum(ev[i][0].elapsed_time(ev[i][1]) for ev in evs) / args.steps
        by_proj[t["p"].name] = 2.0 * TOKENS * t["p"].N * t["p"].K / (ms_i / 1e3) / 1e12
    for t in work:
        assert mq.mq_read_status(t["lws"]) == mq.MQ_OK

    flops = _flops_per_step()
    ms_per_step = elapsed_ms / args.steps
    value = world * flops * args.steps / (elapsed_ms / 1e3) / 1e12

    quant = _quantizer_pass(args, work, device, stream)
    gemm = _gemm_pass(args, work, device, stream)
    e2e = _e2e(args, work, device, stream)
    del work
    torch.cuda.empty_cache()
    # the latency-bound legs first, before the long prefill sequences heat the GPU
    decode = None if args.no_sequence else _decode_figure(device)
    small = None if args.no_sequence else _small_linear(device)
    sequence = None if args.no_sequence else _prefill_sequence(args, device)
    sequence_mlp = None if args.no_sequence else _prefill_sequence(args, device, mlp=True)
    mlp = None if args.no_sequence else _mlp_figure(device)
    scale_stats = None if args.no_sequence else _scale_stats(device)
    bf16_ctx = None if args.no_sequence else _bf16_context(device, value / world)
    long32k = None if args.no_sequence else _long_context_32k(device)
    sweep = None if args.no_sequence else _shape_sweep(device)

    peaks, peaks_src = _peaks()
    num_sms = torch.cuda.get_device_properties(device).multi_processor_count
    # k_gemm is timed alone, in a region of a few tens of ms: the burst peak
    gemm_peaks = _fp4_peaks(peaks, gemm["clocks"]["sm_mhz"], num_sms)
    fp4_peak = gemm_peaks["burst"]
    main_clocks = clocks.summary()
    lin_peaks = _fp4_peaks(peaks, main_clocks["sm_mhz"], num_sms)
    lin_tflops = flops / (lin_ms / 1e3) / 1e12
    hbm = peaks["hbm_gbs"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": TOKENS, "parallelism": f"replicas{world}",
                   "l2": "no flush: per-step working set ~1.1 GB (bf16 X 384 MB, FP4 W 92 MB, bf16 Y 608 MB) > 126 MB L2"},
        "fp4_frac_of_nominal_9pf": value / 9000.0,
        "linear_tflops_by_projection": by_proj,
        "quant_gbs": quant["gbs"],
        "gemm_tflops_by_projection": gemm["by_proj"],
        # the dominant kernel: k_gemm, ~0.8 of each linear's time
        "roofline": {"bound": "tensor", "achieved": gemm["tflops"], "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm["tflops"] / fp4_peak, "traffic": _gemm_traffic(),
                     "traffic_unit": "bytes per launch (mean of the four projections; ncu dram read+write)",
                     "kernel": "k_gemm (mq_nvfp4_gemm on the four projections, pre-quantized X)",
                     "flops_per_launch": "2*8192*N*K", "ms_per_launch": gemm["ms_per_launch"],
                     "launches_timed": gemm["launches_timed"], "timed_region_ms": gemm["timed_region_ms"],
                     "peak_source": f"{peaks_src}: 4 x bf16_tflops (burst: the kernel is timed alone in a "
                                    f"region of a few tens of ms; nominal fp4:bf16 = 9:2.25)",
                     "frac_of_sustained": gemm["tflops"] / gemm_peaks["sustained"],
                     "frac_of_nominal_9pf": gemm["tflops"] / NOMINAL_FP4_TFLOPS,
                     "frac_at_sampled_clock": (gemm["tflops"] / gemm_peaks["at_sampled_clock"]
                                               if "at_sampled_clock" in gemm_peaks else None),
                     "peak_at_sampled_clock": gemm_peaks.get("at_sampled_clock"),
                     "clocks": gemm["clocks"]},
        "linear_roofline": {"bound": "tensor", "achieved": lin_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                            "frac": lin_tflops / fp4_peak,
                            "frac_of_nominal_9pf": lin_tflops / NOMINAL_FP4_TFLOPS,
                            "frac_at_sampled_clock": (lin_tflops / lin_peaks["at_sampled_clock"]
                                                      if "at_sampled_clock" in lin_peaks else None),
                            "peak_source": f"{peaks_src}: 4 x bf16_tflops (burst)",
                            "kernel": "mq_linear_w4a4 = k_quantize_onepass_ws + k_gemm"},
        "quant_roofline": {"bound": "hbm", "achieved": quant["gbs"], "peak": hbm, "unit": "GB/s",
                           "frac": quant["gbs"] / hbm, "traffic": _quant_traffic(),
                           "traffic_unit": "bytes per activation (k_amax + k_quantize_ws; mean of the four "
                                           "activations, algorithmic 4.5625 B/element = 211.8 MB; ncu dram read+write)",
                           "kernel": "k_amax + k_quantize_ws (mq_tensor_scale + mq_nvfp4_quantize)",
                           "bytes_per_element": 4.5625, "peak_source": f"{peaks_src}: hbm_gbs"},
        "gpu_launches": 8 * args.steps,
        "clocks": main_clocks,
        "e2e": e2e,
        "prefill_sequence": sequence,
        "prefill_sequence_mlp": sequence_mlp,
        "decode_gemm": decode,
        "mlp": mlp,
        "block_scale_stats": scale_stats,
        "bf16_matmul_context": bf16_ctx,
        "small_linear_128x1024x1024": small,
        "long_context_32k": long32k,
        "sweep": sweep,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)


def _quantizer_pass(args, work, device, stream):
    """The stand-alone quantizer (A1-A4) on the four activations: per element
    2 B read for alpha, 2 B read + 0.5 B codes + 1/16 B scales for the codes."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    bufs = []
    for t in work:
        qx = mq.QuantizedTensor(TOKENS, t["p"].K, device)
        bufs.append((t["x"], qx, mq.workspace(mq.mq_workspace_bytes(), device)))

    def run():
        for x, qx, ws in bufs:
            mq.mq_tensor_scale(x, qx.alpha, ws, stream)
            mq.mq_nvfp4_quantize(x, qx.alpha, qx.codes, qx.scales, stream)

    for _ in range(3):
        run()
    steps = max(5, min(args.steps, 50))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(steps):
        run()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    elems = sum(x.numel() for x, _, _ in bufs)
    return {"gbs": elems * 4.5625 / (ms / 1e3) / 1e9, "ms": ms}


def _gemm_pass(args, work, device, stream):
    """k_gemm alone: mq_nvfp4_gemm of the quantized X against the quantized
    weight, the launch mq_linear_w4a4 makes after quantizing X.  CUDA events
    around every launch on the launching stream."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    bufs = []
    for t in work:
        qx = mq.quantize(t["x"])
        bufs.append((t, qx, mq.workspace(mq.mq_workspace_bytes(), device)))

    def run(ev=None):
        for i, (t, qx, ws) in enumerate(bufs):
            if ev is not None:
                ev[i][0].record(stream)
            mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, t["qw"].codes, t["qw"].scales, t["qw"].alpha,
                             TOKENS, t["p"].N, t["p"].K, t["y"], ws, stream)
            if ev is not None:
                ev[i][1].record(stream)

    for _ in range(3):
        run()
    steps = max(5, min(args.steps, 50))
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in bufs] for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clocks:
        for k in range(steps):
            run(evs[k])
        torch.cuda.synchronize()
    for _, _, ws in bufs:
        assert mq.mq_read_status(ws) == mq.MQ_OK
    by_proj, total_ms = {}, 0.0
    for i, (t, _, _) in enumerate(bufs):
        ms_i = sum(ev[i][0].elapsed_time(ev[i][1]) for ev in evs) / steps
        total_ms += ms_i
        by_proj[t["p"].name] = 2.0 * TOKENS * t["p"].N * t["p"].K / (ms_i / 1e3) / 1e12
    return {"tflops": _flops_per_step() / (total_ms / 1e3) / 1e12, "by_proj": by_proj,
            "ms_per_launch": total_ms / len(bufs), "launches_timed": steps * len(bufs),
            "timed_region_ms": total_ms * steps, "clocks": clocks.summary()}


def _prefill_sequence(args, device, mlp=False):
    """The 36-layer decoder stack's prefill linears at 131072 tokens (four
    Qwen3-8B-shaped projections per layer, fixed activations, weights
    N(0, 0.02) quantized offline), recorded once as a CUDA graph and replayed;
    CUDA events around each replay.  With `mlp`, each layer's gate/up and
    down linears are its MLP in one mq_mlp_w4a4 call (SwiGLU and H's
    quantization between them), the same GEMM flops."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    from nvfp4_w4a4_quantized_03_b200.sequence import PrefillSequence
    layers, tokens = 36, 131072
    seq = PrefillSequence(layers, tokens, device, mlp=mlp)
    seq.capture()
    seq.replay()                      # warm-up
    torch.cuda.synchronize()
    reps = 3
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    stream = torch.cuda.current_stream()
    for e0, e1 in evs:
        e0.record(stream)
        seq.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    assert seq.status() == mq.MQ_OK
    ms = min(e0.elapsed_time(e1) for e0, e1 in evs)
    what = "(qkv, o, MLP: gate/up + SwiGLU + down)" if mlp else "(qkv, o, gate_up, down)"
    out = {"workload": f"{layers} layers x {what} at {tokens} tokens, one CUDA graph",
           "tflops": seq.flops() / (ms / 1e3) / 1e12, "ms": ms, "ms_per_layer": ms / layers,
           "tflop_per_layer": seq.flops() / layers / 1e12, "graph_kernel_launches": seq.launches(),
           "replays_timed": reps, "timing": "best of the timed replays"}
    del seq
    torch.cuda.empty_cache()
    return out


def _decode_figure(device):
    """Decode-shaped GEMMs (M tokens, the split-K weight-streaming kernel
    mq_nvfp4_gemm takes for M <= 64): the four Qwen3-8B-shaped projections of
    8 layers (weights rotate, ~0.8 GB > L2), pre-quantized operands, one CUDA
    graph per M; weight bytes (codes + scales) per second against HBM, the
    median of 5 rounds of 5 replays."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    layers = 8
    projs = inputs.QWEN3_8B_PROJECTIONS
    weights = [[mq.quantize(inputs.weight_bf16(p.N, p.K, seed=3000 + 16 * l + i, device="cuda"))
                for i, p in enumerate(projs)] for l in range(layers)]
    wbytes = sum(mq.mq_nvfp4_codes_bytes(p.N, p.K) + mq.mq_nvfp4_scales_bytes(p.N, p.K) for p in projs)
    ws = mq.workspace(mq.mq_workspace_bytes(), device)
    out = {"workload": "qwen3-8b projections (qkv, o, gate_up, down), 8 layers of weights in rotation, one CUDA graph",
           "weight_bytes_per_layer": wbytes}
    for M in (1, 16, 64):
        xs = [mq.quantize(inputs.activation_bf16(M, p.K, seed=M + i, outlier_channels=inputs.outlier_count(p.K),
                                                 device="cuda")) for i, p in enumerate(projs)]
        ys = [torch.empty(M, p.N, dtype=torch.bfloat16, device=device) for p in projs]

        def run(stream=None):
            for l in range(layers):
                for i, p in enumerate(projs):
                    q = weights[l][i]
                    mq.mq_nvfp4_gemm(xs[i].codes, xs[i].scales, xs[i].alpha, q.codes, q.scales, q.alpha, M, p.N,
                                     p.K, ys[i], ws, stream)
        run()
        torch.cuda.synchronize()
        s = torch.cuda.Stream(device=device)
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                run(s)
        torch.cuda.current_stream().wait_stream(s)
        g.replay()
        torch.cuda.synchronize()
        rounds = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(5):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            rounds.append(e0.elapsed_time(e1) / (5 * layers) * 1e3)
        us = statistics.median(rounds)
        out[f"M{M}"] = {"us_per_layer": us, "weight_gbs": wbytes / us / 1e3,
                        "tflops": 2.0 * M * sum(p.N * p.K for p in projs) / us / 1e6,
                        "us_per_layer_min": min(rounds), "rounds": len(rounds)}
        del g
    assert mq.mq_read_status(ws) == mq.MQ_OK
    return out


def _bf16_context(device, w4a4_tflops):
    """Context point, not part of the method: torch's BF16 matmul (cuBLAS)
    on the same four projections, X bf16 [8192, K] times W bf16 [N, K]
    transposed, CUDA events around 10 launches each after 3 warm-up ones.
    Beside it the pages' own figure, measured on another GPU."""
    by_proj, tot_ms = {}, 0.0
    for i, p in enumerate(inputs.QWEN3_8B_PROJECTIONS):
        x = inputs.activation_bf16(TOKENS, p.K, seed=5000 + i, outlier_channels=inputs.outlier_count(p.K),
                                   outlier_scale=50.0, device="cuda")
        w = inputs.weight_bf16(p.N, p.K, seed=5100 + i, device="cuda")
        y = torch.empty(TOKENS, p.N, dtype=torch.bfloat16, device=device)
        for _ in range(3):
            torch.matmul(x, w.t(), out=y)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            torch.matmul(x, w.t(), out=y)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 10
        tot_ms += ms
        by_proj[p.name] = 2.0 * TOKENS * p.N * p.K / ms / 1e9
        del x, w, y
    torch.cuda.empty_cache()
    tflops = _flops_per_step() / tot_ms / 1e9
    return {"impl": "torch.matmul bf16 (cuBLAS), same four projections at 8192 tokens", "tflops": tflops,
            "tflops_by_projection": by_proj, "w4a4_linear_speedup": w4a4_tflops / tflops,
            "pages_figure": "NVFP4 W4A4 prefill 2-3.74x faster than BF16, end to end in vLLM on an RTX 5090 "
                            "(another GPU and a whole model: context, not a target)"}


def _time_calls(fn, reps: int, warm: int = 3) -> float:
    """ms per call of fn: CUDA events on the current stream around `reps`
    back-to-back calls, after `warm` untimed ones."""
    for _ in range(warm):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def _small_linear(device):
    """The single small W4A4 linear: X bf16 [128, 1024] N(0, 1) with 4 outlier
    channels x20, W [1024, 1024] N(0, 0.02), seed 0, through mq_linear_w4a4
    (0.268 GFLOP: launch-bound, so microseconds matter more than TFLOP/s).
    Timed as 200 back-to-back calls, and as the same calls replayed from one
    CUDA graph."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    M, K, N = 128, 1024, 1024
    x = inputs.activation_bf16(M, K, seed=0, outlier_channels=4, outlier_scale=20.0, device=device)
    lin = mq.LinearW4A4(inputs.weight_bf16(N, K, seed=0, device=device))
    y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    reps = 200
    ms = _time_calls(lambda: lin(x, y), reps)
    s = torch.cuda.Stream(device=device)
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        lin(x, y, stream=s)
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                lin(x, y, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    ms_graph = _time_calls(g.replay, 5, warm=1) / reps
    assert mq.mq_read_status(lin._ws) == mq.MQ_OK
    del g
    flops = 2.0 * M * N * K
    return {"workload": "single W4A4 linear, X [128, 1024] (4 outlier channels x20), W [1024, 1024], seed 0",
            "us_per_call": ms * 1e3, "tflops": flops / ms / 1e9, "us_per_call_graph": ms_graph * 1e3,
            "tflops_graph": flops / ms_graph / 1e9, "calls_timed": reps, "gpu_launches_per_call": 2}


def _long_context_32k(device):
    """The four Qwen3-8B-shaped projections at 32768 tokens with heavy-tailed
    activations (Student-t(4) times a LogNormal(0, 1) scale per channel),
    through mq_linear_w4a4 (activation quantized inside the call); CUDA events
    around 5 steps of the four linears after 2 warm-up ones."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    T = 32768
    work = []
    for i, p in enumerate(inputs.QWEN3_8B_PROJECTIONS):
        x = inputs.student_t_activation_bf16(T, p.K, seed=300 + p.K + i, device=device)
        lin = mq.LinearW4A4(inputs.weight_bf16(p.N, p.K, seed=400 + p.N, device=device))
        work.append((p, x, lin, torch.empty(T, p.N, dtype=torch.bfloat16, device=device)))

    def step():
        for p, x, lin, y in work:
            lin(x, y)
    ms = _time_calls(step, 5, warm=2)
    for _, _, lin, _ in work:
        assert mq.mq_read_status(lin._ws) == mq.MQ_OK
    flops = sum(2.0 * T * p.N * p.K for p in inputs.QWEN3_8B_PROJECTIONS)
    by_proj = {p.name: 2.0 * T * p.N * p.K / _time_calls(lambda: lin(x, y), 3, warm=1) / 1e9
               for p, x, lin, y in work}
    del work
    torch.cuda.empty_cache()
    return {"workload": "qwen3-8b projections at 32768 tokens, Student-t(4) x LogNormal(0,1) per-channel "
                        "activations, mq_linear_w4a4", "ms_per_step": ms, "tflops": flops / ms / 1e9,
            "tflop_per_step": flops / 1e12, "tflops_by_projection": by_proj}


def _shape_sweep(device):
    """W4A4 linear (mq_linear_w4a4) against torch's BF16 matmul (cuBLAS,
    context) over tokens M in {512 .. 131072} x (K, N) in {(4096, 4096),
    (4096, 12288), (12288, 4096), (5120, 25600)}; activations N(0, 1) with 1%
    outlier channels x50, weights N(0, 0.02).  Each shape is timed over
    enough calls for ~0.5 PFLOP of work (1 to 50), after a warm-up call
    (the smallest M of each (K, N) warms the kernels up first)."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    rows = []
    for K, N in inputs.SWEEP_KN:
        w = inputs.weight_bf16(N, K, seed=N + 7, device=device)
        lin = mq.LinearW4A4(w)
        for M in inputs.SWEEP_M:
            x = inputs.activation_bf16(M, K, seed=M % 9973 + K, outlier_channels=inputs.outlier_count(K),
                                       outlier_scale=50.0, device=device)
            y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            flops = 2.0 * M * N * K
            reps = max(1, min(50, int(5e14 // flops)))
            ms_fp4 = _time_calls(lambda: lin(x, y), reps, warm=1)
            assert mq.mq_read_status(lin._ws) == mq.MQ_OK
            ms_bf16 = _time_calls(lambda: torch.matmul(x, w.t(), out=y), reps, warm=1)
            rows.append({"M": M, "K": K, "N": N, "w4a4_tflops": flops / ms_fp4 / 1e9,
                         "bf16_tflops": flops / ms_bf16 / 1e9, "w4a4_over_bf16": ms_bf16 / ms_fp4,
                         "w4a4_ms": ms_fp4, "bf16_ms": ms_bf16, "calls_timed": reps})
            del x, y
        lin._ws = None
        del w, lin
        torch.cuda.empty_cache()
    return {"workload": "M x (K, N) sweep, W4A4 linear vs torch bf16 matmul", "shapes": rows,
            "pages_figure": "NVFP4 W4A4 prefill 2-3.74x faster than BF16 across sequence lengths and batch sizes, "
                            "end to end in vLLM on an RTX 5090 (context, not a target)"}


def _scale_stats(device):
    """Share of the E4M3 block scales that are zero (the block quantizes to
    all-zero codes) or subnormal (below 2^-6), on the heavy-tailed long-context
    activation (32768 x 4096: Student-t(4) times a LogNormal(0, 1) scale per
    channel) and on the 8192-token activation of the timed step; counted on
    the quantizer's output scale buffer, outside any timed region."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    out = {}
    cases = (("student_t_32768x4096", lambda: inputs.student_t_activation_bf16(32768, 4096, seed=300 + 4096,
                                                                             device=device)),
             ("gaussian_outliers_8192x4096",
              lambda: inputs.activation_bf16(TOKENS, 4096, seed=1, outlier_channels=inputs.outlier_count(4096),
                                             outlier_scale=50.0)))
    for name, make in cases:
        x = make().to(device)
        q = mq.quantize(x)
        torch.cuda.synchronize()
        sc = q.scales            # no padding at these shapes: every byte is a block scale
        n = sc.numel()
        zero = int((sc == 0).sum().item())
        sub = int(((sc & 0x78) == 0).sum().item()) - zero
        out[name] = {"blocks": n, "zero_frac": zero / n, "subnormal_frac": sub / n}
        del x, q, sc
    torch.cuda.empty_cache()
    return out


def _mlp_figure(device):
    """The Qwen3-8B-shaped MLP at 8192 tokens (K 4096, inter 12288, N 4096):
    mq_mlp_w4a4 (x quantized, gate/up GEMM with SwiGLU and max|h| in its
    epilogue, alpha_h, H quantized, down GEMM) against the two linears alone
    (mq_linear_w4a4 on gate/up writing [M, 2 inter], then on the down
    projection with a fixed input), which do not compute the activation."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    M, K, inter, N = TOKENS, 4096, 12288, 4096
    x = inputs.activation_bf16(M, K, seed=4000, outlier_channels=inputs.outlier_count(K), outlier_scale=50.0,
                               device="cuda")
    wgu = inputs.weight_bf16(2 * inter, K, seed=4001, device="cuda")
    wd = inputs.weight_bf16(N, inter, seed=4002, device="cuda")
    mlp = mq.MLPW4A4(wgu, wd)
    lin_gu, lin_d = mq.LinearW4A4(wgu), mq.LinearW4A4(wd)
    del wgu, wd
    y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    y_gu = torch.empty(M, 2 * inter, dtype=torch.bfloat16, device=device)
    mlp(x, y)
    h = mlp.h_view(M).clone()

    def timed(fn, reps=10):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    ms_mlp = timed(lambda: mlp(x, y))
    ms_two = timed(lambda: (lin_gu(x, y_gu), lin_d(h, y)))
    assert mq.mq_read_status(mlp._ws) == mq.MQ_OK
    flops = 2.0 * M * K * 2 * inter + 2.0 * M * inter * N
    return {"workload": "qwen3-8b MLP at 8192 tokens: x [8192, 4096], gate/up [24576, 4096], down [4096, 12288]",
            "ms": ms_mlp, "tflops": flops / ms_mlp / 1e9,
            "two_linears_without_activation_ms": ms_two,
            "launches": 5, "flops": flops}


def _e2e(args, work, device, stream):
    """Pinned host X -> device, mq_linear_w4a4, device -> pinned host Y, every
    step and every projection.  The copies run on their own streams (one per
    direction, so PCIe carries both at once) and overlap the linears of the
    other projections; events order each X copy before its linear, and each
    linear after the copies that still read or write its buffers."""
    from nvfp4_w4a4_quantized_03_b200 import mq
    host_x = [t["x"].cpu().pin_memory() for t in work]
    host_y = [torch.empty(t["y"].shape, dtype=torch.bfloat16).pin_memory() for t in work]
    dx = [torch.empty_like(t["x"]) for t in work]
    lws = [mq.workspace(mq.mq_linear_w4a4_workspace_bytes(TOKENS, t["p"].K), device) for t in work]
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    n = len(work)
    ev_in = [torch.cuda.Event() for _ in range(n)]      # X_i is on the device
    ev_done = [torch.cuda.Event() for _ in range(n)]    # linear i finished: dx[i] free, y_i written
    ev_out = [torch.cuda.Event() for _ in range(n)]     # y_i is on the host: y_i free

    def step():
        for i, t in enumerate(work):
            s_in.wait_event(ev_done[i])
            with torch.cuda.stream(s_in):
                dx[i].copy_(host_x[i], non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            stream.wait_event(ev_out[i])
            mq.mq_linear_w4a4(dx[i], t["qw"].codes, t["qw"].scales, t["qw"].alpha, t["p"].N, t["y"], lws[i], stream)
            ev_done[i].record(stream)
            s_out.wait_event(ev_done[i])
            with torch.cuda.stream(s_out):
                host_y[i].copy_(t["y"], non_blocking=True)
            ev_out[i].record(s_out)

    steps = max(3, min(args.steps, 20))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    s_in.wait_event(s)
    s_out.wait_event(s)
    for _ in range(steps):
        step()
    stream.wait_event(ev_out[n - 1])
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    for i, t in enumerate(work):
        assert torch.equal(host_y[i], t["y"].cpu()), "the host copy of Y differs from Y"
    h2d = sum(h.numel() * 2 for h in host_x)
    d2h = sum(h.numel() * 2 for h in host_y)
    return {"value": _flops_per_step() / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "overlap": "X copies, linears and Y copies on three streams (per-projection events)"}


def profile_target(which: str):
    """One gate/up-shaped (8192 x 24576 x 4096) launch inside an NVTX range
    "gemm", after 3 unmarked ones, for `ncu --nvtx --nvtx-include gemm/`:
    `ours` is mq_nvfp4_gemm on quantized operands, `linear` the linear
    mq_linear_w4a4 (k_quantize_onepass_ws + k_gemm), `ingemm` the linear with
    the activation quantized by the GEMM's own quantizer warps (k_amax +
    k_gemm with quantizer warps), `library` the library NVFP4 GEMM (cuBLASLt
    through torch._scaled_mm; context for the profile comparison only, on
    random codes and unit scales)."""
    M, N, K = TOKENS, 24576, 4096
    if which in ("linear", "ingemm"):
        from nvfp4_w4a4_quantized_03_b200 import mq
        if which == "ingemm":
            mq.mq_set_switch("linear_path", "ingemm")
        x = inputs.activation_bf16(M, K, seed=1, outlier_channels=inputs.outlier_count(K), device="cuda")
        lin = mq.LinearW4A4(inputs.weight_bf16(N, K, seed=2, device="cuda"))
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        f = lambda: lin(x, y)
    elif which == "library":
        a = torch.randint(0, 255, (M, K // 2), dtype=torch.uint8, device="cuda").view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 255, (N, K // 2), dtype=torch.uint8, device="cuda").view(torch.float4_e2m1fn_x2)
        sa = torch.full((M * K // 16,), 1.0, device="cuda").to(torch.float8_e4m3fn)
        sb = torch.full((N * K // 16,), 1.0, device="cuda").to(torch.float8_e4m3fn)
        f = lambda: torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
    else:
        from nvfp4_w4a4_quantized_03_b200 import mq
        x = inputs.activation_bf16(M, K, seed=1, outlier_channels=inputs.outlier_count(K), device="cuda")
        w = inputs.weight_bf16(N, K, seed=2, device="cuda")
        qx, qw = mq.quantize(x), mq.quantize(w)
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        f = lambda: mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, qw.codes, qw.scales, qw.alpha, M, N, K, y)
    for _ in range(3):
        f()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("gemm")
    f()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sequence", action="store_true",
                    help="skip the figures beside the metric (36-layer x 131072-token prefill sequence, decode, "
                         "MLP, small linear, 32768-token projections, shape sweep)")
    ap.add_argument("--profile-target", choices=["ours", "linear", "ingemm", "library"], default=None,
                    help="run one gate/up-shaped GEMM or linear in an NVTX range for ncu and exit (no timing)")
    args = ap.parse_args()
    if args.profile_target:
        profile_target(args.profile_target)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    world, rank, local = _dist()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
