#!/usr/bin/env python
"""Benchmark of the NVFP4 linear-layer training step on B200.

One step = the whole hot path for both linears of the 12B-class hybrid
Mamba-Transformer MLP shapes (tokens 16384, hidden 5120, FFN 20480: the
up-projection W[20480 x 5120] and the down-projection W[5120 x 20480]):
  quantise W (16x16 blocks, row + col layouts)
  fprop:  quantise X (row, RNE; col with 16x16 RHT, RNE)   + GEMM  Y  = X W^T
  dgrad:  quantise dY (row, SR; col with RHT + SR)          + GEMM  dX = dY W
  wgrad:                                                      GEMM  dW = dY^T X (FP32)
Inputs are seeded synthetic BF16 tensors resident in HBM (each larger than the
126 MB L2, so no flush is needed between steps).

Prints one JSON line (rank 0).  `value` is the step's NVFP4 GEMM work (6 GEMMs,
2MNK each) divided by the device time of the whole step, quantisers included.
`e2e` is the same metric through the public C-ABI linear calls with the step's
activations and gradients copied from pinned host memory and the weight
gradients read back, inside the timed region.  `roofline` covers the dominant
kernel (the GEMM) against the FP4 tensor peak; `quantizer` the HBM side.
`targets` times the two single-kernel goals alone: the GEMM at 16384^3 and the
quantiser on the 16384^2 sweep tensor in its three modes.
`--impl reference` times the CPU oracle on a bounded sample of the same step.
Multi-GPU: data parallel, each rank runs the full per-GPU step on its own tokens
and each linear's FP32 weight gradient is all-reduced with NCCL as soon as its
wgrad is enqueued (weak scaling).  Under torchrun every rank reads RANK /
WORLD_SIZE / LOCAL_RANK; `bench.py --gpus N` started as one process launches the
N ranks itself.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS & % FP4 peak; quantizer GB/s & % HBM (1×B200)"
UNIT = "TFLOP/s"
WORKLOAD = "hybrid12b-mlp-linear-step"
FP4_OVER_BF16 = 4.0          # nominal dense ratio (9 / 2.25 PFLOP/s)
RHT_SIGNS = 0x5A3C
SR_SEED = 1234
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peak_number(v):
    """A peak figure from MEASURED_PEAKS.json: a number, or a record holding one."""
    if isinstance(v, bool):
        return None
    if isinstance(v, (int, float)):
        return float(v) if v > 0 else None
    if isinstance(v, dict):
        for k in ("value", "median", "mean", "gbs", "tflops"):
            if k in v:
                return _peak_number(v[k])
    return None


def load_peaks(path=None):
    """The roofline denominators: MEASURED_PEAKS.json where it holds them (per key),
    else the fallback figures; the source says which."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"
    peaks, missing = {}, []
    for key, fb in FALLBACK_PEAKS.items():
        v = _peak_number(d.get(key)) if isinstance(d, dict) else None
        if v is None:
            missing.append(key)
            v = fb
        peaks[key] = v
    if not missing:
        return peaks, "measured"
    if len(missing) == len(FALLBACK_PEAKS):
        return peaks, "fallback"
    return peaks, "measured (fallback for %s)" % ", ".join(missing)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------- traffic

GEMM_SOURCE = os.path.join(ROOT, "nvfp4_pretraining_linear_b200", "csrc", "gemm.cuh")
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "gemm_pair_hybrid12b_step_traffic.txt")


def gemm_traffic_per_launch():
    """DRAM bytes (read + write) per GEMM launch of this step, from the committed ncu
    summary; None when there is none or when the GEMM source changed since it was taken
    (the summary records the SHA-256 of gemm.cuh it was measured with)."""
    import hashlib
    try:
        fields = {}
        with open(TRAFFIC_PROFILE) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        with open(GEMM_SOURCE, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        if fields.get("gemm_source_sha256") != sha:
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms (read-only query)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-i", uuid, "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.t_start = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- workload


class Linear:
    """Buffers of one NVFP4 linear layer step (all device-resident, preallocated)."""

    def __init__(self, name, x, w, dy):
        from nvfp4_pretraining_linear_b200.api import QTensor, SCALE_MMA
        self.name = name
        self.x, self.w, self.dy = x, w, dy
        M, K = x.shape
        N = w.shape[0]
        self.M, self.K, self.N = M, K, N
        dev = x.device
        self.wq_row = QTensor.empty(N, K, SCALE_MMA, dev)
        self.wq_col = QTensor.empty(K, N, SCALE_MMA, dev)
        self.xq_row = QTensor.empty(M, K, SCALE_MMA, dev)
        self.xq_col = QTensor.empty(K, M, SCALE_MMA, dev)
        self.dyq_row = QTensor.empty(M, N, SCALE_MMA, dev)
        self.dyq_col = QTensor.empty(N, M, SCALE_MMA, dev)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.dw = torch.empty((N, K), dtype=torch.float32, device=dev)   # FP32 partials, summed over ranks in FP32

    def gemm_flops(self):
        return 3 * 2.0 * self.M * self.N * self.K

    def quant_bytes(self):
        # two-pass quantiser: 2 B/elem amax read + 2 B/elem quantise read + 0.5625 B/elem per layout
        elems = self.M * self.K + self.N * self.K + self.M * self.N
        return elems * (4.0 + 2 * 0.5625)


def build_workload(device, rank):
    from nvfp4_pretraining_linear_b200 import synthetic as syn
    T, H, F = syn.HYBRID12B["tokens"], syn.HYBRID12B["hidden"], syn.HYBRID12B["ffn"]
    s = 1000 * rank  # each data-parallel rank draws its own tokens
    up = Linear("up", syn.normal((T, H), 1.0, seed=12 + s, device=device, outlier_frac=0.001, outlier_mult=100.0),
                syn.normal((F, H), 0.014, seed=10, device=device),
                syn.normal((T, F), 1e-3, seed=14 + s, device=device))
    down = Linear("down", syn.normal((T, F), 1.0, seed=13 + s, device=device, outlier_frac=0.001, outlier_mult=100.0),
                  syn.normal((H, F), 0.014, seed=11, device=device),
                  syn.normal((T, H), 1e-3, seed=15 + s, device=device))
    return [up, down]


def instrumented_step(linears, ev, offset, reducer=None):
    """One step from the quantiser and GEMM entry points, with CUDA events
    bracketing each GEMM and each quantiser call (same kernels, same order as
    the linear_fwd / linear_dgrad / linear_wgrad entry points).  With a reducer
    (data parallel), each linear's FP32 weight gradient starts its all-reduce as
    soon as its wgrad is enqueued; the caller waits for them at the end."""
    from nvfp4_pretraining_linear_b200 import api
    for L in linears:
        ev.mark("q")
        api.quantize(L.w, emit_row=True, emit_col=True, block_2d=True, out_row=L.wq_row, out_col=L.wq_col)
        api.quantize(L.x, emit_row=True, emit_col=True, rht_col=True, rht_signs=RHT_SIGNS, out_row=L.xq_row,
                     out_col=L.xq_col)
        ev.mark("g")
        api.gemm(L.xq_row, L.wq_row, out=L.y)
        ev.mark("q")
        api.quantize(L.dy, emit_row=True, emit_col=True, stochastic=True, rht_col=True, seed=SR_SEED, offset=offset,
                     rht_signs=RHT_SIGNS, out_row=L.dyq_row, out_col=L.dyq_col)
        ev.mark("g")
        api.gemm(L.dyq_row, L.wq_col, out=L.dx)
        api.gemm(L.dyq_col, L.xq_col, out=L.dw)
        if reducer is not None:
            reducer.start(L.dw)
    ev.mark("end")


class PhaseEvents:
    """Records an event at each phase boundary; sums device time per phase."""

    def __init__(self, enabled=True):
        self.enabled = enabled
        self.marks = []

    def mark(self, phase):
        if not self.enabled:
            return
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.marks.append((phase, e))

    def totals(self):
        out = {}
        for (ph, e0), (_, e1) in zip(self.marks, self.marks[1:]):
            if ph == "end":
                continue
            out[ph] = out.get(ph, 0.0) + e0.elapsed_time(e1)
        return out


def public_step(linears, offset, reducer=None):
    """One step through the public linear entry points (as a user calls them)."""
    from nvfp4_pretraining_linear_b200 import api
    for L in linears:
        api.quantize(L.w, emit_row=True, emit_col=True, block_2d=True, out_row=L.wq_row, out_col=L.wq_col)
        api.linear_fwd(L.x, L.wq_row, rht_signs=RHT_SIGNS, out=L.y, xq_row=L.xq_row, xq_col=L.xq_col)
        api.linear_dgrad(L.dy, L.wq_col, seed=SR_SEED, offset=offset, rht_signs=RHT_SIGNS, out=L.dx,
                         dyq_row=L.dyq_row, dyq_col=L.dyq_col)
        api.linear_wgrad(L.dyq_col, L.xq_col, out=L.dw)
        if reducer is not None:
            reducer.start(L.dw)


LAUNCHES_PER_LINEAR = 2 + 2 + 1 + 2 + 1 + 1   # W quant (amax+quant), X quant, fprop, dY quant, dgrad, wgrad


# ----------------------------------------------------------------------------- CPU oracle sample


def oracle_sample_step(state):
    """The oracle on a bounded sample of the step: the up-projection linear restricted
    to 64 tokens and 256 output features (full hidden width 5120)."""
    from oracle import nvfp4_oracle as O
    x, w, dy = state
    wq = O.quantize_weight(w)
    y, _, xq = O.linear_fwd_ref(x, wq, rht_signs=RHT_SIGNS)
    dx, _, dyq = O.linear_dgrad_ref(dy, wq, seed=SR_SEED, offset=0, rht_signs=RHT_SIGNS)
    dw, _ = O.linear_wgrad_ref(dyq, xq)
    return y, dx, dw


def oracle_sample_inputs():
    from nvfp4_pretraining_linear_b200 import synthetic as syn
    T, N, K = 64, 256, syn.HYBRID12B["hidden"]
    x = syn.normal((T, K), 1.0, seed=12, device="cpu", outlier_frac=0.001, outlier_mult=100.0).float().numpy()
    w = syn.normal((N, K), 0.014, seed=10, device="cpu").float().numpy()
    dy = syn.normal((T, N), 1e-3, seed=14, device="cpu").float().numpy()
    flops = 3 * 2.0 * T * N * K
    return (x, w, dy), flops, "up-projection linear step restricted to 64 tokens x 256 outputs x 5120 hidden"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def blas_threads():
    """Threads of the BLAS library NumPy uses for the oracle's FP64 products (None if unknown)."""
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def time_oracle(min_seconds=10.0, min_steps=3):
    state, flops, desc = oracle_sample_inputs()
    times = []
    t_all = time.perf_counter()
    while len(times) < min_steps or time.perf_counter() - t_all < min_seconds:
        t0 = time.perf_counter()
        oracle_sample_step(state)
        times.append(time.perf_counter() - t0)
        if len(times) >= 50:
            break
    t = statistics.median(times)
    return {"value": flops / t / 1e12, "unit": UNIT, "cores": cpu_cores(), "blas_threads": blas_threads(),
            "kind": "oracle", "sample": desc + "; median of %d steps, %.2f s each" % (len(times), t)}


def step_config(world):
    """The `config` of the bench line: the 12B hybrid MLP step, the same for both arms."""
    from nvfp4_pretraining_linear_b200 import synthetic as syn
    return {"workload": WORKLOAD, "tokens_per_gpu": syn.HYBRID12B["tokens"], "hidden": syn.HYBRID12B["hidden"],
            "ffn": syn.HYBRID12B["ffn"], "linears": ["up 5120->20480", "down 20480->5120"],
            "gemms_per_step": 6, "parallelism": "dp%d" % world,
            "l2": "every input larger than the 126 MB L2; no flush"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    state, flops, desc = oracle_sample_inputs()
    for _ in range(args.warmup):
        oracle_sample_step(state)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(state)
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantise / f64 GEMM",
            "data": "synthetic", "config": step_config(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "blas_threads": blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm


def flushed_median_ms(fn, flush, warmup=3, steps=10):
    """Median device time of fn() over `steps` launches, L2 flushed (a 256 MB write)
    before each, CUDA events on the current stream."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


TARGET_QUANT_MODES = {
    "1d_rne": dict(emit_row=True, emit_col=True),
    "1d_sr_rht": dict(emit_row=True, emit_col=True, stochastic=True, rht_row=True, rht_col=True, seed=SR_SEED,
                      rht_signs=RHT_SIGNS),
    "2d": dict(emit_row=True, emit_col=True, block_2d=True),
}


def measure_targets(fp4_burst, hbm):
    """The two single-kernel targets, each timed alone (L2 flushed, medians of 10):
    the NVFP4 GEMM at M = N = K = 16384 (BF16 output) against the dense FP4 peak, and
    the quantiser on the 16384 x 16384 sweep tensor (Student-t nu = 3 x 0.1) in its
    three modes with both layouts, two passes (amax, then quantise), against HBM."""
    from nvfp4_pretraining_linear_b200 import api, synthetic as syn
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    n = 16384
    a, b = syn.square(n, 2, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    del a, b
    c = torch.empty((n, n), dtype=torch.bfloat16, device="cuda")
    ms = flushed_median_ms(lambda: api.gemm(qa, qb, out=c), flush)
    tflops = 2.0 * n ** 3 / (ms * 1e-3) / 1e12
    gemm = {"shape": [n, n, n], "ms": ms, "tflops": tflops, "frac_fp4_burst": tflops / fp4_burst,
            "frac_fp4_nominal_9000": tflops / 9000.0, "target_frac_nominal": 0.60}
    del qa, qb, c
    x = syn.qsweep(n, device="cuda")
    rq, cq = api.QTensor.empty(n, n), api.QTensor.empty(n, n)
    quant = {}
    for mode, kw in TARGET_QUANT_MODES.items():
        ms = flushed_median_ms(lambda: api.quantize(x, out_row=rq, out_col=cq, **kw), flush)
        gbs = n * n * 5.125 / (ms * 1e-3) / 1e9
        quant[mode] = {"ms": ms, "gbs": gbs, "frac_hbm": gbs / hbm, "frac_hbm_nominal_8000": gbs / 8000.0}
    api.get_status()
    return {"gemm_16384": gemm,
            "quantizer_16384": dict(quant, bytes_per_elem="5.125 (two passes, row + col)", target_frac=0.70)}


def run_ours(args):
    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE is %d" % (args.gpus, world))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    group = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        group = dist.group.WORLD
    from nvfp4_pretraining_linear_b200 import api
    from nvfp4_pretraining_linear_b200.parallel import GradReducer, sr_offset

    peaks, peak_src = load_peaks()
    linears = build_workload(device, rank)
    offset = sr_offset(0, rank, world)

    def barrier():
        torch.cuda.synchronize()
        if group is not None:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    def device_step(ev):
        reducer = GradReducer(group)
        instrumented_step(linears, ev, offset, reducer)
        reducer.wait()

    for _ in range(args.warmup):
        device_step(PhaseEvents(False))
    api.get_status()

    # ---- device-timed region
    evs = [PhaseEvents(True) for _ in range(args.steps)]
    barrier()
    clocks = ClockSampler(local)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        device_step(evs[i])
    t_end.record()
    barrier()
    clock_info = clocks.stop()
    api.get_status()
    ms_total = t_start.elapsed_time(t_end)
    if group is not None:
        t = torch.tensor([ms_total], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / args.steps
    gemm_ms = sum(e.totals().get("g", 0.0) for e in evs) / args.steps
    quant_ms = sum(e.totals().get("q", 0.0) for e in evs) / args.steps
    flops = sum(L.gemm_flops() for L in linears)
    qbytes = sum(L.quant_bytes() for L in linears)
    value = flops * world / (ms_step * 1e-3) / 1e12

    # The timed region lasts well under a second, so the GEMM's roofline is the burst
    # figure (a kernel timed alone, clocks at their maximum); the sustained figure (a
    # seconds-long loop under the power cap) is reported beside it.
    bf16_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    bf16_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    fp4_burst, fp4_sust = bf16_burst * FP4_OVER_BF16, bf16_sust * FP4_OVER_BF16
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    quant_gbs = qbytes / (quant_ms * 1e-3) / 1e9
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    traffic = gemm_traffic_per_launch()

    # ---- end to end through the public API, host buffers, copies inside the timed region
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    # Every step copies its activations and output gradients from pinned host memory
    # and reads its weight gradients back.  Two device sets of those buffers let the
    # copies of neighbouring steps run on their own streams while a step computes, as a
    # training loop prefetches its next batch: step i computes on set i % 2 once its
    # inputs have landed; the inputs of step i + 2 overwrite that set only after step i
    # has computed, and its weight gradients only after they have been read back.
    sets = [linears, [Linear(L.name, torch.empty_like(L.x), L.w, torch.empty_like(L.dy)) for L in linears]]
    host_in = []
    for L in linears:
        for dev_t in (L.x, L.dy):
            host_t = torch.empty(dev_t.shape, dtype=dev_t.dtype, pin_memory=True)
            host_t.copy_(dev_t)
            host_in.append(host_t)
    host_out = [torch.empty(L.dw.shape, dtype=L.dw.dtype, pin_memory=True) for L in linears]
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(h.numel() * h.element_size() for h in host_out)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in (s_in, s_comp, s_out):
        s.wait_event(e0)
    for i in range(e2e_steps):
        k = i % 2
        dev_in = [t for L in sets[k] for t in (L.x, L.dy)]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[k])
            for dev_t, host_t in zip(dev_in, host_in):
                dev_t.copy_(host_t, non_blocking=True)
            in_done[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[k])
            if i >= 2:
                s_comp.wait_event(out_done[k])
            reducer = GradReducer(group)
            public_step(sets[k], offset, reducer)
            reducer.wait()
            comp_done[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            for L, host_t in zip(sets[k], host_out):
                host_t.copy_(L.dw, non_blocking=True)
            out_done[k].record(s_out)
    for s in (s_in, s_comp, s_out):
        torch.cuda.current_stream().wait_stream(s)
    e1.record()
    barrier()
    api.get_status()
    e2e_ms = e0.elapsed_time(e1)
    if group is not None:
        t = torch.tensor([e2e_ms], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = flops * world / (e2e_ms / e2e_steps * 1e-3) / 1e12
    del sets, host_in, host_out

    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3 block scales, fp32 accumulate), bf16 in/out, "
                                          "fp32 weight gradients",
            "data": "synthetic",
            "config": step_config(world),
            "gpu_launches": LAUNCHES_PER_LINEAR * len(linears) * args.steps,
            "quantizer": {"gbs": quant_gbs, "frac_hbm": quant_gbs / hbm, "hbm_peak_gbs": hbm,
                          "peak_source": peak_src, "ms_per_step": quant_ms,
                          "bytes_per_elem": "4.5625 / layout-pair 5.125 (two-pass)"},
            "gemm": {"tflops": gemm_tflops, "frac_fp4_burst": gemm_tflops / fp4_burst,
                     "frac_fp4_sustained": gemm_tflops / fp4_sust, "frac_fp4_nominal_9000": gemm_tflops / 9000.0,
                     "ms_per_step": gemm_ms},
            "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_burst, "unit": "TFLOP/s",
                         "frac": gemm_tflops / fp4_burst, "traffic": traffic,
                         "kernel": "nvfp4::gemm::gemm_kernel_pair",
                         "peak_source": "%s bf16 burst x %.0f (nominal FP4/BF16 ratio), of %s; the timed region "
                                        "is under a second" % (peak_src, FP4_OVER_BF16, peak_src)},
            "clocks": clock_info,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "path": "nvfp4_linear_fwd/dgrad/wgrad via the C ABI, pinned host buffers, "
                    "copies of neighbouring steps overlapped with compute on separate streams"},
        }
        if world == 1 and not args.no_targets:
            del linears
            torch.cuda.empty_cache()
            line["targets"] = dict(measure_targets(fp4_burst, hbm), peak_source=peak_src)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = time_oracle(args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if group is not None:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


QUANT_MODES = {
    "rne_row": dict(emit_row=True),
    "rne_row_col": dict(emit_row=True, emit_col=True),
    "act": dict(emit_row=True, emit_col=True, rht_col=True, rht_signs=RHT_SIGNS),
    "grad": dict(emit_row=True, emit_col=True, stochastic=True, rht_col=True, seed=SR_SEED, rht_signs=RHT_SIGNS),
    "sr_rht_both": dict(emit_row=True, emit_col=True, stochastic=True, rht_row=True, rht_col=True, seed=SR_SEED,
                        rht_signs=RHT_SIGNS),
    "weight": dict(emit_row=True, emit_col=True, block_2d=True),
}


def run_kernel(args):
    """Single-kernel timing (GEMM or quantiser) on one GPU; used for sweeps and ncu captures."""
    from nvfp4_pretraining_linear_b200 import api, synthetic as syn
    torch.cuda.set_device(0)
    dims = [int(v) for v in args.shape.split(",")]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    if args.kernel == "chain":
        return run_chain(args, dims, flush)
    if args.kernel == "ns":
        return run_ns(args, dims, flush)
    if args.kernel == "lora":
        return run_lora(args, dims, flush)
    if args.kernel == "gemm":
        M, N, K = dims
        qa, _ = api.quantize(syn.normal((M, K), 1.0, seed=30, device="cuda"))
        qb, _ = api.quantize(syn.normal((N, K), 1.0, seed=31, device="cuda"))
        out = torch.empty((M, N), dtype=torch.float32 if args.out == "f32" else torch.bfloat16, device="cuda")
        if args.accumulate:
            out.zero_()
        fn = lambda: api.gemm(qa, qb, out=out, accumulate=args.accumulate)  # noqa: E731
        work, unit = 2.0 * M * N * K, "TFLOP/s"
    else:
        R, C = dims
        kw = dict(QUANT_MODES[args.mode])
        x = syn.student_t((R, C), 3, 0.1, seed=1, device="cuda")
        rq = api.QTensor.empty(R, C) if kw.get("emit_row") else None
        cq = api.QTensor.empty(C, R) if kw.get("emit_col") else None
        layouts = int(bool(kw.get("emit_row"))) + int(bool(kw.get("emit_col")))
        if args.amax_in:
            # given maxima (delayed scaling, or the previous GEMM's epilogue): no amax pass
            amax = torch.zeros(3, dtype=torch.float32, device="cuda")
            api.quantize(x, out_row=rq, out_col=cq, amax_out=amax, **kw)
            fn = lambda: api.quantize(x, out_row=rq, out_col=cq, amax_in=amax, **kw)  # noqa: E731
            work, unit = R * C * (2.0 + 0.5625 * layouts), "GB/s"
        else:
            fn = lambda: api.quantize(x, out_row=rq, out_col=cq, **kw)  # noqa: E731
            work, unit = R * C * (4.0 + 0.5625 * layouts), "GB/s"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    clocks = ClockSampler(0)
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    clock_info = clocks.stop()
    api.get_status()
    ms = statistics.median(times)
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"kernel": args.kernel, "shape": dims, "mode": args.mode if args.kernel == "quantize" else None,
                      "out": args.out if args.kernel == "gemm" else None,
                      "accumulate": bool(args.accumulate) if args.kernel == "gemm" else None,
                      "amax_in": bool(args.amax_in) if args.kernel == "quantize" else None,
                      "ms": ms, "value": rate, "unit": unit, "steps": args.steps, "l2": "flushed (256 MB write)",
                      "clocks": clock_info}),
          flush=True)
    return 0


def run_chain(args, dims, flush):
    """A GEMM whose BF16 output is quantised next (row + RHT col, as the next linear's
    activations): nvfp4_gemm then the two-pass quantiser, against nvfp4_gemm_amax then
    the quantiser given the epilogue's maxima (no amax pass)."""
    from nvfp4_pretraining_linear_b200 import api, synthetic as syn
    M, N, K = dims
    qa, _ = api.quantize(syn.normal((M, K), 1.0, seed=30, device="cuda"))
    qb, _ = api.quantize(syn.normal((N, K), 1.0, seed=31, device="cuda"))
    c = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    amax = torch.empty(3, dtype=torch.float32, device="cuda")
    rq, cq = api.QTensor.empty(M, N), api.QTensor.empty(N, M)
    qkw = dict(emit_row=True, emit_col=True, rht_col=True, rht_signs=RHT_SIGNS, out_row=rq, out_col=cq)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    t_gemm = timed(lambda: api.gemm(qa, qb, out=c))
    t_gemm_amax = timed(lambda: api.gemm_amax(qa, qb, rht_signs=RHT_SIGNS, out=c, amax=amax))
    t_quant = timed(lambda: api.quantize(c, **qkw))
    t_quant_in = timed(lambda: api.quantize(c, amax_in=amax, **qkw))
    t_plain = timed(lambda: (api.gemm(qa, qb, out=c), api.quantize(c, **qkw)))
    t_fused = timed(lambda: (api.gemm_amax(qa, qb, rht_signs=RHT_SIGNS, out=c, amax=amax),
                             api.quantize(c, amax_in=amax, **qkw)))
    api.get_status()
    flops = 2.0 * M * N * K
    print(json.dumps({"kernel": "chain", "shape": dims, "gemm_ms": t_gemm, "gemm_amax_ms": t_gemm_amax,
                      "gemm_tflops": flops / t_gemm / 1e9, "gemm_amax_tflops": flops / t_gemm_amax / 1e9,
                      "quantize_two_pass_ms": t_quant, "quantize_amax_in_ms": t_quant_in,
                      "chain_plain_ms": t_plain, "chain_fused_ms": t_fused,
                      "steps": args.steps, "l2": "flushed (256 MB write)"}), flush=True)
    return 0


def run_ns(args, dims, flush):
    """nvfp4_newton_schulz on a Gaussian [m x n] matrix: the whole call (normalisation and
    --iters steps, L2 flushed before each call) and, from the final iterate, each stage of
    one step timed alone: quantise X (row + col), the GEMM adding -X X^T into R, quantise
    R (row), the GEMM adding R X / 2 into X; the two GEMMs also 20 launches back to back
    without a flush, as they run inside the loop (their operands fit in L2)."""
    from nvfp4_pretraining_linear_b200 import api, synthetic as syn
    m, n = dims[:2]
    iters = args.iters
    g = syn.normal((m, n), 1.0, seed=44, device="cuda")
    x = torch.empty_like(g)
    ws = api.newton_schulz_workspace(m, n)
    norm = torch.empty(1, dtype=torch.float32, device="cuda")

    def timed(fn, flush_each=True):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            if flush_each:
                flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    clocks = ClockSampler(0)
    t_ns = timed(lambda: api.newton_schulz(g, iters, out=x, norm=norm, workspace=ws))
    clock_info = clocks.stop()
    xs = x.clone()
    xr, xc = api.QTensor.empty(m, n), api.QTensor.empty(n, m)
    r = torch.eye(m, dtype=torch.bfloat16, device="cuda")
    rr = api.QTensor.empty(m, m)
    api.quantize(xs, emit_row=True, emit_col=True, out_row=xr, out_col=xc)
    t_qx = timed(lambda: api.quantize(xs, emit_row=True, emit_col=True, out_row=xr, out_col=xc))
    t_g1 = timed(lambda: api.gemm(xr, xr, alpha=-1.0, accumulate=True, out=r))
    api.quantize(r, out_row=rr)
    t_qr = timed(lambda: api.quantize(r, out_row=rr))
    t_g2 = timed(lambda: api.gemm(rr, xc, alpha=0.5, accumulate=True, out=xs))

    def back_to_back(fn, reps=20):
        # as inside the iteration loop: launches queued back to back, operands warm in L2
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b) / reps

    b_g1 = back_to_back(lambda: api.gemm(xr, xr, alpha=-1.0, accumulate=True, out=r))
    b_g2 = back_to_back(lambda: api.gemm(rr, xc, alpha=0.5, accumulate=True, out=xs))
    api.get_status()
    step_flops = 4.0 * m * m * n
    print(json.dumps({
        "kernel": "ns", "shape": [m, n], "iters": iters, "ms": t_ns, "ms_per_iter": t_ns / max(iters, 1),
        "value": step_flops * iters / (t_ns * 1e-3) / 1e12, "unit": "TFLOP/s (4 m^2 n per step)",
        "stages_ms": {"quantize_x_row_col": t_qx, "gemm_x_xt": t_g1,
                      "quantize_r_row": t_qr, "gemm_r_x": t_g2},
        "gemm_tflops": {"x_xt": 2.0 * m * m * n / t_g1 / 1e9, "r_x": 2.0 * m * m * n / t_g2 / 1e9},
        "gemm_back_to_back_ms": {"x_xt": b_g1, "r_x": b_g2},
        "gemm_back_to_back_tflops": {"x_xt": 2.0 * m * m * n / b_g1 / 1e9, "r_x": 2.0 * m * m * n / b_g2 / 1e9},
        "quantize_gbs": {"x": m * n * 5.125 / t_qx / 1e6, "r": m * m * 4.5625 / t_qr / 1e6},
        "steps": args.steps, "l2": "flushed (256 MB write) before each timed call", "clocks": clock_info}),
        flush=True)
    return 0


def run_lora(args, dims, flush):
    """The LoRA-SVD linear against the plain NVFP4 linear on one layer shape (M tokens,
    N outputs, K inputs, --rank): fprop and dgrad each way (the LoRA-SVD calls add the
    rank-r term inside the NVFP4 GEMM's accumulator), and the low-rank kernels alone
    (residual, projections, the GEMM with and without its low-rank stage, the separate
    expansion), L2 flushed before each timed call."""
    from nvfp4_pretraining_linear_b200 import api, synthetic as syn
    M, N, K = dims
    rank = args.rank
    x = syn.normal((M, K), 1.0, seed=12, device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    w = syn.normal((N, K), 0.014, seed=10, device="cuda")
    dy = syn.normal((M, N), 1e-3, seed=14, device="cuda")
    l = syn.normal((N, rank), 0.05, seed=15, device="cuda")
    r = syn.normal((rank, K), 0.05, seed=16, device="cuda")
    rt = syn.normal((K, rank), 0.05, seed=17, device="cuda")       # R^T as the dgrad call takes it
    w_res = api.lora_residual(w, l, r)
    wq_row, wq_col = api.quantize_weight(w_res)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    u = torch.empty((M, rank), dtype=torch.bfloat16, device="cuda")
    xr, xc = api.QTensor.empty(M, K), api.QTensor.empty(K, M)
    dr, dc = api.QTensor.empty(M, N), api.QTensor.empty(N, M)
    fkw = dict(rht_signs=RHT_SIGNS, out=y, xq_row=xr, xq_col=xc)
    dkw = dict(seed=SR_SEED, rht_signs=RHT_SIGNS, out=dx, dyq_row=dr, dyq_col=dc)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    res = {
        "fwd_plain_ms": timed(lambda: api.linear_fwd(x, wq_row, **fkw)),
        "fwd_lora_ms": timed(lambda: api.lora_linear_fwd(x, wq_row, l, r, u=u, **fkw)),
        "dgrad_plain_ms": timed(lambda: api.linear_dgrad(dy, wq_col, **dkw)),
        "dgrad_lora_ms": timed(lambda: api.lora_linear_dgrad(dy, wq_col, l, rt, u=u, **dkw)),
        "residual_ms": timed(lambda: api.lora_residual(w, l, r, out=w_res)),
        "project_ms": timed(lambda: api.lowrank_project(x, r, out=u)),
        "project_scaled_ms": timed(lambda: api.lowrank_project_scaled(x, r, xr.tensor_scale, wq_row.tensor_scale,
                                                                      out=u)),
        "project_dgrad_ms": timed(lambda: api.lowrank_project(dy, l, b_trans=True, out=u)),
        "gemm_plain_ms": timed(lambda: api.gemm(xr, wq_row, out=y)),
        "gemm_lowrank_ms": timed(lambda: api.gemm_lowrank(xr, wq_row, u, l, out=y)),
        "expand_ms": timed(lambda: api.lowrank_expand_add(y, u, l)),
    }
    api.get_status()
    res["project_gbs"] = (2.0 * M * K + 2.0 * M * rank) / res["project_ms"] / 1e6
    res["project_dgrad_gbs"] = (2.0 * M * N + 2.0 * M * rank) / res["project_dgrad_ms"] / 1e6
    res["expand_gbs"] = 4.0 * M * N / res["expand_ms"] / 1e6
    res["residual_gbs"] = 4.0 * N * K / res["residual_ms"] / 1e6
    res["fwd_overhead"] = res["fwd_lora_ms"] / res["fwd_plain_ms"] - 1.0
    res["dgrad_overhead"] = res["dgrad_lora_ms"] / res["dgrad_plain_ms"] - 1.0
    print(json.dumps({"kernel": "lora", "shape": dims, "rank": rank, **res, "steps": args.steps,
                      "l2": "flushed (256 MB write)"}), flush=True)
    return 0


def run_layer(args):
    """The four linears of a 3B-class decoder layer at 32768 tokens (QKV 3072->9216, O
    3072->3072, gate-up 3072->16384, down 8192->3072): forward through the layer, then
    backward in reverse, every linear with W quantised (2D), fprop, dgrad and wgrad.
    Timed three ways on one GPU: everything in order on one stream; each wgrad on a
    second stream so it can fill the SMs that the next dgrad's quantiser and GEMM leave
    idle; and the four wgrads deferred to the end of the backward pass and run as one
    grouped launch (nvfp4_gemm_grouped).  The four wgrad GEMMs alone are also timed
    separately and grouped.  Inputs are resident and each larger than L2."""
    from nvfp4_pretraining_linear_b200 import api, synthetic as syn
    torch.cuda.set_device(0)
    names = list(syn.LAYER3B["linears"])
    linears = [Linear(n, *syn.layer3b_linear(n, device="cuda")) for n in names]
    flops = sum(L.gemm_flops() for L in linears)
    side = torch.cuda.Stream()

    def forward(ev):
        for L in linears:
            ev.mark("q")
            api.quantize(L.w, emit_row=True, emit_col=True, block_2d=True, out_row=L.wq_row, out_col=L.wq_col)
            api.quantize(L.x, emit_row=True, emit_col=True, rht_col=True, rht_signs=RHT_SIGNS, out_row=L.xq_row,
                         out_col=L.xq_col)
            ev.mark("g")
            api.gemm(L.xq_row, L.wq_row, out=L.y)

    def step_in_order(ev):
        forward(ev)
        for L in reversed(linears):
            ev.mark("q")
            api.quantize(L.dy, emit_row=True, emit_col=True, stochastic=True, rht_col=True, seed=SR_SEED,
                         rht_signs=RHT_SIGNS, out_row=L.dyq_row, out_col=L.dyq_col)
            ev.mark("g")
            api.gemm(L.dyq_row, L.wq_col, out=L.dx)
            api.gemm(L.dyq_col, L.xq_col, out=L.dw)
        ev.mark("end")

    def step_side_stream(ev):
        main = torch.cuda.current_stream()
        forward(PhaseEvents(False))
        for L in reversed(linears):
            api.linear_dgrad(L.dy, L.wq_col, seed=SR_SEED, rht_signs=RHT_SIGNS, out=L.dx, dyq_row=L.dyq_row,
                             dyq_col=L.dyq_col)
            ready = torch.cuda.Event()
            ready.record(main)
            side.wait_event(ready)
            api.linear_wgrad(L.dyq_col, L.xq_col, out=L.dw, stream=side)
        done = torch.cuda.Event()
        done.record(side)
        main.wait_event(done)

    def step_grouped(ev):
        forward(PhaseEvents(False))
        for L in reversed(linears):
            api.linear_dgrad(L.dy, L.wq_col, seed=SR_SEED, rht_signs=RHT_SIGNS, out=L.dx, dyq_row=L.dyq_row,
                             dyq_col=L.dyq_col)
        # the four weight gradients in one persistent launch over all their tiles
        api.gemm_grouped([(L.dyq_col, L.xq_col) for L in linears], outs=[L.dw for L in linears])

    def timed(fn):
        for _ in range(args.warmup):
            fn(PhaseEvents(False))
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn(PhaseEvents(False))
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def timed_wgrads(grouped):
        def fn():
            if grouped:
                api.gemm_grouped([(L.dyq_col, L.xq_col) for L in linears], outs=[L.dw for L in linears])
            else:
                for L in linears:
                    api.gemm(L.dyq_col, L.xq_col, out=L.dw)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    clocks = ClockSampler(0)
    t_seq = timed(step_in_order)
    clock_info = clocks.stop()
    t_side = timed(step_side_stream)
    t_grouped = timed(step_grouped)
    t_wg_sep, t_wg_grp = timed_wgrads(False), timed_wgrads(True)
    ev = PhaseEvents(True)
    step_in_order(ev)
    torch.cuda.synchronize()
    phases = ev.totals()
    api.get_status()
    print(json.dumps({
        "kernel": "layer", "workload": "layer3b-decoder-linears-32768-tokens", "gemm_tflop_per_step": flops / 1e12,
        "ms_in_order": t_seq, "ms_wgrad_side_stream": t_side, "ms_wgrad_grouped": t_grouped,
        "wgrads_ms_separate": t_wg_sep, "wgrads_ms_grouped": t_wg_grp, "value": flops / (t_seq * 1e-3) / 1e12,
        "unit": "TFLOP/s (12 GEMMs, 2MNK each, per step time)", "phase_ms": phases,
        "gemm_tflops_in_step": flops / (phases.get("g", float("nan")) * 1e-3) / 1e12,
        "steps": args.steps, "l2": "inputs larger than L2, no flush", "clocks": clock_info}), flush=True)
    return 0


def relaunch_with_ranks(args):
    """`bench.py --gpus N` started as one process: start N ranks on this node with
    torch.distributed.run (one per GPU) and return their exit status."""
    import socket
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(args.gpus),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the single-kernel target measurements (GEMM 16384^3, quantiser 16384^2)")
    ap.add_argument("--kernel", choices=["step", "gemm", "quantize", "chain", "ns", "layer", "lora"],
                    default="step",
                    help="step: the contract benchmark; gemm/quantize: one kernel on --shape; chain: GEMM then "
                         "quantise its output, plain against epilogue-fused amax (--shape M,N,K); ns: NVFP4 "
                         "Newton-Schulz on a Gaussian --shape m,n for --iters steps; layer: the four linears of a "
                         "3B decoder layer at 32768 tokens, in order and with wgrad on a side stream; lora: the LoRA-SVD "
                         "linear against the plain one (--shape M,N,K, --rank)")
    ap.add_argument("--iters", type=int, default=16, help="--kernel ns: Newton-Schulz steps per call")
    ap.add_argument("--rank", type=int, default=32, help="--kernel lora: rank of the BF16 branch")
    ap.add_argument("--shape", default="16384,16384,16384")
    ap.add_argument("--mode", choices=sorted(QUANT_MODES), default="grad")
    ap.add_argument("--out", choices=["bf16", "f32"], default="bf16", help="--kernel gemm: output type")
    ap.add_argument("--accumulate", action="store_true", help="--kernel gemm: add into the output")
    ap.add_argument("--amax-in", action="store_true",
                    help="--kernel quantize: given maxima, no amax pass (2 B read + 0.5625 B per layout per element)")
    args = ap.parse_args()
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.kernel == "layer":
        return run_layer(args)
    if args.kernel != "step":
        return run_kernel(args)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_with_ranks(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
