"""Benchmark of the KDA hot path on B200.

One step = one kda_chunk_fwd over the K3-shaped prefill workload
(B=1, H=96, T=8192, d=128, bf16 inputs, fp32 state, S0=0): every row of the
prefill path (tile loads, gate and decay scaling, intra-chunk transform,
chunk products, state scan, output stores) runs inside the timed region.
The decode workload (256 sequences x 96 heads, fp32 state, one
kda_decode_step per step) is timed in the same run and reported under
"decode".

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch under torch.distributed.run: every rank runs the same
per-GPU workload on its own GPU (weak scaling; heads and sequences are
independent, so there is no collective on the data path); the step time is
the max over ranks.

Timing: CUDA events on the stream the kernels are launched on, a barrier and
a synchronize on both sides of the timed region, inputs (about 1 GB) larger
than L2 so no flush is needed.  SM clocks are sampled with nvidia-smi during
the timed region.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "KDA prefill Mtok/s (H=96,d=128,bf16) + % roofline; decode tok/s + HBM GB/s"

# algorithmic bytes per (token, head) for bf16 q, k, v, g in, o out, beta
BYTES_PER_TOKEN_HEAD = (4 * 128 + 128) * 2 + 2          # 1282
FLOPS_PER_TOKEN_HEAD = 2 * 128 * 128 * 3 + 2 * 16 * 128 * 5   # 118,784
STATE_BYTES = 128 * 128 * 4


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "chunk_fwd_sm100_k3_prefill.json")
PREFILL_SOURCES = ("kda_chunk_sm100.cuh", "sm100_ptx.cuh", "kda_common.cuh")


def _prefill_source_hash():
    import hashlib
    srcs = [os.path.join(ROOT, "gated_delta_rule_60_b200", "csrc", f) for f in PREFILL_SOURCES]
    return hashlib.sha256(b"".join(open(f, "rb").read() for f in srcs)).hexdigest()[:16]


def _measured_traffic():
    """DRAM bytes (read + write) per launch of the prefill kernel, from the
    committed ncu record, or None when the kernel sources changed since that
    capture."""
    try:
        rec = json.load(open(TRAFFIC_JSON))
        if rec.get("kernel_source_sha256_16") != _prefill_source_hash():
            return None
        return float(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def record_traffic(csv_path, command):
    """Write the ncu DRAM counters of one prefill launch (an ncu --csv log of
    dram__bytes_read.sum and dram__bytes_write.sum) to the traffic record,
    keyed by the current kernel source hash."""
    import csv
    vals = {}
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f) if len(r) > 5]
    hdr = rows[0]
    for r in rows[1:]:
        d = dict(zip(hdr, r))
        if "chunk_fwd_sm100" not in d.get("Kernel Name", ""):
            continue
        name, unit = d["Metric Name"], d.get("Metric Unit", "")
        if not name.startswith("dram__bytes_"):
            continue
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(unit)
        if scale is None:
            raise ValueError("unexpected unit %r for %s" % (unit, name))
        vals[name] = float(d["Metric Value"].replace(",", "")) * scale
    rd, wr = vals["dram__bytes_read.sum"], vals["dram__bytes_write.sum"]
    rec = {"kernel": "chunk_fwd_sm100_kernel (K3 prefill: B=1 H=96 T=8192 d=128 bf16)",
           "kernel_source_sha256_16": _prefill_source_hash(),
           "dram_bytes_read": rd, "dram_bytes_write": wr,
           "traffic_bytes_per_launch": rd + wr, "command": command}
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="kda_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap")
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
            os.unlink(self.path)
        except OSError:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _config(T, H, d):
    """The workload both arms report (the reference arm runs a head sample
    of it and says so in its cpu_baseline)."""
    return {"workload": "k3_prefill B=1 H=96 T=8192 d=128 bf16 S0=0, "
                        "chunk 16, one kda_chunk_fwd per step",
            "tokens_per_gpu": T, "heads": H, "head_dim": d,
            "l2": "inputs ~1 GB > L2 (126 MB), no flush",
            "parallelism": "replicas: independent heads/sequences per GPU"}


def _oracle_sample(seconds_target=12.0):
    """Time the fp64 oracle on a bounded sample of the K3 workload: a few
    heads over the full 8192 tokens.  Returns (tokens/s full-H equivalent,
    cores, sample description)."""
    import oracle
    from gated_delta_rule_60_b200 import workloads
    w = workloads.K3_PREFILL
    cores = oracle.threads()
    heads = max(1, min(w.H, cores))
    inp = w.make()
    q, k, v, g, b = (x[:, :heads].contiguous() for x in (inp.q, inp.k, inp.v,
                                                          inp.g, inp.beta))
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.forward(q, k, v, g, b, inp.cu_seqlens, None)
        reps += 1
        if time.perf_counter() - t0 >= seconds_target or reps >= 64:
            break
    dt = time.perf_counter() - t0
    token_heads = reps * heads * w.T_tot
    tok_s = token_heads / w.H / dt
    return tok_s, cores, ("%d of 96 heads x 8192 tokens, %d pass(es), %.1f s; "
                          "value in full-96-head tokens/s" % (heads, reps, dt))


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from gated_delta_rule_60_b200 import workloads
    w = workloads.K3_PREFILL
    cores = oracle.threads()
    heads = max(1, min(w.H, cores))
    inp = w.make()
    q, k, v, g, b = (x[:, :heads].contiguous() for x in (inp.q, inp.k, inp.v,
                                                          inp.g, inp.beta))
    for _ in range(args.warmup):
        oracle.forward(q[:256], k[:256], v[:256], g[:256], b[:256], [0, 256], None)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward(q, k, v, g, b, inp.cu_seqlens, None)
        times.append(time.perf_counter() - t0)
    dt = statistics.median(times)
    value = heads * w.T_tot / w.H / dt / 1e6
    sample = "%d of 96 heads x 8192 tokens per step (full-96-head tokens/s)" % heads
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w.T_tot, w.H, w.dk),
        "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def run_gpu(args):
    from gated_delta_rule_60_b200 import binding, inputs, workloads

    world, rank, local = _dist_init(args.gpus)
    dev = torch.device("cuda", local)
    binding.load_library()
    hbm_peak, tc_peak, peak_kind = _peaks()

    if args.only == "decode":
        stream = torch.cuda.Stream(device=dev)
        torch.cuda.synchronize()
        decode = _measure_decode(dev, stream, args, world, hbm_peak, binding, inputs, workloads)
        if rank == 0:
            print(json.dumps({"only": "decode", "decode": decode}))
        return 0

    if args.only == "backward":
        stream = torch.cuda.Stream(device=dev)
        torch.cuda.synchronize()
        backward = _measure_backward(dev, stream, args, world, binding, inputs)
        if rank == 0:
            print(json.dumps({"only": "backward", "backward": backward}))
        return 0

    # ---------------- prefill workload ----------------
    w = workloads.K3_PREFILL
    inp = w.make()
    T, H, d = w.T_tot, w.H, w.dk
    dq, dk_, dv_, dg, db = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    cu = inp.cu_seqlens.to(dev)
    o = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    hT = torch.empty(1, H, d, d, dtype=torch.float32, device=dev)
    ws_n = binding.kda_chunk_fwd_workspace_size(1, T, H, d, d, torch.bfloat16)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev) if ws_n else None
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    launches_per_step = 1

    def step():
        binding.kda_chunk_fwd(dq, dk_, dv_, dg, db, None, cu, o=o, hT=hT,
                              workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            step()
    stream.synchronize()
    assert binding.kda_stream_status(stream) == binding.KDA_OK

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]

    def keep_busy(seconds):
        # untimed steps of the same work, so that the clock samples (every
        # 100 ms) bracket a timed region that may be only tens of ms long
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            while time.perf_counter() - t0 < seconds:
                for _ in range(4):
                    step()
                stream.synchronize()

    with ClockSampler(local) as clk:
        keep_busy(0.6)
        _barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for i in range(args.steps):
                step()
                ev[i + 1].record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        keep_busy(0.3)
    _barrier(world)
    per_launch = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = _max_over_ranks(total_ms, world)
    ms_step = total_ms / args.steps
    st = binding.kda_stream_status(stream)
    if st != binding.KDA_OK:
        raise RuntimeError("kernel status: " + binding.kda_status_string(st))
    clocks = clk.summary()

    alg_bytes = T * H * BYTES_PER_TOKEN_HEAD + H * STATE_BYTES
    kern_ms = statistics.mean(per_launch)
    achieved = alg_bytes / (kern_ms * 1e-3) / 1e9
    value = world * T / (ms_step * 1e-3) / 1e6

    if args.only == "prefill":
        if rank == 0:
            print(json.dumps({"only": "prefill", "ms": kern_ms, "Mtok_s": value,
                              "hbm_frac": achieved / hbm_peak}))
        return 0

    # ---------------- end to end, host buffers ----------------
    e2e = None
    if not args.skip_e2e:
        e2e = _measure_e2e(inp, dev, cu, o, hT, ws, stream, args, world, T, H, d, binding)
    del dq, dk_, dv_, dg, db, o
    torch.cuda.empty_cache()
    extra = {}
    if not args.skip_workloads:
        for wl in (workloads.VARLEN, workloads.LONG):
            extra[wl.name] = _measure_workload(wl, dev, stream, args, world, hbm_peak, binding,
                                               inputs)
            torch.cuda.empty_cache()
        extra["backward_2k"] = _measure_backward(dev, stream, args, world, binding, inputs)
        torch.cuda.empty_cache()
        extra.update(_measure_layer_rows(dev, stream, world, hbm_peak, kern_ms, binding,
                                         inputs))
    decode = None
    if not args.skip_decode:
        decode = _measure_decode(dev, stream, args, world, hbm_peak, binding, inputs, workloads)
    return _report(args, world, rank, value, ms_step, achieved, hbm_peak, peak_kind, alg_bytes,
                   kern_ms, T, H, d, tc_peak, e2e, decode, clocks, launches_per_step, extra)


def _measure_workload(w, dev, stream, args, world, hbm_peak, binding, inputs):
    """One prefill workload (drawn on the device), timed like the headline."""
    pre = inputs.make_prefill(list(w.lengths), w.H, w.dk, w.dv, w.dtype, w.seed,
                              w.h0_std, device=dev)
    torch.cuda.synchronize()
    N, T = len(w.lengths), w.T_tot
    o = torch.empty(T, w.H, w.dv, dtype=w.dtype, device=dev)
    hT = torch.empty(N, w.H, w.dk, w.dv, dtype=torch.float32, device=dev)
    ws_n = binding.kda_chunk_fwd_workspace_size(N, T, w.H, w.dk, w.dv, w.dtype)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev) if ws_n else None

    def step():
        binding.kda_chunk_fwd(pre.q, pre.k, pre.v, pre.g, pre.beta, pre.h0, pre.cu_seqlens,
                              o=o, hT=hT, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    steps = max(2, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
    stream.synchronize()
    assert binding.kda_stream_status(stream) == binding.KDA_OK
    ms = _max_over_ranks(e0.elapsed_time(e1) / steps, world)
    alg = T * w.H * BYTES_PER_TOKEN_HEAD + N * w.H * STATE_BYTES * (2 if w.h0_std else 1)
    gbs = alg / (ms * 1e-3) / 1e9
    return {"tokens": T, "heads": w.H, "sequences": N, "ms": ms,
            "Mtok_s": world * T / (ms * 1e-3) / 1e6, "hbm_gbs": gbs,
            "frac_of_peak": gbs / hbm_peak, "launches_per_step": 1 if not ws_n else 3}


# fp32 operations per (token, head) of the backward kernel at d = 128: the
# checkpoint sweep and the chunk recompute (6 d^2 each: the decayed read and
# the state update) and the reverse token derivative (18 d^2)
BWD_FLOPS_PER_TOKEN_HEAD = 30 * 128 * 128
# fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flops x 1.965 GHz
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def _measure_backward(dev, stream, args, world, binding, inputs):
    """The prefill's gradient (kda_chunk_bwd) on 96 heads x 2,048 tokens, bf16,
    with dO and dhT given: a correctness-first fp32 CUDA-core kernel, timed
    for reference."""
    T, H, d = 2048, 96, 128
    pre = inputs.make_prefill([T], H, d, d, torch.bfloat16, 1009, 0.02, device=dev)
    gen = torch.Generator(device=dev).manual_seed(5)
    dO = torch.randn(T, H, d, generator=gen, device=dev).to(torch.bfloat16)
    dhT = torch.randn(1, H, d, d, generator=gen, device=dev) * 0.1
    torch.cuda.synchronize()

    def step():
        return binding.kda_chunk_bwd(pre.q, pre.k, pre.v, pre.g, pre.beta, dO, pre.h0,
                                     pre.cu_seqlens, dhT, stream=stream)

    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    steps = 3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
    stream.synchronize()
    assert binding.kda_stream_status(stream) == binding.KDA_OK
    ms = _max_over_ranks(e0.elapsed_time(e1) / steps, world)
    tflops = T * H * BWD_FLOPS_PER_TOKEN_HEAD / (ms * 1e-3) / 1e12
    return {"tokens": T, "heads": H, "sequences": 1, "ms": ms,
            "Mtok_s": world * T / (ms * 1e-3) / 1e6, "fp32_tflops": tflops,
            "frac_of_fp32_peak": tflops / FP32_PEAK_TFLOPS, "launches_per_step": 1}


def _events_ms(stream, fn, warmup, steps):
    """Mean device time of fn() over `steps` launches on `stream` (CUDA
    events), after `warmup` untimed launches."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / steps


# (tokens, heads, head size) of the rows around the operator
LAYER_ROW_SHAPES = {"prologue_k3": (8192, 96, 128), "gated_k3": (8192, 96, 128),
                    "softplus_2k": (2048, 96, 128)}


def _prologue_local(dev, stream, binding, inputs):
    T, H, d = LAYER_ROW_SHAPES["prologue_k3"]
    li = inputs.make_layer([T], H, d, torch.bfloat16, seed=1011, device=dev)
    torch.cuda.synchronize()
    ms = _events_ms(stream, lambda: binding.kda_prologue(
        li.xq, li.xk, li.xv, li.wq, li.wk, li.wv, li.beta_raw, li.cu_seqlens,
        stream=stream), 3, 10)
    # xq, xk, xv, beta_raw read and q, k, v, beta written (bf16; 1,540 B per
    # (token, head) at d = 128), plus the fp32 taps
    alg = T * H * (2 * 3 * d * 2 + 2 * 2) + 3 * H * d * 4 * 4
    return ms, alg, T, H


def _gated_local(dev, stream, binding, inputs):
    T, H, d = LAYER_ROW_SHAPES["gated_k3"]
    pre = inputs.make_prefill([T], H, d, d, torch.bfloat16, 1012, device=dev)
    gen = torch.Generator(device=dev).manual_seed(6)
    z = torch.randn(T, H, d, generator=gen, device=dev).to(torch.bfloat16)
    o = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    hT = torch.empty(1, H, d, d, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    ms = _events_ms(stream, lambda: binding.kda_chunk_fwd_gated(
        pre.q, pre.k, pre.v, pre.g, pre.beta, z, None, pre.cu_seqlens, o=o, hT=hT,
        stream=stream), 3, 10)
    # the prefill's bytes plus z (1,538 B per (token, head) at d = 128) and hT
    alg = T * H * ((5 * d + d) * 2 + 2) + H * d * d * 4
    return ms, alg, T, H


def _softplus_local(dev, stream, binding, inputs):
    T, H, d = LAYER_ROW_SHAPES["softplus_2k"]
    pre = inputs.make_prefill([T], H, d, d, torch.bfloat16, 1013, 0.02, device=dev)
    o = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    hT = torch.empty(1, H, d, d, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    ms = _events_ms(stream, lambda: binding.kda_chunk_fwd_softplus(
        pre.q, pre.k, pre.v, pre.g, pre.beta, pre.h0, pre.cu_seqlens, o=o, hT=hT,
        stream=stream), 1, 3)
    # the prefill's bytes (1,282 B per (token, head) at d = 128), h0 and hT
    alg = T * H * ((4 * d + d) * 2 + 2) + 2 * H * d * d * 4
    return ms, alg, T, H


def _measure_layer_rows(dev, stream, world, hbm_peak, plain_ms, binding, inputs):
    """The rows around the operator, each in one launch per step:
    - prologue_k3: kda_prologue on the K3 shape (96 heads x 8,192 tokens,
      d = 128, bf16), a memory-bound pass;
    - gated_k3: kda_chunk_fwd_gated on the K3 shape (the output gate fused
      into the tensor-core prefill), with its cost over the plain launch;
    - softplus_2k: kda_chunk_fwd_softplus on 96 heads x 2,048 tokens (the
      unbounded gate on the fp32 CUDA-core kernel, a correctness path).
    Each rank measures on its own; a failure is reported in the row instead
    of ending the run, and every rank takes the same collective steps."""
    rows = {}
    for name, fn in (("prologue_k3", _prologue_local), ("gated_k3", _gated_local),
                     ("softplus_2k", _softplus_local)):
        _barrier(world)
        err = None
        try:
            ms, alg, T, H = fn(dev, stream, binding, inputs)
            st = binding.kda_stream_status(stream)
            if st != binding.KDA_OK:
                err = "kernel status: " + binding.kda_status_string(st)
        except Exception as e:                      # reported in the JSON line
            err = "%s: %s" % (type(e).__name__, e)
        ms = _max_over_ranks(float("inf") if err else ms, world)
        if err or ms == float("inf"):
            rows[name] = {"error": err or "failed on another rank"}
        else:
            gbs = alg / (ms * 1e-3) / 1e9
            rows[name] = {"tokens": T, "heads": H, "ms": ms,
                          "Mtok_s": world * T / (ms * 1e-3) / 1e6, "hbm_gbs": gbs,
                          "frac_of_peak": gbs / hbm_peak,
                          "algorithmic_bytes_per_launch": alg, "launches_per_step": 1}
        torch.cuda.empty_cache()
    if "ms" in rows.get("gated_k3", {}):
        rows["gated_k3"]["cost_over_plain"] = rows["gated_k3"]["ms"] / plain_ms - 1.0
    return rows


def _measure_e2e(inp, dev, cu, o, hT, ws, stream, args, world, T, H, d, binding):
    """End to end through the public API: every step copies its inputs from
    pinned host memory, runs kda_chunk_fwd and reads o and hT back.  Steps are
    pipelined over two buffer sets: the host-to-device copy of step i+1 and the
    device-to-host copy of step i-1 run on their own streams while step i
    computes (events order each buffer's reuse)."""
    names = ("q", "k", "v", "g", "beta")
    host = {n: getattr(inp, n).pin_memory() for n in names}
    o_host = [torch.empty(T, H, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h_host = [torch.empty(1, H, d, d, dtype=torch.float32).pin_memory() for _ in range(2)]
    dev_in = [{n: torch.empty_like(t, device=dev) for n, t in host.items()} for _ in range(2)]
    dev_o = [o, torch.empty_like(o)]
    dev_h = [hT, torch.empty_like(hT)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host[0].numel() * 2 + h_host[0].numel() * 4
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    n_steps = max(2, min(args.steps, 10))
    ev = lambda: torch.cuda.Event()
    in_ready = [ev() for _ in range(n_steps + 1)]
    done = [ev() for _ in range(n_steps + 1)]
    out_read = [ev() for _ in range(n_steps + 1)]

    def run(n, t0=None):
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[i - 2])          # the kernel of step i-2 read buffer b
                for name in names:
                    dev_in[b][name].copy_(host[name], non_blocking=True)
                in_ready[i].record(s_in)
            stream.wait_event(in_ready[i])
            if i >= 2:
                stream.wait_event(out_read[i - 2])        # o, hT of buffer b were read back
            x = dev_in[b]
            binding.kda_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], None, cu,
                                  o=dev_o[b], hT=dev_h[b], workspace=ws, stream=stream)
            done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i])
                o_host[b].copy_(dev_o[b], non_blocking=True)
                h_host[b].copy_(dev_h[b], non_blocking=True)
                out_read[i].record(s_out)

    run(2)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    run(n_steps)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / n_steps, world)
    e2e_val = world * T / (e2e_ms * 1e-3) / 1e6
    del dev_in
    return {"value": e2e_val, "unit": "Mtok/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "pipelined": "2 buffer sets; H2D, compute, D2H on 3 streams"}


def _measure_decode(dev, stream, args, world, hbm_peak, binding, inputs, workloads):
    B, Hd, D = workloads.DECODE_B, workloads.DECODE_H, workloads.DECODE_D
    # the state: a 512-token prefill of every sequence (drawn on the device)
    pre = inputs.make_prefill([workloads.DECODE_PREFILL] * B, Hd, D, D,
                              torch.bfloat16, workloads.DECODE_SEED, device=dev)
    torch.cuda.synchronize()
    S = torch.empty(B, Hd, D, D, dtype=torch.float32, device=dev)
    od_pre = torch.empty(B * workloads.DECODE_PREFILL, Hd, D, dtype=torch.bfloat16,
                         device=dev)
    ws_pre_n = binding.kda_chunk_fwd_workspace_size(
        B, B * workloads.DECODE_PREFILL, Hd, D, D, torch.bfloat16)
    ws_pre = torch.empty(ws_pre_n, dtype=torch.uint8, device=dev) if ws_pre_n else None
    binding.kda_chunk_fwd(pre.q, pre.k, pre.v, pre.g, pre.beta, None,
                          pre.cu_seqlens, o=od_pre, hT=S, workspace=ws_pre,
                          stream=stream)
    stream.synchronize()
    del pre, od_pre, ws_pre
    torch.cuda.empty_cache()
    xs = [inputs.make_decode_step(B, Hd, D, D, torch.bfloat16,
                                  workloads.DECODE_STEP_SEED0 + s, device=dev)
          for s in range(4)]
    xs = [{n: getattr(x, n) for n in ("q", "k", "v", "g", "beta")} for x in xs]
    torch.cuda.synchronize()
    od = torch.empty(B, Hd, D, dtype=torch.bfloat16, device=dev)

    def dstep(i):
        x = xs[i % len(xs)]
        binding.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S,
                                o=od, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            dstep(i)
    stream.synchronize()
    dsteps = max(args.steps, 10)
    dev_ev = [torch.cuda.Event(enable_timing=True) for _ in range(dsteps + 1)]
    _barrier(world)
    with torch.cuda.stream(stream):
        dev_ev[0].record(stream)
        for i in range(dsteps):
            dstep(i)
            dev_ev[i + 1].record(stream)
    stream.synchronize()
    dms = [dev_ev[i].elapsed_time(dev_ev[i + 1]) for i in range(dsteps)]
    d_ms = _max_over_ranks(statistics.median(dms), world)
    d_bytes = 2 * B * Hd * D * D * 4 + B * Hd * (4 * D + D) * 2 + B * Hd * 2
    d_gbs = d_bytes / (d_ms * 1e-3) / 1e9
    assert binding.kda_stream_status(stream) == binding.KDA_OK
    return {"workload": "256 seqs x 96 heads, d=128, fp32 state built by a 512-token "
                        "prefill, one kda_decode_step per step",
            "tok_s": world * B / (d_ms * 1e-3), "ms_per_step": d_ms,
            "hbm_gbs": d_gbs, "frac_of_peak": d_gbs / hbm_peak,
            "algorithmic_bytes_per_step": d_bytes}


def _report(args, world, rank, value, ms_step, achieved, hbm_peak, peak_kind, alg_bytes,
            kern_ms, T, H, d, tc_peak, e2e, decode, clocks, launches_per_step, extra):
    if rank != 0:
        _barrier(world)
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        tok_s, cores, sample = _oracle_sample()
        cpu = {"value": tok_s / 1e6, "unit": "Mtok/s", "cores": cores,
               "kind": "oracle", "sample": sample}

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "Mtok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": _config(T, H, d),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak,
                     "unit": "GB/s", "frac": achieved / hbm_peak,
                     "traffic": _measured_traffic(), "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "kernel_ms": kern_ms,
                     "tensor_tflops": T * H * FLOPS_PER_TOKEN_HEAD / (kern_ms * 1e-3) / 1e12,
                     "tensor_peak_tflops": tc_peak},
        "e2e": e2e,
        "decode": decode,
        "workloads": extra,
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "gpu_launches": args.steps * launches_per_step,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))
    if world > 1:
        _barrier(world)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="libkda", choices=["libkda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true",
                    help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--skip-decode", action="store_true",
                    help="skip the decode measurement")
    ap.add_argument("--skip-workloads", action="store_true",
                    help="skip the varlen and long-context prefill measurements")
    ap.add_argument("--only", choices=["prefill", "decode", "backward"], default=None,
                    help="run one part only (for profiling): the K3 prefill, the decode "
                         "or the backward")
    ap.add_argument("--record-traffic", metavar="NCU_CSV", default=None,
                    help="write the prefill DRAM traffic record from an ncu --csv log of "
                         "dram__bytes_read.sum and dram__bytes_write.sum (no GPU needed)")
    ap.add_argument("--record-command", default="",
                    help="the ncu command line that produced NCU_CSV (kept in the record)")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic, args.record_command)
        return 0
    if args.impl == "reference":
        return run_reference(args)
    rc = run_gpu(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
