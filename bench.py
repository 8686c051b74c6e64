"""Benchmark of the routed MoE expert FFN layer (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME|all]

A step is one pass of the whole layer -- routing, gather (+ FP8 quantisation),
the w1/w3 + SwiGLU group GEMM, the w2 + scatter group GEMM and the bf16
finalize -- over one batch of T tokens whose inputs are already resident in
HBM.  The headline workload is the Mixtral-8x7B-shaped FP8 decode layer
(T=16, d_model=4096, d_ff=14336, E=8, top-2); by default (``--config all``)
the same run also times every other workload of the Mixtral expert shape
(prefill T=4096 FP8, skewed-routing T=8192 BF16, the FP8 batch sweep
T = 1, 128, 1024, 16384, decode / prefill with MX FP4 expert weights, and a
BF16 training step at T=4096: forward and backward) and reports
each as a sub-record under ``configs`` with its own step time, roofline, CPU
baseline and end-to-end number.

With N > 1, one process per GPU (under torch.distributed.run; ``--gpus N``
without a launcher starts one itself) runs its own token batch against its
own copy of the weights (weak scaling); the only collectives are the timing
barriers and the max over ranks.

``--impl reference`` times the CPU oracle (fp64, the host's CPU cores) on a
bounded sample of the headline workload; under N ranks rank 0 alone runs it.
"""
import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (Mixtral-8x7B shape FP8, T=16 and T=4096); % of roofline"

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)

HEADLINE = "decode"
# the workloads of one default run, headline first; the sweep points share one weight set
ALL_CONFIGS = ["decode", "prefill", "skewed", "sweep_T1", "sweep_T128", "sweep_T1024", "sweep_T16384",
               "decode_mxfp4", "prefill_mxfp4", "train_prefill"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", default="all", help="a workload name, or 'all' (headline + every other workload)")
    p.add_argument("--cpu-sample-seconds", type=float, default=12.0, help="oracle sample of the headline workload")
    p.add_argument("--sub-cpu-sample-seconds", type=float, default=4.0, help="oracle sample of each other workload")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true", help="skip the end-to-end pass (profiling runs)")
    p.add_argument("--fp8-peak-probe", action="store_true",
                   help="measure the dense e4m3 GEMM rate of torch._scaled_mm (context for the FP8 roofline) and exit")
    return p.parse_args(argv)


def fp8_peak_probe(n=8192, burst_reps=10, sustained_s=3.0):
    """Dense e4m3 x e4m3 -> bf16 GEMM rate of the library GEMM (torch._scaled_mm,
    per-tensor scales) at n^3: best of `burst_reps` single calls (burst) and
    the average over a loop of about `sustained_s` seconds (under the power
    cap), CUDA events on the current stream, clocks sampled meanwhile.  A
    reference figure for the FP8 fractions, beside bf16 x 2."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    g = torch.Generator(device=dev).manual_seed(0)
    a = (torch.randn(n, n, device=dev, generator=g) * 0.5).to(torch.float8_e4m3fn)
    b = (torch.randn(n, n, device=dev, generator=g) * 0.5).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)  # noqa: E731
    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    best = float("inf")
    for _ in range(burst_reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    reps = max(10, int(sustained_s * 1e3 / best))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        mm()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    sust = e0.elapsed_time(e1) / reps
    return {"probe": "torch._scaled_mm e4m3 x e4m3 -> bf16, per-tensor scales", "n": n,
            "burst_tflops": flop / (best / 1e3) / 1e12, "burst_ms": best,
            "sustained_tflops": flop / (sust / 1e3) / 1e12, "sustained_ms": sust, "sustained_reps": reps,
            "clocks": clk}


def config_names(arg):
    if arg == "all":
        return list(ALL_CONFIGS)
    names = [n.strip() for n in arg.split(",") if n.strip()]
    import moe_inputs
    known = {**moe_inputs.CONFIGS, **moe_inputs.BWD_CONFIGS}
    for n in names:
        if n not in known:
            raise SystemExit(f"unknown workload {n!r}; known: {sorted(known)}")
    return names


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(spec, name):
    return (f"{name}: T={spec['T']} tokens, d_model={spec['H']}, d_ff={spec['F']}, E={spec['E']}, "
            f"top-{spec['k']}, {spec['dtype']}" + (", skewed routing" if spec["skew"] else ""))


def weight_bytes(dtype, rows, cols):
    """Bytes of one expert matrix [rows, cols] with its scales: bf16; e4m3 +
    one fp32 scale per row; MX FP4 = half a byte per code + one byte per 32."""
    if dtype == "bf16":
        return 2 * rows * cols
    if dtype == "fp8":
        return rows * cols + 4 * rows
    return rows * cols // 2 + rows * cols // 32


def algorithmic(spec, counts):
    """Algorithmic FLOPs and bytes of the layer and of each GEMM kernel, from
    the routed expert counts (experts with no tokens read no weights)."""
    T, H, F, E, k = spec["T"], spec["H"], spec["F"], spec["E"], spec["k"]
    dt = spec["dtype"]
    ba = 2 if dt == "bf16" else 1  # activation / h bytes per element
    sf = (lambda n: n // 32) if dt != "bf16" else (lambda n: 0)  # h's block scales
    A = T * k
    active = sum(1 for c in counts if c > 0)
    s1_bytes = active * weight_bytes(dt, 2 * F, H) + A * H * ba + A * F * ba + sf(A * F)
    s2_bytes = active * weight_bytes(dt, H, F) + A * F * ba + sf(A * F) + T * H * 4
    layer_bytes = active * (weight_bytes(dt, 2 * F, H) + weight_bytes(dt, H, F)) + T * H * 2 * 2 + 4 * T * E
    return dict(s1_flops=4.0 * H * F * A, s2_flops=2.0 * H * F * A, layer_flops=6.0 * H * F * A + 2.0 * T * E,
                s1_bytes=float(s1_bytes), s2_bytes=float(s2_bytes), layer_bytes=float(layer_bytes), active=active)


def power_capped(window_ms, clk):
    """Whether the timed work ran in the sustained regime: a timed region of a
    second or more, or SM clocks sampled well below their maximum (the power
    cap pulls a long tensor-core run to about 1.3 GHz).  The sustained GEMM
    peak is the denominator then, the burst one otherwise."""
    if window_ms >= 1000.0:
        return True
    return bool(clk) and clk.get("sm_mhz", 0) < 0.9 * clk.get("sm_max_mhz", 0)


def roofline(spec, alg, dom, dom_ms, window_ms, peaks, peak_kind, name, clk=None):
    """Roofline record of the dominant kernel: algorithmic bytes (HBM-bound
    shapes) or FLOPs (tensor-bound shapes) per launch over its average launch
    time, against the measured peak."""
    H, F = spec["H"], spec["F"]
    fp8 = spec["dtype"] != "bf16"  # e4m3 activations: the FP8 tensor rate (MX FP4 weights too)
    wb = weight_bytes(spec["dtype"], 3 * H, F)
    decode_like = alg["active"] * wb / 6.5e12 > alg["layer_flops"] / ((2 * 2.25e15) if fp8 else 2.25e15)
    if not dom.startswith("stage"):
        return {"bound": "hbm", "achieved": None, "peak": float(peaks.get("hbm_gbs", 6650.0)), "unit": "GB/s",
                "frac": None, "traffic": None, "kernel": dom, "kernel_ms": dom_ms}
    per = "s1" if dom.startswith("stage1") else "s2"
    if decode_like:
        ach = alg[per + "_bytes"] / (dom_ms / 1e3) / 1e9
        peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "traffic": recorded_traffic(dom, name), "peak_source": f"{peak_kind} HBM copy bandwidth",
                "algorithmic_per_launch": alg[per + "_bytes"]}
    else:
        ach = alg[per + "_flops"] / (dom_ms / 1e3) / 1e12
        long_run = power_capped(window_ms, clk)
        key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
        base = float(peaks.get(key, FALLBACK_PEAKS[key]))
        peak = base * (FP8_PER_BF16 if fp8 else 1.0)
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": recorded_traffic(dom, name),
                "peak_source": f"{peak_kind} {'sustained' if long_run else 'burst'} bf16 cuBLAS"
                               + (" x 2 (fp8/bf16 nominal ratio)" if fp8 else ""),
                "algorithmic_per_launch": alg[per + "_flops"]}
    roof["kernel"] = dom
    roof["kernel_ms"] = dom_ms
    return roof


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while GPU work runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.t0 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        self.t0 = time.perf_counter()

    def stop(self):
        if self.proc is None:
            return None
        window = (time.perf_counter() - self.t0) * 1e3 if self.t0 else None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sms:
            return None
        rec = {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
               "samples": len(sms)}
        if window is not None:
            rec["window_ms"] = round(window, 1)
        return rec


def source_sha(kernel="stage1_w13_swiglu", workload=""):
    """Hash of the code a kernel is compiled from (the grouped GEMMs of the
    forward: gemm.cu; of the backward and of the training forward -- every
    GEMM of a train_* workload: bwd.cu and bwd.cuh; both with the library
    headers they include -- the public header gives them only status codes),
    comments and blank space removed, so that an edit to a comment keeps the
    recorded counters."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_routed_02_b200", "csrc")
    files = ("bwd.cu", "bwd.cuh", "kernels.cuh", "ptx.cuh") if kernel.startswith("bwd") or workload.startswith(
        "train") else ("gemm.cu", "kernels.cuh", "ptx.cuh")
    for path in [os.path.join(csrc, n) for n in files]:
        with open(path) as f:
            code = f.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        code = " ".join(code.split())
        h.update(os.path.basename(path).encode() + code.encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f)
    except (OSError, ValueError):
        return None
    sha = source_sha(kernel, workload)
    for r in recs:
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_sha") == sha:
            return r.get("dram_bytes_per_launch")
    return None


def host_cores():
    """CPU cores this process may run on (the oracle's thread count; a launcher
    such as torch.distributed.run sets OMP_NUM_THREADS=1, which the oracle
    would otherwise inherit)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_baseline(case, spec, name, seconds):
    """Time the oracle (as it stands) on whole-token samples of the workload."""
    import numpy as np

    import moe_inputs
    import oracle
    nc = moe_inputs.to_numpy(case)
    T = spec["T"]
    batch = max(1, min(T, 8))
    cores = host_cores()
    tokens_done = 0
    t0 = time.perf_counter()
    i = 0
    while True:
        tok = (np.arange(batch) + i * batch) % T
        oracle.moe_ffn_tokens(nc, tok.astype(np.int32), nthreads=cores)
        tokens_done += batch
        i += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens_done / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{tokens_done} tokens of the {name} workload ({batch}-token batches, whole layer per token: "
                      f"routing, both expert GEMMs, combine), {dt:.1f} s"}


def rank_batch(spec, rank):
    """Seed of rank r's token batch under weak scaling (the weights are shared)."""
    return spec["seed"] + 100 * rank


def max_over_ranks(value_ms, world, device=None):
    """Largest elapsed time over all ranks (the timing of a multi-GPU run)."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(argv, n):
    """Re-run this script as n ranks (one per GPU) under torch.distributed.run
    on 127.0.0.1; returns the exit status of the launcher."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_reference(args, rank):
    """The oracle as it stands, on the host cores: each step is one oracle call on
    a small batch of the headline workload's tokens (sized so the run stays
    within a couple of minutes)."""
    if rank != 0:
        return 0
    import numpy as np

    import moe_inputs
    import oracle
    names = config_names(args.config)
    name = HEADLINE if HEADLINE in names else names[0]
    spec = moe_inputs.CONFIGS[name]
    case = moe_inputs.make_case(spec["T"], spec["H"], spec["F"], spec["E"], spec["k"], spec["dtype"], spec["seed"],
                                spec["skew"])
    nc = moe_inputs.to_numpy(case)
    T = spec["T"]
    batch = max(1, min(T, 8))
    cores = host_cores()
    t0 = time.perf_counter()
    oracle.moe_ffn_tokens(nc, np.arange(batch, dtype=np.int32), nthreads=cores)
    per_call = time.perf_counter() - t0
    budget = 120.0
    while batch > 1 and per_call * (args.steps + args.warmup) > budget:
        batch //= 2
        per_call /= 2
    calls = [((np.arange(batch) + i * batch) % T).astype(np.int32) for i in range(args.warmup + args.steps)]
    for tok in calls[:args.warmup]:
        oracle.moe_ffn_tokens(nc, tok, nthreads=cores)
    t0 = time.perf_counter()
    for tok in calls[args.warmup:]:
        oracle.moe_ffn_tokens(nc, tok, nthreads=cores)
    dt = time.perf_counter() - t0
    value = batch * args.steps / dt
    cb = {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
          "sample": f"{args.steps} oracle calls of {batch} tokens each from the {name} workload (whole layer per "
                    f"token), {dt:.1f} s"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(spec, name), "T": spec["T"], "d_model": spec["H"], "d_ff": spec["F"],
                       "experts": spec["E"], "top_k": spec["k"], "weights": spec["dtype"]},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


class Weights:
    """Device weights of one (shape, dtype, seed), prepared once and shared by
    every workload drawn from the same weight seed (the sweep points)."""

    def __init__(self):
        self.key = None
        self.w = None

    def get(self, moe, case, spec, dev):
        import torch
        key = (spec["H"], spec["F"], spec["E"], spec["dtype"], spec["seed"])
        if key != self.key:
            self.w = None
            torch.cuda.empty_cache()
            fp8 = spec["dtype"] == "fp8"
            if spec["dtype"] == "mxfp4":
                w13, s13, w2, s2 = moe.prepare_weights_mx(*(case[n].to(dev) for n in ("w1", "w3", "s1", "s3", "w2",
                                                                                        "s2")))
            else:
                w13, s13, w2 = moe.prepare_weights(case["w1"].to(dev), case["w3"].to(dev),
                                                   case["s1"].to(dev) if fp8 else None,
                                                   case["s3"].to(dev) if fp8 else None, case["w2"].to(dev))
                s2 = case["s2"].to(dev) if fp8 else None
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            self.key, self.w = key, (w13, s13, w2, s2)
        return self.w


def run_gpu_config(args, moe, name, spec, case, weights, dev, world, rank, cpu_seconds):
    """Time one workload: the device-timed region (K steps, inputs resident),
    a per-kernel pass, and the end-to-end pass through the public call with
    host buffers.  Returns its record."""
    import torch
    import torch.distributed as dist
    T, H, F, E, k = spec["T"], spec["H"], spec["F"], spec["E"], spec["k"]
    fp8 = {"bf16": False, "fp8": True, "mxfp4": "mxfp4"}[spec["dtype"]]  # the binding's dtype argument

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and cpu_seconds > 0:
        cb = cpu_baseline(case, spec, name, cpu_seconds)

    w13, s13, w2, s2 = weights.get(moe, case, spec, dev)
    if rank > 0:  # weak scaling: each rank its own batch (seed offset by rank), the same weights
        import moe_inputs
        x_cpu = moe_inputs.make_x(T, H, rank_batch(spec, rank))
        lg_cpu = moe_inputs.make_logits(T, E, rank_batch(spec, rank), spec["skew"])
    else:
        x_cpu, lg_cpu = case["x"], case["logits"]
    x = x_cpu.to(dev)
    logits = lg_cpu.to(dev)
    dt_code = moe.dtype_code(spec["dtype"])
    ws = moe.workspace(T, H, F, E, k, dt_code, dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        moe.ffn_forward(x, logits, w13, s13, w2, s2, k, F, fp8, out=out, ws=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = moe.moe_get_status(None)
    if st != 0:
        raise RuntimeError(f"{name}: device status {moe.STATUS_NAMES.get(st, st)} after warm-up")
    counts = moe.ws_view(ws, T, H, F, E, k, dt_code, "counts", torch.int32).cpu().tolist()

    # ---------------- device-timed region (inputs resident in HBM).  No events
    # between the kernels here: an event recorded between two kernels would
    # stop the next one from starting while the previous one drains.  The
    # clock sampler runs from just before this region to the end of the
    # end-to-end pass (all of this workload's GPU work).
    clocks = ClockSampler(torch.cuda.current_device())
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)  # let the sampler start
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, dev)

    # ---------------- per-kernel durations: the same K steps again, with a CUDA
    # event pair around every kernel on its launch stream (moe_profile_*)
    moe.moe_profile_read(reset=True)
    moe.moe_profile_enable(1)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    moe.moe_profile_enable(0)
    kern = moe.moe_profile_read(reset=True)
    st = moe.moe_get_status(None)
    if st != 0:
        raise RuntimeError(f"{name}: device status {moe.STATUS_NAMES.get(st, st)} in the timed region")
    ms_step = ms_total / args.steps
    value = T * world * args.steps / (ms_total / 1e3)

    # ---------------- end to end through the public API: pinned host in, result back to host.
    # A serving loop's pipeline: two sets of device buffers; step i's inputs go
    # up on one copy stream and step i-1's result comes down on another while
    # the layer runs, each step waiting only for the copies it needs.
    e2e = None
    if not args.no_e2e:
        x_h = x.cpu().pin_memory()
        lg_h = logits.cpu().pin_memory()
        outs_h = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        xs_d, lgs_d, outs_d = [x, x.clone()], [logits, logits.clone()], [out, torch.empty_like(out)]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        for e in comp_done + d2h_done:
            e.record(stream)

        def e2e_step(i):
            b = i % 2
            h2d_s.wait_event(comp_done[b])  # the layer two steps back has read these inputs
            with torch.cuda.stream(h2d_s):
                xs_d[b].copy_(x_h, non_blocking=True)
                lgs_d[b].copy_(lg_h, non_blocking=True)
            h2d_done[b].record(h2d_s)
            stream.wait_event(h2d_done[b])
            stream.wait_event(d2h_done[b])  # the result two steps back has been read out
            moe.ffn_forward(xs_d[b], lgs_d[b], w13, s13, w2, s2, k, F, fp8, out=outs_d[b], ws=ws, stream=stream)
            comp_done[b].record(stream)
            d2h_s.wait_event(comp_done[b])
            with torch.cuda.stream(d2h_s):
                outs_h[b].copy_(outs_d[b], non_blocking=True)
            d2h_done[b].record(d2h_s)

        for i in range(max(3, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ev0.record(stream)
        h2d_s.wait_event(ev0)  # no copy of the timed steps starts before the clock does
        d2h_s.wait_event(ev0)
        for i in range(args.steps):
            e2e_step(i)
        for e in d2h_done:
            stream.wait_event(e)
        ev1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
        last = (args.steps - 1) % 2
        if not torch.equal(outs_h[last], outs_d[last].cpu()):
            raise RuntimeError(f"{name}: the result read back to the host is not the last step's output")
        e2e = {"value": T * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": T * H * 2 + T * E * 4, "d2h_bytes_per_step": T * H * 2,
               "ms_per_step": e2e_ms / args.steps}
        st = moe.moe_get_status(None)
        if st != 0:
            raise RuntimeError(f"{name}: device status {moe.STATUS_NAMES.get(st, st)} in the end-to-end pass")
    clk = clocks.stop()

    # ---------------- roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    alg = algorithmic(spec, counts)
    names = moe.FWD_KERNELS
    dom = max(names, key=lambda n: kern[n][0])
    dom_ms = kern[dom][0] / max(1, kern[dom][1])
    roof = roofline(spec, alg, dom, dom_ms, ms_total, peaks, peak_kind, name, clk)
    launches = sum(v[1] for v in kern.values())  # K steps, the same count as the timed region
    rec = {
        "value": value, "unit": "tokens/s", "ms_per_step": ms_step, "steps": args.steps, "warmup": args.warmup,
        "dtype": {"fp8": "fp8_e4m3 (fp32 accumulate)", "bf16": "bf16 (fp32 accumulate)",
                  "mxfp4": "e2m1 weights with UE8M0 block scales x fp8_e4m3 activations (fp32 accumulate)"}[
                      spec["dtype"]],
        "config": {"workload": workload_desc(spec, name), "T": T, "d_model": H, "d_ff": F, "experts": E, "top_k": k,
                   "weights": spec["dtype"], "parallelism": f"weak-scaling replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2 (expert weights %.2f GB per step)" % (
                       alg["active"] * weight_bytes(spec["dtype"], 3 * H, F) / 1e9),
                   "expert_counts": counts},
        "roofline": roof,
        "layer": {"tflops": alg["layer_flops"] / (ms_step / 1e3) / 1e12,
                  "gbs": alg["layer_bytes"] / (ms_step / 1e3) / 1e9,
                  "hbm_frac": alg["layer_bytes"] / (ms_step / 1e3) / 1e9 / float(peaks.get("hbm_gbs", 6650.0))},
        "kernels_ms_per_step": {n: kern[n][0] / args.steps for n in names},
        "kernel_timing": "separate pass of the same K steps with an event pair around each kernel",
        "cpu_baseline": cb,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    del ws, out, x, logits
    return rec


def train_cpu_baseline(case, dy, spec, name, seconds):
    """Time the oracle's backward (as it stands) on sampled tokens of the
    training workload: per token the forward of its k assignments, dh, the
    SwiGLU derivative, dx and the router gradient (the sampled form leaves out
    the weight-gradient outer products)."""
    import numpy as np

    import moe_inputs
    import oracle
    nc = moe_inputs.to_numpy(case)
    f = oracle.bf16_bits_to_f64
    args64 = (f(nc["x"]), nc["logits"].astype(np.float64), f(nc["w1"]), f(nc["w3"]), f(nc["w2"]),
              f(moe_inputs.to_numpy({"dy": dy})["dy"]))
    T = spec["T"]
    cores = host_cores()
    batch = max(1, min(T, cores))
    done = 0
    feats = np.zeros((0, 2), dtype=np.int32)
    t0 = time.perf_counter()
    i = 0
    while True:
        tok = ((np.arange(batch) + i * batch) % T).astype(np.int32)
        oracle.ffn_bwd64_sampled(*args64, spec["k"], tok, feats, round_h=True, nthreads=cores)
        done += batch
        i += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} tokens of the {name} workload ({batch}-token batches): the oracle's sampled backward "
                      f"(forward of the token's experts, dh, SwiGLU derivative, dx, router gradient; no weight "
                      f"gradients), {dt:.1f} s"}


def run_gpu_train(args, moe, name, spec, case, dev, world, rank, cpu_seconds):
    """Time one BF16 training step of the layer: the training forward (from
    the row-major weights, which change every step, keeping routing, x, g, u
    and h) and the backward from what it kept (custom VJP: dx, dw1, dw3, dw2,
    dlogits).  Same structure of record as run_gpu_config."""
    import torch
    import torch.distributed as dist

    import moe_inputs
    T, H, F, E, k = spec["T"], spec["H"], spec["F"], spec["E"], spec["k"]
    seed = rank_batch(spec, rank)
    dy_cpu = moe_inputs.make_dy(T, H, seed)
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and cpu_seconds > 0:
        cb = train_cpu_baseline(case, dy_cpu, spec, name, cpu_seconds)
    if rank > 0:
        x_cpu, lg_cpu = moe_inputs.make_x(T, H, seed), moe_inputs.make_logits(T, E, seed, spec["skew"])
    else:
        x_cpu, lg_cpu = case["x"], case["logits"]
    x, logits, dy = x_cpu.to(dev), lg_cpu.to(dev), dy_cpu.to(dev)
    w1, w3, w2 = case["w1"].to(dev), case["w3"].to(dev), case["w2"].to(dev)
    ws = moe.backward_workspace(T, H, F, E, k, dev)
    y, _ = moe.ffn_forward_train(x, logits, w1, w3, w2, k, ws=ws)
    grads = moe.ffn_backward_saved(w1, w3, w2, dy, k, ws)
    stream = torch.cuda.current_stream(dev)

    def step(xx=x, lgg=logits, dyy=dy, g=grads):
        moe.ffn_forward_train(xx, lgg, w1, w3, w2, k, ws=ws, out=y, stream=stream)
        moe.ffn_backward_saved(w1, w3, w2, dyy, k, ws, out=g, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = moe.moe_get_status(None)
    if st != 0:
        raise RuntimeError(f"{name}: device status {moe.STATUS_NAMES.get(st, st)} after warm-up")
    counts = moe.ws_view(ws, T, H, F, E, k, "bf16", "counts", torch.int32).cpu().tolist()

    clocks = ClockSampler(torch.cuda.current_device())
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, dev)

    moe.moe_profile_read(reset=True)
    moe.moe_profile_enable(1)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    moe.moe_profile_enable(0)
    kern = moe.moe_profile_read(reset=True)
    st = moe.moe_get_status(None)
    if st != 0:
        raise RuntimeError(f"{name}: device status {moe.STATUS_NAMES.get(st, st)} in the timed region")
    ms_step = ms_total / args.steps
    value = T * world * args.steps / (ms_total / 1e3)

    # end to end: x, logits and dy up from pinned host memory, dx and dlogits back, every step
    e2e = None
    if not args.no_e2e:
        x_h, lg_h, dy_h = (t.cpu().pin_memory() for t in (x_cpu, lg_cpu, dy_cpu))
        dx_h = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
        dl_h = torch.empty(T, E, dtype=torch.float32).pin_memory()
        xd, lgd, dyd = torch.empty_like(x), torch.empty_like(logits), torch.empty_like(dy)

        def e2e_step():
            xd.copy_(x_h, non_blocking=True)
            lgd.copy_(lg_h, non_blocking=True)
            dyd.copy_(dy_h, non_blocking=True)
            step(xd, lgd, dyd, grads)
            dx_h.copy_(grads["dx"], non_blocking=True)
            dl_h.copy_(grads["dlogits"], non_blocking=True)

        for _ in range(max(3, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        ev1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
        if not torch.equal(dx_h, grads["dx"].cpu()):
            raise RuntimeError(f"{name}: the dx read back to the host is not the last step's")
        e2e = {"value": T * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": T * H * 2 * 2 + T * E * 4, "d2h_bytes_per_step": T * H * 2 + T * E * 4,
               "ms_per_step": e2e_ms / args.steps}
    clk = clocks.stop()

    # roofline of the dominant kernel (tensor-bound at this size): algorithmic
    # FLOPs per launch from the routed assignments A = T k (padding rows excluded)
    A = T * k
    kflops = {"stage1_w13_swiglu": 4.0 * A * F * H, "stage2_w2_scatter": 2.0 * A * F * H,  # the training forward
              "bwd_gu_recompute": 4.0 * A * F * H, "bwd_dh_swiglu": 2.0 * A * F * H,
              "bwd_dx_scatter": 4.0 * A * F * H, "bwd_dw2": 2.0 * A * F * H, "bwd_dw13": 4.0 * A * F * H}
    dom = max(kflops, key=lambda n: kern[n][0])
    dom_ms = kern[dom][0] / max(1, kern[dom][1])
    peaks, peak_kind = load_peaks()
    long_run = power_capped(ms_total, clk)
    key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
    peak = float(peaks.get(key, FALLBACK_PEAKS[key]))
    ach = kflops[dom] / (dom_ms / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "traffic": recorded_traffic(dom, name),
            "peak_source": f"{peak_kind} {'sustained' if long_run else 'burst'} bf16 cuBLAS",
            "algorithmic_per_launch": kflops[dom], "kernel": dom, "kernel_ms": dom_ms}
    step_flops = 18.0 * A * F * H  # forward 6 (g, u, h kept), dh 2, dx 4, dW2 2, dW1/dW3 4
    launches = sum(v[1] for v in kern.values())
    wbytes = 3 * E * F * H * 2
    return {
        "value": value, "unit": "tokens/s", "ms_per_step": ms_step, "steps": args.steps, "warmup": args.warmup,
        "dtype": "bf16 (fp32 accumulate)",
        "config": {"workload": workload_desc(spec, name) + "; training step: forward from the row-major weights "
                   "keeping g/u/h, backward from them (dx, dw1, dw3, dw2, dlogits)", "T": T, "d_model": H, "d_ff": F,
                   "experts": E, "top_k": k,
                   "weights": "bf16", "parallelism": f"weak-scaling replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2 (expert weights %.2f GB, read by several kernels per step)" % (
                       wbytes / 1e9),
                   "expert_counts": counts},
        "roofline": roof,
        "layer": {"tflops": step_flops / (ms_step / 1e3) / 1e12, "flops_per_step": step_flops},
        "kernels_ms_per_step": {n: kern[n][0] / args.steps for n in moe.KERNELS if kern[n][1]},
        "kernel_timing": "separate pass of the same K steps with an event pair around each kernel",
        "cpu_baseline": cb,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }


def main(argv=None):
    raw_argv = sys.argv[1:] if argv is None else list(argv)
    args = parse(raw_argv)
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        # no launcher: start one process per GPU ourselves
        return launch_ranks(raw_argv, args.gpus)
    world = int(env_world or "1")
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} does not match WORLD_SIZE={world}")
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)

    import moe_inputs
    import torch
    import torch.distributed as dist
    if args.fp8_peak_probe:
        torch.cuda.set_device(local_rank)
        if rank == 0:
            print(json.dumps(fp8_peak_probe()), flush=True)
        return 0
    names = config_names(args.config)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import mixture_experts_routed_02_b200 as moe
    weights = Weights()
    host_w = {}  # host weights of the last (shape, dtype, seed): the sweep points share them
    records = {}
    for i, name in enumerate(names):
        train = name in moe_inputs.BWD_CONFIGS
        spec = moe_inputs.BWD_CONFIGS[name] if train else moe_inputs.CONFIGS[name]
        t0 = time.perf_counter()
        wkey = (spec["H"], spec["F"], spec["E"], spec["dtype"], spec["seed"])
        if wkey not in host_w:
            host_w = {wkey: moe_inputs.make_weights(spec["H"], spec["F"], spec["E"], spec["dtype"], spec["seed"])}
        case = moe_inputs.make_case(spec["T"], spec["H"], spec["F"], spec["E"], spec["k"], spec["dtype"],
                                    spec["seed"], spec["skew"], weights=host_w[wkey])
        log(f"[rank {rank}] {name}: inputs generated in {time.perf_counter() - t0:.1f} s")
        cpu_s = args.cpu_sample_seconds if i == 0 else args.sub_cpu_sample_seconds
        if train:
            weights.w = weights.key = None  # the forward workloads' device weights are not needed here
            torch.cuda.empty_cache()
            records[name] = run_gpu_train(args, moe, name, spec, case, dev, world, rank, cpu_s)
        else:
            records[name] = run_gpu_config(args, moe, name, spec, case, weights, dev, world, rank, cpu_s)
        del case
        r = records[name]
        frac = r["roofline"]["frac"]
        log(f"[rank {rank}] {name}: {r['ms_per_step'] * 1e3:.1f} us/step, {r['value']:.0f} tokens/s, "
            f"{r['roofline']['kernel']} at " + (f"{frac:.3f}" if frac is not None else "n/a") +
            f" of {r['roofline']['unit']} peak")

    head = names[0]
    h = records[head]
    line = {
        "metric": METRIC, "value": h["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": h["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": h["dtype"],
        "data": "synthetic (seeded; random-init weights of the Mixtral-8x7B expert shape)",
        "config": h["config"], "roofline": h["roofline"], "layer": h["layer"],
        "kernels_ms_per_step": h["kernels_ms_per_step"], "kernel_timing": h["kernel_timing"],
        "cpu_baseline": h["cpu_baseline"], "e2e": h["e2e"], "gpu_launches": h["gpu_launches"], "clocks": h["clocks"],
    }
    if len(names) > 1:
        line["configs"] = {n: records[n] for n in names[1:]}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
