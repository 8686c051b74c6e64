"""Benchmark of the routed MoE expert FFN layer (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

A step is one pass of the whole layer -- routing, gather (+ FP8 quantisation),
the w1/w3 + SwiGLU group GEMM, the w2 + scatter group GEMM and the bf16
finalize -- over one batch of T tokens whose inputs are already resident in
HBM.  The default workload is the Mixtral-8x7B-shaped FP8 decode layer
(T=16, d_model=4096, d_ff=14336, E=8, top-2).  With N > 1 (one process per GPU
under torch.distributed.run) every rank runs its own batch against its own copy
of the weights (weak scaling); the only collectives are the timing barrier and
the max over ranks.

``--impl reference`` times the CPU oracle (fp64, the host's CPU cores) on a
bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (Mixtral-8x7B shape FP8, T=16 and T=4096); % of roofline"

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", default="decode")
    p.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


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


def algorithmic(spec, counts):
    """Algorithmic FLOPs and bytes of the layer and of each GEMM kernel, from
    the routed expert counts (experts with no tokens read no weights)."""
    T, H, F, E, k = spec["T"], spec["H"], spec["F"], spec["E"], spec["k"]
    bw = 1 if spec["dtype"] == "fp8" else 2
    A = T * k
    active = sum(1 for c in counts if c > 0)
    s1_bytes = active * (2 * F * H * bw + (8 * F if bw == 1 else 0)) + A * H * bw + A * F * bw + (A * F // 32 if bw == 1 else 0)
    s2_bytes = active * (H * F * bw + (4 * H if bw == 1 else 0)) + A * F * bw + (A * F // 32 if bw == 1 else 0) + T * H * 4
    layer_bytes = active * (3 * H * F * bw + (4 * (2 * F + H) if bw == 1 else 0)) + T * H * 2 * 2 + 4 * T * E
    return dict(s1_flops=4.0 * H * F * A, s2_flops=2.0 * H * F * A, layer_flops=6.0 * H * F * A + 2.0 * T * E,
                s1_bytes=float(s1_bytes), s2_bytes=float(s2_bytes), layer_bytes=float(layer_bytes), active=active)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
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
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "samples": len(sms)}


def source_sha():
    """Hash of the code the grouped-GEMM kernels are compiled from (their
    translation unit and the headers it includes), comments and blank space
    removed, so that an edit to a comment keeps the recorded counters."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_routed_02_b200", "csrc")
    for path in [os.path.join(csrc, n) for n in ("gemm.cu", "kernels.cuh", "ptx.cuh")] + \
            [os.path.join(ROOT, "include", "moe.h")]:
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
    sha = source_sha()
    for r in recs:
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_sha") == sha:
            return r.get("dram_bytes_per_launch")
    return None


def cpu_baseline(spec, name, seconds):
    """Time the oracle (as it stands) on whole-token samples of the workload."""
    import numpy as np

    import moe_inputs
    import oracle
    case = moe_inputs.make_case(spec["T"], spec["H"], spec["F"], spec["E"], spec["k"], spec["dtype"], spec["seed"],
                                spec["skew"])
    nc = moe_inputs.to_numpy(case)
    T = spec["T"]
    batch = max(1, min(T, 8))
    tokens_done = 0
    t0 = time.perf_counter()
    i = 0
    while True:
        tok = (np.arange(batch) + i * batch) % T
        oracle.moe_ffn_tokens(nc, tok.astype(np.int32))
        tokens_done += batch
        i += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens_done / dt, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
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


def run_reference(args, spec, name, rank):
    """The oracle as it stands, on the host cores: each step is one oracle call on
    a small batch of the workload's tokens (sized so the run stays within a
    couple of minutes)."""
    if rank != 0:
        return 0
    import numpy as np

    import moe_inputs
    import oracle
    case = moe_inputs.make_case(spec["T"], spec["H"], spec["F"], spec["E"], spec["k"], spec["dtype"], spec["seed"],
                                spec["skew"])
    nc = moe_inputs.to_numpy(case)
    T = spec["T"]
    batch = max(1, min(T, 8))
    t0 = time.perf_counter()
    oracle.moe_ffn_tokens(nc, np.arange(batch, dtype=np.int32))
    per_call = time.perf_counter() - t0
    budget = 120.0
    while batch > 1 and per_call * (args.steps + args.warmup) > budget:
        batch //= 2
        per_call /= 2
    calls = [((np.arange(batch) + i * batch) % T).astype(np.int32) for i in range(args.warmup + args.steps)]
    for tok in calls[:args.warmup]:
        oracle.moe_ffn_tokens(nc, tok)
    t0 = time.perf_counter()
    for tok in calls[args.warmup:]:
        oracle.moe_ffn_tokens(nc, tok)
    dt = time.perf_counter() - t0
    value = batch * args.steps / dt
    cb = {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
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


def main():
    args = parse()
    import moe_inputs
    name = args.config
    spec = moe_inputs.CONFIGS[name]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, spec, name, rank)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # the CPU baseline runs first, before the GPU is busy (rank 0, one GPU only)
    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(spec, name, args.cpu_sample_seconds)

    import mixture_experts_routed_02_b200 as moe
    t0 = time.perf_counter()
    # weak scaling: each rank its own batch (seed offset by rank), the same weights
    case = moe_inputs.make_case(spec["T"], spec["H"], spec["F"], spec["E"], spec["k"], spec["dtype"], spec["seed"],
                                spec["skew"])
    if rank > 0:
        case["x"] = moe_inputs.make_x(spec["T"], spec["H"], rank_batch(spec, rank))
        case["logits"] = moe_inputs.make_logits(spec["T"], spec["E"], rank_batch(spec, rank), spec["skew"])
    log(f"[rank {rank}] inputs generated in {time.perf_counter() - t0:.1f} s")
    T, H, F, E, k = spec["T"], spec["H"], spec["F"], spec["E"], spec["k"]
    fp8 = spec["dtype"] == "fp8"
    x = case["x"].to(dev)
    logits = case["logits"].to(dev)
    s2 = case["s2"].to(dev) if fp8 else None
    w13, s13, w2 = moe.prepare_weights(case["w1"].to(dev), case["w3"].to(dev),
                                       case["s1"].to(dev) if fp8 else None, case["s3"].to(dev) if fp8 else None,
                                       case["w2"].to(dev))
    del case
    torch.cuda.empty_cache()
    dt_code = moe.MOE_FP8_E4M3 if fp8 else moe.MOE_BF16
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
        raise RuntimeError(f"device status {moe.STATUS_NAMES.get(st, st)} after warm-up")
    counts = moe.ws_view(ws, T, H, F, E, k, dt_code, "counts", torch.int32).cpu().tolist()

    # ---------------- device-timed region (inputs resident in HBM).  No events
    # between the kernels here: an event recorded between two kernels would
    # stop the next one from starting while the previous one drains.
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
    clk = clocks.stop()
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
        raise RuntimeError(f"device status {moe.STATUS_NAMES.get(st, st)} in the timed region")
    ms_step = ms_total / args.steps
    value = T * world * args.steps / (ms_total / 1e3)

    # ---------------- end to end through the public API: pinned host in, result back to host.
    # A serving loop's pipeline: two sets of device buffers; step i's inputs go
    # up on one copy stream and step i-1's result comes down on another while
    # the layer runs, each step waiting only for the copies it needs.
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
    e2e_value = T * world * args.steps / (e2e_ms / 1e3)
    last = (args.steps - 1) % 2
    if not torch.equal(outs_h[last], outs_d[last].cpu()):
        raise RuntimeError("the result read back to the host is not the last step's output")

    # ---------------- roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    alg = algorithmic(spec, counts)
    names = moe.KERNELS
    dom = max(names, key=lambda n: kern[n][0])
    dom_ms = kern[dom][0] / max(1, kern[dom][1])
    decode_like = alg["active"] * 3 * H * F * (1 if fp8 else 2) / 6.5e12 > alg["layer_flops"] / (
        (2 * 2.25e15) if fp8 else 2.25e15)
    if dom.startswith("stage"):
        per = "s1" if dom.startswith("stage1") else "s2"
        if decode_like:
            ach = alg[per + "_bytes"] / (dom_ms / 1e3) / 1e9
            peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
            roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                    "traffic": recorded_traffic(dom, name),
                    "peak_source": f"{peak_kind} HBM copy bandwidth"}
        else:
            ach = alg[per + "_flops"] / (dom_ms / 1e3) / 1e12
            # a timed region of a second or more runs under the power cap: sustained peak; else burst
            long_run = ms_total >= 1000.0
            key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
            base = float(peaks.get(key, FALLBACK_PEAKS[key]))
            peak = base * (FP8_PER_BF16 if fp8 else 1.0)
            roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                    "traffic": recorded_traffic(dom, name),
                    "peak_source": f"{peak_kind} {'sustained' if long_run else 'burst'} bf16 cuBLAS"
                                   + (" x 2 (fp8/bf16 nominal ratio)" if fp8 else "")}
    else:
        roof = {"bound": "hbm", "achieved": None, "peak": float(peaks.get("hbm_gbs", 6650.0)), "unit": "GB/s",
                "frac": None, "traffic": None}
    roof["kernel"] = dom
    roof["kernel_ms"] = dom_ms

    launches = sum(v[1] for v in kern.values())  # K steps, the same count as the timed region
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3 (fp32 accumulate)" if fp8 else "bf16 (fp32 accumulate)",
        "data": "synthetic (seeded; random-init weights of the Mixtral-8x7B expert shape)",
        "config": {"workload": workload_desc(spec, name), "T": T, "d_model": H, "d_ff": F, "experts": E, "top_k": k,
                   "weights": spec["dtype"], "parallelism": f"weak-scaling replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2 (expert weights %.2f GB per step)" % (alg["active"] * 3 * H * F * (1 if fp8 else 2) / 1e9),
                   "expert_counts": counts},
        "roofline": roof,
        "layer": {"tflops": alg["layer_flops"] / (ms_step / 1e3) / 1e12,
                  "gbs": alg["layer_bytes"] / (ms_step / 1e3) / 1e9,
                  "hbm_frac": alg["layer_bytes"] / (ms_step / 1e3) / 1e9 / float(peaks.get("hbm_gbs", 6650.0))},
        "kernels_ms_per_step": {n: kern[n][0] / args.steps for n in names},
        "kernel_timing": "separate pass of the same K steps with an event pair around each kernel",
        "cpu_baseline": cb,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * H * 2 + T * E * 4,
                "d2h_bytes_per_step": T * H * 2},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
