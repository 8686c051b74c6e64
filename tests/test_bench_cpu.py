"""Host-side measurement logic of bench.py (no GPU): the algorithmic work the
roofline divides by, the lookup of recorded ncu traffic, and the parsing of
the clock samples taken during the timed region."""
import os
import shutil

import pytest

import bench

DECODE = dict(T=16, H=4096, F=14336, E=8, k=2, dtype="fp8", skew=False)


def test_algorithmic_work_of_the_decode_layer():
    # all 8 experts active: per expert 3*H*F e4m3 weight bytes plus 4*(2F+H)
    # bytes of fp32 channel scales; bf16 tokens in and out; fp32 logits
    w = bench.algorithmic(DECODE, [4, 4, 4, 4, 4, 4, 4, 4])
    H, F, T, E = 4096, 14336, 16, 8
    assert w["layer_bytes"] == 8 * (3 * H * F + 4 * (2 * F + H)) + T * H * 4 + 4 * T * E
    assert abs(w["layer_bytes"] - 1.4106e9) < 1e6
    # 6*H*F FLOP per assignment (3.523e8), 32 assignments, plus the router's T*E
    assert w["layer_flops"] == 6.0 * H * F * 32 + 2.0 * T * E
    assert abs(6.0 * H * F - 3.523e8) < 1e5
    assert w["s1_flops"] == 2 * w["s2_flops"]
    # stage 1 streams w1 and w3, stage 2 streams w2: 2:1 in weight bytes
    assert abs(w["s1_bytes"] / w["s2_bytes"] - 2.0) < 0.01


def test_experts_without_tokens_read_no_weights():
    full = bench.algorithmic(DECODE, [4] * 8)
    two = bench.algorithmic(DECODE, [16, 16, 0, 0, 0, 0, 0, 0])
    assert two["active"] == 2
    per_expert = 3 * 4096 * 14336 + 4 * (2 * 14336 + 4096)
    assert full["layer_bytes"] - two["layer_bytes"] == 6 * per_expert
    assert full["layer_flops"] == two["layer_flops"]  # same assignments, same work


def test_bf16_weights_count_two_bytes_and_no_scales():
    spec = dict(DECODE, dtype="bf16")
    w = bench.algorithmic(spec, [4] * 8)
    assert w["layer_bytes"] == 8 * 3 * 4096 * 14336 * 2 + 16 * 4096 * 4 + 4 * 16 * 8


def test_recorded_traffic_needs_the_same_kernel_code(monkeypatch):
    assert bench.recorded_traffic("stage1_w13_swiglu", "no-such-workload") is None
    monkeypatch.setattr(bench, "source_sha", lambda kernel="", workload="": "0000000000000000")
    assert bench.recorded_traffic("stage1_w13_swiglu", "decode") is None


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    for d in ("mixture_experts_routed_02_b200/csrc", "include"):
        (root / d).mkdir(parents=True)
    for rel in ("mixture_experts_routed_02_b200/csrc/gemm.cu", "mixture_experts_routed_02_b200/csrc/kernels.cuh",
                "mixture_experts_routed_02_b200/csrc/ptx.cuh"):
        shutil.copy(os.path.join(bench.ROOT, rel), root / rel)
    monkeypatch.setattr(bench, "ROOT", str(root))
    base = bench.source_sha()
    gemm = root / "mixture_experts_routed_02_b200/csrc/gemm.cu"
    text = gemm.read_text()
    gemm.write_text("// a new comment line\n" + text.replace("\n", "\n\n", 3))
    assert bench.source_sha() == base
    gemm.write_text(text.replace("kBlockM", "kBlockM ", 1) + "\nstatic int extra_code = 1;\n")
    assert bench.source_sha() != base


class _FakeSmi:
    def __init__(self, lines):
        self.out = "\n".join(lines)

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


@pytest.mark.parametrize("lines,reasons,median", [
    (["0, 1965, 1965, 700, 0x0, Not Active, Not Active, Not Active, Not Active"] * 3, [], 1965.0),
    (["0, 1400, 1965, 1000, 0x4, Not Active, Not Active, Not Active, Active",
      "0, 1350, 1965, 1000, 0x4, Not Active, Not Active, Not Active, Active",
      "0, 1965, 1965, 900, 0x0, Not Active, Not Active, Not Active, Not Active"], ["sw_power_cap"], 1400.0),
    (["0, 1200, 1965, 600, 0x40, Not Active, Active, Not Active, Not Active", "garbage"],
     ["hw_thermal_slowdown"], 1200.0),
])
def test_clock_samples(lines, reasons, median):
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi(lines)
    clk = s.stop()
    assert clk["reasons"] == reasons
    assert clk["sm_mhz"] == median
    assert clk["sm_max_mhz"] == 1965.0


def test_default_run_times_every_mixtral_workload():
    """The default bench run (`--config all`) times the headline decode layer
    first and every other Mixtral-shaped workload after it, the training step
    (forward + backward) included."""
    import moe_inputs
    names = bench.config_names("all")
    assert names[0] == bench.HEADLINE == "decode"
    assert set(names) == (set(moe_inputs.CONFIGS) - {"tiny"}) | {"train_prefill"}
    assert bench.config_names("prefill,sweep_T1") == ["prefill", "sweep_T1"]
    assert bench.config_names("train_small") == ["train_small"]  # the profiler's small training case
    with pytest.raises(SystemExit):
        bench.config_names("no-such-workload")


def test_tensor_bound_roofline_uses_fp8_peak_from_bf16():
    spec = dict(T=4096, H=4096, F=14336, E=8, k=2, dtype="fp8", skew=False)
    alg = bench.algorithmic(spec, [1024] * 8)
    peaks = {"hbm_gbs": 6540.0, "bf16_tflops": 1633.0, "bf16_tflops_sustained": 1374.0}
    r = bench.roofline(spec, alg, "stage1_w13_swiglu", 1.0, 30.0, peaks, "measured", "prefill")
    assert r["bound"] == "tensor" and r["peak"] == 2 * 1633.0
    assert abs(r["achieved"] - alg["s1_flops"] / 1e-3 / 1e12) < 1e-6
    r = bench.roofline(spec, alg, "stage1_w13_swiglu", 1.0, 2000.0, peaks, "measured", "prefill")
    assert r["peak"] == 2 * 1374.0  # a long timed region runs under the power cap
    d = bench.roofline(dict(spec, T=16), bench.algorithmic(dict(spec, T=16), [4] * 8), "stage1_w13_swiglu", 0.15,
                       5.0, peaks, "measured", "decode")
    assert d["bound"] == "hbm" and d["unit"] == "GB/s"


def test_mxfp4_weight_bytes():
    """MX FP4 expert weights: half a byte per code plus one exponent byte per
    32 codes -- 0.53125 bytes per weight, against 1 (+ channel scales) for e4m3."""
    H, F = 4096, 14336
    assert bench.weight_bytes("mxfp4", 3 * H, F) == 3 * H * F * 17 // 32
    assert bench.weight_bytes("fp8", 3 * H, F) == 3 * H * F + 4 * 3 * H
    assert bench.weight_bytes("bf16", 3 * H, F) == 6 * H * F
    spec = dict(DECODE, dtype="mxfp4")
    w = bench.algorithmic(spec, [4] * 8)
    fp8 = bench.algorithmic(DECODE, [4] * 8)
    assert 0.5 < w["layer_bytes"] / fp8["layer_bytes"] < 0.55
    assert w["layer_flops"] == fp8["layer_flops"]


def test_training_kernels_hash_the_backward_sources():
    """Every GEMM of a training workload (the training forward's too) comes
    from the backward's translation unit: its recorded counters are keyed to
    that unit's hash, the forward layer's to the forward GEMM's."""
    fwd = bench.source_sha("stage1_w13_swiglu", "prefill")
    assert bench.source_sha("stage1_w13_swiglu", "train_prefill") == bench.source_sha("bwd_dw13", "train_prefill")
    assert bench.source_sha("stage1_w13_swiglu", "train_prefill") != fwd


def test_power_capped_clocks_select_the_sustained_peak():
    """A tensor-bound run whose sampled SM clock sat well below its maximum
    (the power cap) is measured against the sustained GEMM rate even when its
    timed region is short; at full clock against the burst rate."""
    spec = dict(T=4096, H=4096, F=14336, E=8, k=2, dtype="fp8", skew=False)
    alg = bench.algorithmic(spec, [1024] * 8)
    peaks = {"hbm_gbs": 6540.0, "bf16_tflops": 1633.0, "bf16_tflops_sustained": 1374.0}
    capped = {"sm_mhz": 1263.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    full = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.roofline(spec, alg, "stage1_w13_swiglu", 1.0, 300.0, peaks, "measured", "prefill",
                          capped)["peak"] == 2 * 1374.0
    assert bench.roofline(spec, alg, "stage1_w13_swiglu", 1.0, 300.0, peaks, "measured", "prefill",
                          full)["peak"] == 2 * 1633.0
    assert bench.power_capped(1500.0, None) and not bench.power_capped(10.0, None)
