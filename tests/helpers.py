"""Shared helpers of the test-suite: device copies of seeded cases, the
tolerance of the layer's output, and oracle comparison utilities."""
import numpy as np
import torch

import moe_inputs

# |gpu - ref| <= REL * |ref| + ABS_RMS * rms(ref), element by element: the
# tolerance stated for this layer (fp32 tensor-core accumulation and bf16/e4m3
# rounding of intermediates against an fp64 reference).
REL = 1e-2
ABS_RMS = 2e-3


def bf16_bits_to_f64(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_close(gpu, ref, what=""):
    """gpu, ref: float64 arrays of the same shape.  Returns (max_err/allowed, stats)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    allowed = REL * np.abs(ref) + ABS_RMS * rms
    err = np.abs(gpu - ref)
    bad = err > allowed
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; worst "
                           f"err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}, rms(ref) {rms:.3e}")
    return float((err / np.maximum(allowed, 1e-300)).max()) if err.size else 0.0


def to_device(case, device="cuda"):
    """Copy a moe_inputs case to the GPU and prepare the weights there."""
    import mixture_experts_routed_02_b200 as moe
    d = {}
    for key in ("x", "logits", "w1", "w3", "w2", "s1", "s3", "s2"):
        v = case.get(key)
        d[key] = None if v is None else v.to(device)
    d["w13"], d["s13"] = moe.prepare_weights(d["w1"], d["w3"], d["s1"], d["s3"])
    for key in ("T", "H", "F", "E", "k", "dtype"):
        d[key] = case[key]
    return d


def run_layer(dcase, ws=None):
    import mixture_experts_routed_02_b200 as moe
    if ws is None:
        ws = moe.workspace(dcase["T"], dcase["H"], dcase["F"], dcase["E"], dcase["k"], dcase["dtype"])
    out = moe.ffn_forward(dcase["x"], dcase["logits"], dcase["w13"], dcase["s13"], dcase["w2"], dcase["s2"],
                          dcase["k"], ws=ws)
    st = moe.moe_get_status(None)
    assert st == 0, f"device status {moe.STATUS_NAMES.get(st, st)}"
    return out, ws


def out_as_f64(out):
    return out.float().double().cpu().numpy()


def small_case(T, H=256, F=512, E=8, k=2, dtype="bf16", seed=0, skew=False):
    return moe_inputs.make_case(T, H, F, E, k, dtype, seed, skew)
