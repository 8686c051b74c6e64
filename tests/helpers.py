"""Shared helpers of the test-suite: device copies of seeded cases, the
tolerance of the layer's output, and oracle comparison utilities."""
import numpy as np
import torch

import moe_inputs
import oracle

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
    if case["dtype"] == "mxfp4":
        d["w13"], d["s13"], d["w2p"], d["s2p"] = moe.prepare_weights_mx(d["w1"], d["w3"], d["s1"], d["s3"], d["w2"],
                                                                         d["s2"])
    else:
        d["w13"], d["s13"], d["w2p"] = moe.prepare_weights(d["w1"], d["w3"], d["s1"], d["s3"], d["w2"])
        d["s2p"] = d["s2"]
    for key in ("T", "H", "F", "E", "k", "dtype"):
        d[key] = case[key]
    return d


def run_layer(dcase, ws=None):
    import mixture_experts_routed_02_b200 as moe
    if ws is None:
        ws = moe.workspace(dcase["T"], dcase["H"], dcase["F"], dcase["E"], dcase["k"], dcase["dtype"])
    out = moe.ffn_forward(dcase["x"], dcase["logits"], dcase["w13"], dcase["s13"], dcase["w2p"], dcase["s2p"],
                          dcase["k"], dcase["F"], dcase["dtype"], ws=ws)
    st = moe.moe_get_status(None)
    assert st == 0, f"device status {moe.STATUS_NAMES.get(st, st)}"
    return out, ws


def out_as_f64(out):
    return out.float().double().cpu().numpy()


def small_case(T, H=256, F=512, E=8, k=2, dtype="bf16", seed=0, skew=False):
    return moe_inputs.make_case(T, H, F, E, k, dtype, seed, skew)


# ---------------------------------------------------------------- flip-aware layer check
#
# The intermediate h is rounded (bf16, and in FP8 mode e4m3 with a per-32
# power-of-two scale) from a value the GPU forms with fp32 tensor-core
# accumulation and the oracle in fp64.  Where that value lies within rounding
# noise of a decision boundary both neighbouring codes are correct, and one
# flipped e4m3 code moves the outputs of its row by |w2| * (one e4m3 step).
# verify_layer therefore (1) compares the GPU's h with the oracle's h element
# by element and accepts a difference only when it is such a flip -- the
# oracle's exact value lies within RHO (relative) of the boundary between the
# two codes -- and only when flips are rare; (2) checks every output element
# against the stated tolerance plus the exact effect of the validated flips of
# its token, computed from the oracle's w2 and routing weights.

RHO = 2.0 ** -12          # admissible distance of a flipped decision from its boundary (relative) ...
ABS_FLOOR = 2.0 ** -14    # ... plus this fraction of the row's rms: g and u are sums of ~K terms, so
                          # fp32 accumulation leaves an absolute error that is large relative to h
                          # wherever g or u cancels to nearly zero
MAX_FLIP_FRACTION = 1e-2  # flips allowed per h row (a real defect changes most of a row)


def w2_columns(nc, dtype, e, cols):
    """Dequantised columns `cols` (d_ff indices) of expert e's w2 [H, len(cols)],
    from the oracle's number formats."""
    cols = np.asarray(cols)
    if dtype == "fp8":
        return _e4m3_values()[nc["w2"][e][:, cols]] * nc["s2"][e][:, None].astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(nc["w2"][e][:, cols])
    byte = nc["w2"][e][:, cols // 2]
    code = np.where(cols % 2 == 1, byte >> 4, byte & 15)
    vals = np.array([oracle.e2m1_to_double(c) for c in range(16)])[code]
    return vals * np.array([oracle.ue8m0_to_double(v) for v in range(256)])[nc["s2"][e][:, cols // 32]]


def _e4m3_values():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def gpu_h_rows(moe, ws, case, assignments):
    """Dequantised GPU intermediate (float64 [n, F]) and, in FP8 mode, the block
    exponents ([n, F/32]) of the given assignments."""
    T, H, F, E, k, dt = (case[x] for x in ("T", "H", "F", "E", "k", "dtype"))
    dc = moe.dtype_code(dt)
    A = T * k
    slot_of = moe.ws_view(ws, T, H, F, E, k, dc, "slot_of", torch.int32)[:A].cpu().numpy()
    slots = torch.from_numpy(slot_of[np.asarray(assignments)].astype(np.int64)).to(ws.device)
    hreg = moe.ws_view(ws, T, H, F, E, k, dc, "h")
    eb = 2 if dt == "bf16" else 1
    pitch = F * eb + 128  # rows of h are 128 bytes longer than their data
    hrows = hreg.view(-1, pitch)[slots][:, :F * eb].contiguous()
    if dt == "bf16":
        return hrows.view(torch.bfloat16).double().cpu().numpy(), None
    codes = hrows.cpu().numpy()
    sf = moe.ws_view(ws, T, H, F, E, k, dc, "h_sf").cpu().numpy()
    s = slots.cpu().numpy()
    m, row = s // 128, s % 128
    b = np.arange(F // 32)
    idx = ((m[:, None] * (F // 128) + b[None, :] // 4) * 512 + (row[:, None] % 32) * 16 + (row[:, None] // 32) * 4
           + b[None, :] % 4)
    exps = sf[idx].astype(np.int64) - 127
    vals = _e4m3_values()[codes] * np.repeat(2.0 ** exps, 32, axis=1)
    return vals, exps


def _quant_h(v, e, fp8):
    """The oracle's rounding of one exact value: bf16, then (FP8) e4m3 at block exponent e."""
    b = oracle.bf16_to_double(oracle.bf16_from_double(v))
    if not fp8:
        return b
    return oracle.e4m3_to_double(oracle.e4m3_from_float(np.float32(b / 2.0 ** e))) * 2.0 ** e


def _admissible(v, gpu_val, e_gpu, fp8, floor):
    """Is gpu_val the rounding of some value within RHO of v?  (Rounding is
    monotone, so it suffices to bracket gpu_val between the roundings of the
    window's ends.)"""
    w = RHO * abs(v) + RHO * floor
    lo, hi = _quant_h(v - w, e_gpu, fp8), _quant_h(v + w, e_gpu, fp8)
    return min(lo, hi) <= gpu_val <= max(lo, hi)


def verify_layer(moe, ws, out, case, tokens=None, what=""):
    """Check the GPU layer output (and its intermediate h) for the given tokens
    against the oracle.  Returns a dict of statistics."""
    nc = moe_inputs.to_numpy(case)
    T, F, k = case["T"], case["F"], case["k"]
    fp8 = case["dtype"] in ("fp8", "mxfp4")  # h is e4m3 with block scales
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ref = oracle.moe_ffn_tokens(nc, tokens.astype(np.int32), want_h=True)
    r = oracle.route(nc["logits"], k)
    assigns = (tokens[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    gh, gexp = gpu_h_rows(moe, ws, case, assigns)
    rh, rx = ref["h_deq"], ref["h_exact"]
    allow = np.zeros((len(tokens), case["H"]))
    flips = 0
    for q in range(len(assigns)):
        d = np.nonzero(gh[q] != rh[q])[0]
        if d.size == 0:
            continue
        assert d.size <= max(2, MAX_FLIP_FRACTION * F), f"{what}: {d.size} h elements differ in assignment {assigns[q]}"
        floor = (ABS_FLOOR / RHO) * float(np.sqrt(np.mean(rx[q] ** 2)))
        for n in d:
            e_gpu = int(gexp[q, n // 32]) if fp8 else 0
            if fp8:
                blk = slice(32 * (n // 32), 32 * (n // 32) + 32)
                amax_i = 32 * (n // 32) + int(np.argmax(np.abs(rx[q, blk])))
                e_ref = oracle.mx_exponent(max(abs(oracle.bf16_to_double(oracle.bf16_from_double(v)))
                                               for v in rx[q, blk]))
                if e_gpu != e_ref:
                    # a block-scale flip: the block's absmax must sit at the exponent boundary
                    va = rx[q, amax_i]
                    wa = RHO * abs(va)
                    cand = {oracle.mx_exponent(abs(oracle.bf16_to_double(oracle.bf16_from_double(va + s * wa))))
                            for s in (-1, 1)}
                    assert e_gpu in cand, f"{what}: block exponent {e_gpu} vs {e_ref} not at a boundary"
            assert _admissible(rx[q, n], gh[q, n], e_gpu, fp8, floor), (
                f"{what}: h[{assigns[q]}, {n}] gpu {gh[q, n]!r} oracle {rh[q, n]!r} exact {rx[q, n]!r}: not a "
                f"rounding flip")
        flips += d.size
        # exact effect of the flips of this assignment on the token's outputs
        t_i, j = divmod(q, k)
        e = int(r["ids"][tokens[t_i], j])
        wgt = float(r["w"][tokens[t_i], j])
        col = w2_columns(nc, case["dtype"], e, d)
        allow[t_i] += wgt * (np.abs(col) @ np.abs(gh[q, d] - rh[q, d]))
    gpu = out.float().double().cpu().numpy()[tokens]
    refv = bf16_bits_to_f64(ref["out"])
    rms = float(np.sqrt(np.mean(refv ** 2)))
    allowed = REL * np.abs(refv) + ABS_RMS * rms + allow
    err = np.abs(gpu - refv)
    bad = err > allowed
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outputs out of tolerance; worst err "
                           f"{err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}, rms(ref) {rms:.3e}, "
                           f"h flips {flips}")
    strict = err <= REL * np.abs(refv) + ABS_RMS * rms
    return dict(flips=flips, h_elements=len(assigns) * F, outputs_needing_allowance=int((~strict).sum()),
                max_err_over_tol=float((err / (REL * np.abs(refv) + ABS_RMS * rms)).max()))
