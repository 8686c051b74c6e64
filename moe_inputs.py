"""Seeded synthetic inputs for the routed MoE expert FFN.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests.  It holds none of the method's arithmetic: it only draws random numbers
and stores them in the input formats the layer consumes.  Expert weights in the
FP8 configurations are *given* to the layer as e4m3 codes with one fp32 scale
per output channel; producing those codes from N(0, 0.02^2) bf16 draws
(scale = row absmax / 448, code = e4m3(w / scale)) is input preparation and is
done here with torch's own float8 conversion.

Workloads (Mixtral-8x7B expert shapes, rocketrecap.com "FlyDSL kernels in
JAX", paragraph 2 and timestamp 8:14: Mixtral 8x7B, FP8, top-2 routing):

=============  =====  =====  =====  ==  =  =====  ====  =================================
name           T      H      F      E   k  dtype  seed  notes
=============  =====  =====  =====  ==  =  =====  ====  =================================
tiny           64     256    512    8   2  bf16   0
decode         16     4096   14336  8   2  fp8    1     weight-streaming shape
prefill        4096   4096   14336  8   2  fp8    2     tensor-core shape
skewed         8192   4096   14336  8   2  bf16   3     logits + 2*log(1/(e+1))
sweep_T<n>     n      4096   14336  8   2  fp8    4     n in {1, 128, 1024, 16384}
decode_mxfp4   16     4096   14336  8   2  mxfp4  5     MX FP4 expert weights
prefill_mxfp4  4096   4096   14336  8   2  mxfp4  6     MX FP4 expert weights
train_prefill  4096   4096   14336  8   2  bf16   7     backward pass (BWD_CONFIGS)
train_small    1024   1024   3584   8   2  bf16   8     backward, small case for profiler captures
=============  =====  =====  =====  ==  =  =====  ====  =================================

Distributions: x ~ N(0,1) rounded to bf16; router logits ~ N(0,1) fp32;
upstream gradient of the backward pass dy ~ N(0,1) rounded to bf16;
weights ~ N(0, 0.02^2) rounded to bf16 (and quantised per output channel for
fp8).  Every draw comes from its own torch CPU generator seeded with
``seed * 1000 + stream`` so that each tensor can be regenerated alone.
"""
import math

import numpy as np
import torch

H_MIXTRAL = 4096
F_MIXTRAL = 14336


def _spec(T, H, F, E, k, dtype, seed, skew=False):
    return dict(T=T, H=H, F=F, E=E, k=k, dtype=dtype, seed=seed, skew=skew)


CONFIGS = {
    "tiny": _spec(64, 256, 512, 8, 2, "bf16", 0),
    "decode": _spec(16, H_MIXTRAL, F_MIXTRAL, 8, 2, "fp8", 1),
    "prefill": _spec(4096, H_MIXTRAL, F_MIXTRAL, 8, 2, "fp8", 2),
    "skewed": _spec(8192, H_MIXTRAL, F_MIXTRAL, 8, 2, "bf16", 3, skew=True),
}
for _n in (1, 128, 1024, 16384):
    CONFIGS[f"sweep_T{_n}"] = _spec(_n, H_MIXTRAL, F_MIXTRAL, 8, 2, "fp8", 4)
# MX-scaled FP4 expert weights (e2m1 with a power-of-two scale per 32 values)
CONFIGS["decode_mxfp4"] = _spec(16, H_MIXTRAL, F_MIXTRAL, 8, 2, "mxfp4", 5)
CONFIGS["prefill_mxfp4"] = _spec(4096, H_MIXTRAL, F_MIXTRAL, 8, 2, "mxfp4", 6)

# backward pass (training) workloads: BF16 weights, an upstream gradient dy
BWD_CONFIGS = {
    "train_prefill": _spec(4096, H_MIXTRAL, F_MIXTRAL, 8, 2, "bf16", 7),
    # a quarter-width expert shape: the small case for detailed profiler captures
    "train_small": _spec(1024, 1024, 3584, 8, 2, "bf16", 8),
}

# stream ids of the generators
_S_X, _S_LOGITS, _S_W1, _S_W3, _S_W2, _S_DY = range(6)


def _gen(seed, stream):
    return torch.Generator().manual_seed(int(seed) * 1000 + stream)


def skew_bias(E):
    """Per-expert logit bias of the skewed workload: b_e = 2*log(1/(e+1))."""
    return torch.tensor([2.0 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=torch.float32)


def make_x(T, H, seed):
    return torch.randn(T, H, generator=_gen(seed, _S_X)).to(torch.bfloat16)


def make_dy(T, H, seed):
    """Upstream gradient of the layer output for the backward pass: N(0,1) -> bf16 [T,H]."""
    return torch.randn(T, H, generator=_gen(seed, _S_DY)).to(torch.bfloat16)


def make_logits(T, E, seed, skew=False):
    lg = torch.randn(T, E, generator=_gen(seed, _S_LOGITS))
    if skew:
        lg = lg + skew_bias(E)
    return lg.contiguous()


def _weight(E, rows, cols, seed, stream, dtype):
    """[E, rows, cols] weights ~ N(0, 0.02^2) -> bf16; fp8: per-row e4m3 + fp32 scale."""
    g = _gen(seed, stream)
    if dtype == "bf16":
        out = torch.empty(E, rows, cols, dtype=torch.bfloat16)
        for e in range(E):
            out[e] = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16)
        return out, None
    codes = torch.empty(E, rows, cols, dtype=torch.float8_e4m3fn)
    scales = torch.empty(E, rows, dtype=torch.float32)
    for e in range(E):
        wb = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16).float()
        amax = wb.abs().amax(dim=1)
        s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        codes[e] = (wb / s[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
        scales[e] = s
    return codes, scales


def _weight_mxfp4(E, rows, cols, seed, stream):
    """[E, rows, cols] weights ~ N(0, 0.02^2) -> bf16, then the MX FP4 format
    (OCP Microscaling): each block of 32 consecutive elements along `cols`
    (the contraction dimension) shares the power of two X = 2^(floor(log2
    amax) - 2) (2 = the exponent of e2m1's largest value, 6 = 1.5 * 2^2; X = 1
    for an all-zero block), and each element is the e2m1 code of w / X
    (round to nearest, ties to even, saturating at +-6; ml_dtypes' float4
    conversion).  Returns (codes uint8 [E, rows, cols/2], two per byte, the
    even column in the low 4 bits; exponents uint8 [E, rows, cols/32] biased
    by 127)."""
    import ml_dtypes
    g = _gen(seed, stream)
    codes = torch.empty(E, rows, cols // 2, dtype=torch.uint8)
    exps = torch.empty(E, rows, cols // 32, dtype=torch.uint8)
    for e in range(E):
        wb = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16).float().numpy()
        blk = wb.reshape(rows, cols // 32, 32)
        amax = np.abs(blk).max(axis=2)
        with np.errstate(divide="ignore"):
            ex = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, 0).astype(np.int32)
        ex = np.clip(ex, -127, 127)
        q = (blk / np.ldexp(np.float32(1.0), ex)[:, :, None]).astype(np.float32)  # exact: a power of two
        c4 = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8).reshape(rows, cols) & 0xF
        codes[e] = torch.from_numpy((c4[:, 0::2] | (c4[:, 1::2] << 4)).astype(np.uint8))
        exps[e] = torch.from_numpy((ex + 127).astype(np.uint8))
    return codes, exps


def make_weights(H, F, E, dtype="bf16", seed=0):
    """The expert weights of a case alone: dict(w1, w3, s1, s3, w2, s2) as in
    ``make_case`` (the same draws for the same shape, dtype and seed)."""
    if dtype not in ("bf16", "fp8", "mxfp4"):
        raise ValueError(dtype)
    if dtype == "mxfp4":
        w1, s1 = _weight_mxfp4(E, F, H, seed, _S_W1)
        w3, s3 = _weight_mxfp4(E, F, H, seed, _S_W3)
        w2, s2 = _weight_mxfp4(E, H, F, seed, _S_W2)
        return dict(w1=w1, w3=w3, w2=w2, s1=s1, s3=s3, s2=s2)
    w1, s1 = _weight(E, F, H, seed, _S_W1, dtype)
    w3, s3 = _weight(E, F, H, seed, _S_W3, dtype)
    w2, s2 = _weight(E, H, F, seed, _S_W2, dtype)
    return dict(w1=w1, w3=w3, w2=w2, s1=s1, s3=s3, s2=s2)


def make_case(T, H, F, E, k, dtype="bf16", seed=0, skew=False, weights=None):
    """All inputs of one layer call as torch CPU tensors.

    Returns dict(x bf16 [T,H], logits f32 [T,E], w1/w3 [E,F,H], w2 [E,H,F]
    (bf16 or float8_e4m3fn), s1/s3 f32 [E,F], s2 f32 [E,H] (fp8 only, else
    None), and the scalars T,H,F,E,k,dtype,seed).  mxfp4: w1/w3 uint8
    [E,F,H/2], w2 uint8 [E,H,F/2] (packed e2m1), s1/s3 uint8 [E,F,H/32], s2
    uint8 [E,H,F/32] (block exponents, see ``_weight_mxfp4``).  ``weights``, if given, is
    the result of ``make_weights(H, F, E, dtype, seed)`` (reused, not redrawn)."""
    if dtype not in ("bf16", "fp8", "mxfp4"):
        raise ValueError(dtype)
    w = weights if weights is not None else make_weights(H, F, E, dtype, seed)
    return dict(x=make_x(T, H, seed), logits=make_logits(T, E, seed, skew), **w,
                T=T, H=H, F=F, E=E, k=k, dtype=dtype, seed=seed)


def make_config(name):
    s = CONFIGS[name]
    return make_case(s["T"], s["H"], s["F"], s["E"], s["k"], s["dtype"], s["seed"], s["skew"])


def to_numpy(case):
    """Bit-level numpy view for the oracle: bf16 -> uint16, e4m3 -> uint8."""
    def bits(t):
        if t is None:
            return None
        t = t.contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8).numpy()
        return t.numpy()
    out = {k: bits(v) if isinstance(v, torch.Tensor) else v for k, v in case.items()}
    return out
