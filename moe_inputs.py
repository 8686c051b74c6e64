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
=============  =====  =====  =====  ==  =  =====  ====  =================================

Distributions: x ~ N(0,1) rounded to bf16; router logits ~ N(0,1) fp32;
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

# stream ids of the generators
_S_X, _S_LOGITS, _S_W1, _S_W3, _S_W2 = range(5)


def _gen(seed, stream):
    return torch.Generator().manual_seed(int(seed) * 1000 + stream)


def skew_bias(E):
    """Per-expert logit bias of the skewed workload: b_e = 2*log(1/(e+1))."""
    return torch.tensor([2.0 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=torch.float32)


def make_x(T, H, seed):
    return torch.randn(T, H, generator=_gen(seed, _S_X)).to(torch.bfloat16)


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


def make_weights(H, F, E, dtype="bf16", seed=0):
    """The expert weights of a case alone: dict(w1, w3, s1, s3, w2, s2) as in
    ``make_case`` (the same draws for the same shape, dtype and seed)."""
    if dtype not in ("bf16", "fp8"):
        raise ValueError(dtype)
    w1, s1 = _weight(E, F, H, seed, _S_W1, dtype)
    w3, s3 = _weight(E, F, H, seed, _S_W3, dtype)
    w2, s2 = _weight(E, H, F, seed, _S_W2, dtype)
    return dict(w1=w1, w3=w3, w2=w2, s1=s1, s3=s3, s2=s2)


def make_case(T, H, F, E, k, dtype="bf16", seed=0, skew=False, weights=None):
    """All inputs of one layer call as torch CPU tensors.

    Returns dict(x bf16 [T,H], logits f32 [T,E], w1/w3 [E,F,H], w2 [E,H,F]
    (bf16 or float8_e4m3fn), s1/s3 f32 [E,F], s2 f32 [E,H] (fp8 only, else
    None), and the scalars T,H,F,E,k,dtype,seed).  ``weights``, if given, is
    the result of ``make_weights(H, F, E, dtype, seed)`` (reused, not redrawn)."""
    if dtype not in ("bf16", "fp8"):
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
