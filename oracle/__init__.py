"""CPU oracle for the routed MoE expert FFN -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does, and this
package never imports the CUDA library: the two share nothing but the seeded
input bytes produced by ``moe_inputs``.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64); this module builds it
with gcc and marshals numpy arrays through ctypes.  Each wrapper names the
step it follows:

* ``quant_x``      -- per-token FP8 activation quantisation (R0);
* ``e2m1_to_double``, ``ue8m0_to_double`` -- the MX FP4 element and block
                      scale formats (MX-scaled FP4 expert weights);
* ``route``        -- top-k, renormalised softmax, histogram, scan and stable
                      permutation (R1/R2; rocketrecap.com "FlyDSL kernels in
                      JAX", timestamps 5:56 "dynamic expert sizes" and 8:14
                      "top-2 routing");
* ``moe_ffn``      -- the whole layer, routed or masked-dense form (paragraph 2
                      and timestamp 5:56: gather, group GEMM, SwiGLU, scatter
                      versus the masked dense GEMM path);
* ``moe_ffn_tokens`` -- the same layer evaluated on a subset of tokens;
* ``ffn64``, ``ffn_bwd64``, ``ffn_bwd64_sampled`` -- the BF16 layer on fp64
                      inputs and its gradients (the custom VJP for training
                      that timestamp 10:07 names as the next step): dx, dw1,
                      dw3, dw2 and the router logits' gradient, in full or
                      sampled at full size.

Parity of these functions with the pages is pinned by ``tests/test_oracle.py``.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

BF16 = 0
FP8 = 1
MXFP4 = 2


def build(force=False):
    """Compile liboracle.so next to its source (gcc, OpenMP, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-fno-fast-math", "-ffp-contract=off",
           _SRC, "-o", _LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.oracle_bf16_from_double.restype = ctypes.c_uint16
        lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        lib.oracle_e2m1_to_double.restype = ctypes.c_double
        lib.oracle_e2m1_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_ue8m0_to_double.restype = ctypes.c_double
        lib.oracle_ue8m0_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_mx_exponent.restype = I
        lib.oracle_mx_exponent.argtypes = [ctypes.c_double]
        lib.oracle_mx_quant_block.restype = I
        lib.oracle_mx_quant_block.argtypes = [P, I, P]
        lib.oracle_quant_x.restype = None
        lib.oracle_quant_x.argtypes = [P, I, I, P, P]
        lib.oracle_route.restype = I
        lib.oracle_route.argtypes = [P, I, I, I, P, P, P, P, P, P]
        lib.oracle_moe_ffn.restype = I
        lib.oracle_moe_ffn.argtypes = [I, P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, I]
        lib.oracle_moe_ffn_tokens.restype = I
        lib.oracle_moe_ffn_tokens.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, P, P, P, I]
        lib.oracle_max_threads.restype = I
        lib.oracle_max_threads.argtypes = []
        lib.oracle_moe_ffn64.restype = I
        lib.oracle_moe_ffn64.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, I]
        lib.oracle_moe_ffn_bwd64.restype = I
        lib.oracle_moe_ffn_bwd64.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P,
                                             I]
        lib.oracle_moe_ffn_bwd64_sampled.restype = I
        lib.oracle_moe_ffn_bwd64_sampled.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, P, P, I, P, P, P,
                                                     P, P, P, P, P, I]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def max_threads():
    return _load().oracle_max_threads()


# -- number formats ---------------------------------------------------------

def e4m3_to_double(code):
    return _load().oracle_e4m3_to_double(int(code) & 0xFF)


def e4m3_from_float(v):
    return _load().oracle_e4m3_from_float(float(v))


def e2m1_to_double(code):
    return _load().oracle_e2m1_to_double(int(code) & 0xF)


def ue8m0_to_double(e):
    return _load().oracle_ue8m0_to_double(int(e) & 0xFF)


def bf16_from_double(v):
    return _load().oracle_bf16_from_double(float(v))


def bf16_to_double(b):
    return _load().oracle_bf16_to_double(int(b) & 0xFFFF)


def mx_exponent(amax):
    return _load().oracle_mx_exponent(float(amax))


def mx_quant_block(hb):
    """Quantise one block of bf16 values (given as float64): (exponent, codes)."""
    hb = _c(hb, np.float64)
    codes = np.zeros(hb.shape[0], dtype=np.uint8)
    e = _load().oracle_mx_quant_block(_ptr(hb), hb.shape[0], _ptr(codes))
    return e, codes


# -- R0 --------------------------------------------------------------------

def quant_x(x_bf16_bits):
    """x: uint16 [T,H] bf16 bit patterns -> (xq uint8 [T,H], sx float32 [T])."""
    x = _c(x_bf16_bits, np.uint16)
    T, H = x.shape
    xq = np.zeros((T, H), dtype=np.uint8)
    sx = np.zeros(T, dtype=np.float32)
    _load().oracle_quant_x(_ptr(x), T, H, _ptr(xq), _ptr(sx))
    return xq, sx


# -- R1/R2 -----------------------------------------------------------------

def route(logits, k):
    """logits float32 [T,E] -> dict(ids, w, counts, offsets, perm, inv_perm)."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    A = T * k
    ids = np.zeros(max(A, 1), dtype=np.int32)
    w = np.zeros(max(A, 1), dtype=np.float64)
    counts = np.zeros(E, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    perm = np.zeros(max(A, 1), dtype=np.int32)
    inv = np.zeros(max(A, 1), dtype=np.int32)
    rc = _load().oracle_route(_ptr(lg), T, E, k, _ptr(ids), _ptr(w), _ptr(counts), _ptr(offsets),
                              _ptr(perm), _ptr(inv))
    if rc != 0:
        raise ValueError("oracle_route: bad arguments")
    return dict(ids=ids[:A].reshape(T, k), w=w[:A].reshape(T, k), counts=counts, offsets=offsets,
                perm=perm[:A], inv_perm=inv[:A])


# -- the layer --------------------------------------------------------------

def _weights(case):
    """Weights and scales of a case: bf16 bits; e4m3 codes + fp32 channel
    scales (fp8); packed e2m1 codes + uint8 block exponents (mxfp4)."""
    dt = case["dtype"]
    wt = np.uint16 if dt == "bf16" else np.uint8
    st = {"bf16": None, "fp8": np.float32, "mxfp4": np.uint8}[dt]
    w1 = _c(case["w1"], wt)
    w3 = _c(case["w3"], wt)
    w2 = _c(case["w2"], wt)
    s1, s3, s2 = ((_c(case.get(n), st) if st is not None else None) for n in ("s1", "s3", "s2"))
    return w1, w3, w2, s1, s3, s2, {"bf16": BF16, "fp8": FP8, "mxfp4": MXFP4}[dt]



def moe_ffn(case, mode="routed", nthreads=0, want_h=False):
    """Whole layer on a case dict of numpy arrays (see ``moe_inputs.to_numpy``).

    Returns dict(out=uint16 [T,H] bf16 bits, out64=float64 [T,H], h=optional
    float64 [T*k,F] dequantised intermediate in sorted order)."""
    x = _c(case["x"], np.uint16)
    lg = _c(case["logits"], np.float32)
    T, H = x.shape
    E = lg.shape[1]
    k = int(case["k"])
    w1, w3, w2, s1, s3, s2, dt = _weights(case)
    F = w1.shape[1]
    out = np.zeros((T, H), dtype=np.uint16)
    out64 = np.zeros((T, H), dtype=np.float64)
    h = np.zeros((T * k, F), dtype=np.float64) if want_h else None
    rc = _load().oracle_moe_ffn(0 if mode == "routed" else 1, _ptr(x), _ptr(lg), _ptr(w1), _ptr(w3),
                                _ptr(s1), _ptr(s3), _ptr(w2), _ptr(s2), T, H, F, E, k, dt, _ptr(out),
                                _ptr(out64), _ptr(h), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_moe_ffn: bad arguments")
    return dict(out=out, out64=out64, h=h)


def moe_ffn_tokens(case, tokens, nthreads=0, want_h=False):
    """Output rows for the given token ids only: dict(out [n,H] bf16 bits, out64),
    plus with want_h the per-assignment intermediates h_deq and h_exact
    [n*k, F] (row i*k + j = j-th expert of the i-th listed token)."""
    x = _c(case["x"], np.uint16)
    lg = _c(case["logits"], np.float32)
    T, H = x.shape
    E = lg.shape[1]
    k = int(case["k"])
    w1, w3, w2, s1, s3, s2, dt = _weights(case)
    F = w1.shape[1]
    tok = _c(tokens, np.int32)
    n = tok.shape[0]
    out = np.zeros((n, H), dtype=np.uint16)
    out64 = np.zeros((n, H), dtype=np.float64)
    h_deq = np.zeros((n * k, F), dtype=np.float64) if want_h else None
    h_exact = np.zeros((n * k, F), dtype=np.float64) if want_h else None
    rc = _load().oracle_moe_ffn_tokens(_ptr(x), _ptr(lg), _ptr(w1), _ptr(w3), _ptr(s1), _ptr(s3),
                                       _ptr(w2), _ptr(s2), T, H, F, E, k, dt, _ptr(tok), n, _ptr(out),
                                       _ptr(out64), _ptr(h_deq), _ptr(h_exact), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_moe_ffn_tokens: bad arguments")
    return dict(out=out, out64=out64, h_deq=h_deq, h_exact=h_exact)


def bf16_bits_to_float(b):
    """uint16 bf16 bit patterns -> float64 values (exact widening)."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# -- backward (custom VJP) of the BF16 layer -------------------------------

def bf16_bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _round(round_h, round_inter=False):
    return (1 if round_h else 0) | (2 if round_inter else 0)


def _dims64(x, w1, logits, k):
    T, H = x.shape
    E, F, H1 = w1.shape
    if H1 != H or logits.shape != (T, E) or not 1 <= k <= E:
        raise ValueError("inconsistent shapes")
    return T, H, F, E


def ffn64(x, logits, w1, w3, w2, k, round_h=False, nthreads=0):
    """The layer on fp64 inputs: y [T,H] fp64 (not rounded); h rounded to bf16
    when round_h, as the BF16 forward does."""
    x, lg, w1, w3, w2 = (_c(a, np.float64) for a in (x, logits, w1, w3, w2))
    T, H, F, E = _dims64(x, w1, lg, k)
    y = np.zeros((T, H))
    rc = _load().oracle_moe_ffn64(_ptr(x), _ptr(lg), _ptr(w1), _ptr(w3), _ptr(w2), T, H, F, E, k, _round(round_h),
                                  _ptr(y), nthreads)
    if rc != 0:
        raise ValueError("oracle_moe_ffn64: bad arguments")
    return y


def ffn_bwd64(x, logits, w1, w3, w2, dy, k, round_h=True, round_inter=False, want_abs=False, nthreads=0):
    """Gradients of <dy, layer(x)>: dict(dx [T,H], dw1 [E,F,H], dw3 [E,F,H],
    dw2 [E,H,F], dlogits [T,E], dwa [T,k] routing-weight gradients), fp64.
    round_h: h rounded to bf16 as the forward does; round_inter: also dg, du
    and the w_a dy_t entering dW2 (a bf16 implementation's storage points).
    want_abs: also each entry's sum of absolute terms ("<name>_abs")."""
    x, lg, w1, w3, w2, dy = (_c(a, np.float64) for a in (x, logits, w1, w3, w2, dy))
    T, H, F, E = _dims64(x, w1, lg, k)
    out = dict(dx=np.zeros((T, H)), dw1=np.zeros((E, F, H)), dw3=np.zeros((E, F, H)), dw2=np.zeros((E, H, F)),
               dlogits=np.zeros((T, E)), dwa=np.zeros(max(T * k, 1)))
    names = ("dx", "dw1", "dw3", "dw2", "dlogits")
    if want_abs:
        for n in names:
            out[n + "_abs"] = np.zeros_like(out[n])
    ab = [_ptr(out[n + "_abs"]) if want_abs else None for n in names]
    rc = _load().oracle_moe_ffn_bwd64(_ptr(x), _ptr(lg), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(dy), T, H, F, E, k,
                                      _round(round_h, round_inter), _ptr(out["dx"]), _ptr(out["dw1"]), _ptr(out["dw3"]),
                                      _ptr(out["dw2"]), _ptr(out["dlogits"]), _ptr(out["dwa"]), *ab, nthreads)
    if rc != 0:
        raise ValueError("oracle_moe_ffn_bwd64: bad arguments")
    out["dwa"] = out["dwa"][:T * k].reshape(T, k)
    return out


def ffn_bwd64_sampled(x, logits, w1, w3, w2, dy, k, tokens, feats, round_h=True, round_inter=False, want_abs=False,
                      nthreads=0):
    """Sampled gradients: dx [ntok,H] and dlogits [ntok,E] of the listed
    tokens; for each (e, n) in feats, dw1[e, n, :], dw3[e, n, :] and
    dw2[e, :, n] ([nfeat,H] each); with want_abs their error scales too."""
    x, lg, w1, w3, w2, dy = (_c(a, np.float64) for a in (x, logits, w1, w3, w2, dy))
    T, H, F, E = _dims64(x, w1, lg, k)
    tok = _c(tokens, np.int32).reshape(-1)
    ft = _c(feats, np.int32).reshape(-1, 2)
    out = dict(dx=np.zeros((len(tok), H)), dlogits=np.zeros((len(tok), E)), dw1=np.zeros((len(ft), H)),
               dw3=np.zeros((len(ft), H)), dw2=np.zeros((len(ft), H)))
    names = ("dx", "dlogits", "dw1", "dw3", "dw2")
    if want_abs:
        for n in names:
            out[n + "_abs"] = np.zeros_like(out[n])
    ab = [_ptr(out[n + "_abs"]) if want_abs else None for n in names]
    rc = _load().oracle_moe_ffn_bwd64_sampled(_ptr(x), _ptr(lg), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(dy), T, H, F, E,
                                              k, _round(round_h, round_inter), _ptr(tok), len(tok), _ptr(out["dx"]),
                                              _ptr(out["dlogits"]), _ptr(ft), len(ft), _ptr(out["dw1"]),
                                              _ptr(out["dw3"]), _ptr(out["dw2"]), *ab, nthreads)
    if rc != 0:
        raise ValueError("oracle_moe_ffn_bwd64_sampled: bad arguments")
    return out
