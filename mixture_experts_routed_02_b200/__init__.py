"""Routed MoE expert FFN on one B200 (sm_100a): Python binding of libmoe.

The layer (rocketrecap.com "FlyDSL kernels in JAX", paragraph 2 and
timestamps 5:56 and 8:14): top-k routing, gather of each expert's tokens, group
GEMM with w1/w3 fused with SwiGLU, group GEMM with w2 fused with the
routing-weighted scatter back to token order; FP8 (e4m3 with fp32 scales) or
BF16.

This module only marshals arguments: every step of the layer runs in the CUDA
kernels of ``libmoe.so`` (built in tree by ``build.py``).  The C entry points
keep their names (``moe_route``, ``moe_ffn_forward``, ...) and take raw device
pointers; the ``route``/``ffn_forward``/``prepare_weights`` helpers accept
torch tensors and pass their pointers and the current CUDA stream.  There is no
fallback: if the library cannot be loaded, importing this package fails.

Use (FP8: e4m3 weights with fp32 per-output-channel scales)::

    import mixture_experts_routed_02_b200 as moe
    w13, s13, w2p = moe.prepare_weights(w1, w3, s1, s3, w2)   # once, at load time
    ws = moe.workspace(T, H, F, E, k, "fp8")                    # reusable scratch
    out = moe.ffn_forward(x, logits, w13, s13, w2p, s2, k, F, True, ws=ws)
    assert moe.moe_get_status(None) == moe.MOE_OK             # device-side checks

``moe_set_option(OPT_PATH, n)`` forces the tile configuration (0 = by size,
1 = CTA pairs, 2 = weight streaming, 3 = 128 x 256 tiles, 4 = tiny batches);
``moe_profile_enable``/``moe_profile_read`` time each kernel of the layer.

Training (BF16, the row-major weights as they are)::

    out, ws = moe.ffn_forward_train(x, logits, w1, w3, w2, k)   # keeps g, u, h in ws
    grads = moe.ffn_backward_saved(w1, w3, w2, dy, k, ws)         # dx, dw1, dw3, dw2, dlogits
    grads = moe.ffn_backward(x, logits, w1, w3, w2, dy, k)        # the same, recomputing g and u
"""
import ctypes
import os

__all__ = [
    "lib", "MOE_OK", "MOE_BF16", "MOE_FP8_E4M3", "WS", "MoeError", "moe_workspace_size", "moe_workspace_region",
    "moe_prepare_weights", "moe_route", "moe_ffn_forward", "moe_get_status", "moe_set_option", "prepare_weights",
    "route", "ffn_forward", "workspace", "ws_view", "EXPORTS", "KERNELS", "moe_profile_enable",
    "moe_profile_read", "backward_workspace", "ffn_backward", "ffn_forward_train", "ffn_backward_saved",
    "moe_backward_workspace_size", "moe_ffn_backward", "moe_ffn_forward_train", "moe_ffn_backward_saved",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_ALIGNMENT",
                -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA", -6: "MOE_ERR_DEVICE_TIMEOUT",
                -7: "MOE_ERR_DEVICE_BOUNDS"}
MOE_BF16 = 0
MOE_FP8_E4M3 = 1
MOE_MXFP4 = 2
OPT_PATH, OPT_SPLITK, OPT_TIMEOUT_MS, OPT_TEST_STALL, OPT_TEST_CORRUPT, OPT_GATHER = range(6)

# workspace regions (moe_ws_region)
WS = dict(topk_ids=0, topk_w=1, counts=2, offsets=3, perm=4, inv_perm=5, slot_of=6, xs=7, sx=8, h=9, h_sf=10,
          out32=11, num_mtiles=12, slot_assign=13, mtile_expert=14, route_blocks=15, xg=16, sx_slot=17)

# every symbol include/moe.h declares
EXPORTS = ["moe_workspace_size", "moe_prepare_weights", "moe_route", "moe_ffn_forward", "moe_get_status",
           "moe_workspace_region", "moe_set_option", "moe_profile_enable", "moe_profile_read",
           "moe_ffn_forward_static", "moe_static_workspace_bytes", "moe_ffn_forward_dff", "moe_dff_finalize",
           "moe_prepare_weights_mx", "moe_backward_workspace_size", "moe_ffn_backward", "moe_ffn_forward_train",
           "moe_ffn_backward_saved"]
# kernel ids of moe_profile_read: the forward's five, then the backward's
FWD_KERNELS = ["route", "quantize", "stage1_w13_swiglu", "stage2_w2_scatter", "finalize"]
BWD_KERNELS = ["bwd_gu_recompute", "bwd_dh_swiglu", "bwd_dx_scatter", "bwd_dw2", "bwd_dw13", "bwd_aux"]
KERNELS = FWD_KERNELS + BWD_KERNELS + ["prepare_weights"]


class MoeError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run `python mixture_experts_routed_02_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
lib.moe_workspace_size.restype = _Z
lib.moe_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I]
lib.moe_workspace_region.restype = ctypes.c_longlong
lib.moe_workspace_region.argtypes = [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_Z)]
lib.moe_prepare_weights.restype = _I
lib.moe_prepare_weights.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]
lib.moe_prepare_weights_mx.restype = _I
lib.moe_prepare_weights_mx.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P]
lib.moe_route.restype = _I
lib.moe_route.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _Z, _P]
lib.moe_ffn_forward.restype = _I
lib.moe_ffn_forward.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P]
lib.moe_get_status.restype = _I
lib.moe_get_status.argtypes = [_P]
lib.moe_set_option.restype = _I
lib.moe_set_option.argtypes = [_I, _I]
lib.moe_ffn_forward_static.restype = _I
lib.moe_ffn_forward_static.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]
lib.moe_static_workspace_bytes.restype = _Z
lib.moe_static_workspace_bytes.argtypes = []
lib.moe_ffn_forward_dff.restype = _I
lib.moe_ffn_forward_dff.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _Z, _P]
lib.moe_dff_finalize.restype = _I
lib.moe_dff_finalize.argtypes = [_P, _P, _I, _I, _P, ctypes.c_uint, _P]
lib.moe_profile_enable.restype = _I
lib.moe_profile_enable.argtypes = [_I]
lib.moe_profile_read.restype = _I
lib.moe_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I), _I]
lib.moe_backward_workspace_size.restype = _Z
lib.moe_backward_workspace_size.argtypes = [_I, _I, _I, _I, _I]
lib.moe_ffn_backward.restype = _I
lib.moe_ffn_backward.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P]
lib.moe_ffn_forward_train.restype = _I
lib.moe_ffn_forward_train.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _Z, _P]
lib.moe_ffn_backward_saved.restype = _I
lib.moe_ffn_backward_saved.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _P]

# raw entry points, same names as the C ABI
moe_workspace_size = lib.moe_workspace_size
moe_prepare_weights = lib.moe_prepare_weights
moe_prepare_weights_mx = lib.moe_prepare_weights_mx
moe_route = lib.moe_route
moe_ffn_forward = lib.moe_ffn_forward
moe_get_status = lib.moe_get_status
moe_set_option = lib.moe_set_option
moe_profile_enable = lib.moe_profile_enable
moe_ffn_forward_static = lib.moe_ffn_forward_static
moe_static_workspace_bytes = lib.moe_static_workspace_bytes
moe_ffn_forward_dff = lib.moe_ffn_forward_dff
moe_dff_finalize = lib.moe_dff_finalize
moe_backward_workspace_size = lib.moe_backward_workspace_size
moe_ffn_backward = lib.moe_ffn_backward
moe_ffn_forward_train = lib.moe_ffn_forward_train
moe_ffn_backward_saved = lib.moe_ffn_backward_saved


def moe_profile_read(reset=True):
    """{kernel name: (total ms, launches)} of the calls recorded while profiling was on."""
    ms = (ctypes.c_double * len(KERNELS))()
    n = (ctypes.c_int * len(KERNELS))()
    _check("moe_profile_read", lib.moe_profile_read(ms, n, 1 if reset else 0))
    return {name: (ms[i], n[i]) for i, name in enumerate(KERNELS)}


def moe_workspace_region(T, H, F, E, k, dtype, which):
    """(byte offset, byte size) of a workspace region (``WS`` names or ints)."""
    n = ctypes.c_size_t(0)
    w = WS[which] if isinstance(which, str) else int(which)
    off = lib.moe_workspace_region(T, H, F, E, k, dtype, w, ctypes.byref(n))
    if off < 0:
        raise MoeError("moe_workspace_region", -1)
    return int(off), int(n.value)


# ---------------------------------------------------------------- torch helpers

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, rc):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def dtype_code(dtype):
    """"bf16" / "fp8" / "mxfp4" (or True = fp8, False = bf16, or the codes) -> the moe_dtype code."""
    if dtype in ("mxfp4", MOE_MXFP4) and dtype is not True:
        return MOE_MXFP4
    if dtype is True or dtype in ("fp8", MOE_FP8_E4M3):
        return MOE_FP8_E4M3
    return MOE_BF16


def workspace(T, H, F, E, k, dtype, device="cuda"):
    """Allocate (with torch) a workspace large enough for one layer call."""
    import torch
    n = moe_workspace_size(T, H, F, E, k, dtype_code(dtype))
    if n == 0:
        raise MoeError("moe_workspace_size", -1)
    return torch.empty(n, dtype=torch.uint8, device=device)


def ws_view(ws, T, H, F, E, k, dtype, which, torch_dtype=None):
    """A tensor view of one workspace region (for inspection)."""
    import torch
    off, n = moe_workspace_region(T, H, F, E, k, dtype_code(dtype), which)
    v = ws[off:off + n]
    return v.view(torch_dtype) if torch_dtype is not None else v


def prepare_weights_mx(w1, w3, s1, s3, w2, s2, stream=None):
    """One-time preparation of MX FP4 weights (uint8 tensors: packed e2m1
    w1/w3 [E,F,H/2], w2 [E,H,F/2]; UE8M0 exponents s1/s3 [E,F,H/32], s2
    [E,H,F/32]); returns (w13, s13, w2p, s2p) for ffn_forward(..., "mxfp4")."""
    import torch
    E, F, Hh = w1.shape
    H = 2 * Hh
    for t in (w1, w3, s1, s3, w2, s2):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise ValueError("prepare_weights_mx takes contiguous uint8 tensors (packed e2m1 codes, UE8M0 exponents)")
    if (w3.shape != (E, F, Hh) or w2.shape != (E, H, F // 2) or s1.shape != (E, F, H // 32)
            or s3.shape != (E, F, H // 32) or s2.shape != (E, H, F // 32)):
        raise ValueError("MX FP4 weight or scale shapes do not match")
    dev = w1.device
    w13 = torch.empty(E * 2 * F * Hh, dtype=torch.uint8, device=dev)
    s13 = torch.empty(E * 2 * F * (H // 32), dtype=torch.uint8, device=dev)
    w2p = torch.empty_like(w2).view(-1)
    s2p = torch.empty_like(s2).view(-1)
    rc = moe_prepare_weights_mx(_ptr(w1), _ptr(w3), _ptr(s1), _ptr(s3), _ptr(w2), _ptr(s2), _ptr(w13), _ptr(s13),
                                _ptr(w2p), _ptr(s2p), E, F, H, _stream(stream))
    _check("moe_prepare_weights_mx", rc)
    return w13, s13, w2p, s2p


def prepare_weights(w1, w3, s1, s3, w2, stream=None, out=None):
    """One-time preshuffle: returns (w13, s13, w2p) in the blocked layouts the
    kernels stream (w13/w2p are flat byte tensors; s13 [E,2F] or None).
    ``out``: an earlier result to write into (training: every step)."""
    import torch
    for t in (w1, w3, w2):
        if t.dtype not in (torch.bfloat16, torch.float8_e4m3fn) or t.dtype != w1.dtype or not t.is_contiguous():
            raise ValueError("prepare_weights takes contiguous bf16 or float8_e4m3fn weights of one dtype "
                             "(MX FP4 weights: prepare_weights_mx)")
    E, F, H = w1.shape
    if w3.shape != (E, F, H) or w2.shape != (E, H, F):
        raise ValueError(f"weight shapes {tuple(w1.shape)}, {tuple(w3.shape)}, {tuple(w2.shape)} do not match")
    fp8 = w1.dtype == torch.float8_e4m3fn
    if out is not None:
        w13, s13, w2p = out
    else:
        w13 = torch.empty(E * 2 * F * H * w1.element_size(), dtype=torch.uint8, device=w1.device)
        w2p = torch.empty(w2.numel() * w2.element_size(), dtype=torch.uint8, device=w2.device)
        s13 = torch.empty(E, 2 * F, dtype=torch.float32, device=w1.device) if fp8 else None
    rc = moe_prepare_weights(_ptr(w1), _ptr(w3), _ptr(s1) if fp8 else None, _ptr(s3) if fp8 else None, _ptr(w2),
                             _ptr(w13), _ptr(s13), _ptr(w2p), E, F, H, MOE_FP8_E4M3 if fp8 else MOE_BF16,
                             _stream(stream))
    _check("moe_prepare_weights", rc)
    return w13, s13, w2p


def route(logits, k, stream=None):
    """Routing alone; returns dict of device tensors (ids, w, counts, offsets, perm, inv_perm)."""
    import torch
    T, E = logits.shape
    dev = logits.device
    A = T * k
    out = dict(ids=torch.empty(T, k, dtype=torch.int32, device=dev), w=torch.empty(T, k, dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev), offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               perm=torch.empty(max(A, 1), dtype=torch.int32, device=dev),
               inv_perm=torch.empty(max(A, 1), dtype=torch.int32, device=dev))
    rc = moe_route(_ptr(logits), T, E, k, _ptr(out["ids"]), _ptr(out["w"]), _ptr(out["counts"]), _ptr(out["offsets"]),
                   _ptr(out["perm"]), _ptr(out["inv_perm"]), None, 0, _stream(stream))
    _check("moe_route", rc)
    out["perm"] = out["perm"][:A]
    out["inv_perm"] = out["inv_perm"][:A]
    return out


def ffn_forward(x, logits, w13, s13, w2p, s2, k, F, fp8, out=None, ws=None, stream=None):
    """The whole layer on prepared weights; returns the bf16 output [T,H] (and
    fills ``ws``).  ``fp8``: True (e4m3 weights), False (bf16) or "mxfp4"."""
    import torch
    T, H = x.shape
    E = logits.shape[1]
    dt = dtype_code(fp8)
    fp8 = dt != MOE_BF16
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = workspace(T, H, F, E, k, dt, x.device)
    rc = moe_ffn_forward(_ptr(x), _ptr(logits), _ptr(w13), _ptr(s13) if fp8 else None, _ptr(w2p),
                         _ptr(s2) if fp8 else None, T, H, F, E, k, dt, _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    _check("moe_ffn_forward", rc)
    return out


# ---------------------------------------------------------------- d_ff-sharded layer

def dff_rows(T, n_ranks, rank):
    """(first token, number of tokens) that rank `rank` owns in the d_ff-sharded
    layer: blocks of ceil(T / n_ranks) tokens, the last one possibly shorter."""
    per = -(-T // n_ranks) if T > 0 else 0
    first = min(T, rank * per)
    return first, max(0, min(per, T - first))


def dff_shard(w1, w3, s1, s3, w2, n_ranks, rank):
    """This rank's d_ff slice of the expert weights (slicing only): rows
    [r*Fs, (r+1)*Fs) of w1, w3 (and s1, s3) and the same columns of w2,
    Fs = d_ff / n_ranks (a multiple of 128).  Works on torch tensors on any
    device; returns contiguous copies (w1, w3, s1, s3, w2)."""
    F = w1.shape[1]
    if F % n_ranks or (F // n_ranks) % 128:
        raise ValueError(f"d_ff={F} does not split into {n_ranks} shards of a multiple of 128")
    fs = F // n_ranks
    sl = slice(rank * fs, (rank + 1) * fs)
    c = lambda t: None if t is None else t.contiguous()  # noqa: E731
    return (c(w1[:, sl]), c(w3[:, sl]), c(None if s1 is None else s1[:, sl]), c(None if s3 is None else s3[:, sl]),
            c(w2[:, :, sl]))


def ffn_forward_dff(x, logits, w13, s13, w2p, s2, k, F_shard, fp8, n_ranks, rank, peer_out32, peer_counter,
                    ws=None, stream=None):
    """One rank's part of a d_ff-sharded layer step (see moe_ffn_forward_dff):
    ``peer_out32`` / ``peer_counter`` are lists of n_ranks device tensors (or
    raw device addresses) of every rank's combine rows and arrival counter."""
    T, H = x.shape
    E = logits.shape[1]
    dt = MOE_FP8_E4M3 if fp8 else MOE_BF16
    if ws is None:
        ws = workspace(T, H, F_shard, E, k, dt, x.device)
    addr = lambda t: t if isinstance(t, int) else t.data_ptr()  # noqa: E731
    outs = (ctypes.c_void_p * n_ranks)(*[addr(t) for t in peer_out32])
    ctrs = (ctypes.c_void_p * n_ranks)(*[addr(t) for t in peer_counter])
    rc = moe_ffn_forward_dff(_ptr(x), _ptr(logits), _ptr(w13), _ptr(s13) if fp8 else None, _ptr(w2p),
                             _ptr(s2) if fp8 else None, T, H, F_shard, E, k, dt, n_ranks, rank, outs, ctrs, _ptr(ws),
                             ws.numel(), _stream(stream))
    _check("moe_ffn_forward_dff", rc)
    return ws


def dff_finalize(out32_rows, out, counter, target, stream=None):
    """Round this rank's combine rows to bf16 once every rank has signalled
    (see moe_dff_finalize); ``out32_rows`` [rows, H] fp32, ``out`` [rows, H] bf16."""
    rows, H = out.shape
    rc = moe_dff_finalize(_ptr(out32_rows), _ptr(out), rows, H, _ptr(counter), int(target) & 0xFFFFFFFF,
                          _stream(stream))
    _check("moe_dff_finalize", rc)
    return out


# ---------------------------------------------------------------- backward pass (BF16)

def backward_workspace(T, H, F, E, k, device="cuda"):
    import torch
    n = moe_backward_workspace_size(T, H, F, E, k)
    if n == 0:
        raise MoeError("moe_backward_workspace_size", -1)
    return torch.empty(n, dtype=torch.uint8, device=device)


def ffn_backward(x, logits, w1, w3, w2, dy, k, ws=None, out=None, stream=None):
    """Gradients of the BF16 layer for the upstream gradient dy: returns
    dict(dx [T,H] bf16, dw1 [E,F,H], dw3 [E,F,H], dw2 [E,H,F] bf16, dlogits
    [T,E] fp32).  w1, w3 [E,F,H], w2 [E,H,F]: the row-major bf16 weights (no
    preparation).  ``out``: an earlier result dict to write into."""
    import torch
    T, H = x.shape
    E, F, _ = w1.shape
    dev = x.device
    if ws is None:
        ws = backward_workspace(T, H, F, E, k, dev)
    if out is None:
        out = dict(dx=torch.empty(T, H, dtype=torch.bfloat16, device=dev),
                   dw1=torch.empty(E, F, H, dtype=torch.bfloat16, device=dev),
                   dw3=torch.empty(E, F, H, dtype=torch.bfloat16, device=dev),
                   dw2=torch.empty(E, H, F, dtype=torch.bfloat16, device=dev),
                   dlogits=torch.empty(T, E, dtype=torch.float32, device=dev))
    for t in (w1, w3, w2):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("ffn_backward takes contiguous bf16 weights")
    if w3.shape != (E, F, H) or w2.shape != (E, H, F):
        raise ValueError("weight shapes do not match")
    rc = moe_ffn_backward(_ptr(x), _ptr(logits), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(dy), T, H, F, E, k,
                          _ptr(out["dx"]), _ptr(out["dw1"]), _ptr(out["dw3"]), _ptr(out["dw2"]), _ptr(out["dlogits"]),
                          _ptr(ws), ws.numel(), _stream(stream))
    _check("moe_ffn_backward", rc)
    return out


def _bf16_weights(w1, w3, w2, fn):
    import torch
    for t in (w1, w3, w2):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{fn} takes contiguous bf16 weights")
    E, F, H = w1.shape
    if w3.shape != (E, F, H) or w2.shape != (E, H, F):
        raise ValueError("weight shapes do not match")
    return E, F, H


def ffn_forward_train(x, logits, w1, w3, w2, k, ws=None, out=None, stream=None):
    """The BF16 layer from the row-major weights (no preparation), keeping in
    ``ws`` (a backward workspace) what ffn_backward_saved needs; returns
    (out [T,H] bf16, ws)."""
    import torch
    T, H = x.shape
    E, F, _ = _bf16_weights(w1, w3, w2, "ffn_forward_train")
    if ws is None:
        ws = backward_workspace(T, H, F, E, k, x.device)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    _check("moe_ffn_forward_train", moe_ffn_forward_train(_ptr(x), _ptr(logits), _ptr(w1), _ptr(w3), _ptr(w2), T, H, F,
                                                          E, k, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out, ws


def ffn_backward_saved(w1, w3, w2, dy, k, ws, out=None, stream=None):
    """The backward of the last ffn_forward_train on ``ws``: same result dict
    as ffn_backward."""
    import torch
    T, H = dy.shape
    E, F, _ = _bf16_weights(w1, w3, w2, "ffn_backward_saved")
    dev = dy.device
    if out is None:
        out = dict(dx=torch.empty(T, H, dtype=torch.bfloat16, device=dev),
                   dw1=torch.empty(E, F, H, dtype=torch.bfloat16, device=dev),
                   dw3=torch.empty(E, F, H, dtype=torch.bfloat16, device=dev),
                   dw2=torch.empty(E, H, F, dtype=torch.bfloat16, device=dev),
                   dlogits=torch.empty(T, E, dtype=torch.float32, device=dev))
    rc = moe_ffn_backward_saved(_ptr(w1), _ptr(w3), _ptr(w2), _ptr(dy), T, H, F, E, k, _ptr(out["dx"]),
                                _ptr(out["dw1"]), _ptr(out["dw3"]), _ptr(out["dw2"]), _ptr(out["dlogits"]), _ptr(ws),
                                ws.numel(), _stream(stream))
    _check("moe_ffn_backward_saved", rc)
    return out
