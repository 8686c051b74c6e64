"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Routing (ids, counts, offsets, permutation) and the FP8 activation codes and
scales must match bit for bit; the layer output must satisfy
|gpu - ref| <= 1e-2*|ref| + 2e-3*rms(ref) element by element.  Small cases span
several 128-row tiles, ragged tails, empty experts and both tile paths; the
full-size workloads are checked on sampled tokens.
"""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle
from helpers import bf16_bits_to_f64, check_close, out_as_f64, run_layer, small_case, to_device, verify_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import mixture_experts_routed_02_b200 as m
    assert torch.cuda.is_available()
    return m


@pytest.fixture(autouse=True)
def _reset_options(moe):
    yield
    moe.moe_set_option(moe.OPT_PATH, 0)
    moe.moe_set_option(moe.OPT_SPLITK, 0)
    moe.moe_set_option(moe.OPT_GATHER, 0)


GATHER = pytest.mark.parametrize("gather", [2, 1], ids=["gather_pass", "tma_gather"])


def check_r0(moe, ws, case, nc, gather):
    """R0 bitwise: the per-token e4m3 codes (in the rows the first GEMM reads:
    per-token rows for the TMA gather, gather = 1; the padded layout written by
    the gather pass otherwise) and the per-token scales equal the oracle's."""
    T, H, F, E, k, dt = (case[n] for n in ("T", "H", "F", "E", "k", "dtype"))
    dtc = moe.dtype_code(dt)
    xq_ref, sx_ref = oracle.quant_x(nc["x"])
    sx = moe.ws_view(ws, T, H, F, E, k, dtc, "sx", torch.float32)[:T].cpu().numpy()
    np.testing.assert_array_equal(sx.view(np.uint32), sx_ref.view(np.uint32))
    if gather == 1:
        xs = moe.ws_view(ws, T, H, F, E, k, dtc, "xs").cpu().numpy().reshape(T, H)
        np.testing.assert_array_equal(xs, xq_ref)
    else:
        A = T * k
        slot_of = moe.ws_view(ws, T, H, F, E, k, dtc, "slot_of", torch.int32)[:A].cpu().numpy()
        xg = moe.ws_view(ws, T, H, F, E, k, dtc, "xg").cpu().numpy().reshape(-1, H + 128)[:, :H]
        np.testing.assert_array_equal(xg[slot_of], xq_ref[np.arange(A) // k])


# ---------------------------------------------------------------- routing

def _route_cases():
    rng = np.random.default_rng(0)
    cases = []
    for T, E, k in [(1, 8, 2), (5, 3, 3), (64, 8, 2), (1000, 8, 2), (333, 64, 8), (77, 16, 1), (4096, 8, 2)]:
        cases.append((f"normal_T{T}_E{E}_k{k}", rng.normal(0, 1, (T, E)).astype(np.float32), k))
    ties = rng.integers(-2, 3, (500, 8)).astype(np.float32)  # many exact ties
    ties[::7, 3] = np.nan
    ties[::11, :] = 0.0
    ties[1::11, ::2] = -0.0
    cases.append(("ties_nan_zeros", ties, 2))
    # at most 32 assignments: the one-warp router (more than 16 experts, every
    # k up to 8, and the tie / NaN / signed-zero ordering)
    cases.append(("warp_T4_E64_k8", rng.normal(0, 1, (4, 64)).astype(np.float32), 8))
    cases.append(("warp_T32_E20_k1", rng.normal(0, 1, (32, 20)).astype(np.float32), 1))
    cases.append(("warp_ties_nan_zeros_T16", ties[:16].copy(), 2))
    wt = rng.integers(-1, 2, (8, 24)).astype(np.float32)
    wt[::3, 5] = np.nan
    wt[1::4, ::3] = -0.0
    cases.append(("warp_ties_T8_E24_k4", wt, 4))
    cases.append(("skewed_T8192", moe_inputs.make_logits(8192, 8, 3, skew=True).numpy(), 2))
    cases.append(("sweep_T16384", moe_inputs.make_logits(16384, 8, 4).numpy(), 2))
    return cases


@pytest.mark.parametrize("name,logits,k", _route_cases(), ids=lambda v: v if isinstance(v, str) else "")
def test_route_bit_exact(moe, name, logits, k):
    ref = oracle.route(logits, k)
    out = moe.route(torch.from_numpy(logits).cuda(), k)
    assert moe.moe_get_status(None) == 0
    np.testing.assert_array_equal(out["ids"].cpu().numpy(), ref["ids"])
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(out["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(out["perm"].cpu().numpy(), ref["perm"])
    np.testing.assert_array_equal(out["inv_perm"].cpu().numpy(), ref["inv_perm"])
    np.testing.assert_allclose(out["w"].cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)


def test_route_deterministic(moe):
    lg = torch.from_numpy(moe_inputs.make_logits(16384, 8, 9).numpy()).cuda()
    runs = [moe.route(lg, 2) for _ in range(3)]
    for key in ("ids", "counts", "offsets", "perm", "inv_perm", "w"):
        for r in runs[1:]:
            assert torch.equal(r[key], runs[0][key]), key


# ---------------------------------------------------------------- the layer, small sizes

SMALL = [
    # (T, H, F, E, k, dtype, seed, skew)
    (64, 256, 512, 8, 2, "bf16", 0, False),     # the tiny workload
    (64, 256, 512, 8, 2, "fp8", 0, False),
    (1, 256, 512, 8, 2, "fp8", 5, False),
    (3, 256, 256, 8, 2, "bf16", 6, False),
    (200, 256, 512, 8, 2, "bf16", 7, False),    # several 128-row tiles, ragged tails
    (300, 256, 512, 8, 2, "fp8", 8, True),      # skewed: big and empty experts
    (37, 128, 256, 1, 1, "fp8", 9, False),      # E = 1, k = 1 (dense SwiGLU MLP)
    (50, 128, 384, 4, 4, "bf16", 10, False),    # k = E
    (129, 384, 640, 16, 3, "fp8", 11, False),   # odd multiples of 128
    (16, 256, 512, 8, 2, "fp8", 12, False),     # a decode-shaped batch (32 assignments)
    (16, 256, 512, 8, 2, "bf16", 13, False),
    (1000, 256, 512, 4, 2, "fp8", 14, False),   # 4 tiles per expert: whole CTA pairs
    (700, 256, 512, 4, 2, "bf16", 15, False),   # 3 tiles per expert: a pair and a lone tile
]


def _ids(p):
    T, H, F, E, k, dt, seed, skew = p
    return f"T{T}_H{H}_F{F}_E{E}_k{k}_{dt}" + ("_skew" if skew else "")


@GATHER
@pytest.mark.parametrize("path", [1, 2, 3, 4], ids=["pair_tiles", "streaming_tiles", "wide_tiles", "tiny_tiles"])
@pytest.mark.parametrize("p", SMALL, ids=_ids)
def test_layer_small(moe, p, path, gather):
    T, H, F, E, k, dt, seed, skew = p
    if path == 4 and T * k > 32:
        pytest.skip("the tiny-batch tiles take at most 32 assignments")
    moe.moe_set_option(moe.OPT_PATH, path)
    moe.moe_set_option(moe.OPT_GATHER, gather)
    case = small_case(T, H, F, E, k, dt, seed, skew)
    nc = moe_inputs.to_numpy(case)
    dcase = to_device(case)
    out, ws = run_layer(dcase)
    verify_layer(moe, ws, out, case, what=f"layer {_ids(p)} path {path}")

    # routing inside the layer is bit-exact too
    r = oracle.route(nc["logits"], k)
    A = T * k
    dtc = moe.dtype_code(dt)
    ids = moe.ws_view(ws, T, H, F, E, k, dtc, "topk_ids", torch.int32)[:A].cpu().numpy()
    perm = moe.ws_view(ws, T, H, F, E, k, dtc, "perm", torch.int32)[:A].cpu().numpy()
    np.testing.assert_array_equal(ids, r["ids"].reshape(-1))
    np.testing.assert_array_equal(perm, r["perm"])
    if dt in ("fp8", "mxfp4"):
        check_r0(moe, ws, case, nc, gather)


MXFP4 = [
    # (T, H, F, E, k, seed, skew): MX FP4 weights run on 128 x 128 one-CTA tiles
    (64, 256, 512, 8, 2, 30, False),
    (1, 256, 512, 8, 2, 31, False),
    (16, 256, 512, 8, 2, 32, False),       # decode-shaped (32 assignments)
    (200, 384, 640, 8, 2, 33, False),      # several m-tiles, ragged tails, odd multiples of 128
    (300, 256, 512, 8, 2, 34, True),       # skewed: big and empty experts
    (37, 128, 256, 1, 1, 35, False),       # E = 1, k = 1
    (16, 256, 2560, 8, 2, 36, False),      # last wave cut into 64-row slices (half-block scales)
]


@GATHER
@pytest.mark.parametrize("path", [0, 4], ids=["auto_tiles", "tiny_tiles"])
@pytest.mark.parametrize("p", MXFP4, ids=lambda p: f"T{p[0]}_H{p[1]}_F{p[2]}_E{p[3]}_k{p[4]}" + ("_skew" if p[6] else ""))
def test_layer_small_mxfp4(moe, p, path, gather):
    T, H, F, E, k, seed, skew = p
    if path == 4 and T * k > 32:
        pytest.skip("the tiny-batch tiles take at most 32 assignments")
    moe.moe_set_option(moe.OPT_PATH, path)
    moe.moe_set_option(moe.OPT_GATHER, gather)
    case = small_case(T, H, F, E, k, "mxfp4", seed, skew)
    nc = moe_inputs.to_numpy(case)
    out, ws = run_layer(to_device(case))
    verify_layer(moe, ws, out, case, what=f"mxfp4 layer T={T} H={H} F={F}")
    check_r0(moe, ws, case, nc, gather)


def test_layer_mxfp4_sliced_last_wave(moe):
    """MX FP4 at a decode shape whose last wave of first-GEMM tiles is lightly
    filled, so that wave runs as 64-row slices: each slice's packed rows are
    half of a 128-row block and its B scales half of a 128-row chunk."""
    T, H, F, E, k = 16, 256, 2560, 8, 2
    case = small_case(T, H, F, E, k, "mxfp4", 38)
    out, ws = run_layer(to_device(case))
    verify_layer(moe, ws, out, case, what="mxfp4 sliced last wave")


def test_prepare_weights_mx_layout(moe):
    """moe_prepare_weights_mx: w13 rows interleaved in groups of 32 (w1 then
    w3), still packed, in contiguous blocks of 128 rows x 64 bytes ordered
    [expert][row block][K block]; the scales regrouped into 512-byte chunks
    per (expert, 128-row block, 128-column block), byte (r%32)*16 + (r/32)*4 + b."""
    E, F, H = 2, 256, 384
    case = small_case(3, H, F, E, 2, "mxfp4", 37)
    d = to_device(case)
    unblock = lambda t, rows, cols: (t.cpu().numpy().reshape(E, rows // 128, cols // 128, 128, 64)  # noqa: E731
                                     .transpose(0, 1, 3, 2, 4).reshape(E, rows, cols // 2))
    w13 = unblock(d["w13"], 2 * F, H)
    w1, w3 = case["w1"].numpy(), case["w3"].numpy()
    src_rows = lambda R: (w3 if R % 64 >= 32 else w1, 32 * (R // 64) + R % 32)  # noqa: E731
    for R in range(2 * F):
        src, r = src_rows(R)
        np.testing.assert_array_equal(w13[:, R], src[:, r])
    np.testing.assert_array_equal(unblock(d["w2p"], H, F), case["w2"].numpy())
    s13 = d["s13"].cpu().numpy().reshape(E, 2 * F // 128, H // 128, 512)
    s1, s3 = case["s1"].numpy(), case["s3"].numpy()
    for R in range(2 * F):
        src, r = (s3 if R % 64 >= 32 else s1), 32 * (R // 64) + R % 32
        nb, rr = divmod(R, 128)
        for kt in range(H // 128):
            for b in range(4):
                assert s13[:, nb, kt, (rr % 32) * 16 + (rr // 32) * 4 + b].tolist() == src[:, r, 4 * kt + b].tolist()
    s2p = d["s2p"].cpu().numpy().reshape(E, H // 128, F // 128, 512)
    s2 = case["s2"].numpy()
    for R in range(0, H, 7):
        nb, rr = divmod(R, 128)
        for kt in range(F // 128):
            np.testing.assert_array_equal(s2p[:, nb, kt, (rr % 32) * 16 + (rr // 32) * 4 + np.arange(4)],
                                          s2[:, R, 4 * kt:4 * kt + 4])


def _expected_layout(r, T, E, k):
    """The expert-padded row layout from the oracle's routing: expert e owns
    whole 128-row tiles, its assignments first in sorted order, then padding."""
    counts = r["counts"].astype(np.int64)
    tiles = -(-counts // 128)
    mt_start = np.concatenate([[0], np.cumsum(tiles)])
    A = T * k
    slot_of = np.empty(A, np.int64)
    slot_assign = np.full(int(mt_start[-1]) * 128, -1, np.int64)
    for e in range(E):
        members = r["perm"][r["offsets"][e]:r["offsets"][e + 1]]
        slots = mt_start[e] * 128 + np.arange(len(members))
        slot_of[members] = slots
        slot_assign[slots] = members
    mtile_expert = np.repeat(np.arange(E), tiles)
    return slot_of, slot_assign, mtile_expert, int(mt_start[-1])


@pytest.mark.parametrize("T,E,k,seed", [(1024, 8, 2, 51), (1300, 16, 3, 52), (5000, 64, 8, 53), (3000, 8, 1, 54)])
def test_layer_routing_layout_many_ctas(moe, T, E, k, seed):
    """Large batches route on many SMs: every routing and layout array of the
    layer's workspace equals the oracle's routing and the padding rule."""
    H = F = 128
    case = small_case(T, H, F, E, k, "fp8", seed)
    out, ws = run_layer(to_device(case))
    nc = moe_inputs.to_numpy(case)
    r = oracle.route(nc["logits"], k)
    A = T * k
    view = lambda name: moe.ws_view(ws, T, H, F, E, k, 1, name, torch.int32).cpu().numpy()
    np.testing.assert_array_equal(view("topk_ids")[:A], r["ids"].reshape(-1))
    np.testing.assert_allclose(moe.ws_view(ws, T, H, F, E, k, 1, "topk_w", torch.float32)[:A].cpu().numpy(),
                               r["w"].reshape(-1), rtol=2e-6, atol=1e-7)
    np.testing.assert_array_equal(view("counts")[:E], r["counts"])
    np.testing.assert_array_equal(view("offsets")[:E + 1], r["offsets"])
    np.testing.assert_array_equal(view("perm")[:A], r["perm"])
    np.testing.assert_array_equal(view("inv_perm")[:A], r["inv_perm"])
    slot_of, slot_assign, mtile_expert, n_mt = _expected_layout(r, T, E, k)
    assert int(view("num_mtiles")[0]) == n_mt
    np.testing.assert_array_equal(view("slot_of")[:A], slot_of)
    np.testing.assert_array_equal(view("slot_assign")[:n_mt * 128], slot_assign)
    np.testing.assert_array_equal(view("mtile_expert")[:n_mt], mtile_expert)
    verify_layer(moe, ws, out, case, tokens=np.array([0, T // 2, T - 1]), what=f"many-CTA routing T={T}")


def test_layer_largest_batch(moe):
    """The largest batch the library takes (T*k = 262144 assignments): routing
    of every token is bit-exact, the padded layout is complete, and sampled
    outputs match the oracle."""
    T, H, F, E, k = 131072, 128, 256, 8, 2
    case = small_case(T, H, F, E, k, "fp8", 71)
    out, ws = run_layer(to_device(case))
    nc = moe_inputs.to_numpy(case)
    r = oracle.route(nc["logits"], k)
    A = T * k
    view = lambda name: moe.ws_view(ws, T, H, F, E, k, 1, name, torch.int32).cpu().numpy()
    np.testing.assert_array_equal(view("topk_ids")[:A], r["ids"].reshape(-1))
    np.testing.assert_array_equal(view("perm")[:A], r["perm"])
    slot_of, slot_assign, mtile_expert, n_mt = _expected_layout(r, T, E, k)
    np.testing.assert_array_equal(view("slot_of")[:A], slot_of)
    np.testing.assert_array_equal(view("slot_assign")[:n_mt * 128], slot_assign)
    rng = np.random.default_rng(72)
    tokens = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 12)]))
    verify_layer(moe, ws, out, case, tokens=tokens, what="largest batch")


@pytest.mark.parametrize("splits", [2, 4])
def test_layer_split_k(moe, splits):
    moe.moe_set_option(moe.OPT_PATH, 2)
    moe.moe_set_option(moe.OPT_SPLITK, splits)
    case = small_case(40, 256, 1024, 8, 2, "fp8", 21)
    out, ws = run_layer(to_device(case))
    verify_layer(moe, ws, out, case, what=f"split-K {splits}")


def _last_wave_sliced(num_mt, T, F, E, k, bn, num_sms):
    """Whether the first GEMM cuts its last wave into 64-row slices: one CTA per
    SM at most; a last wave that, cut into bn/64 slices per tile, still fits
    in the grid."""
    n_tiles = 2 * F // bn
    grid = min((-(-T * k // 128) + E) * n_tiles, num_sms)
    tail = (num_mt * n_tiles) % grid
    return tail > 0 and tail * (bn // 64) <= grid


@GATHER
@pytest.mark.parametrize("path,dt", [(3, "fp8"), (3, "bf16"), (2, "fp8"), (2, "bf16")],
                         ids=["wide_fp8", "wide_bf16", "streaming_fp8", "streaming_bf16"])
def test_layer_last_wave_slices(moe, path, dt, gather):
    """The first GEMM's last, lightly filled wave runs as 64-row weight slices
    (MMA N = 64); every slice's SwiGLU columns land in the right place."""
    T, H, F, E, k = 16, 256, 2560, 8, 2
    moe.moe_set_option(moe.OPT_PATH, path)
    moe.moe_set_option(moe.OPT_GATHER, gather)
    case = small_case(T, H, F, E, k, dt, 61)
    out, ws = run_layer(to_device(case))
    num_mt = int(moe.ws_view(ws, T, H, F, E, k, moe.dtype_code(dt), "num_mtiles", torch.int32)[0])
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert _last_wave_sliced(num_mt, T, F, E, k, 256 if path == 3 else 128, sms)
    verify_layer(moe, ws, out, case, what=f"last-wave slices path {path} {dt}")


def test_layer_repeat_and_empty(moe):
    case = small_case(70, 256, 512, 8, 2, "fp8", 22)
    dcase = to_device(case)
    a, ws = run_layer(dcase)
    b, _ = run_layer(dcase, ws)  # the workspace is reused: nothing may leak from the first call
    c, _ = run_layer(dcase, ws)
    assert torch.equal(b, c)
    verify_layer(moe, ws, c, case, what="repeat")
    import mixture_experts_routed_02_b200 as moe_mod
    # T = 0: valid, nothing to do
    rc = moe_mod.moe_ffn_forward(None, None, dcase["w13"].data_ptr(), dcase["s13"].data_ptr(),
                                 dcase["w2p"].data_ptr(), dcase["s2"].data_ptr(), 0, 256, 512, 8, 2, 1, None,
                                 ws.data_ptr(), ws.numel(), None)
    assert rc == 0


def _unblock(blocks, E, rows, row_bytes):
    """Invert the blocked, swizzled weight layout: [E][rows/128][row_bytes/128][128 x 128 B]."""
    nb, kt = rows // 128, row_bytes // 128
    b = blocks.reshape(E, nb, kt, 128, 8, 16)
    r = np.arange(128)[:, None]
    pc = np.arange(8)[None, :] ^ (r % 8)              # stored position of logical chunk c
    logical = b[:, :, :, np.arange(128)[:, None], pc, :]  # [E, nb, kt, 128, 8, 16]
    return logical.transpose(0, 1, 3, 2, 4, 5).reshape(E, rows, row_bytes)


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_preshuffle_layout(moe, dtype):
    case = small_case(4, 256, 384, 3, 2, dtype, 23)
    d = to_device(case)
    eb = 1 if dtype == "fp8" else 2
    E, F, H = 3, 384, 256
    w13 = _unblock(d["w13"].cpu().numpy(), E, 2 * F, H * eb)
    w2 = _unblock(d["w2p"].cpu().numpy(), E, H, F * eb)
    raw = lambda t: t.contiguous().view(torch.uint8).numpy().reshape(t.shape[0], t.shape[1], -1)  # noqa: E731
    w1, w3, w2_ref = raw(case["w1"]), raw(case["w3"]), raw(case["w2"])
    np.testing.assert_array_equal(w2, w2_ref)
    for r in range(2 * F):
        b, i = divmod(r, 64)
        src = (w3 if i >= 32 else w1)[:, 32 * b + (i % 32)]
        np.testing.assert_array_equal(w13[:, r], src)
        if dtype == "fp8":
            np.testing.assert_array_equal(d["s13"][:, r].cpu().numpy(),
                                          (case["s3"] if i >= 32 else case["s1"])[:, 32 * b + (i % 32)].numpy())


def test_host_errors(moe):
    x = torch.zeros(16, 100, dtype=torch.bfloat16, device="cuda")
    rc = moe.moe_ffn_forward(x.data_ptr(), x.data_ptr(), x.data_ptr(), None, x.data_ptr(), None, 16, 100, 256, 8, 2,
                             0, x.data_ptr(), x.data_ptr(), 1 << 30, None)
    assert rc == -2  # H % 128 != 0
    rc = moe.moe_ffn_forward(x.data_ptr() + 2, x.data_ptr(), x.data_ptr(), None, x.data_ptr(), None, 16, 128, 256, 8,
                             2, 0, x.data_ptr(), x.data_ptr(), 1 << 30, None)
    assert rc == -3  # misaligned
    rc = moe.moe_ffn_forward(x.data_ptr(), x.data_ptr(), x.data_ptr(), None, x.data_ptr(), None, 16, 128, 256, 8, 2,
                             0, x.data_ptr(), x.data_ptr(), 16, None)
    assert rc == -4  # workspace too small
    assert moe.moe_get_status(None) == 0


# ---------------------------------------------------------------- full-size workloads, sampled tokens

FULL = ["decode", "prefill", "skewed", "sweep_T1", "sweep_T128", "sweep_T1024", "sweep_T16384", "decode_mxfp4",
        "prefill_mxfp4"]


def _tokens_per_mtile(r, k, T, rng):
    """One token from every 128-row tile of the expert-padded layout (so every
    tile, and both halves of every CTA pair, is compared), plus the first and
    last token.  Rows of a tile are the sorted assignments of one expert."""
    picks = [0, T - 1]
    for e in range(len(r["counts"])):
        members = r["perm"][r["offsets"][e]:r["offsets"][e + 1]]
        for m0 in range(0, len(members), 128):
            tile = members[m0:m0 + 128]
            picks.append(int(tile[rng.integers(0, len(tile))]) // k)
    return np.unique(np.array(picks))


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_layer_full_size_sampled(moe, name):
    """Full-size workloads: routing of every token is bit-exact; outputs of one
    token per 128-row tile of every expert (every token when there are at most
    32) match the oracle; the outputs that need the rounding-flip allowance
    are counted (printed) and must stay below 0.1%."""
    case = moe_inputs.make_config(name)
    T = case["T"]
    dcase = to_device(case)
    out, ws = run_layer(dcase)
    nc = moe_inputs.to_numpy(case)
    r = oracle.route(nc["logits"], case["k"])
    # routing over every token is bit-exact
    A = T * case["k"]
    dtc = moe.dtype_code(case["dtype"])
    ids = moe.ws_view(ws, T, case["H"], case["F"], case["E"], case["k"], dtc, "topk_ids", torch.int32)[:A]
    perm = moe.ws_view(ws, T, case["H"], case["F"], case["E"], case["k"], dtc, "perm", torch.int32)[:A]
    np.testing.assert_array_equal(ids.cpu().numpy(), r["ids"].reshape(-1))
    np.testing.assert_array_equal(perm.cpu().numpy(), r["perm"])
    rng = np.random.default_rng(1234)
    tokens = np.arange(T) if T <= 32 else _tokens_per_mtile(r, case["k"], T, rng)
    stats = verify_layer(moe, ws, out, case, tokens, what=f"{name} sampled tokens")
    print(name, len(tokens), "tokens", stats)
    # outputs that meet the stated tolerance only with the exact effect of a
    # validated rounding flip of h added: recorded, and rare
    assert stats["outputs_needing_allowance"] <= 1e-3 * len(tokens) * case["H"], stats
