"""Pins for the CPU oracle: each test checks it against something other than
itself -- library routines (torch's float8/bfloat16 casts, torch.softmax,
fp64 matmuls, Python's stable sort), closed forms, invariants and brute force.

The method is the routed MoE expert FFN of rocketrecap.com "FlyDSL kernels in
JAX" (paragraph 2; timestamps 5:56 and 8:14).  Numeric readings the pages leave
open (tie-break, softmax over the selected logits, FP8 quantisation points) are
the ones stated in the oracle's header.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import moe_inputs
import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def e4m3_lib(v):
    """torch's float32 -> float8_e4m3fn cast (round to nearest even)."""
    return int(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item())


def bf16_lib(v):
    return int(torch.tensor([v], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF


# ---------------------------------------------------------------- formats

def test_e4m3_decode_all_codes_match_library():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).float().double().numpy()
    for c in range(256):
        mine = oracle.e4m3_to_double(c)
        if math.isnan(lib[c]):
            assert math.isnan(mine), c
        else:
            assert mine == lib[c], (c, mine, lib[c])
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9  # smallest subnormal


def test_e4m3_encode_matches_library_in_range():
    rng = np.random.default_rng(1)
    vals = list(rng.normal(0, 50, 4000).astype(np.float32)) + list(rng.normal(0, 0.01, 2000).astype(np.float32))
    # exact midpoints between neighbouring codes (ties) and values just beside them
    pos = [oracle.e4m3_to_double(c) for c in range(0x7F)]
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32((a + b) / 2)
        vals += [m, -m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))]
    for v in vals:
        v = np.float32(v)
        if abs(v) > 448:
            continue
        assert oracle.e4m3_from_float(v) == e4m3_lib(v), v


def test_e4m3_ties_to_even_and_saturation():
    assert oracle.e4m3_from_float(1.0625) == 0x38      # 1.0 (mantissa 000) beats 1.125
    assert oracle.e4m3_from_float(1.1875) == 0x3A      # 1.25 (mantissa 010) beats 1.125
    assert oracle.e4m3_from_float(448.0) == 0x7E
    assert oracle.e4m3_from_float(470.0) == 0x7E       # satfinite clamps
    assert oracle.e4m3_from_float(1e30) == 0x7E
    assert oracle.e4m3_from_float(-1e30) == 0xFE
    assert oracle.e4m3_from_float(float("inf")) == 0x7E
    assert oracle.e4m3_from_float(float("nan")) == 0x7F
    assert oracle.e4m3_from_float(-0.0) == 0x80
    assert oracle.e4m3_from_float(2.0 ** -10) == 0x00  # half the smallest subnormal: tie to even (0)


def test_bf16_round_matches_library_for_binary32_inputs():
    rng = np.random.default_rng(2)
    vals = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-30, 200), rng.normal(0, 1e30, 200)])
    vals = vals.astype(np.float32)
    # binary32 values halfway between two bf16 values
    halfway = (rng.integers(0, 2 ** 15, 500, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    for v in list(vals) + list(halfway):
        if not np.isfinite(v):
            continue
        assert oracle.bf16_from_double(float(v)) == bf16_lib(float(v)), v


def test_bf16_round_from_double_is_single_rounding():
    # a double just above a bf16 tie must round up (a binary32 detour would
    # land exactly on the tie and round to even = down)
    lo = 1.0
    ulp = 2.0 ** -7
    v = lo + ulp / 2 + 2.0 ** -40
    assert Fraction(v) > Fraction(lo) + Fraction(ulp) / 2
    assert oracle.bf16_to_double(oracle.bf16_from_double(v)) == lo + ulp
    assert oracle.bf16_to_double(oracle.bf16_from_double(lo + ulp / 2)) == lo   # exact tie -> even
    assert oracle.bf16_to_double(oracle.bf16_from_double(lo + 3 * ulp / 2)) == lo + 2 * ulp


# ---------------------------------------------------------------- R0

def test_quant_x_properties():
    rng = np.random.default_rng(3)
    x = torch.tensor(rng.normal(0, 1, (6, 64)), dtype=torch.float32).to(torch.bfloat16)
    x[2] = 0
    x[3, 5] = -7.5  # dominating negative absmax
    bits = x.view(torch.int16).numpy().view(np.uint16)
    xq, sx = oracle.quant_x(bits)
    xf = x.float().numpy()
    assert sx[2] == 1.0 and np.all(xq[2] == 0)
    for t in (0, 1, 3, 4, 5):
        amax = np.abs(xf[t]).max()
        # sx is the binary32 quotient absmax / 448
        assert abs(float(sx[t]) * 448.0 - amax) <= amax * 2.0 ** -23
        i = int(np.abs(xf[t]).argmax())
        assert xq[t, i] in (0x7E, 0xFE)  # the absmax element maps to +-448
        deq = np.array([oracle.e4m3_to_double(c) for c in xq[t]]) * float(sx[t])
        # nearest-value rounding: error at most half the spacing of e4m3 at that magnitude
        for v, d in zip(xf[t], deq):
            mag = abs(v) / float(sx[t])
            spacing = 2.0 ** (max(math.floor(math.log2(mag)), -6) - 3) if mag > 0 else 2.0 ** -9
            assert abs(d - v) <= 0.5 * spacing * float(sx[t]) * (1 + 1e-6) + 1e-30
    assert xq[3, 5] == 0xFE


def _quant_x_torch(x_bf16):
    """R0 restated with torch's IEEE binary32 arithmetic and float8 conversion:
    sx = fp32(absmax / 448) (1 for a zero row), codes = e4m3(fp32(x / sx))."""
    xf = x_bf16.float()
    amax = xf.abs().amax(dim=1)
    sx = torch.where(amax > 0, amax / torch.tensor(448.0, dtype=torch.float32), torch.ones_like(amax))
    q = (xf / sx[:, None]).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).numpy(), sx.numpy()


def test_quant_x_bitwise_against_binary32_division():
    """Codes and scales equal, bit for bit, a division in binary32 followed by
    a round-to-nearest-even e4m3 conversion -- on random rows of many
    magnitudes, and on rows whose scale is a power of two so that quotients
    land exactly on e4m3 ties (normal and subnormal), where a wrong rounding
    rule, a reciprocal multiply or a scale computed in another precision
    would show."""
    rng = np.random.default_rng(31)
    rows = [rng.normal(0, 10.0 ** rng.uniform(-8, 4), 256) for _ in range(60)]
    rows += [rng.uniform(-1, 1, 256) * 10.0 ** rng.uniform(-3, 3) for _ in range(20)]
    ties = []
    for j in (-3, 0, 5):
        scale = 2.0 ** j  # absmax 448 * 2^j gives sx = 2^j exactly
        mids = []
        for ex in range(-6, 8):      # normal e4m3 binades: spacing 2^(ex-3), ties at odd multiples of half of it
            step = 2.0 ** (ex - 3)
            mids += [(2.0 ** ex) + (i + 0.5) * step for i in range(8)]
        mids += [(i + 0.5) * 2.0 ** -9 for i in range(8)]  # subnormal ties
        row = np.array([448.0] + mids + [-m for m in mids[:40]]) * scale
        ties.append(row)
    x = torch.zeros(len(rows) + len(ties), 256, dtype=torch.float32)
    for i, r in enumerate(rows + ties):
        x[i, :len(r)] = torch.tensor(r[:256], dtype=torch.float32)
    x = x.to(torch.bfloat16)
    # the tie rows are exactly representable in bf16
    for i, r in enumerate(ties):
        np.testing.assert_array_equal(x[len(rows) + i, :len(r)].double().numpy(), r)
    x[3] = 0  # a zero row: scale 1, all codes zero
    bits = x.view(torch.int16).numpy().view(np.uint16)
    xq, sx = oracle.quant_x(bits)
    xq_t, sx_t = _quant_x_torch(x)
    np.testing.assert_array_equal(sx.view(np.uint32), sx_t.view(np.uint32))
    np.testing.assert_array_equal(xq, xq_t)
    assert sx[3] == 1.0 and not xq[3].any()
    # the ties did round to even: e.g. 1.0625 -> 1.0 (code 0x38), 1.1875 -> 1.25 (0x3A)
    t0 = len(rows) + 1  # scale 2^0
    vals = x[t0].double().numpy()
    i1 = int(np.nonzero(vals == 1.0625)[0][0])
    i2 = int(np.nonzero(vals == 1.1875)[0][0])
    assert xq[t0, i1] == 0x38 and xq[t0, i2] == 0x3A


# ---------------------------------------------------------------- MX block quantisation of h

@pytest.mark.parametrize("amax,expected", [
    (448.0, 0), (224.0, -1), (896.0, 1), (448.0 * 2 ** -10, -10), (449.0, 1), (447.0, 0),
    (1.0, -8), (1.75, -8), (1.7578125, -7), (0.0, 0), (1e-40, -127), (3e38, 120)])
def test_mx_exponent_closed_form(amax, expected):
    assert oracle.mx_exponent(amax) == expected


def test_mx_quant_block_properties():
    rng = np.random.default_rng(4)
    for trial in range(50):
        hb = torch.tensor(rng.normal(0, 10.0 ** rng.uniform(-6, 3), 32), dtype=torch.float32)
        hb = hb.to(torch.bfloat16).double().numpy()
        e, codes = oracle.mx_quant_block(hb)
        amax = np.abs(hb).max()
        assert amax / 2.0 ** e <= 448.0
        assert amax / 2.0 ** e > 224.0  # smallest power of two that fits
        for v, c in zip(hb, codes):
            assert c == e4m3_lib(np.float32(v / 2.0 ** e))
    e, codes = oracle.mx_quant_block(np.zeros(32))
    assert e == 0 and np.all(codes == 0)


# ---------------------------------------------------------------- R1/R2 routing

def _brute_topk(l, k):
    key = lambda e: (-(-math.inf if math.isnan(l[e]) else float(l[e])), e)  # noqa: E731
    return sorted(range(len(l)), key=key)[:k]


def _check_routing(logits, k):
    r = oracle.route(logits, k)
    T, E = logits.shape
    for t in range(T):
        assert list(r["ids"][t]) == _brute_topk(logits[t], k), t
        sel = np.array([logits[t, e] for e in r["ids"][t]], dtype=np.float64)
        if np.all(np.isfinite(sel)):
            ref = torch.softmax(torch.tensor(sel), dim=0).numpy()
            np.testing.assert_allclose(r["w"][t], ref, rtol=1e-14, atol=1e-15)
        assert abs(r["w"][t].sum() - 1.0) < 1e-12
    flat = r["ids"].reshape(-1)
    np.testing.assert_array_equal(r["counts"], np.bincount(flat, minlength=E))
    assert r["counts"].sum() == T * k
    np.testing.assert_array_equal(r["offsets"], np.concatenate([[0], np.cumsum(r["counts"])]))
    # stable sort of assignments by expert (Python's sort is stable)
    np.testing.assert_array_equal(r["perm"], sorted(range(T * k), key=lambda a: flat[a]))
    np.testing.assert_array_equal(r["inv_perm"][r["perm"]], np.arange(T * k))
    return r


@pytest.mark.parametrize("T,E,k", [(8, 4, 2), (8, 4, 1), (5, 3, 3), (7, 8, 2), (64, 8, 2), (33, 64, 8)])
def test_route_matches_brute_force(T, E, k):
    rng = np.random.default_rng(T * 100 + E * 10 + k)
    _check_routing(rng.normal(0, 1, (T, E)).astype(np.float32), k)


def test_route_ties_nan_and_signed_zero():
    lg = np.array([
        [1.0, 1.0, 1.0, 1.0],          # all equal -> experts 0, 1
        [0.0, -0.0, 0.5, -1.0],        # 0.5 first, then +0 vs -0 tie -> lower index 0
        [np.nan, -5.0, np.nan, -6.0],  # NaN ranks as -inf
        [-np.inf, np.nan, -np.inf, np.nan],  # nothing finite -> index order
        [2.0, 3.0, 3.0, 1.0],          # tie on the max -> 1 then 2
    ], dtype=np.float32)
    r = _check_routing(lg, 2)
    assert r["ids"].tolist() == [[0, 1], [2, 0], [1, 3], [0, 1], [1, 2]]
    np.testing.assert_allclose(r["w"][0], [0.5, 0.5])
    np.testing.assert_allclose(r["w"][3], [0.5, 0.5])   # limit reading: equal shares
    np.testing.assert_allclose(r["w"][4], [0.5, 0.5])


def test_route_random_shapes_with_ties():
    """Random shapes (T from 0, E up to 16, every k) with logits drawn from a
    small set that forces ties, signed zeros, infinities and NaN."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    values = st.sampled_from([0.0, -0.0, 1.0, -1.0, 0.5, 2.0, math.inf, -math.inf, math.nan])

    @settings(max_examples=150, deadline=None, derandomize=True)
    @given(st.data())
    def check(data):
        E = data.draw(st.integers(1, 16))
        k = data.draw(st.integers(1, min(E, 8)))
        T = data.draw(st.integers(0, 40))
        flat = data.draw(st.lists(values, min_size=T * E, max_size=T * E))
        _check_routing(np.array(flat, dtype=np.float32).reshape(T, E), k)

    check()


def test_route_k_equals_e_and_k1():
    rng = np.random.default_rng(7)
    lg = rng.normal(0, 1, (9, 4)).astype(np.float32)
    r = _check_routing(lg, 4)
    np.testing.assert_array_equal(r["counts"], [9, 9, 9, 9])
    r1 = _check_routing(lg, 1)
    assert np.all(r1["w"] == 1.0)


def test_route_skewed_shares():
    lg = moe_inputs.make_logits(8192, 8, 3, skew=True).numpy()
    r = oracle.route(lg, 2)
    share = r["counts"] / r["counts"].sum()
    assert share[0] > 0.40 and share[7] < 0.01 and np.all(np.diff(share) < 0)


# ---------------------------------------------------------------- MX FP4 weight formats

def test_e2m1_decode_all_codes():
    """The 16 e2m1 codes against ml_dtypes' float4_e2m1fn (magnitudes 0, 0.5,
    1, 1.5, 2, 3, 4, 6 and their negatives; -0 keeps its sign)."""
    import ml_dtypes
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.array([oracle.e2m1_to_double(c) for c in range(16)])
    np.testing.assert_array_equal(got, ref)
    assert math.copysign(1.0, oracle.e2m1_to_double(8)) == -1.0
    assert oracle.e2m1_to_double(0x17) == oracle.e2m1_to_double(0x07) == 6.0  # only the low 4 bits count


def test_ue8m0_decode_all_codes():
    import ml_dtypes
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = np.array([oracle.ue8m0_to_double(c) for c in range(256)])
    np.testing.assert_array_equal(got[:255], ref[:255])
    assert math.isnan(got[255]) and math.isnan(ref[255])
    assert got[127] == 1.0 and got[0] == 2.0 ** -127 and got[254] == 2.0 ** 127


def test_mxfp4_weights_are_an_mx_block_quantisation():
    """The MX FP4 input format (OCP Microscaling): the block scale is
    2^(floor(log2 amax) - 2), so a block's largest magnitude sits in [4, 8)
    before rounding; every weight is within half an e2m1 step of the bf16
    draw it encodes, except magnitudes above 6, which saturate at 6."""
    E, rows, cols = 2, 64, 256
    codes, exps = moe_inputs._weight_mxfp4(E, rows, cols, seed=21, stream=0)
    g = moe_inputs._gen(21, 0)
    for e in range(E):
        wb = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16).double().numpy()
        deq = _mx_fp4_dequant(codes[e], exps[e]).numpy()
        scale = np.repeat(2.0 ** (exps[e].numpy().astype(np.int64) - 127), 32, axis=1)
        q = deq / scale
        assert np.abs(q).max() <= 6.0
        # error at most half the e2m1 spacing at that magnitude (0.5 below 2, 1 in [2, 4), 2 in [4, 6])
        mag = np.abs(wb / scale)
        assert mag.max() < 8.0
        spacing = np.where(mag < 2, 0.5, np.where(mag < 4, 1.0, 2.0))
        allowed = np.where(mag > 6, mag - 6, 0.5 * spacing)
        assert np.all(np.abs(q - wb / scale) <= allowed + 1e-12)
        bmax = np.abs(q).reshape(rows, cols // 32, 32).max(axis=2)
        assert np.all((bmax >= 4.0) & (bmax <= 6.0))


# ---------------------------------------------------------------- the layer

def _bf16_round_vec(a):
    return np.array([oracle.bf16_to_double(oracle.bf16_from_double(float(v))) for v in a.reshape(-1)]).reshape(a.shape)


def _mx_fp4_dequant(codes, exps):
    """Packed e2m1 codes [rows, K/2] and block exponents [rows, K/32] -> float64
    [rows, K], decoded by ml_dtypes (an independent implementation of both
    formats); the even column sits in the low 4 bits of each byte."""
    import ml_dtypes
    c = codes.numpy()
    nib = np.empty((c.shape[0], c.shape[1] * 2), dtype=np.uint8)
    nib[:, 0::2] = c & 0xF
    nib[:, 1::2] = c >> 4
    vals = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    scale = exps.numpy().view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    return torch.tensor(vals * np.repeat(scale, 32, axis=1))


def _dense_swiglu_reference(case, tok):
    """E=1, k=1: the layer is a dense SwiGLU MLP; fp64 torch matmuls."""
    fp8 = case["dtype"] in ("fp8", "mxfp4")
    x = case["x"].double()
    if fp8:
        xq, sx = oracle.quant_x(moe_inputs.to_numpy(case)["x"])
        xd = torch.tensor(xq).view(torch.float8_e4m3fn).double() * torch.tensor(sx).double()[:, None]
        if case["dtype"] == "fp8":
            deq = lambda w, s: w.double() * s.double()[..., None]  # noqa: E731
        else:
            deq = _mx_fp4_dequant
        W1, W3, W2 = deq(case["w1"][0], case["s1"][0]), deq(case["w3"][0], case["s3"][0]), deq(case["w2"][0], case["s2"][0])
    else:
        xd = x
        W1, W3, W2 = case["w1"][0].double(), case["w3"][0].double(), case["w2"][0].double()
    xd = xd[tok]
    g = xd @ W1.T
    u = xd @ W3.T
    h = _bf16_round_vec((g * torch.sigmoid(g) * u).numpy())
    if fp8:
        hq = np.empty_like(h)
        for r in range(h.shape[0]):
            for b in range(0, h.shape[1], 32):
                e, codes = oracle.mx_quant_block(h[r, b:b + 32])
                hq[r, b:b + 32] = [oracle.e4m3_to_double(c) * 2.0 ** e for c in codes]
        h = hq
    return (torch.tensor(h) @ W2.T).numpy()


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "mxfp4"])
def test_single_expert_equals_dense_swiglu_mlp(dtype):
    case = moe_inputs.make_case(T=6, H=64, F=96, E=1, k=1, dtype=dtype, seed=11)
    r = oracle.moe_ffn(moe_inputs.to_numpy(case))
    ref = _dense_swiglu_reference(case, np.arange(6))
    scale = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(r["out64"] - ref)) <= 1e-12 * scale
    np.testing.assert_array_equal(r["out"], np.array([[oracle.bf16_from_double(v) for v in row] for row in ref]))


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "mxfp4"])
def test_routed_equals_masked_dense(dtype):
    case = moe_inputs.make_case(T=12, H=64, F=64, E=4, k=2, dtype=dtype, seed=12)
    nc = moe_inputs.to_numpy(case)
    a = oracle.moe_ffn(nc, mode="routed")
    b = oracle.moe_ffn(nc, mode="masked_dense")
    scale = np.sqrt(np.mean(a["out64"] ** 2))
    assert np.max(np.abs(a["out64"] - b["out64"])) <= 1e-12 * scale
    np.testing.assert_array_equal(a["out"], b["out"])


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_token_permutation_permutes_output(dtype):
    case = moe_inputs.make_case(T=10, H=32, F=64, E=4, k=2, dtype=dtype, seed=13)
    nc = moe_inputs.to_numpy(case)
    base = oracle.moe_ffn(nc)
    p = np.random.default_rng(5).permutation(10)
    nc2 = dict(nc)
    nc2["x"] = nc["x"][p]
    nc2["logits"] = nc["logits"][p]
    perm_out = oracle.moe_ffn(nc2)
    np.testing.assert_array_equal(perm_out["out"], base["out"][p])
    r1, r2 = oracle.route(nc["logits"], 2), oracle.route(nc2["logits"], 2)
    np.testing.assert_array_equal(r2["ids"], r1["ids"][p])


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_token_subset_matches_full_layer(dtype):
    case = moe_inputs.make_case(T=9, H=32, F=64, E=4, k=2, dtype=dtype, seed=14)
    nc = moe_inputs.to_numpy(case)
    full = oracle.moe_ffn(nc)
    tok = np.array([7, 0, 3])
    sub = oracle.moe_ffn_tokens(nc, tok)
    np.testing.assert_array_equal(sub["out"], full["out"][tok])


def test_one_hot_closed_form():
    """x_t = v_t * onehot(i_t); w1 = a_e I, w3 = b_e I, w2 = c_e P (P a cyclic
    shift, not an involution).  Then Y(e,t)[P(i_t)] = c_e * bf16(silu(a_e v) b_e v)
    and every other output is zero."""
    D, E, k, T = 16, 3, 2, 5
    a = [0.5, 1.5, -2.0]
    b = [0.25, -1.0, 3.0]
    c = [2.0, 0.5, -1.0]
    shift = lambda n: (n + 3) % D  # noqa: E731
    w1 = torch.zeros(E, D, D)
    w3 = torch.zeros(E, D, D)
    w2 = torch.zeros(E, D, D)
    for e in range(E):
        for n in range(D):
            w1[e, n, n] = a[e]
            w3[e, n, n] = b[e]
            w2[e, shift(n), n] = c[e]
    idx = [1, 4, 9, 15, 0]
    vals = [1.0, -0.5, 2.0, 0.75, -3.0]
    x = torch.zeros(T, D)
    for t in range(T):
        x[t, idx[t]] = vals[t]
    logits = torch.tensor([[0.1, 0.7, 0.3], [1.0, 1.0, -1.0], [-2.0, 0.0, 2.0], [0.0, 0.0, 0.0], [5.0, -5.0, 4.0]])
    case = dict(x=x.to(torch.bfloat16), logits=logits, w1=w1.to(torch.bfloat16), w3=w3.to(torch.bfloat16),
                w2=w2.to(torch.bfloat16), k=k, dtype="bf16")
    r = oracle.moe_ffn(moe_inputs.to_numpy(case))
    for t in range(T):
        lg = logits[t].tolist()
        sel = sorted(range(E), key=lambda e: (-lg[e], e))[:k]
        ex = [math.exp(lg[e] - lg[sel[0]]) for e in sel]
        wts = [v / sum(ex) for v in ex]
        expect = np.zeros(D)
        v = vals[t]
        for wj, e in sorted(zip(wts, sel), key=lambda p: p[1]):
            g = a[e] * v
            hval = oracle.bf16_to_double(oracle.bf16_from_double(g / (1 + math.exp(-g)) * (b[e] * v)))
            expect[shift(idx[t])] += wj * c[e] * hval
        np.testing.assert_allclose(r["out64"][t], expect, rtol=1e-15, atol=1e-300)


def test_golden_regression_record():
    """The stored record was written by tests/golden/make_golden.py (oracle only)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_routing_and_rows.json")
    with open(path) as f:
        g = json.load(f)
    nc = moe_inputs.to_numpy(moe_inputs.make_config("tiny"))
    r = oracle.route(nc["logits"], nc["k"])
    assert r["ids"].tolist() == g["topk_ids"]
    assert r["counts"].tolist() == g["counts"]
    assert r["perm"].tolist() == g["perm"]
    rows = oracle.moe_ffn_tokens(nc, g["tokens"])
    assert rows["out"].tolist() == g["out_bits"]


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_per_assignment_intermediates(dtype):
    """h_deq of the per-token form equals the routed form's h (sorted order), and
    rounding h_exact (bf16, then the block quantiser) reproduces h_deq."""
    case = moe_inputs.make_case(T=7, H=64, F=96, E=4, k=2, dtype=dtype, seed=15)
    nc = moe_inputs.to_numpy(case)
    full = oracle.moe_ffn(nc, want_h=True)
    tok = np.arange(7)
    sub = oracle.moe_ffn_tokens(nc, tok, want_h=True)
    r = oracle.route(nc["logits"], 2)
    for a in range(14):
        np.testing.assert_array_equal(sub["h_deq"][a], full["h"][r["inv_perm"][a]])
        hb = _bf16_round_vec(sub["h_exact"][a])
        if dtype == "bf16":
            np.testing.assert_array_equal(hb, sub["h_deq"][a])
        else:
            for b in range(0, 96, 32):
                e, codes = oracle.mx_quant_block(hb[b:b + 32])
                np.testing.assert_array_equal([oracle.e4m3_to_double(c) * 2.0 ** e for c in codes],
                                              sub["h_deq"][a][b:b + 32])


# ---------------------------------------------------------------- backward (custom VJP)

def _bwd_inputs(T, H, F, E, seed, wscale=0.3):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((T, H)), logits=rng.standard_normal((T, E)),
                w1=rng.standard_normal((E, F, H)) * wscale, w3=rng.standard_normal((E, F, H)) * wscale,
                w2=rng.standard_normal((E, H, F)) * wscale, dy=rng.standard_normal((T, H)))


def test_ffn64_equals_forward_oracle_on_bf16_inputs():
    """The fp64-input layer with h rounded to bf16 is the BF16 forward oracle
    (pinned above) on bf16-representable inputs: the same sums in the same
    order, so equal to the last bit."""
    case = moe_inputs.make_case(23, 128, 256, 8, 2, "bf16", 41)
    nc = moe_inputs.to_numpy(case)
    ref = oracle.moe_ffn(nc)["out64"]
    f = oracle.bf16_bits_to_f64
    y = oracle.ffn64(f(nc["x"]), nc["logits"].astype(np.float64), f(nc["w1"]), f(nc["w3"]), f(nc["w2"]), 2,
                     round_h=True)
    np.testing.assert_array_equal(y, ref)


@pytest.mark.parametrize("T,H,F,E,k", [(5, 8, 12, 4, 2), (3, 6, 10, 3, 3), (4, 8, 8, 1, 1)])
def test_bwd_matches_finite_differences(T, H, F, E, k):
    """Every entry of dx, dw1, dw3, dw2 and dlogits against a central
    difference of L = <dy, layer(x)> (fp64, h not rounded), step 1e-6: a
    dropped term, a sign, a transposed operand or a wrong index fails."""
    d = _bwd_inputs(T, H, F, E, seed=7 * T + E)
    g = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], k, round_h=False)
    names = ["x", "logits", "w1", "w3", "w2"]
    grads = {"x": "dx", "logits": "dlogits", "w1": "dw1", "w3": "dw3", "w2": "dw2"}
    eps = 1e-6

    def loss(args):
        return float((oracle.ffn64(*(args[n] for n in names), k) * d["dy"]).sum())

    for n in names:
        for idx in np.ndindex(d[n].shape):
            p = {m: d[m] for m in names}
            p[n] = d[n].copy()
            p[n][idx] += eps
            lp = loss(p)
            p[n][idx] -= 2 * eps
            lm = loss(p)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[grads[n]][idx]) < 1e-7 * (1 + abs(fd)), (n, idx, fd, g[grads[n]][idx])


def test_bwd_dense_mlp_against_autograd():
    """E = 1, k = 1: the layer is a dense SwiGLU MLP with routing weight 1;
    its gradients from torch.autograd (fp64) and dlogits = 0."""
    T, H, F = 9, 16, 24
    d = _bwd_inputs(T, H, F, 1, seed=3)
    g = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 1, round_h=False)
    x, w1, w3, w2 = (torch.tensor(d[n], requires_grad=True) for n in ("x", "w1", "w3", "w2"))
    y = (torch.nn.functional.silu(x @ w1[0].T) * (x @ w3[0].T)) @ w2[0].T
    (y * torch.tensor(d["dy"])).sum().backward()
    for mine, lib in ((g["dx"], x.grad), (g["dw1"], w1.grad), (g["dw3"], w3.grad), (g["dw2"], w2.grad)):
        np.testing.assert_allclose(mine, lib.numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(g["dlogits"] == 0.0)


def test_bwd_all_experts_chosen_against_autograd():
    """k = E: every expert is chosen and the weights are the softmax over all
    logits, so the layer is sum_e softmax(l)_e FFN_e(x); torch.autograd of
    that (fp64) gives every gradient, the logits' included."""
    T, H, F, E = 7, 12, 20, 3
    d = _bwd_inputs(T, H, F, E, seed=11)
    g = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], E, round_h=False)
    x, lg, w1, w3, w2 = (torch.tensor(d[n], requires_grad=True) for n in ("x", "logits", "w1", "w3", "w2"))
    p = torch.softmax(lg, dim=1)
    y = sum(p[:, e:e + 1] * ((torch.nn.functional.silu(x @ w1[e].T) * (x @ w3[e].T)) @ w2[e].T) for e in range(E))
    (y * torch.tensor(d["dy"])).sum().backward()
    for mine, lib in ((g["dx"], x.grad), (g["dlogits"], lg.grad), (g["dw1"], w1.grad), (g["dw3"], w3.grad),
                      (g["dw2"], w2.grad)):
        np.testing.assert_allclose(mine, lib.numpy(), rtol=1e-11, atol=1e-12)


def test_bwd_router_gradient_invariants():
    """Softmax is invariant to a shift of the chosen logits: each token's
    logit gradients sum to 0; experts not chosen get exactly 0; and dlogit_j =
    w_j (dw_j - sum_i w_i dw_i) with dw_a = <dy_t, expert output>."""
    T, H, F, E, k = 40, 16, 32, 8, 2
    d = _bwd_inputs(T, H, F, E, seed=5)
    g = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], k)
    np.testing.assert_allclose(g["dlogits"].sum(axis=1), 0.0, atol=1e-12)
    r = oracle.route(d["logits"].astype(np.float32), k)
    for t in range(T):
        chosen = set(r["ids"][t].tolist())
        for e in range(E):
            if e not in chosen:
                assert g["dlogits"][t, e] == 0.0
    # dw_a from the expert outputs y_e computed by the forward with one-hot logits
    big = 1e4
    for t in range(0, T, 7):
        for j in range(k):
            e = int(r["ids"][t, j])
            onehot = np.full((1, E), -big)
            onehot[0, e] = 0.0
            ye = oracle.ffn64(d["x"][t:t + 1], onehot, d["w1"], d["w3"], d["w2"], 1, round_h=True)
            assert abs(g["dwa"][t, j] - float(ye[0] @ d["dy"][t])) < 1e-12 * (1 + abs(g["dwa"][t, j]))


def test_bwd_rounded_h_close_to_exact():
    """Rounding h to bf16 (the forward's intermediate) moves the gradients by
    about the bf16 unit (2^-9 relative) and no more."""
    d = _bwd_inputs(30, 16, 32, 4, seed=9)
    a = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 2, round_h=True)
    b = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 2, round_h=False)
    for n in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        rel = np.linalg.norm(a[n] - b[n]) / np.linalg.norm(b[n])
        assert rel < 2.0 ** -8, (n, rel)
    # dx, dw1 and dw3 see h only through dw_a (the router) -- not at all with k = 1 and E = 1
    d1 = _bwd_inputs(10, 8, 16, 1, seed=2)
    a1 = oracle.ffn_bwd64(d1["x"], d1["logits"], d1["w1"], d1["w3"], d1["w2"], d1["dy"], 1, round_h=True)
    b1 = oracle.ffn_bwd64(d1["x"], d1["logits"], d1["w1"], d1["w3"], d1["w2"], d1["dy"], 1, round_h=False)
    for n in ("dx", "dw1", "dw3"):
        np.testing.assert_array_equal(a1[n], b1[n])


def test_bwd_sampled_equals_full():
    """The sampled form (used at full size) gives the full form's values for
    the rows and columns it samples, to the last bit."""
    T, H, F, E, k = 33, 16, 24, 4, 2
    d = _bwd_inputs(T, H, F, E, seed=13)
    full = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], k)
    tok = np.array([0, 5, 32, 17], dtype=np.int32)
    feats = np.array([[0, 0], [3, 23], [2, 7], [1, 11]], dtype=np.int32)
    s = oracle.ffn_bwd64_sampled(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], k, tok, feats)
    np.testing.assert_array_equal(s["dx"], full["dx"][tok])
    np.testing.assert_array_equal(s["dlogits"], full["dlogits"][tok])
    for q, (e, n) in enumerate(feats):
        np.testing.assert_array_equal(s["dw1"][q], full["dw1"][e, n])
        np.testing.assert_array_equal(s["dw3"][q], full["dw3"][e, n])
        np.testing.assert_array_equal(s["dw2"][q], full["dw2"][e, :, n])


def test_bwd_rounding_points_move_little():
    """Rounding the backward's stored intermediates (g, u, dg, du, w_a dy_t)
    to bf16 moves the gradients by about the bf16 unit, and rounds exactly
    the values it names: with E = 1 and k = 1, dw1 from the rounded form is
    the product of bf16 dg and x."""
    d = _bwd_inputs(30, 16, 32, 4, seed=19)
    a = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 2, round_h=True, round_inter=True)
    b = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 2, round_h=True)
    for n in ("dx", "dw1", "dw3", "dw2"):
        rel = np.linalg.norm(a[n] - b[n]) / np.linalg.norm(b[n])
        assert 0 < rel < 2.0 ** -7, (n, rel)
    np.testing.assert_array_equal(a["dlogits"], b["dlogits"])  # dw_a sees neither rounding
    # one token, one expert: dw1 = dg x^T with dg a bf16 value
    d1 = _bwd_inputs(1, 8, 16, 1, seed=23)
    g1 = oracle.ffn_bwd64(d1["x"], d1["logits"], d1["w1"], d1["w3"], d1["w2"], d1["dy"], 1, round_h=True,
                          round_inter=True)
    x = d1["x"][0]
    i = int(np.argmax(np.abs(x)))
    dg = g1["dw1"][0][:, i] / x[i]
    bits = torch.tensor(dg, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    np.testing.assert_allclose(dg, bits, rtol=1e-15, atol=0)


def test_bwd_error_scales():
    """The error scales are sums of absolute terms: at least |gradient|
    everywhere, equal to it where a sum has one term (one token, one expert:
    dW1 = dg x^T, dW3 = du x^T, dW2 = dO h^T), and the sampled form gives the
    full form's scales."""
    d = _bwd_inputs(25, 16, 24, 4, seed=29)
    g = oracle.ffn_bwd64(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 2, round_inter=True, want_abs=True)
    for n in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        assert np.all(g[n + "_abs"] >= np.abs(g[n]) * (1 - 1e-12)), n
    assert np.all(g["dx_abs"] > 0)
    one = _bwd_inputs(1, 8, 16, 1, seed=31)
    g1 = oracle.ffn_bwd64(one["x"], one["logits"], one["w1"], one["w3"], one["w2"], one["dy"], 1, want_abs=True)
    for n in ("dw1", "dw3", "dw2"):
        np.testing.assert_allclose(g1[n + "_abs"], np.abs(g1[n]), rtol=1e-14)
    tok = np.array([3, 24], dtype=np.int32)
    feats = np.array([[1, 5], [3, 23]], dtype=np.int32)
    s = oracle.ffn_bwd64_sampled(d["x"], d["logits"], d["w1"], d["w3"], d["w2"], d["dy"], 2, tok, feats,
                                 round_inter=True, want_abs=True)
    np.testing.assert_allclose(s["dx_abs"], g["dx_abs"][tok], rtol=1e-13)
    np.testing.assert_allclose(s["dlogits_abs"], g["dlogits_abs"][tok], rtol=1e-13)
    for q, (e, n) in enumerate(feats):
        np.testing.assert_allclose(s["dw1_abs"][q], g["dw1_abs"][e, n], rtol=1e-13)
        np.testing.assert_allclose(s["dw3_abs"][q], g["dw3_abs"][e, n], rtol=1e-13)
        np.testing.assert_allclose(s["dw2_abs"][q], g["dw2_abs"][e, :, n], rtol=1e-13)
