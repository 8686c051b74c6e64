"""Parity of the backward pass (custom VJP) of the BF16 layer with the fp64
oracle: dx, dw1, dw3, dw2 and the router-logit gradients, element by element
at small sizes (several tiles, ragged tails, empty experts, k = E, E = 1,
d_ff not a multiple of 256), sampled rows and columns at the Mixtral expert
shape, and results independent of stale workspace contents.

The oracle rounds to bf16 where the GPU stores bf16 between its kernels (h,
as the forward does; dg, du and the w_a dy_t entering dW2: round_h and
round_inter) and is exact otherwise.  What separates the two is then: the
bf16 rounding of the GPU's outputs (dx and the weight gradients; at most half
a unit, 2^-9 of the value); an intermediate that the GPU (fp32) and the oracle
(fp64) round to neighbouring bf16 values, which moves that term of a sum by
one unit (at most 2^-7 of the term; dW2's terms have two rounded factors);
and the GPU's fp32 sums (K up to 2F terms: about 2^-9 of the sum of the
absolute terms).  Tolerance, element by element:

    |gpu - ref| <= REL |ref| + C |ref|_abs,

|ref|_abs the oracle's sum of the absolute values of the entry's terms,
REL = 2^-8, C = 2^-6 (2^-5 for dW2): twice the unit-flip and summation terms."""
import numpy as np
import pytest
import torch

import moe_inputs
import oracle

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8
C_ABS = {"dx": 2.0 ** -6, "dw1": 2.0 ** -6, "dw3": 2.0 ** -6, "dw2": 2.0 ** -5, "dlogits": 2.0 ** -6}


@pytest.fixture(scope="module")
def moe():
    import mixture_experts_routed_02_b200 as m
    return m


def close(gpu, ref, ref_abs, name, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape == ref_abs.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    if ref.size == 0:
        return
    err = np.abs(gpu - ref)
    allowed = REL * np.abs(ref) + C_ABS[name] * ref_abs
    ratio = err / np.maximum(allowed, 1e-300)
    bad = err > allowed
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} out of tolerance; worst {ratio.max():.2f}x "
                           f"the allowance, at {np.unravel_index(ratio.argmax(), err.shape)}")


def f64(t):
    """A bf16 or fp32 torch tensor (any device) -> float64 numpy."""
    return t.detach().float().cpu().double().numpy()


def run_bwd(moe, case, dy):
    dev = "cuda"
    x, lg = case["x"].to(dev), case["logits"].to(dev)
    w1, w3, w2 = case["w1"].to(dev), case["w3"].to(dev), case["w2"].to(dev)
    out = moe.ffn_backward(x, lg, w1, w3, w2, dy.to(dev), case["k"])
    torch.cuda.synchronize()
    st = moe.moe_get_status(None)
    assert st == 0, moe.STATUS_NAMES.get(st, st)
    return out


def oracle_inputs(case, dy):
    nc = moe_inputs.to_numpy(case)
    f = oracle.bf16_bits_to_f64
    return (f(nc["x"]), nc["logits"].astype(np.float64), f(nc["w1"]), f(nc["w3"]), f(nc["w2"]),
            f(moe_inputs.to_numpy({"dy": dy})["dy"]))


SMALL = [
    # (T, H, F, E, k, seed, skew)
    (64, 256, 512, 8, 2, 50, False),
    (200, 256, 512, 8, 2, 51, False),     # several m-tiles per expert, ragged tails
    (300, 256, 512, 8, 2, 52, True),      # skewed: big and empty experts (zero weight gradients)
    (129, 384, 640, 4, 3, 53, False),     # d_ff and d_model not multiples of 256: 128-wide tiles
    (37, 128, 256, 1, 1, 54, False),      # E = 1, k = 1: a dense SwiGLU MLP (dlogits = 0)
    (50, 128, 384, 4, 4, 55, False),      # k = E
    (1, 256, 512, 8, 2, 56, False),       # one token
    (700, 256, 512, 4, 2, 57, False),     # several full tiles per expert
]


@pytest.fixture(autouse=True)
def _reset_path(moe):
    yield
    moe.moe_set_option(moe.OPT_PATH, 0)


@pytest.mark.parametrize("path", [0, 3], ids=["pair_tiles", "one_sm_tiles"])
@pytest.mark.parametrize("p", SMALL, ids=lambda p: f"T{p[0]}_H{p[1]}_F{p[2]}_E{p[3]}_k{p[4]}" + ("_skew" if p[6] else ""))
def test_backward_small(moe, p, path):
    """Pairs of SMs on 256 x 256 tiles where the tile is 256 wide (an expert
    with an odd number of 128-row tiles repeats its last one in the second
    CTA; an odd number of 128-row weight-gradient tiles keeps one-SM tiles),
    or one-SM tiles throughout."""
    T, H, F, E, k, seed, skew = p
    moe.moe_set_option(moe.OPT_PATH, path)
    case = moe_inputs.make_case(T, H, F, E, k, "bf16", seed, skew)
    dy = moe_inputs.make_dy(T, H, seed)
    out = run_bwd(moe, case, dy)
    ref = oracle.ffn_bwd64(*oracle_inputs(case, dy), k, round_h=True, round_inter=True, want_abs=True)
    for name in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        close(f64(out[name]), ref[name], ref[name + "_abs"], name, f"{name} T={T} H={H} F={F} E={E} k={k}")
    if skew:
        counts = np.bincount(oracle.route(case["logits"].numpy(), k)["ids"].reshape(-1), minlength=E)
        for e in np.flatnonzero(counts == 0):
            for name in ("dw1", "dw3", "dw2"):
                assert torch.count_nonzero(out[name][e]).item() == 0, (name, e)


def test_backward_no_tokens(moe):
    """T = 0: every weight gradient is zero (written, not left as it was)."""
    H, F, E, k = 128, 256, 4, 2
    case = moe_inputs.make_case(0, H, F, E, k, "bf16", 58)
    dev = "cuda"
    w1, w3, w2 = case["w1"].to(dev), case["w3"].to(dev), case["w2"].to(dev)
    out = {n: torch.full(s, 7.0, dtype=torch.bfloat16, device=dev)
           for n, s in (("dw1", (E, F, H)), ("dw3", (E, F, H)), ("dw2", (E, H, F)))}
    out["dx"] = torch.empty(0, H, dtype=torch.bfloat16, device=dev)
    out["dlogits"] = torch.empty(0, E, dtype=torch.float32, device=dev)
    x = torch.empty(0, H, dtype=torch.bfloat16, device=dev)
    lg = torch.empty(0, E, dtype=torch.float32, device=dev)
    moe.ffn_backward(x, lg, w1, w3, w2, x, k, out=out)
    torch.cuda.synchronize()
    for n in ("dw1", "dw3", "dw2"):
        assert torch.count_nonzero(out[n]).item() == 0, n


def test_backward_stale_workspace(moe):
    """The weight gradients sum over every slot of an expert, padding slots
    included: the backward writes those rows as zeros itself, so a workspace
    full of NaN patterns from earlier use changes nothing."""
    T, H, F, E, k = 37, 256, 512, 4, 2
    case = moe_inputs.make_case(T, H, F, E, k, "bf16", 60)
    dy = moe_inputs.make_dy(T, H, 60)
    dev = "cuda"
    x, lg = case["x"].to(dev), case["logits"].to(dev)
    w1, w3, w2 = case["w1"].to(dev), case["w3"].to(dev), case["w2"].to(dev)
    clean = moe.backward_workspace(T, H, F, E, k)
    clean.zero_()
    stale = moe.backward_workspace(T, H, F, E, k)
    stale.fill_(0xFF)  # bf16 and fp32 NaN bit patterns everywhere
    a = moe.ffn_backward(x, lg, w1, w3, w2, dy.to(dev), k, ws=clean)
    b = moe.ffn_backward(x, lg, w1, w3, w2, dy.to(dev), k, ws=stale)
    torch.cuda.synchronize()
    assert moe.moe_get_status(None) == 0
    for n in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        assert torch.equal(a[n], b[n]), n


def test_backward_full_size_sampled(moe):
    """The Mixtral expert shape at the training workload's size (T = 4096,
    d_model 4096, d_ff 14336, 8 experts, top-2), in the launch configuration
    the benchmark times: dx and dlogits of sampled tokens, rows of dW1/dW3
    and columns of dW2 of sampled (expert, feature) pairs, against the
    oracle's sampled form."""
    spec = moe_inputs.BWD_CONFIGS["train_prefill"]
    T, H, F, E, k = spec["T"], spec["H"], spec["F"], spec["E"], spec["k"]
    case = moe_inputs.make_case(T, H, F, E, k, "bf16", spec["seed"])
    dy = moe_inputs.make_dy(T, H, spec["seed"])
    out = run_bwd(moe, case, dy)
    tokens = np.array([0, 1, 1023, 2048, T - 1], dtype=np.int32)
    feats = np.array([[0, 0], [1, 7000], [3, F - 1], [5, 4097], [7, 128]], dtype=np.int32)
    ref = oracle.ffn_bwd64_sampled(*oracle_inputs(case, dy), k, tokens, feats, round_h=True, round_inter=True,
                                   want_abs=True)
    idx = torch.from_numpy(tokens).long()
    close(f64(out["dx"][idx]), ref["dx"], ref["dx_abs"], "dx", "dx (sampled tokens)")
    close(f64(out["dlogits"][idx]), ref["dlogits"], ref["dlogits_abs"], "dlogits", "dlogits (sampled tokens)")
    for q, (e, n) in enumerate(feats):
        close(f64(out["dw1"][e, n]), ref["dw1"][q], ref["dw1_abs"][q], "dw1", f"dw1[{e}, {n}, :]")
        close(f64(out["dw3"][e, n]), ref["dw3"][q], ref["dw3_abs"][q], "dw3", f"dw3[{e}, {n}, :]")
        close(f64(out["dw2"][e, :, n]), ref["dw2"][q], ref["dw2_abs"][q], "dw2", f"dw2[{e}, :, {n}]")


TRAIN = [
    # (T, H, F, E, k, seed, skew)
    (64, 256, 512, 8, 2, 61, False),
    (300, 256, 512, 8, 2, 62, True),      # big and empty experts
    (129, 384, 640, 4, 3, 63, False),     # 128-wide tiles
    (700, 256, 512, 4, 2, 64, False),
]


@pytest.mark.parametrize("path", [0, 3], ids=["pair_tiles", "one_sm_tiles"])
@pytest.mark.parametrize("p", TRAIN, ids=lambda p: f"T{p[0]}_H{p[1]}_F{p[2]}_E{p[3]}_k{p[4]}" + ("_skew" if p[6] else ""))
def test_training_pair(moe, p, path):
    """moe_ffn_forward_train: the BF16 layer from the row-major weights, held
    to the forward's own check (every output against the oracle, h flips
    validated); moe_ffn_backward_saved from what it kept: the backward's
    check against the oracle, and the same gradients as moe_ffn_backward."""
    from helpers import verify_layer
    T, H, F, E, k, seed, skew = p
    moe.moe_set_option(moe.OPT_PATH, path)
    case = moe_inputs.make_case(T, H, F, E, k, "bf16", seed, skew)
    dy = moe_inputs.make_dy(T, H, seed).cuda()
    x, lg = case["x"].cuda(), case["logits"].cuda()
    w1, w3, w2 = case["w1"].cuda(), case["w3"].cuda(), case["w2"].cuda()
    out, ws = moe.ffn_forward_train(x, lg, w1, w3, w2, k)
    torch.cuda.synchronize()
    assert moe.moe_get_status(None) == 0
    verify_layer(moe, ws, out, case, what=f"training forward T={T} F={F}")
    saved = moe.ffn_backward_saved(w1, w3, w2, dy, k, ws)
    again = moe.ffn_backward(x, lg, w1, w3, w2, dy, k)
    torch.cuda.synchronize()
    assert moe.moe_get_status(None) == 0
    ref = oracle.ffn_bwd64(*oracle_inputs(case, dy.cpu()), k, round_h=True, round_inter=True, want_abs=True)
    for name in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        close(f64(saved[name]), ref[name], ref[name + "_abs"], name, f"saved {name} T={T} F={F}")
        close(f64(again[name]), ref[name], ref[name + "_abs"], name, f"recomputed {name} T={T} F={F}")
    # the same g, u, h either way: the weight gradients without cross-tile
    # atomics match bit for bit
    for name in ("dw1", "dw3", "dw2"):
        assert torch.equal(saved[name], again[name]), name


def test_training_pair_in_a_cuda_graph(moe):
    """The training forward and the saved backward allocate nothing and
    synchronise nothing: a CUDA graph captured from them replays the same
    step, bit for bit on the outputs without cross-tile atomics."""
    T, H, F, E, k = 200, 256, 512, 8, 2
    case = moe_inputs.make_case(T, H, F, E, k, "bf16", 65)
    x, lg = case["x"].cuda(), case["logits"].cuda()
    w1, w3, w2 = case["w1"].cuda(), case["w3"].cuda(), case["w2"].cuda()
    dy = moe_inputs.make_dy(T, H, 65).cuda()
    out, ws = moe.ffn_forward_train(x, lg, w1, w3, w2, k)
    grads = moe.ffn_backward_saved(w1, w3, w2, dy, k, ws)
    torch.cuda.synchronize()
    eager = {n: v.clone() for n, v in grads.items()}
    eager_out = out.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        moe.ffn_forward_train(x, lg, w1, w3, w2, k, ws=ws, out=out, stream=s)  # warm up on the capture stream
        moe.ffn_backward_saved(w1, w3, w2, dy, k, ws, out=grads, stream=s)
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            moe.ffn_forward_train(x, lg, w1, w3, w2, k, ws=ws, out=out, stream=s)
            moe.ffn_backward_saved(w1, w3, w2, dy, k, ws, out=grads, stream=s)
    for v in list(grads.values()) + [out]:
        v.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_status(None) == 0
    assert torch.equal(out, eager_out)
    for n in ("dw1", "dw3", "dw2"):
        assert torch.equal(grads[n], eager[n]), n
    for n in ("dx", "dlogits"):
        torch.testing.assert_close(grads[n], eager[n], rtol=1e-6, atol=1e-6)
    del g


@pytest.mark.parametrize("table", [1, 3], ids=["slot_assign", "num_mtiles"])
@pytest.mark.parametrize("path", [0, 3], ids=["pair_tiles", "one_sm_tiles"])
def test_backward_catches_corrupted_routing(moe, table, path):
    """A routing-table entry far out of range (written on the host side of the
    call, after routing) is caught by the backward's kernels: the status word
    says MOE_ERR_DEVICE_BOUNDS, nothing faults, and the next call is correct."""
    T, H, F, E, k = 64, 256, 512, 8, 2
    case = moe_inputs.make_case(T, H, F, E, k, "bf16", 66)
    dy = moe_inputs.make_dy(T, H, 66)
    moe.moe_set_option(moe.OPT_PATH, path)
    x, lg = case["x"].cuda(), case["logits"].cuda()
    w1, w3, w2 = case["w1"].cuda(), case["w3"].cuda(), case["w2"].cuda()
    old = moe.moe_set_option(moe.OPT_TEST_CORRUPT, table)
    try:
        moe.ffn_backward(x, lg, w1, w3, w2, dy.cuda(), k)
        st = moe.moe_get_status(None)
        assert st == -7, f"expected MOE_ERR_DEVICE_BOUNDS, got {moe.STATUS_NAMES.get(st, st)}"
    finally:
        moe.moe_set_option(moe.OPT_TEST_CORRUPT, old)
    out = run_bwd(moe, case, dy)
    ref = oracle.ffn_bwd64(*oracle_inputs(case, dy), k, round_h=True, round_inter=True, want_abs=True)
    for name in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        close(f64(out[name]), ref[name], ref[name + "_abs"], name, f"{name} after a corrupted table {table}")
