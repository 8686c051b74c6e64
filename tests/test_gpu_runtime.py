"""Runtime behaviour of the CUDA path: failure detection through the device
status word (a wait that runs out ends the kernel cleanly and leaves the
context usable; a routing-table index out of range is caught by the kernel
that reads it, which skips the access), capture of a layer call in a CUDA
graph, and run-to-run determinism."""
import numpy as np
import pytest
import torch

from helpers import run_layer, small_case, to_device, verify_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import mixture_experts_routed_02_b200 as m
    return m


PATHS = pytest.mark.parametrize("path", [2, 1, 3, 4], ids=["streaming_tiles", "pair_tiles", "wide_tiles", "tiny_tiles"])


@pytest.fixture(autouse=True)
def _reset_path(moe):
    yield
    moe.moe_set_option(moe.OPT_PATH, 0)


@PATHS
def test_stalled_wait_times_out_and_context_survives(moe, path):
    case = small_case(16 if path == 4 else 64, 256, 512, 8, 2, "fp8", 41)
    d = to_device(case)
    moe.moe_set_option(moe.OPT_PATH, path)
    old_t = moe.moe_set_option(moe.OPT_TIMEOUT_MS, 50)
    old_s = moe.moe_set_option(moe.OPT_TEST_STALL, 1)
    try:
        moe.ffn_forward(d["x"], d["logits"], d["w13"], d["s13"], d["w2p"], d["s2"], 2, 512, True)
        st = moe.moe_get_status(None)
        assert st == -6, f"expected MOE_ERR_DEVICE_TIMEOUT, got {moe.STATUS_NAMES.get(st, st)}"
        assert moe.moe_get_status(None) == 0  # reading clears the status word
    finally:
        moe.moe_set_option(moe.OPT_TEST_STALL, old_s)
        moe.moe_set_option(moe.OPT_TIMEOUT_MS, old_t)
    torch.cuda.synchronize()  # no sticky CUDA error: the kernel unwound by itself
    out, ws = run_layer(d)    # the next call is correct
    verify_layer(moe, ws, out, case, what="after a timed-out call")


@PATHS
@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_cuda_graph_capture_and_replay(moe, dtype, path):
    moe.moe_set_option(moe.OPT_PATH, path)
    T, H, F, E, k = (16 if path == 4 else 48), 256, 512, 8, 2
    case = small_case(T, H, F, E, k, dtype, 42)
    d = to_device(case)
    fp8 = dtype == "fp8"
    ws = moe.workspace(T, H, F, E, k, dtype)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):  # first call outside capture (one-time set-up)
        moe.ffn_forward(d["x"], d["logits"], d["w13"], d["s13"], d["w2p"], d["s2"], k, F, fp8, out=out, ws=ws)
    torch.cuda.synchronize()
    ref = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.ffn_forward(d["x"], d["logits"], d["w13"], d["s13"], d["w2p"], d["s2"], k, F, fp8, out=out, ws=ws)
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_status(None) == 0
    assert torch.equal(out, ref)
    # new inputs in the same buffers flow through the captured graph
    case2 = small_case(T, H, F, E, k, dtype, 43)
    d["x"].copy_(case2["x"].cuda())
    d["logits"].copy_(case2["logits"].cuda())
    g.replay()
    torch.cuda.synchronize()
    case2.update(w1=case["w1"], w3=case["w3"], w2=case["w2"], s1=case["s1"], s3=case["s3"], s2=case["s2"])
    verify_layer(moe, ws, out, case2, what="graph replay with new inputs")


def test_output_deterministic_without_k_splits(moe):
    case = small_case(200, 256, 512, 8, 2, "fp8", 44)
    d = to_device(case)
    outs = [run_layer(d)[0].clone() for _ in range(3)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


CORRUPT = pytest.mark.parametrize("table", [1, 2, 3], ids=["slot_assign", "mtile_expert", "num_mtiles"])


@CORRUPT
@PATHS
def test_corrupted_routing_index_is_caught(moe, table, path):
    """A routing-table entry far out of range (written on the host side of the
    call, after routing) is caught by the kernel that reads it: the status word
    says MOE_ERR_DEVICE_BOUNDS, nothing faults, and the next call is correct."""
    T = 16 if path == 4 else 64
    case = small_case(T, 256, 512, 8, 2, "fp8", 45)
    d = to_device(case)
    moe.moe_set_option(moe.OPT_PATH, path)
    old = moe.moe_set_option(moe.OPT_TEST_CORRUPT, table)
    try:
        moe.ffn_forward(d["x"], d["logits"], d["w13"], d["s13"], d["w2p"], d["s2"], 2, 512, True)
        st = moe.moe_get_status(None)
        assert st == -7, f"expected MOE_ERR_DEVICE_BOUNDS, got {moe.STATUS_NAMES.get(st, st)}"
    finally:
        moe.moe_set_option(moe.OPT_TEST_CORRUPT, old)
    torch.cuda.synchronize()
    out, ws = run_layer(d)
    verify_layer(moe, ws, out, case, what=f"after a corrupted table {table}")
