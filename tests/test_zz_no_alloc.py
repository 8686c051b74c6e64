"""moe_ffn_forward_static -- the layer for callers that cannot allocate device
memory (for example code running while a stream is captured into a CUDA graph)
-- against the ordinary entry point with a caller-allocated workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes on its own in a
fresh process as well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import check_close, small_case, to_device

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_static_workspace_matches_allocated_workspace(dtype):
    import mixture_experts_routed_02_b200 as moe
    T, H, F, E, k = 48, 512, 1024, 8, 2
    case = small_case(T, H, F, E, k, dtype, seed=31)
    d = to_device(case)
    dt = moe.dtype_code(dtype)
    assert moe.moe_workspace_size(T, H, F, E, k, dt) <= moe.moe_static_workspace_bytes()
    stream = torch.cuda.current_stream()
    ref = moe.ffn_forward(d["x"], d["logits"], d["w13"], d["s13"], d["w2p"], d["s2"], k, F, dtype == "fp8")
    assert moe.moe_get_status(None) == 0
    ref64 = ref.float().double().cpu().numpy()
    for call in range(2):  # two calls in a row share the built-in workspace
        out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = moe.moe_ffn_forward_static(_p(d["x"]), _p(d["logits"]), _p(d["w13"]), _p(d["s13"]), _p(d["w2p"]),
                                        _p(d["s2"]), T, H, F, E, k, dt, _p(out), ctypes.c_void_p(stream.cuda_stream))
        assert rc == 0, f"call {call}: {moe.STATUS_NAMES.get(rc, rc)}"
        assert moe.moe_get_status(None) == 0
        check_close(out.float().double().cpu().numpy(), ref64, f"static workspace, call {call}")


def test_static_workspace_rejects_oversized_problem():
    import mixture_experts_routed_02_b200 as moe
    T, H, F, E, k = 4096, 4096, 14336, 8, 2  # needs far more than the built-in buffer
    assert moe.moe_workspace_size(T, H, F, E, k, 1) > moe.moe_static_workspace_bytes()
    x = torch.zeros(16, dtype=torch.uint8, device="cuda")
    rc = moe.moe_ffn_forward_static(_p(x), _p(x), _p(x), _p(x), _p(x), _p(x), T, H, F, E, k, 1, _p(x), None)
    assert rc == -4  # MOE_ERR_WORKSPACE, nothing enqueued
    assert moe.moe_get_status(None) == 0


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_static_workspace_in_a_captured_graph(dtype):
    """Code under stream capture cannot allocate: the first call (outside the
    capture) looks up the built-in array, later calls are captured into a CUDA
    graph whose replays match the allocated-workspace output."""
    import mixture_experts_routed_02_b200 as moe
    T, H, F, E, k = 24, 256, 512, 8, 2
    case = small_case(T, H, F, E, k, dtype, seed=32)
    d = to_device(case)
    dt = moe.dtype_code(dtype)
    ref = moe.ffn_forward(d["x"], d["logits"], d["w13"], d["s13"], d["w2p"], d["s2"], k, F, dtype == "fp8")
    assert moe.moe_get_status(None) == 0
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()

    def call():
        return moe.moe_ffn_forward_static(_p(d["x"]), _p(d["logits"]), _p(d["w13"]), _p(d["s13"]), _p(d["w2p"]),
                                          _p(d["s2"]), T, H, F, E, k, dt, _p(out), ctypes.c_void_p(s.cuda_stream))

    with torch.cuda.stream(s):
        assert call() == 0  # first call in this context: outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        rc = call()
    assert rc == 0
    for _ in range(2):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_status(None) == 0
        check_close(out.float().double().cpu().numpy(), ref.float().double().cpu().numpy(), "captured static call")
