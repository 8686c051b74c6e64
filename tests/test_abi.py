"""The C ABI on the host (no GPU needed): the library loads, exports every
entry point include/moe.h declares, and rejects bad arguments before touching
the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:size_t|int|long long)\s+(moe_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def moe():
    import mixture_experts_routed_02_b200 as m
    return m


def test_exports_every_declared_symbol(moe):
    declared = _declared_functions()
    assert set(declared) >= {"moe_route", "moe_ffn_forward", "moe_workspace_size", "moe_prepare_weights",
                             "moe_get_status"}
    raw = ctypes.CDLL(moe.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert sorted(moe.EXPORTS) == declared


def test_workspace_layout(moe):
    for (T, H, F, E, k, dt) in [(64, 256, 512, 8, 2, 0), (16, 4096, 14336, 8, 2, 1), (4096, 4096, 14336, 8, 2, 1),
                                (8192, 4096, 14336, 8, 2, 0), (1, 128, 128, 1, 1, 1)]:
        total = moe.moe_workspace_size(T, H, F, E, k, dt)
        assert total > 0
        regions = sorted(moe.moe_workspace_region(T, H, F, E, k, dt, w) for w in moe.WS)
        end = 0
        for off, n in regions:
            assert off % 1024 == 0 and off >= end
            end = off + n
        assert end <= total
    # assignment-sized regions grow with T
    assert moe.moe_workspace_size(2000, 256, 512, 8, 2, 1) > moe.moe_workspace_size(1000, 256, 512, 8, 2, 1)


@pytest.mark.parametrize("T,H,F,E,k,dt", [(16, 4096, 14336, 8, 2, 1), (4096, 4096, 14336, 8, 2, 1),
                                          (300, 384, 640, 16, 3, 0), (1, 128, 128, 1, 1, 1)])
def test_workspace_region_sizes(moe, T, H, F, E, k, dt):
    """Each region has the size its description in moe.h gives: routing arrays
    of T*k ints, per-token e4m3 rows and scales (FP8 only), h in the padded
    layout of S = 128*(ceil(T*k/128) + E) rows with a row pitch of row bytes
    + 128, h's block scales as 512-byte chunks per (128-row tile, 128-column
    block) in FP8, the fp32 combine buffer [T, H]."""
    A = T * k
    eb = 1 if dt == 1 else 2
    mt_max = -(-A // 128) + E
    S = 128 * mt_max
    want = dict(topk_ids=4 * A, topk_w=4 * A, counts=4 * E, offsets=4 * (E + 1), perm=4 * A, inv_perm=4 * A,
                slot_of=4 * A, xs=T * H if dt == 1 else 0, sx=4 * T if dt == 1 else 0, h=S * (F * eb + 128),
                h_sf=mt_max * (F // 128) * 512 if dt == 1 else 0, out32=4 * T * H, num_mtiles=4,
                slot_assign=4 * S, mtile_expert=4 * mt_max, route_blocks=4 * (-(-T // 256)) * E,
                xg=S * (H * eb + 128), sx_slot=4 * S if dt == 1 else 0)
    assert set(want) == set(moe.WS)
    for name, n in want.items():
        off, size = moe.moe_workspace_region(T, H, F, E, k, dt, moe.WS[name])
        assert size == n, name


@pytest.mark.parametrize("args", [
    (16, 4096, 14336, 0, 2, 1),     # E = 0
    (16, 4096, 14336, 65, 2, 1),    # E > 64
    (16, 4096, 14336, 8, 0, 1),     # k = 0
    (16, 4096, 14336, 8, 9, 1),     # k > E
    (16, 4096, 14336, 8, 2, 7),     # unknown dtype
    (-1, 4096, 14336, 8, 2, 1),     # T < 0
])
def test_bad_dimensions(moe, args):
    assert moe.moe_workspace_size(*args) == 0
    T, H, F, E, k, dt = args
    rc = moe.moe_ffn_forward(None, None, None, None, None, None, T, H, F, E, k, dt, None, None, 0, None)
    assert rc == -1


def test_null_and_unsupported_before_device(moe):
    P = 4096  # a fake, 16-byte aligned address: never dereferenced on these paths
    # null weights
    assert moe.moe_ffn_forward(P, P, None, None, P, None, 4, 128, 128, 2, 1, 0, P, P, 1 << 40, None) == -1
    # FP8 without scales
    assert moe.moe_ffn_forward(P, P, P, None, P, None, 4, 128, 128, 2, 1, 1, P, P, 1 << 40, None) == -1
    # H not a multiple of 128
    assert moe.moe_ffn_forward(P, P, P, None, P, None, 4, 200, 128, 2, 1, 0, P, P, 1 << 40, None) == -2
    # too many assignments
    assert moe.moe_ffn_forward(P, P, P, None, P, None, 200000, 128, 128, 8, 2, 0, P, P, 1 << 40, None) == -2
    # misaligned pointer
    assert moe.moe_ffn_forward(P + 4, P, P, None, P, None, 4, 128, 128, 2, 1, 0, P, P, 1 << 40, None) == -3
    # workspace too small
    assert moe.moe_ffn_forward(P, P, P, None, P, None, 4, 128, 128, 2, 1, 0, P, P, 10, None) == -4
    # routing and preshuffle argument checks
    assert moe.moe_route(None, 4, 0, 1, None, None, None, None, None, None, None, 0, None) == -1
    assert moe.moe_route(P, 4, 8, 2, None, P, P, P, P, P, None, 0, None) == -1
    assert moe.moe_prepare_weights(None, P, None, None, P, P, None, P, 2, 128, 128, 0, None) == -1
    assert moe.moe_prepare_weights(P, P, None, None, None, P, None, P, 2, 128, 128, 0, None) == -1
    assert moe.moe_prepare_weights(P, P, None, None, P, P, None, P, 2, 128, 128, 1, None) == -1  # FP8 needs scales
    assert moe.moe_prepare_weights(P, P, None, None, P, P, None, P, 2, 100, 128, 0, None) == -2
    assert moe.moe_prepare_weights(P, P, None, None, P + 8, P, None, P, 2, 128, 128, 0, None) == -3


def test_options(moe):
    old = moe.moe_set_option(moe.OPT_PATH, 2)
    assert moe.moe_set_option(moe.OPT_PATH, old) == 2
    assert moe.moe_set_option(moe.OPT_PATH, 5) == -1
    old = moe.moe_set_option(moe.OPT_PATH, 4)
    # tiny-batch tiles are refused, before the device is touched, for more than 32 assignments
    P = 4096
    assert moe.moe_ffn_forward(P, P, P, None, P, None, 64, 128, 128, 8, 2, 0, P, P, 1 << 40, None) == -2
    moe.moe_set_option(moe.OPT_PATH, old)
    assert moe.moe_set_option(99, 0) == -1
    assert moe.moe_set_option(moe.OPT_TIMEOUT_MS, 0) == -1


def test_static_entry_checks_arguments_before_size(moe):
    """moe_ffn_forward_static applies moe_ffn_forward's checks first, in the
    same order, and only then compares the problem with its built-in
    workspace (nothing here touches the device)."""
    P = 4096
    big = (4096, 4096, 14336, 8, 2, 1)  # far more than the built-in workspace
    assert moe.moe_workspace_size(*big) > moe.moe_static_workspace_bytes()
    T, H, F, E, k, dt = big
    # null weights on an oversized problem: invalid argument, not workspace
    assert moe.moe_ffn_forward_static(P, P, None, P, P, P, T, H, F, E, k, dt, P, None) == -1
    # misaligned pointer on an oversized problem: alignment
    assert moe.moe_ffn_forward_static(P + 4, P, P, P, P, P, T, H, F, E, k, dt, P, None) == -3
    # unsupported shape
    assert moe.moe_ffn_forward_static(P, P, P, P, P, P, 4, 200, 128, 2, 1, 1, P, None) == -2
    # bad dimensions
    assert moe.moe_ffn_forward_static(P, P, P, P, P, P, 4, 128, 128, 0, 1, 1, P, None) == -1
    # valid arguments, oversized problem: workspace
    assert moe.moe_ffn_forward_static(P, P, P, P, P, P, T, H, F, E, k, dt, P, None) == -4


def test_static_workspace_holds_the_decode_layer(moe):
    """The built-in workspace (64 MiB) holds the Mixtral-shaped decode layer
    (T = 16) in every weight format; the header's figures for it are about
    22 MB in FP8 and 43 MB in BF16."""
    cap = moe.moe_static_workspace_bytes()
    assert cap == 64 << 20
    need = {d: moe.moe_workspace_size(16, 4096, 14336, 8, 2, moe.dtype_code(d)) for d in ("fp8", "bf16", "mxfp4")}
    assert all(n <= cap for n in need.values())
    assert round(need["fp8"] / 1e6) == 22 and round(need["bf16"] / 1e6) == 43


def test_test_hook_options_range(moe):
    assert moe.moe_set_option(moe.OPT_TEST_CORRUPT, 4) == -1
    assert moe.moe_set_option(moe.OPT_TEST_CORRUPT, -1) == -1
    assert moe.moe_set_option(moe.OPT_TEST_CORRUPT, 0) == 0
    assert moe.moe_set_option(moe.OPT_GATHER, 3) == -1
    assert moe.moe_set_option(moe.OPT_GATHER, 0) == 0
    assert moe.moe_set_option(6, 0) == -1  # no option 6


def test_dff_entry_checks_arguments(moe):
    """The d_ff-sharded entry points reject bad rank arguments and pointers
    before touching the device."""
    import ctypes
    P = 4096
    ptrs = lambda n, v=P: (ctypes.c_void_p * n)(*([v] * n))  # noqa: E731
    args = (P, P, P, P, P, P, 4, 128, 128, 2, 1, 1)
    assert moe.moe_ffn_forward_dff(*args, 0, 0, ptrs(1), ptrs(1), P, 1 << 40, None) == -1    # no ranks
    assert moe.moe_ffn_forward_dff(*args, 17, 0, ptrs(17), ptrs(17), P, 1 << 40, None) == -1  # > 16 ranks
    assert moe.moe_ffn_forward_dff(*args, 2, 2, ptrs(2), ptrs(2), P, 1 << 40, None) == -1    # rank >= n_ranks
    assert moe.moe_ffn_forward_dff(*args, 2, 0, None, ptrs(2), P, 1 << 40, None) == -1
    assert moe.moe_ffn_forward_dff(*args, 2, 0, ptrs(2, P + 8), ptrs(2), P, 1 << 40, None) == -3
    assert moe.moe_ffn_forward_dff(*args, 2, 0, ptrs(2), ptrs(2, P + 2), P, 1 << 40, None) == -3
    assert moe.moe_ffn_forward_dff(*args, 2, 0, ptrs(2), ptrs(2), P, 10, None) == -4          # workspace
    assert moe.moe_dff_finalize(P, P, 4, 100, P, 2, None) == -1                               # H % 128
    assert moe.moe_dff_finalize(P, P, 4, 128, None, 2, None) == -1
    assert moe.moe_dff_finalize(P + 4, P, 4, 128, P, 2, None) == -3


def test_backward_entry_checks(moe):
    """Unsupported shapes and misaligned pointers are refused before any launch."""
    assert moe.moe_backward_workspace_size(16, 4096, 14336, 8, 2) > 0
    assert moe.moe_backward_workspace_size(16, 4000, 14336, 8, 2) == 0   # d_model not a multiple of 128
    assert moe.moe_backward_workspace_size(16, 4096, 14336, 8, 9) == 0   # k > E
    P = 4096
    assert moe.moe_ffn_backward(P, P, P, P, P, P, 16, 4096, 14336, 8, 2, P, P, P, P, P, None, 0, None) == -1
    assert moe.moe_ffn_backward(P, P, P + 8, P, P, P, 16, 4096, 14336, 8, 2, P, P, P, P, P, P, 1 << 40,
                                None) == -3
    n = moe.moe_backward_workspace_size(16, 256, 512, 8, 2)
    assert moe.moe_ffn_backward(P, P, P, P, P, P, 16, 256, 512, 8, 2, P, P, P, P, P, P, n - 1, None) == -4


def test_training_entries_check_arguments(moe):
    """The training forward and the saved backward refuse bad shapes,
    pointers, alignment and a short workspace before any launch."""
    P = 4096
    n = moe.moe_backward_workspace_size(16, 256, 512, 8, 2)
    assert moe.moe_ffn_forward_train(P, P, P, P, P, 16, 4000, 512, 8, 2, P, P, n, None) == -1  # d_model
    assert moe.moe_ffn_forward_train(P, P, P, P, P, 16, 256, 512, 8, 2, None, P, n, None) == -1  # no output
    assert moe.moe_ffn_forward_train(P, P, P + 8, P, P, 16, 256, 512, 8, 2, P, P, n, None) == -3
    assert moe.moe_ffn_forward_train(P, P, P, P, P, 16, 256, 512, 8, 2, P, P, n - 1, None) == -4
    assert moe.moe_ffn_backward_saved(P, P, P, None, 16, 256, 512, 8, 2, P, P, P, P, P, P, n, None) == -1  # no dy
    assert moe.moe_ffn_backward_saved(P, P, P, P, 16, 256, 512, 8, 2, P + 4, P, P, P, P, P, n, None) == -3
    assert moe.moe_ffn_backward_saved(P, P, P, P, 16, 256, 512, 8, 2, P, P, P, P, P, P, n - 1, None) == -4
