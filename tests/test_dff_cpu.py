"""The d_ff-sharded layer's host logic on CPU, two gloo ranks: each rank slices
its d_ff shard of the expert weights with the library's helper, evaluates the
oracle on its slice (the unrounded per-token sums), and the sum over ranks
(the reduce-scatter's arithmetic) equals the oracle's whole layer -- the
sharding splits d_ff at multiples of 128, so the FP8 blocks of 32 channels of
h never straddle two shards and every shard rounds h as the whole layer does.
Token ownership covers every token exactly once."""
import datetime
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, dtype, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    for p in (ROOT, os.path.join(ROOT, "tests")):
        sys.path.insert(0, p)
    import moe_inputs
    import oracle
    import mixture_experts_routed_02_b200 as moe
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, H, F, E, k = 12, 128, 512, 4, 2
        case = moe_inputs.make_case(T, H, F, E, k, dtype, seed=81)
        w1, w3, s1, s3, w2 = moe.dff_shard(case["w1"], case["w3"], case["s1"], case["s3"], case["w2"], world, rank)
        shard = dict(case, w1=w1, w3=w3, s1=s1, s3=s3, w2=w2)
        tokens = np.arange(T, dtype=np.int32)
        part = oracle.moe_ffn_tokens(moe_inputs.to_numpy(shard), tokens)["out64"]
        tot = torch.from_numpy(part.copy())
        dist.all_reduce(tot)  # the reduce-scatter's sums (here: every row everywhere)
        first, n = moe.dff_rows(T, world, rank)
        owned = torch.tensor([first, n], dtype=torch.int64)
        all_owned = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(all_owned, owned)
        if rank == 0:
            full = oracle.moe_ffn_tokens(moe_inputs.to_numpy(case), tokens)["out64"]
            q.put(("sum", float(np.abs(tot.numpy() - full).max()), float(np.abs(full).max())))
            q.put(("rows", [tuple(int(v) for v in o) for o in all_owned]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
def test_dff_shards_sum_to_the_whole_layer(dtype):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + (7 if dtype == "fp8" else 0)) % 900
    procs = [ctx.Process(target=_worker, args=(r, 2, port, dtype, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = dict((item[0], item[1:]) for item in (q.get(timeout=5), q.get(timeout=5)))
    err, scale = res["sum"]
    assert err <= 1e-12 * scale, (err, scale)
    rows = res["rows"][0]
    assert rows == [(0, 6), (6, 6)]


def test_dff_rows_cover_every_token_once():
    import mixture_experts_routed_02_b200 as moe
    for T in (0, 1, 5, 16, 37, 4096):
        for G in (1, 2, 3, 4, 8, 16):
            seen = []
            for r in range(G):
                first, n = moe.dff_rows(T, G, r)
                seen += list(range(first, first + n))
                assert n <= -(-T // G) if T else n == 0
            assert seen == list(range(T)), (T, G)


def test_dff_shard_slices():
    import moe_inputs
    import mixture_experts_routed_02_b200 as moe
    case = moe_inputs.make_case(4, 128, 512, 3, 2, "fp8", seed=82)
    parts = [moe.dff_shard(case["w1"], case["w3"], case["s1"], case["s3"], case["w2"], 4, r) for r in range(4)]
    assert all(p[0].shape == (3, 128, 128) and p[4].shape == (3, 128, 128) for p in parts)
    cat = lambda i, dim: torch.cat([p[i].view(torch.uint8) if p[i].dtype == torch.float8_e4m3fn else p[i]  # noqa: E731
                                    for p in parts], dim=dim)
    assert torch.equal(cat(0, 1), case["w1"].view(torch.uint8))
    assert torch.equal(cat(1, 1), case["w3"].view(torch.uint8))
    assert torch.equal(cat(2, 1), case["s1"]) and torch.equal(cat(3, 1), case["s3"])
    assert torch.equal(cat(4, 2), case["w2"].view(torch.uint8))
    with pytest.raises(ValueError):
        moe.dff_shard(case["w1"], case["w3"], case["s1"], case["s3"], case["w2"], 3, 0)  # 512/3 is no shard
