"""The d_ff-sharded layer on one GPU standing in for G ranks: every rank's
second GEMM adds its partial outputs into the combine rows of the rank that
owns each token (here all in this GPU's memory), signals every rank, and each
rank rounds its own rows once all G signals of the step have arrived.  Every
rank's layer call is enqueued before any rank's finalize, so no kernel ever
waits for one that has not run.  The sharded output equals the whole layer's
up to the order of the fp32 sums, over several steps that alternate two sets
of combine rows."""
import numpy as np
import pytest
import torch

from helpers import run_layer, small_case, to_device, verify_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    import mixture_experts_routed_02_b200 as m
    return m


CASES = [
    # (G, T, H, F, E, k, dtype, path)
    (2, 64, 256, 512, 8, 2, "fp8", 0),
    (4, 37, 256, 1024, 8, 2, "bf16", 0),
    (2, 300, 256, 512, 4, 2, "fp8", 1),   # CTA-pair tiles
    (3, 5, 128, 384, 4, 2, "fp8", 0),     # ragged: 2 tokens per rank, the last one 1
    (1, 16, 256, 512, 8, 2, "fp8", 0),
    (2, 1, 128, 256, 4, 1, "bf16", 0),    # rank 1 owns no token
]


@pytest.mark.parametrize("G,T,H,F,E,k,dtype,path", CASES,
                         ids=[f"G{c[0]}_T{c[1]}_F{c[3]}_{c[6]}_path{c[7]}" for c in CASES])
def test_dff_layer_matches_whole_layer(moe, G, T, H, F, E, k, dtype, path):
    moe.moe_set_option(moe.OPT_PATH, path)
    try:
        fp8 = dtype == "fp8"
        Fs = F // G
        base = small_case(T, H, F, E, k, dtype, seed=90 + G)
        whole = to_device(base)
        shards = []
        for r in range(G):
            w1, w3, s1, s3, w2 = moe.dff_shard(whole["w1"], whole["w3"], whole["s1"], whole["s3"], whole["w2"], G, r)
            shards.append(moe.prepare_weights(w1, w3, s1, s3, w2))
        per = -(-T // G)
        combine = [[torch.zeros(max(per, 1), H, dtype=torch.float32, device="cuda") for _ in range(G)]
                   for _ in range(2)]
        counters = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(G)]
        wss = [moe.workspace(T, H, Fs, E, k, dtype) for _ in range(G)]
        for step in range(1, 4):
            case = small_case(T, H, F, E, k, dtype, seed=100 * step + G)
            case.update({key: base[key] for key in ("w1", "w3", "w2", "s1", "s3", "s2")})
            x, lg = case["x"].cuda(), case["logits"].cuda()
            rows = combine[step % 2]
            for r in range(G):
                w13, s13, w2p = shards[r]
                moe.ffn_forward_dff(x, lg, w13, s13, w2p, whole["s2"], k, Fs, fp8, G, r, rows, counters, ws=wss[r])
            outs = []
            for r in range(G):
                first, n = moe.dff_rows(T, G, r)
                o = torch.empty(n, H, dtype=torch.bfloat16, device="cuda")
                moe.dff_finalize(rows[r][:n], o, counters[r], G * step)
                outs.append(o)
            st = moe.moe_get_status(None)
            assert st == 0, moe.STATUS_NAMES.get(st, st)
            got = torch.cat(outs).float().double().cpu().numpy()
            # the whole layer on the same inputs, itself checked against the oracle
            dcase = dict(whole, x=x, logits=lg)
            ref, ws = run_layer(dcase)
            verify_layer(moe, ws, ref, case, what=f"whole layer step {step}")
            refv = ref.float().double().cpu().numpy()
            rms = float(np.sqrt(np.mean(refv ** 2)))
            # fp32 sums in another order: at most a bf16 rounding step apart
            err = np.abs(got - refv)
            assert (err <= 2.0 ** -7 * np.abs(refv) + 1e-3 * rms).all(), (step, float(err.max()), rms)
            for r in range(G):  # finalize left the rows zero for the step after next
                assert not rows[r].any()
                assert int(counters[r].item()) == G * step
    finally:
        moe.moe_set_option(moe.OPT_PATH, 0)


def test_dff_finalize_wait_runs_out_and_context_survives(moe):
    """A rank whose peers never signal: its bounded wait runs out, the status
    word says MOE_ERR_DEVICE_TIMEOUT, its output is left unwritten, and the
    context stays usable."""
    H = 128
    rows = torch.ones(4, H, dtype=torch.float32, device="cuda")
    out = torch.zeros(4, H, dtype=torch.bfloat16, device="cuda")
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    old = moe.moe_set_option(moe.OPT_TIMEOUT_MS, 50)
    try:
        moe.dff_finalize(rows, out, counter, 2)  # nobody will ever add 2
        st = moe.moe_get_status(None)
        assert st == -6, moe.STATUS_NAMES.get(st, st)
    finally:
        moe.moe_set_option(moe.OPT_TIMEOUT_MS, old)
    assert not out.any() and bool((rows == 1).all())
    counter.fill_(2)
    moe.dff_finalize(rows, out, counter, 2)
    assert moe.moe_get_status(None) == 0
    assert bool((out.float() == 1).all()) and not rows.any()
