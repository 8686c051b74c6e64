"""Writes tests/golden/tiny_routing_and_rows.json from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
The pages print no worked example for the routed MoE layer, so this fixture is
a regression record of the oracle on the tiny workload (T=64, d_model=256,
d_ff=512, E=8, top-2, bf16, seed 0): top-2 ids, expert counts, the stable
permutation, and the bf16 output bits of four tokens.  It pins nothing against
the pages; the pins are in tests/test_oracle.py.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs  # noqa: E402
import oracle  # noqa: E402

TOKENS = [0, 1, 31, 63]


def compute():
    nc = moe_inputs.to_numpy(moe_inputs.make_config("tiny"))
    r = oracle.route(nc["logits"], nc["k"])
    rows = oracle.moe_ffn_tokens(nc, TOKENS)
    return {
        "workload": "tiny: T=64, d_model=256, d_ff=512, E=8, top-2, bf16, seed 0",
        "topk_ids": r["ids"].tolist(),
        "counts": r["counts"].tolist(),
        "perm": r["perm"].tolist(),
        "tokens": TOKENS,
        "out_bits": rows["out"].tolist(),
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_routing_and_rows.json")
    with open(path, "w") as f:
        json.dump(compute(), f)
    print("wrote", path)
