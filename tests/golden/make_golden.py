"""Write tests/golden/tiny_oracle.npz from the CPU oracle only.

The fixture is a regression guard for the oracle: a tiny packed varlen case
(two sequences, ragged tails, GQA, band bias, sinks) with its lse, block
masses, kept sets and outputs.  Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from cross_model_attention_block_b200 import synth  # noqa: E402
from oracle import mapflow_oracle as orc  # noqa: E402

CASE = dict(lengths=[40, 23], Hs=3, Hr=4, Hkv=2, d=16, B=8, tau=0.9,
            band_bias=2.0, band_width=12, dtype="f32", seed=7)


def compute():
    w, x = synth.small_case(CASE["lengths"], CASE["Hs"], CASE["Hr"], CASE["Hkv"],
                            CASE["d"], CASE["B"], CASE["tau"], dtype=CASE["dtype"],
                            band_bias=CASE["band_bias"],
                            band_width=CASE["band_width"], seed=CASE["seed"])
    res, O = orc.run_layer(x.Q, x.K, x.V, x.W, w.lengths, w.Hkv, w.B, w.tau,
                           w.band_bias, w.band_width)
    out = {"O": O}
    for s, r in enumerate(res):
        for qb, rec in r.items():
            out[f"s{s}_qb{qb}_lse"] = rec["lse"]
            out[f"s{s}_qb{qb}_mass"] = rec["mass"]
            out[f"s{s}_qb{qb}_kept"] = rec["kept"]
    return out


if __name__ == "__main__":
    np.savez_compressed(os.path.join(HERE, "tiny_oracle.npz"), **compute())
    print("wrote", os.path.join(HERE, "tiny_oracle.npz"))
