"""Measure the bf16 noise floor of the oracle and write noise_floor.json.

The max-abs relative error between two bf16 evaluations of a deep random
model is bounded below by how far the model moves when a few bf16 rounding
decisions go the other way.  This script moves 0.1% of the entries of every
layer matrix by one bf16 ulp (the kind of difference a different summation
order produces at a rounding point), re-runs the oracle, and records the
max-abs relative error and cosine of the logits against the unmoved run.
Calls only oracle/ and the seeded input generator.

    python tests/golden/make_noise_floor.py [out.json]     (the 9B shape needs ~70 GB of host memory)
"""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
sys.path.insert(0, os.path.dirname(HERE))

import oracle  # noqa: E402
import seeded  # noqa: E402
from seeded import workloads as W  # noqa: E402
from metrics import cosine, rel_err  # noqa: E402


def floor(model, seed, tokens, frac=1e-3):
    o = oracle.Model(oracle.make_config(**model), seed=seed)
    ref = o.prefill(tokens, all_positions=True)
    n_phys = model["n_prelude"] + model["n_block"] + model["n_coda"]
    rng = np.random.default_rng(0)
    ws = []
    for i in range(o.num_weights()):
        x = o.weight(i)
        is_matrix = 2 <= i < 2 + 10 * n_phys and (i - 2) % 10 not in (0, 6)
        if x.size and is_matrix:
            idx = np.flatnonzero(rng.random(x.size) < frac)
            x[idx] = seeded.to_bf16_f32(x[idx] * (1 + 2.0**-8 * np.sign(rng.random(idx.size) - 0.5)))
        ws.append(x)
    o.close()
    alt = oracle.Model(oracle.make_config(**model), weights=ws).prefill(tokens, all_positions=True)
    return {"rel": rel_err(alt, ref), "cos": cosine(alt, ref)}


def main():
    out = {"_source": "written by tests/golden/make_noise_floor.py (oracle only): logits of the oracle vs the "
                      "oracle with 0.1% of its layer-matrix entries moved by one bf16 ulp"}
    mid = dict(W.model_config("tiny_fp32", hidden=512, ffn=512, vocab=2048, n_q=4, n_kv=2, head_dim=128, n_lin=4,
                              lin_dim=128, dtype=1), max_batch=2, max_ctx=700)
    out["mid_b2_s700"] = floor(mid, 5, seeded.tokens(5, 2, 700, 2048))
    w = W.WORKLOADS["loop9b_prefill_b4_s8192"]
    m9 = dict(w["model"], max_batch=1, max_ctx=16)
    out["loop9b_prefix16"] = floor(m9, w["seed"], seeded.tokens(w["seed"], 4, 8192, m9["vocab"])[:1, :16])
    path = sys.argv[1] if len(sys.argv) > 1 else os.path.join(HERE, "noise_floor.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
