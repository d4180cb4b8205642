"""Write the stored expected values under tests/golden/.

Calls only ``oracle`` (and the seeded input generator ``synth``); nothing here
comes from the CUDA path.  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import scores as osc          # noqa: E402
from oracle import select as osel         # noqa: E402
from synth import gen_score_case          # noqa: E402


def score_fp32():
    c = gen_score_case(0)
    q = c.q.reshape(c.S, c.H, c.D)
    k = c.k.reshape(c.S, c.H, c.D)
    sc = osc.block_scores_softmax_mass(q, k, c.blk)
    (idx, n, mask), mean = osel.select_mean_ge(sc.astype("float32"))
    return {
        "workload": "score_fp32 (S=512, 4 heads x 64, block 32, seed 0, 8 salient keys x4)",
        "definition": "Jenga summary 4.2.1 Eq. (1) with softmax probabilities, block-summed (4.2.3); "
                      "threshold = average block score (Algorithm 1, step 1)",
        "salient_rows": [int(v) for v in c.salient],
        "scores": [float(v) for v in sc],
        "mean": float(mean),
        "kept_blocks": [int(v) for v in idx[:n]],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "score_fp32_oracle.json"), "w") as f:
        json.dump(score_fp32(), f, indent=1)
    print("wrote", os.path.join(HERE, "score_fp32_oracle.json"))
