"""Writes tests/golden/tiny_oracle.json from the fp64 oracle only.

The pages print no worked example with numbers, so the stored values here are
the oracle's own output on the seeded `tiny` workload (seed 0), kept as a
regression fixture: a later change to the oracle's arithmetic that moves them
must say which passage or reading justifies it.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_attention_27_b200 import workloads as W  # noqa: E402


def main():
    w = W.make("tiny", 0)
    r = oracle.select(W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                      w.topk.numpy())
    q2, bk2, bv2 = w.step_inputs(2)
    o2, lse2 = oracle.sparse(W.bits(q2), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(),
                             r.idx, r.cnt, W.bits(bk2), W.bits(bv2))
    out = {
        "workload": "tiny", "seed": 0,
        "source": "written by tests/golden/make_golden.py from the fp64 oracle",
        "idx": r.idx[0, 0].tolist(),
        "cnt": int(r.cnt[0, 0]),
        "page_score": [float(x) for x in r.score[0, 0]],
        "select_o_row0": [float(x) for x in r.o[0, 0, 0]],
        "select_lse": [float(x) for x in r.lse.reshape(-1)],
        "step2_o_row0": [float(x) for x in o2[0, 0, 0]],
        "step2_lse": [float(x) for x in lse2.reshape(-1)],
    }
    with open(os.path.join(ROOT, "tests", "golden", "tiny_oracle.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
