"""Writes tests/golden/tiny_oracle.json and tests/golden/variants_oracle.json from the
fp64 oracle only.

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
    with open(os.path.join(ROOT, "tests", "golden", "variants_oracle.json"), "w") as f:
        json.dump(variants(), f, indent=1)


VARIANT_WORKLOAD = dict(n=300, topk=48, B=2, Hq=4, Hkv=2, d=32, needle_count=2)


def variants():
    """Head-adaptive budget and prefix-part reuse on a 2-head `tiny`-shaped workload:
    the shared-budget selection, then a step-2 call with every token active (its
    caches) and a step-3 call with token 1 stable (reusing them)."""
    w = W.make("tiny", 1, **VARIANT_WORKLOAD)
    args = (W.bits(w.q1), W.bits(w.k_cache), W.bits(w.v_cache), w.n_ctx.numpy(), w.topk.numpy())
    g = oracle.select_global(*args, kmax=w.max_pages)
    r = oracle.select(*args)
    import numpy as np
    zeros_o = np.zeros(W.bits(w.q1).shape, np.uint16)
    zeros_l = np.zeros(w.q1.shape[:3])
    q2, bk2, bv2 = w.step_inputs(2)
    o2, _, co2, cl2 = oracle.sparse_losa(W.bits(q2), W.bits(w.k_cache), W.bits(w.v_cache),
                                         w.n_ctx.numpy(), r.idx, r.cnt, W.bits(bk2), W.bits(bv2),
                                         np.ones((w.S, w.B), bool), zeros_o, zeros_l)
    import torch
    cache_bits = W.bits(torch.from_numpy(co2).to(torch.bfloat16))
    q3, bk3, bv3 = w.step_inputs(3)
    mask = np.array([[True, False]])
    o3, lse3, _, _ = oracle.sparse_losa(W.bits(q3), W.bits(w.k_cache), W.bits(w.v_cache),
                                        w.n_ctx.numpy(), r.idx, r.cnt, W.bits(bk3), W.bits(bv3),
                                        mask, cache_bits, cl2)
    return {
        "workload": "tiny", "seed": 1, "overrides": VARIANT_WORKLOAD,
        "source": "written by tests/golden/make_golden.py from the fp64 oracle",
        "global_idx": g.idx[0].tolist(), "global_cnt": g.cnt[0].tolist(),
        "losa_step2_o_row0": [float(x) for x in o2[0, 0, 0]],
        "losa_step2_cache_lse": [float(x) for x in cl2.reshape(-1)],
        "losa_step3_mask": mask.tolist(),
        "losa_step3_o": [float(x) for x in o3.reshape(-1)[:64]],
        "losa_step3_lse": [float(x) for x in lse3.reshape(-1)],
    }


if __name__ == "__main__":
    main()
