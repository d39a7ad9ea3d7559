"""Top-k recall of a reused page selection across the steps of a denoising block.

MAGE ("MAGE: All-[MASK] Block Already Knows Where to Look in Block Diffusion
LLM", Surprising findings) reports that the pages selected at the block's first
step keep a high recall of each later step's own top-k pages.  Step-dLLM's
variant refreshes the selection at anchor steps.  This module measures both on
the GPU path: every selection it needs is a dsa_select call (the exact top-k of
step t is the selection pass run with step t's queries); only the set
comparison happens on the host.

    recall(used, exact) = mean over (sequence, KV head) of |used ∩ exact| / |exact|
"""
from __future__ import annotations

import numpy as np

from . import dsa


def set_recall(used_idx, used_cnt, exact_idx, exact_cnt) -> float:
    """Mean over (sequence, KV head) of |used ∩ exact| / |exact| (1 where exact is empty).

    Index arrays are [S, Hkv, kmax] with the first cnt[s, h] entries valid."""
    used_idx, exact_idx = np.asarray(used_idx), np.asarray(exact_idx)
    used_cnt, exact_cnt = np.asarray(used_cnt), np.asarray(exact_cnt)
    vals = []
    for s in range(exact_idx.shape[0]):
        for h in range(exact_idx.shape[1]):
            e = set(exact_idx[s, h, :exact_cnt[s, h]].tolist())
            u = set(used_idx[s, h, :used_cnt[s, h]].tolist())
            vals.append(1.0 if not e else len(e & u) / len(e))
    return float(np.mean(vals))


def exact_selection(dw: "dsa.DeviceWorkload", q):
    """The selection pass run with queries q: (idx, cnt) copied to the host."""
    idx, cnt, _ = dw.select(q)
    return idx.cpu().numpy().copy(), cnt.cpu().numpy().copy()


def step_recall(dw: "dsa.DeviceWorkload", step_queries, anchor: int | None = None):
    """Recall at steps 1..T of the page set in use against each step's exact top-k.

    step_queries[t - 1] is the block's query tensor at step t (on the GPU).  With
    anchor=None the step-1 set is reused for every step (MAGE); with anchor=a the
    selection is refreshed at steps 1, 1 + a, 1 + 2a, ... and the latest refresh
    is in use.  Returns a list of T floats (step 1 first)."""
    exact = [exact_selection(dw, q) for q in step_queries]
    out = []
    used = exact[0]
    for t in range(1, len(step_queries) + 1):
        if anchor is not None and (t - 1) % anchor == 0:
            used = exact[t - 1]
        out.append(set_recall(used[0], used[1], exact[t - 1][0], exact[t - 1][1]))
    return out
