"""The comparison rules of tests/parity.py, on hand-made results (CPU): what the
tie window lets through and what it must not."""
from types import SimpleNamespace

import numpy as np
import pytest

import parity


def _orc_global(scores, kp):
    """Oracle-like result of the head-adaptive rule on [Hkv, np] scores, one sequence."""
    Hkv, np_ = scores.shape
    flat = scores.reshape(-1)
    order = np.lexsort((np.arange(flat.size), -flat))[:Hkv * kp]
    idx = np.full((1, Hkv, np_), -1, np.int32)
    cnt = np.zeros((1, Hkv), np.int32)
    for h in range(Hkv):
        pages = sorted(int(i) % np_ for i in order if int(i) // np_ == h)
        idx[0, h, :len(pages)] = pages
        cnt[0, h] = len(pages)
    return SimpleNamespace(idx=idx, cnt=cnt, score=scores[None].astype(np.float64))


def _gpu(sets, np_):
    Hkv = len(sets)
    idx = np.full((1, Hkv, np_), -1, np.int32)
    cnt = np.zeros((1, Hkv), np.int32)
    for h, pages in enumerate(sets):
        idx[0, h, :len(pages)] = sorted(pages)
        cnt[0, h] = len(pages)
    return idx, cnt


def test_global_exact_match_passes():
    sc = np.array([[0.5, 0.2, 0.1, 0.05], [0.3, 0.25, 0.01, 0.02]])
    orc = _orc_global(sc, 2)            # budget 4: (0,0) (1,0) (1,1) (0,1)
    idx, cnt = _gpu([[0, 1], [0, 1]], 4)
    assert parity.check_global_selection(idx, cnt, orc, [4], [2]) == 0


def test_global_swap_outside_window_fails():
    sc = np.array([[0.5, 0.2, 0.1, 0.05], [0.3, 0.25, 0.01, 0.02]])
    orc = _orc_global(sc, 2)
    idx, cnt = _gpu([[0, 2], [0, 1]], 4)  # (0,2) instead of (0,1): 0.1 vs 0.2, far apart
    with pytest.raises(AssertionError):
        parity.check_global_selection(idx, cnt, orc, [4], [2])


def test_global_swap_inside_window_passes():
    # the 4th and 5th best pairs, (0, 2) and (1, 1), differ by 1e-7 relative: the
    # oracle keeps (0, 2) (the lower head), the other choice is accepted too
    sc = np.array([[0.5, 0.2, 0.1, 0.05], [0.3, 0.1 * (1 - 1e-7), 0.01, 0.02]])
    orc = _orc_global(sc, 2)
    assert orc.idx[0, 0, :orc.cnt[0, 0]].tolist() == [0, 1, 2]
    idx, cnt = _gpu([[0, 1], [0, 1]], 4)
    assert parity.check_global_selection(idx, cnt, orc, [4], [2]) == 1


def test_global_wrong_count_fails():
    sc = np.array([[0.5, 0.2, 0.1, 0.05], [0.3, 0.25, 0.01, 0.02]])
    orc = _orc_global(sc, 2)
    idx, cnt = _gpu([[0, 1], [0, 1, 2]], 4)
    with pytest.raises(AssertionError):
        parity.check_global_selection(idx, cnt, orc, [4], [2])


def test_per_head_window_rule():
    """check_selection: a tie at the cut may go either way, a clear miss may not."""
    sc = np.array([[[0.4, 0.3, 0.3 * (1 - 1e-7), 0.0]]])  # [S=1, Hkv=1, np=4]
    orc = SimpleNamespace(idx=np.array([[[0, 1, -1, -1]]], np.int32), cnt=np.array([[2]], np.int32),
                          score=sc)
    ok_idx, ok_cnt = np.array([[[0, 2, -1, -1]]], np.int32), np.array([[2]], np.int32)
    assert parity.check_selection(ok_idx, ok_cnt, orc, [4], [2]) == 1
    bad_idx = np.array([[[0, 3, -1, -1]]], np.int32)
    with pytest.raises(AssertionError):
        parity.check_selection(bad_idx, ok_cnt, orc, [4], [2])
