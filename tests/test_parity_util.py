"""The GPU parity comparator on CPU: a selection that differs from the oracle's only on a
near-tie token is accepted, counted and reported; any other difference, or a permutation that
is not the one of the compared selection, fails."""
import numpy as np
import pytest

import oracle
import parity_util
from parity_util import compare_routing


def _case():
    # 6 tokens, 5 experts, top-2; token 3 has an exact tie between experts 1 and 2 for its
    # second slot (gap 0), every other token is well separated
    E, k = 5, 2
    lg = np.array([[5.0, 1.0, 0.0, -1.0, -2.0],
                   [0.0, 4.0, 3.0, 1.0, -1.0],
                   [1.0, 0.0, 0.0, 6.0, 2.0],
                   [3.0, 2.0, 2.0, 0.0, -1.0],
                   [-1.0, 0.0, 2.0, 1.0, 5.0],
                   [2.0, 3.0, 1.0, 0.0, 4.0]])
    idx = oracle.topk_select(lg, k)
    gk, gi = oracle.selection_gaps(lg, k)
    perm, inv = oracle.permutation(idx, E)
    cnt = oracle.expert_histogram(idx, E)
    r = dict(logits=lg, idx=idx, w=oracle.routing_weights(lg, idx), count=cnt,
             offsets=oracle.expert_offsets(cnt), perm=perm, inv_perm=inv, gap_k=gk, gap_in=gi)
    return r, E, k


def _gpu_from(idx, w, E):
    perm, inv = oracle.permutation(idx, E)
    return dict(topk_idx=idx.copy(), topk_w=w.copy(),
                expert_offsets=oracle.expert_offsets(oracle.expert_histogram(idx, E)),
                perm=perm, inv_perm=inv)


def test_identical_selection_passes_and_is_reported():
    r, E, k = _case()
    n0 = len(parity_util.NEAR_TIE_REPORTS)
    rep = compare_routing(_gpu_from(r["idx"], r["w"], E), r, k, E)
    assert rep["mismatched"] == 0 and rep["near_set"] == 1
    assert len(parity_util.NEAR_TIE_REPORTS) == n0 + 1
    assert parity_util.NEAR_TIE_REPORTS[-1]["near_set"] == 1


def test_near_tie_token_may_select_the_other_expert():
    r, E, k = _case()
    idx = r["idx"].copy()
    assert idx[3].tolist() == [0, 1]
    idx[3] = [0, 2]                               # the tied expert with the higher index
    rep = compare_routing(_gpu_from(idx, r["w"], E), r, k, E)
    assert rep["mismatched"] == 1 and rep["set_changed"] == [3]


def test_a_separated_token_may_not_differ():
    r, E, k = _case()
    idx = r["idx"].copy()
    idx[0] = [0, 2]                               # gap 1.0 between the 2nd and 3rd logit
    with pytest.raises(AssertionError):
        compare_routing(_gpu_from(idx, r["w"], E), r, k, E)


def test_permutation_must_be_the_selection_s_own():
    r, E, k = _case()
    g = _gpu_from(r["idx"], r["w"], E)
    a, b = g["expert_offsets"][1], g["expert_offsets"][2]
    assert b - a >= 2
    g["perm"][a:b] = g["perm"][a:b][::-1]         # same rows, not ascending in the segment
    with pytest.raises(AssertionError):
        compare_routing(g, r, k, E)


def test_weights_outside_tolerance_fail():
    r, E, k = _case()
    w = r["w"].copy()
    w[5, 0] += 1e-3
    w[5, 1] -= 1e-3
    with pytest.raises(AssertionError):
        compare_routing(_gpu_from(r["idx"], w, E), r, k, E)
