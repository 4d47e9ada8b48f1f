"""Pins for the oracle's top-k row selection (C-13).

References independent of the oracle's code: planted one-step code updates
whose count per row is known by construction (so the scores, the order and
the tie-break are known), the threshold rule (C-10 / C-11) that top-k must
reduce to when k covers every candidate row, the scores restated with the
search-based E4M3 encoder, and the invariants of a top-k choice (no
unselected candidate outranks a selected one; ties go to the lower index).
"""

import numpy as np
import pytest

import oracle as O
from synthetic import gen

from test_oracle_codec import _brute_encode

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _planted(scores, K=16, seed=0):
    """Wq with 0.5 (code 0x30) everywhere, P with an exact one-code-up step at
    the first scores[n] positions of row n, s_W = 1."""
    N = len(scores)
    wq = np.full((N, K), 0x30, dtype=np.uint8)
    P = np.zeros((N, K), dtype=np.float32)
    step = np.float32(DEC[0x31] - DEC[0x30])  # exact in float32
    for n, s in enumerate(scores):
        P[n, :s] = step
    # an unselectable perturbation elsewhere: far below half a code step
    P[:, K - 1] += np.float32(1e-6) * (np.arange(N, dtype=np.float32) + 1)
    return wq, np.float32(1.0), P


@pytest.mark.parametrize("k,expect", [
    (0, []),
    (1, [1]),               # scores 5, 5, 5 at rows 1, 2, 5: the lowest index wins
    (2, [1, 2]),
    (3, [1, 2, 5]),
    (4, [0, 1, 2, 5]),
    (6, [0, 1, 2, 4, 5]),   # row 3 has no changing code: never selected
    (100, [0, 1, 2, 4, 5]),
])
def test_planted_scores_order_and_ties(k, expect):
    scores = [3, 5, 5, 0, 1, 5]
    wq, s_w, P = _planted(scores)
    wq2, P2, mask, cnt = O.proxy_select_topk(wq, s_w, P, k)
    assert cnt == len(expect)
    assert np.flatnonzero(mask).tolist() == expect
    for n, s in enumerate(scores):
        if n in expect:
            assert np.all(wq2[n, :s] == 0x31) and np.all(wq2[n, s:] == 0x30)
            assert np.all(P2[n].view(np.uint32) == 0)
        else:  # bit-identical code row and accumulated proxy
            assert np.array_equal(wq2[n], wq[n])
            assert np.array_equal(P2[n].view(np.uint32), P[n].view(np.uint32))


def _state(seed, N=48, K=64, p_std=3e-6):
    w = gen.normal_f32(seed, (N, K), 0.02)
    wq, s_w, _, _ = O.quantize(w)
    P = gen.normal_f32(seed + 1, (N, K), p_std)
    return wq, s_w, P


def test_k_covering_every_candidate_is_the_threshold_rule():
    wq, s_w, P = _state(11)
    a = O.proxy_select_topk(wq, s_w, P, wq.shape[0])
    b = O.proxy_select(wq, s_w, P)
    assert a[3] == b[3] > 0
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))


@pytest.mark.parametrize("seed,k", [(12, 1), (13, 5), (14, 17), (15, 40)])
def test_topk_invariants_against_restated_scores(seed, k):
    wq, s_w, P = _state(seed)
    wq2, P2, mask, cnt = O.proxy_select_topk(wq, s_w, P, k)
    # scores restated with the search-based encoder (C-10's c', value compare)
    w = DEC[wq].astype(np.float32)
    t = (w + (np.float32(s_w) * P).astype(np.float32)).astype(np.float32)
    cn = _brute_encode(t.ravel()).reshape(t.shape)
    changed = DEC[cn] != DEC[wq]
    score = changed.sum(axis=1)
    cand = score > 0
    assert 0 < cand.sum(), "data should have candidate rows"
    sel = mask.astype(bool)
    assert cnt == sel.sum() == min(k, cand.sum())
    assert not np.any(sel & ~cand)
    # no unselected candidate outranks a selected row; equal scores: lower index first
    for a in np.flatnonzero(sel):
        for b in np.flatnonzero(cand & ~sel):
            assert score[a] > score[b] or (score[a] == score[b] and a < b)
    # selected rows as in C-11, the others untouched
    expect = np.where(changed, cn, wq)
    assert np.array_equal(wq2[sel], expect[sel])
    assert np.array_equal(wq2[~sel], wq[~sel])
    assert np.all(P2[sel].view(np.uint32) == 0)
    assert np.array_equal(P2[~sel].view(np.uint32), P[~sel].view(np.uint32))


def test_update_topk_composes_accumulate_then_select():
    w = gen.normal_f32(21, (24, 48), 0.02)
    wq, s_w, _, _ = O.quantize(w)
    P = gen.normal_f32(22, (24, 48), 1e-4)
    dB = gen.normal_bf16_bits(23, (24, 8), 1e-2)
    A = gen.normal_bf16_bits(24, (8, 48), 1e-2)
    a = O.proxy_update_topk(wq, s_w, P, dB, A, 7)
    b = O.proxy_select_topk(wq, s_w, O.proxy_accumulate(P, dB, A), 7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[3] == b[3]
