"""Pins for the oracle's top-k selection over the r rank components (C-13).

References independent of the function under test:
  - the accumulation restated as numpy's float32 add of the transposed
    increment;
  - the score against the largest element of the component's outer product,
    formed in full in float64 (not the factored max * max);
  - planted components whose scores, order and ties are known by
    construction, and whose merged codes are known exactly (power-of-two
    operands, so every product and sum is exact);
  - the merge of a set S against the separately pinned threshold path
    (C-9 chain from a zero proxy, then C-10 / C-11) run on the sub-matrices
    Q[S], A[S]: with S every component this is the full r-term update.
"""

import numpy as np
import pytest

import oracle as O
from synthetic import gen

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _bf16(x):
    return gen.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _state(seed, N=40, K=48, r=12, q_std=2e-3, bf16_q=True):
    """Backbone codes of W ~ N(0, 0.02), a proxy Q [r, N] (bfloat16-valued when
    bf16_q, so the threshold path can take it as its increment) and A."""
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed, (N, K), 0.02))
    Q = gen.normal_f32(seed + 1, (r, N), q_std)
    if bf16_q:
        Q = gen.bf16_bits_to_f32(_bf16(Q)).reshape(r, N)
    A = gen.normal_bf16_bits(seed + 2, (r, K), 0.01)
    return wq, s_w, Q, A


def _threshold_merge(wq, s_w, Q, A, S):
    """C-9 chain of Q[S]^T A[S] from a zero proxy, then C-10 / C-11."""
    N, K = wq.shape
    if len(S) == 0:
        return wq.copy()
    D = O.proxy_accumulate(np.zeros((N, K), np.float32), _bf16(Q[S].T.copy()), A[S].copy())
    return O.proxy_select(wq, s_w, D)[0]


def test_accumulate_only_is_a_float32_add():
    wq, s_w, Q, A = _state(1, bf16_q=False)
    N, r = wq.shape[0], A.shape[0]
    dB = gen.normal_bf16_bits(9, (N, r), 1e-3)
    wq2, Q2, mask, cnt, st = O.proxy_update_topk(wq, s_w, Q, dB, A, k=5, accumulate=True, select=False)
    expect = (Q + gen.bf16_bits_to_f32(dB).reshape(N, r).T).astype(np.float32)
    assert np.array_equal(Q2.view(np.uint32), expect.view(np.uint32))
    assert np.array_equal(wq2, wq) and cnt == 0 and not mask.any() and st == 0


def test_scores_are_the_largest_element_of_each_outer_product():
    _, _, Q, A = _state(2, bf16_q=False)
    sc, st = O.proxy_topk_scores(Q, A)
    Af = gen.bf16_bits_to_f32(A).reshape(A.shape).astype(np.float64)
    brute = np.array([np.abs(np.outer(Q[i].astype(np.float64), Af[i])).max() for i in range(Q.shape[0])])
    assert st == 0
    assert np.array_equal(sc, brute)


def _planted(levels, N=16, K=32):
    """Wq = 0.5 everywhere (code 0x30, one step up is 0x31 = 0.5625), s_W = 1.
    Component i has Q[i, :] = levels[i] and A[i, :] = 1, so its score is
    levels[i] and its whole update is levels[i] on every weight."""
    r = len(levels)
    wq = np.full((N, K), 0x30, dtype=np.uint8)
    Q = np.zeros((r, N), dtype=np.float32)
    for i, v in enumerate(levels):
        Q[i, :] = v
    A = _bf16(np.ones((r, K), np.float32))
    return wq, np.float32(1.0), Q, A


@pytest.mark.parametrize("k,expect", [
    (0, []),
    (1, [1]),             # 1/16 at components 1, 3 and 6: the lowest index wins
    (2, [1, 3]),
    (3, [1, 3, 6]),
    (4, [0, 1, 3, 6]),
    (6, [0, 1, 3, 5, 6]),  # component 2 (and 4) score 0: never selected
    (100, [0, 1, 3, 5, 6]),
])
def test_planted_order_ties_and_zero_scores(k, expect):
    step = np.float32(DEC[0x31] - DEC[0x30])  # 1/16
    levels = [step / 4, step, 0.0, step, 0.0, step / 8, step]
    wq, s_w, Q, A = _planted(levels)
    wq2, Q2, mask, cnt, st = O.proxy_update_topk(wq, s_w, Q, None, A, k, accumulate=False)
    assert st == 0 and cnt == len(expect)
    assert np.flatnonzero(mask).tolist() == expect
    merged = sum(levels[i] for i in expect)  # exact: sums of 2^-4, 2^-6, 2^-7
    # 0.5 + merged rounds to the nearest E4M3 value (spacing 1/16 in [0.5, 1))
    want = O.e4m3_encode(np.float32(0.5 + merged))
    assert np.all(wq2 == (want if DEC[want] != 0.5 else 0x30))
    for i in range(len(levels)):
        if i in expect:
            assert np.all(Q2[i].view(np.uint32) == 0)
        else:
            assert np.array_equal(Q2[i].view(np.uint32), Q[i].view(np.uint32))


def test_planted_dominant_component_moves_known_codes():
    """One component carries +3/16 on row 2, columns 5..9 (A = 1 there, 0
    elsewhere); the others are tiny.  k = 1 merges it: exactly those codes go
    from 0.5 to 0.6875 (0x33), nothing else moves."""
    wq, s_w, _, _ = _planted([0.0] * 4)
    N, K = wq.shape
    Q = np.full((4, N), np.float32(2.0 ** -12), dtype=np.float32)
    Q[2, 2] = np.float32(3.0 / 16.0)
    A = np.zeros((4, K), np.float32)
    A[:, :] = 2.0 ** -3
    A[2, :] = 0.0
    A[2, 5:10] = 1.0
    A = _bf16(A)
    wq2, Q2, mask, cnt, st = O.proxy_update_topk(wq, s_w, Q, None, A, 1, accumulate=False)
    assert np.flatnonzero(mask).tolist() == [2] and cnt == 1
    expect = wq.copy()
    expect[2, 5:10] = 0x33
    assert np.array_equal(wq2, expect)
    assert np.all(Q2[2].view(np.uint32) == 0)
    assert np.array_equal(np.delete(Q2, 2, 0).view(np.uint32), np.delete(Q, 2, 0).view(np.uint32))


@pytest.mark.parametrize("seed", [3, 4, 5])
def test_merging_every_component_is_the_full_threshold_update(seed):
    wq, s_w, Q, A = _state(seed)
    r = A.shape[0]
    wq2, Q2, mask, cnt, st = O.proxy_update_topk(wq, s_w, Q, None, A, r, accumulate=False)
    assert cnt == r and mask.all() and st == 0
    ref = _threshold_merge(wq, s_w, Q, A, list(range(r)))
    assert np.array_equal(wq2, ref)
    assert (wq2 != wq).any(), "the update should move some codes"
    assert np.all(Q2.view(np.uint32) == 0)


@pytest.mark.parametrize("seed,k", [(6, 1), (7, 3), (8, 7), (9, 11)])
def test_merging_k_components_is_the_threshold_update_of_their_subset(seed, k):
    wq, s_w, Q, A = _state(seed, q_std=2e-2)
    wq2, Q2, mask, cnt, st = O.proxy_update_topk(wq, s_w, Q, None, A, k, accumulate=False)
    S = np.flatnonzero(mask).tolist()
    assert cnt == len(S) == k
    # the chosen set is the top k of the outer-product maxima, ties to the lower index
    Af = gen.bf16_bits_to_f32(A).reshape(A.shape).astype(np.float64)
    brute = np.array([np.abs(np.outer(Q[i].astype(np.float64), Af[i])).max() for i in range(Q.shape[0])])
    order = sorted(range(len(brute)), key=lambda i: (-brute[i], i))
    assert S == sorted(order[:k])
    assert np.array_equal(wq2, _threshold_merge(wq, s_w, Q, A, S))
    rest = [i for i in range(Q.shape[0]) if i not in S]
    assert np.array_equal(Q2[rest].view(np.uint32), Q[rest].view(np.uint32))
    assert np.all(Q2[S].view(np.uint32) == 0)


def test_accumulate_then_select_composes():
    wq, s_w, Q, A = _state(10, bf16_q=False)
    N, r = wq.shape[0], A.shape[0]
    dB = gen.normal_bf16_bits(11, (N, r), 1e-2)
    a = O.proxy_update_topk(wq, s_w, Q, dB, A, 4)
    q1 = O.proxy_update_topk(wq, s_w, Q, dB, A, 0, select=False)[1]
    b = O.proxy_update_topk(wq, s_w, q1, None, A, 4, accumulate=False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))
    assert np.array_equal(a[2], b[2]) and a[3] == b[3] == 4


def test_zero_proxy_merges_nothing():
    wq, s_w, Q, A = _state(12)
    Z = np.zeros_like(Q)
    wq2, Q2, mask, cnt, st = O.proxy_update_topk(wq, s_w, Z, None, A, Q.shape[0], accumulate=False)
    assert cnt == 0 and not mask.any() and np.array_equal(wq2, wq) and st == 0


def test_nonfinite_component_ranks_first_and_sets_status():
    wq, s_w, Q, A = _state(13)
    Q = Q.copy()
    Q[7, 3] = np.inf
    sc, st = O.proxy_topk_scores(Q, A)
    assert st == O.STATUS_NONFINITE and np.isinf(sc[7]) and np.isfinite(np.delete(sc, 7)).all()
    _, _, mask, cnt, st2 = O.proxy_update_topk(wq, s_w, Q, None, A, 1, accumulate=False)
    assert np.flatnonzero(mask).tolist() == [7] and st2 == O.STATUS_NONFINITE
