"""Pins for the oracle's residual-keeping clear (C-14, error feedback).

References independent of the oracle's code: a planted update of 1.25 code
steps whose residual (a quarter step) is exact; conservation of the decoded
weight plus its proxy (nothing of the accumulated update is dropped); the
codes of C-11, which C-14 must leave unchanged; and bit-identical rows and
unchanged codes."""

import numpy as np
import pytest

import oracle as O
from synthetic import gen

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _state(seed, N=40, K=96, p_std=3e-6):
    wq, s_w, _, _ = O.quantize(gen.normal_f32(seed, (N, K), 0.02))
    P = gen.normal_f32(seed + 1, (N, K), p_std)
    return wq, s_w, P


def test_planted_quarter_step_residual_is_exact():
    N, K = 4, 16
    wq = np.full((N, K), 0x30, dtype=np.uint8)          # 0.5
    P = np.zeros((N, K), dtype=np.float32)
    step = np.float32(DEC[0x31] - DEC[0x30])              # 0.0625
    P[2, 5] = np.float32(1.25) * step                     # rounds to one step up
    P[2, 9] = np.float32(0.25) * step                     # below half a step: no change
    wq2, P2, mask, cnt = O.proxy_select_residual(wq, np.float32(1.0), P)
    assert cnt == 1 and mask.tolist() == [0, 0, 1, 0]
    assert wq2[2, 5] == 0x31 and np.all(np.delete(wq2[2], 5) == 0x30)
    assert P2[2, 5] == np.float32(0.25) * step            # the unapplied quarter step
    assert P2[2, 9] == P[2, 9]                            # unchanged code keeps its proxy
    assert np.array_equal(P2[[0, 1, 3]], P[[0, 1, 3]])


def test_codes_equal_the_clearing_rule_and_nothing_is_dropped():
    wq, s_w, P = _state(31)
    a = O.proxy_select_residual(wq, s_w, P)
    b = O.proxy_select(wq, s_w, P)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2]) and a[3] == b[3] > 0
    # decoded weight + scaled proxy is conserved per element, up to the two roundings
    before = DEC[wq] + np.float64(s_w) * P.astype(np.float64)
    after = DEC[a[0]] + np.float64(s_w) * a[1].astype(np.float64)
    scale = np.abs(DEC[wq]) + np.abs(np.float64(s_w) * P.astype(np.float64)) + 1e-30
    assert np.all(np.abs(after - before) <= 2.0 ** -22 * scale)
    # a clearing rule loses exactly what this one keeps
    lost = np.abs(DEC[b[0]] + np.float64(s_w) * b[1].astype(np.float64) - before)
    assert lost.max() > 0


def test_unchanged_codes_and_unselected_rows_keep_their_proxy():
    wq, s_w, P = _state(32)
    wq2, P2, mask, cnt = O.proxy_select_residual(wq, s_w, P)
    same = DEC[wq2] == DEC[wq]
    assert np.array_equal(P2[same].view(np.uint32), P[same].view(np.uint32))
    sel = mask.astype(bool)
    assert np.array_equal(wq2[~sel], wq[~sel])
