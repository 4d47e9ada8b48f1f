"""Pins for the oracle's row-wise proxy update (C-9 .. C-11).

References independent of the oracle: a numpy restatement with float32
additions (equal to the FMA chain because bf16 x bf16 products are exact in
float32), exact power-of-two rank-1 updates, a brute-force selection rule
written with the search-based E4M3 encoder, and the invariants of the method:
P = 0 selects nothing; a planted one-step update selects exactly its row;
rows not selected keep Wq bit-identical.
"""

import numpy as np

import oracle as O
from synthetic import gen

from test_oracle_codec import _brute_encode

DEC = np.array([O.e4m3_decode(c) for c in range(256)])


def _state(seed, N=24, K=48, r=8, p_std=1e-4):
    w = gen.normal_f32(seed, (N, K), 0.02)
    wq, s_w, _, _ = O.quantize(w)
    P = gen.normal_f32(seed + 1, (N, K), p_std)
    dB = gen.normal_bf16_bits(seed + 2, (N, r), 1e-2)
    A = gen.normal_bf16_bits(seed + 3, (r, K), 1e-2)
    return wq, s_w, P, dB, A


def test_accumulate_equals_float32_sequential_adds():
    _, _, P, dB, A = _state(1)
    got = O.proxy_accumulate(P, dB, A)
    b = gen.bf16_bits_to_f32(dB)
    a = gen.bf16_bits_to_f32(A)
    acc = np.zeros(P.shape, dtype=np.float32)
    for i in range(a.shape[0]):
        prod = (b[:, i:i + 1].astype(np.float64) * a[i:i + 1, :].astype(np.float64))
        assert np.array_equal(prod, prod.astype(np.float32).astype(np.float64))  # exact in fp32
        acc = (acc + prod.astype(np.float32)).astype(np.float32)
    assert np.array_equal(got, (P + acc).astype(np.float32))


def test_accumulate_order_is_index_order():
    # reversing the i order changes float32 rounding somewhere: the pin above
    # must be able to tell the two orders apart on this data
    _, _, P, dB, A = _state(2, r=64)
    b = gen.bf16_bits_to_f32(dB)
    a = gen.bf16_bits_to_f32(A)
    fwd = np.zeros(P.shape, dtype=np.float32)
    rev = np.zeros(P.shape, dtype=np.float32)
    for i in range(64):
        fwd = fwd + (b[:, i:i + 1] * a[i:i + 1, :]).astype(np.float32)
        rev = rev + (b[:, 63 - i:64 - i] * a[63 - i:64 - i, :]).astype(np.float32)
    got = O.proxy_accumulate(np.zeros_like(P), dB, A)
    assert np.array_equal(got, fwd)
    assert not np.array_equal(fwd, rev)


def test_zero_increment_leaves_proxy_bit_identical():
    _, _, P, _, A = _state(3)
    got = O.proxy_accumulate(P, np.zeros((P.shape[0], A.shape[0]), dtype=np.uint16), A)
    assert np.array_equal(got.view(np.uint32), P.view(np.uint32))


def test_rank1_power_of_two_update_is_exact():
    N, K = 16, 32
    e = np.arange(N) % 5
    f = np.arange(K) % 7
    dB = gen.f32_to_bf16_bits((2.0 ** -(e + 3)).astype(np.float32)).reshape(N, 1)
    sgn = np.where(np.arange(K) % 3 == 0, -1.0, 1.0)
    A = gen.f32_to_bf16_bits((sgn * 2.0 ** -(f + 4)).astype(np.float32)).reshape(1, K)
    got = O.proxy_accumulate(np.zeros((N, K), np.float32), dB, A)
    ref = np.outer(2.0 ** -(e + 3), sgn * 2.0 ** -(f + 4))
    assert np.array_equal(got.astype(np.float64), ref)


def test_zero_proxy_selects_nothing():
    wq, s_w, P, _, _ = _state(4)
    wq2, P2, mask, cnt = O.proxy_select(wq, s_w, np.zeros_like(P))
    assert cnt == 0 and not mask.any()
    assert np.array_equal(wq2, wq) and np.all(P2 == 0)


def test_planted_one_step_update_selects_exactly_its_row():
    wq, s_w, P, _, _ = _state(5)
    Pz = np.zeros_like(P)
    n, k = 7, 11
    c = int(wq[n, k])
    if c & 0x7F >= 0x7E or c & 0x80:
        wq[n, k] = c = 0x30
    step = (DEC[c + 1] - DEC[c]) / np.float64(s_w)  # one code up, in weight units
    Pz[n, k] = np.float32(step)
    assert np.float64(Pz[n, k]) * np.float64(s_w) != 0
    wq2, P2, mask, cnt = O.proxy_select(wq, s_w, Pz)
    assert cnt == 1 and mask[n] == 1 and mask.sum() == 1
    assert wq2[n, k] == c + 1
    expect = wq.copy()
    expect[n, k] = c + 1
    assert np.array_equal(wq2, expect)
    assert np.all(P2 == 0)


def test_select_matches_brute_force_restatement():
    wq, s_w, P, _, _ = _state(6, N=40, K=64, p_std=1e-5)
    wq2, P2, mask, cnt = O.proxy_select(wq, s_w, P)
    w = DEC[wq].astype(np.float32)
    upd = (np.float32(s_w) * P).astype(np.float32)
    t = (w + upd).astype(np.float32)
    cn = _brute_encode(t.ravel()).reshape(t.shape)
    changed = DEC[cn] != DEC[wq]
    sel = changed.any(axis=1)
    assert 0 < sel.sum() < len(sel), "data should select some rows but not all"
    assert np.array_equal(mask.astype(bool), sel) and cnt == sel.sum()
    # selected rows: value-changing codes replaced, equal-valued codes kept as they were
    expect = np.where(changed, cn, wq)
    assert np.array_equal(wq2[sel], expect[sel])
    assert np.array_equal(wq2[~sel], wq[~sel])
    assert np.all(P2[sel].view(np.uint32) == 0)
    assert np.array_equal(P2[~sel].view(np.uint32), P[~sel].view(np.uint32))


def test_selected_row_keeps_zero_sign_of_unchanged_codes():
    wq, s_w, P, _, _ = _state(9)
    P[:] = 0
    wq[3, :] = 0x80                       # -0 codes ...
    wq[3, 5] = 0x30                       # ... and one 0.5 that an update moves
    P[3, :] = np.float32(1e-30)           # -0 + tiny -> +0: same value, other bits
    step = (DEC[0x31] - DEC[0x30]) / np.float64(s_w)
    P[3, 5] = np.float32(step)
    wq2, P2, mask, cnt = O.proxy_select(wq, s_w, P)
    assert cnt == 1 and mask[3] == 1
    assert wq2[3, 5] == 0x31
    assert np.all(np.delete(wq2[3], 5) == 0x80)  # -0 kept although t rounds to +0
    assert np.all(P2[3] == 0)


def test_unselected_rows_bit_identical_and_negative_zero_not_a_change():
    wq, s_w, P, _, _ = _state(7)
    wq[:, :] = 0x80  # -0 codes everywhere
    P[:, :] = np.float32(1e-30)  # t = -0 + tiny rounds to +0: a sign flip only
    wq2, P2, mask, cnt = O.proxy_select(wq, s_w, P)
    assert cnt == 0 and np.array_equal(wq2, wq) and np.array_equal(P2, P)


def test_update_composes_accumulate_then_select():
    wq, s_w, P, dB, A = _state(8, p_std=1e-3)
    wq2, P2, mask, cnt = O.proxy_update(wq, s_w, P, dB, A)
    Pn = O.proxy_accumulate(P, dB, A)
    wq3, P3, mask3, cnt3 = O.proxy_select(wq, s_w, Pn)
    assert np.array_equal(wq2, wq3) and np.array_equal(P2, P3) and cnt == cnt3
