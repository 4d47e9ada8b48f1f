"""Plain CPU oracle for the FALQON melded FP8 linear step (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never touches the CUDA library and
the CUDA library never touches it.

The arithmetic lives in ``falqon_oracle.cpp`` (its header lists every reading
of the method); this module only marshals numpy arrays through ctypes.  All
bfloat16 tensors are passed as their uint16 bit patterns.
"""

from __future__ import annotations

import ctypes as C

import numpy as np

from .build import build as _build

STATUS_NONFINITE = 1
STATUS_SCALE_OVERFLOW = 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = C.CDLL(path)
        p = C.c_void_p
        i64 = C.c_int64
        L.fo_e4m3_decode.restype = C.c_double
        L.fo_e4m3_decode.argtypes = [C.c_uint8]
        L.fo_e4m3_encode.restype = C.c_uint8
        L.fo_e4m3_encode.argtypes = [C.c_float]
        L.fo_e4m3_encode_array.argtypes = [p, i64, p]
        L.fo_bf16_round.restype = C.c_uint16
        L.fo_bf16_round.argtypes = [C.c_double]
        L.fo_bf16_round_array.argtypes = [p, i64, p]
        L.fo_amax.restype = C.c_uint32
        L.fo_amax.argtypes = [p, C.c_int, i64, p]
        L.fo_scale.restype = C.c_uint32
        L.fo_scale.argtypes = [C.c_float, C.c_int, p]
        L.fo_quantize.argtypes = [p, C.c_int, i64, C.c_float, C.c_int, p]
        L.fo_e5m2_decode.restype = C.c_double
        L.fo_e5m2_decode.argtypes = [C.c_uint8]
        L.fo_e5m2_encode_array.argtypes = [p, i64, p]
        L.fo_residual.argtypes = [p, C.c_int, p, i64, C.c_float, p, p]
        L.fo_linear_fwd.argtypes = [p, C.c_float, p, C.c_float, i64, i64, i64, i64, i64, p]
        L.fo_linear_dx.argtypes = [p, C.c_float, C.c_int, p, C.c_float, i64, i64, i64, i64, i64, p]
        L.fo_adapter_t.argtypes = [p, C.c_float, p, i64, i64, i64, p, p]
        L.fo_adapter_u.argtypes = [p, C.c_float, C.c_int, p, i64, i64, i64, p, p]
        L.fo_adapter_db.argtypes = [p, C.c_float, C.c_int, p, p, i64, i64, i64, p]
        L.fo_adapter_da.argtypes = [p, p, p, C.c_float, i64, i64, i64, p]
        L.fo_proxy_accumulate.argtypes = [p, p, p, i64, i64, i64]
        L.fo_proxy_select.argtypes = [p, C.c_float, p, i64, i64, p, p]
        L.fo_proxy_topk.restype = C.c_uint32
        L.fo_proxy_topk.argtypes = [p, C.c_float, p, p, p, i64, i64, i64, i64, C.c_int, C.c_int, p, p, p]
        L.fo_proxy_select_residual.argtypes = [p, C.c_float, p, i64, i64, p, p]
        L.fo_matmul_f64.argtypes = [p, p, i64, i64, i64, C.c_int, p]
        L.fo_set_threads.argtypes = [C.c_int]
        L.fo_get_threads.restype = C.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def set_threads(n: int) -> None:
    lib().fo_set_threads(int(n))


def get_threads() -> int:
    return int(lib().fo_get_threads())


# ------------------------------------------------------------------ codecs
def e4m3_decode(c: int) -> float:
    return float(lib().fo_e4m3_decode(int(c)))


def e4m3_decode_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32)
    shape = v.shape
    flat = np.ascontiguousarray(v.reshape(-1))
    out = np.empty(flat.shape, dtype=np.uint8)
    lib().fo_e4m3_encode_array(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(shape)


FORMATS = {"e4m3": 0, "e5m2": 1}


def e5m2_decode(c: int) -> float:
    return float(lib().fo_e5m2_decode(int(c)))


def e5m2_encode(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32)
    shape = v.shape
    flat = np.ascontiguousarray(v.reshape(-1))
    out = np.empty(flat.shape, dtype=np.uint8)
    lib().fo_e5m2_encode_array(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(shape)


def bf16_round(v) -> np.ndarray:
    """float64 -> bfloat16 bits, one rounding (nearest, ties to even)."""
    v = np.asarray(v, dtype=np.float64)
    shape = v.shape
    flat = np.ascontiguousarray(v.reshape(-1))
    out = np.empty(flat.shape, dtype=np.uint16)
    lib().fo_bf16_round_array(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(shape)


def bf16_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ C-2, C-3, C-4
def _xin(x: np.ndarray):
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 1
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), 0
    raise TypeError("x must be bfloat16 bits (uint16) or float32")


def amax(x: np.ndarray):
    x, is_bf16 = _xin(x)
    out = np.zeros(1, dtype=np.float32)
    st = lib().fo_amax(_ptr(x), is_bf16, x.size, _ptr(out))
    return np.float32(out[0]), int(st)


def scale(amax_value, fmt: str = "e4m3") -> tuple:
    out = np.zeros(1, dtype=np.float32)
    st = lib().fo_scale(C.c_float(float(amax_value)), FORMATS[fmt], _ptr(out))
    return np.float32(out[0]), int(st)


def quantize(x: np.ndarray, fmt: str = "e4m3"):
    """Per-tensor FP8 quantization (E4M3, or E5M2 per C-15): returns (codes,
    scale, amax, status)."""
    x, is_bf16 = _xin(x)
    a, st1 = amax(x)
    s, st2 = scale(a, fmt)
    codes = np.empty(x.shape, dtype=np.uint8)
    lib().fo_quantize(_ptr(x), is_bf16, x.size, C.c_float(float(s)), FORMATS[fmt], _ptr(codes))
    return codes, np.float32(s), np.float32(a), st1 | st2


def residual(x: np.ndarray, codes: np.ndarray, s) -> tuple:
    """Eq. 8 quantization error W - DQ(W~): (float64, float32) arrays."""
    x, is_bf16 = _xin(x)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    r64 = np.empty(x.shape, dtype=np.float64)
    r32 = np.empty(x.shape, dtype=np.float32)
    lib().fo_residual(_ptr(x), is_bf16, _ptr(codes), x.size, C.c_float(float(s)),
                      _ptr(r64), _ptr(r32))
    return r64, r32


# ------------------------------------------------------------------ C-5, C-6
def linear_fwd(xq, s_x, wq, s_w, rows=None) -> np.ndarray:
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    m0, m1 = (0, M) if rows is None else rows
    y = np.empty((m1 - m0, N), dtype=np.float64)
    lib().fo_linear_fwd(_ptr(xq), C.c_float(float(s_x)), _ptr(wq), C.c_float(float(s_w)),
                        M, N, K, m0, m1, _ptr(y))
    return y


def linear_dx(dyq, s_dy, wq, s_w, rows=None, dy_fmt: str = "e4m3") -> np.ndarray:
    dyq = np.ascontiguousarray(dyq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    M, N = dyq.shape
    K = wq.shape[1]
    m0, m1 = (0, M) if rows is None else rows
    dx = np.empty((m1 - m0, K), dtype=np.float64)
    lib().fo_linear_dx(_ptr(dyq), C.c_float(float(s_dy)), FORMATS[dy_fmt], _ptr(wq), C.c_float(float(s_w)),
                       M, N, K, m0, m1, _ptr(dx))
    return dx


# ------------------------------------------------------------------ C-7, C-8
def adapter_t(xq, s_x, A):
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    M, K = xq.shape
    r = A.shape[0]
    t64 = np.empty((M, r), dtype=np.float64)
    t16 = np.empty((M, r), dtype=np.uint16)
    lib().fo_adapter_t(_ptr(xq), C.c_float(float(s_x)), _ptr(A), M, K, r, _ptr(t64), _ptr(t16))
    return t64, t16


def adapter_u(dyq, s_dy, B, dy_fmt: str = "e4m3"):
    dyq = np.ascontiguousarray(dyq, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint16)
    M, N = dyq.shape
    r = B.shape[1]
    u64 = np.empty((M, r), dtype=np.float64)
    u16 = np.empty((M, r), dtype=np.uint16)
    lib().fo_adapter_u(_ptr(dyq), C.c_float(float(s_dy)), FORMATS[dy_fmt], _ptr(B), M, N, r, _ptr(u64),
                       _ptr(u16))
    return u64, u16


def adapter_db(dyq, s_dy, t16=None, t64=None, dy_fmt: str = "e4m3"):
    dyq = np.ascontiguousarray(dyq, dtype=np.uint8)
    M, N = dyq.shape
    t = t16 if t16 is not None else t64
    r = t.shape[1]
    t16c = None if t16 is None else np.ascontiguousarray(t16, dtype=np.uint16)
    t64c = None if t64 is None or t16 is not None else np.ascontiguousarray(t64, dtype=np.float64)
    db = np.empty((N, r), dtype=np.float64)
    lib().fo_adapter_db(_ptr(dyq), C.c_float(float(s_dy)), FORMATS[dy_fmt], _ptr(t16c), _ptr(t64c), M, N, r,
                        _ptr(db))
    return db


def adapter_da(xq, s_x, u16=None, u64=None):
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    M, K = xq.shape
    u = u16 if u16 is not None else u64
    r = u.shape[1]
    u16c = None if u16 is None else np.ascontiguousarray(u16, dtype=np.uint16)
    u64c = None if u64 is None or u16 is not None else np.ascontiguousarray(u64, dtype=np.float64)
    da = np.empty((r, K), dtype=np.float64)
    lib().fo_adapter_da(_ptr(u16c), _ptr(u64c), _ptr(xq), C.c_float(float(s_x)), M, K, r, _ptr(da))
    return da


# ------------------------------------------------------------------ C-16
def folded_t(xq, s_x, aq, s_a) -> np.ndarray:
    """C-16: the adapter columns of the folded forward product
    [Y | T] = Xq . [Wq ; A~q]^T, i.e. C-5's sum with the codes of A~ and
    their scale in place of the backbone's (float64, not rounded)."""
    return linear_fwd(xq, s_x, aq, s_a)


def folded_u(dyq, s_dy, bq, s_b, dy_fmt: str = "e4m3") -> np.ndarray:
    """C-16: the adapter columns of the folded dX product
    [dX | U] = dYq . [Wq | B~q], i.e. C-6's sum with B~q [N, r] in place of
    Wq [N, K] (float64, not rounded)."""
    return linear_dx(dyq, s_dy, bq, s_b, dy_fmt=dy_fmt)


def folded_adapter_grads(xq, s_x, dyq, s_dy, aq, s_a, bq=None, s_b=None, dy_fmt: str = "e4m3"):
    """C-16: (T, dB, U, dA) of the folded path; U and dA are None without B~q."""
    t64 = folded_t(xq, s_x, aq, s_a)
    db = adapter_db(dyq, s_dy, t64=t64, dy_fmt=dy_fmt)
    if bq is None:
        return t64, db, None, None
    u64 = folded_u(dyq, s_dy, bq, s_b, dy_fmt=dy_fmt)
    return t64, db, u64, adapter_da(xq, s_x, u64=u64)


# ------------------------------------------------------------------ C-9, C-10, C-11
def proxy_accumulate(P: np.ndarray, dB_inc: np.ndarray, A: np.ndarray) -> np.ndarray:
    """Returns P + (dB_inc . A) with the float32 FMA chain; P is not modified."""
    P = np.array(P, dtype=np.float32, copy=True, order="C")
    dB_inc = np.ascontiguousarray(dB_inc, dtype=np.uint16)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    N, K = P.shape
    r = A.shape[0]
    lib().fo_proxy_accumulate(_ptr(P), _ptr(dB_inc), _ptr(A), N, K, r)
    return P


def proxy_select(wq: np.ndarray, s_w, P: np.ndarray):
    """Returns (new wq, new P, mask, n_selected); the inputs are not modified."""
    wq = np.array(wq, dtype=np.uint8, copy=True, order="C")
    P = np.array(P, dtype=np.float32, copy=True, order="C")
    N, K = wq.shape
    mask = np.zeros(N, dtype=np.uint8)
    cnt = np.zeros(1, dtype=np.int32)
    lib().fo_proxy_select(_ptr(wq), C.c_float(float(s_w)), _ptr(P), N, K, _ptr(mask), _ptr(cnt))
    return wq, P, mask, int(cnt[0])


def proxy_select_residual(wq: np.ndarray, s_w, P: np.ndarray):
    """C-10 with C-14 (residual-keeping clear): returns (new wq, new P, mask,
    n_selected); the inputs are not modified."""
    wq = np.array(wq, dtype=np.uint8, copy=True, order="C")
    P = np.array(P, dtype=np.float32, copy=True, order="C")
    N, K = wq.shape
    mask = np.zeros(N, dtype=np.uint8)
    cnt = np.zeros(1, dtype=np.int32)
    lib().fo_proxy_select_residual(_ptr(wq), C.c_float(float(s_w)), _ptr(P), N, K, _ptr(mask), _ptr(cnt))
    return wq, P, mask, int(cnt[0])


def proxy_update_topk(wq, s_w, Q, dB_inc, A, k, accumulate=True, select=True):
    """C-13: one update of the top-k proxy over the r rank components.

    Q is float32 [r, N] (row i: the unmerged part of B's column i), dB_inc
    bfloat16 bits [N, r] (read when accumulate), A bfloat16 bits [r, K].
    Returns (new wq, new Q, component mask [r], number merged, status); the
    inputs are not modified."""
    wq = np.array(wq, dtype=np.uint8, copy=True, order="C")
    Q = np.array(Q, dtype=np.float32, copy=True, order="C")
    A = np.ascontiguousarray(A, dtype=np.uint16)
    N, K = wq.shape
    r = A.shape[0]
    assert Q.shape == (r, N), "Q must be [r, N]"
    dBc = None if dB_inc is None else np.ascontiguousarray(dB_inc, dtype=np.uint16)
    if accumulate:
        assert dBc is not None and dBc.shape == (N, r)
    mask = np.zeros(r, dtype=np.uint8)
    cnt = np.zeros(1, dtype=np.int32)
    st = lib().fo_proxy_topk(_ptr(wq), C.c_float(float(s_w)), _ptr(Q), _ptr(dBc), _ptr(A), N, K, r, int(k),
                             int(bool(accumulate)), int(bool(select)), None, _ptr(mask), _ptr(cnt))
    return wq, Q, mask, int(cnt[0]), int(st)


def proxy_topk_scores(Q, A):
    """C-13 scores of the r components of Q [r, N] with A [r, K] (float64),
    and the status bits."""
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    A = np.ascontiguousarray(A, dtype=np.uint16)
    r, N = Q.shape
    K = A.shape[1]
    wq = np.zeros((N, K), dtype=np.uint8)
    sc = np.zeros(r, dtype=np.float64)
    st = lib().fo_proxy_topk(_ptr(wq), C.c_float(1.0), _ptr(Q), None, _ptr(A), N, K, r, 0, 0, 0, _ptr(sc),
                             None, None)
    return sc, int(st)


def proxy_update(wq, s_w, P, dB_inc, A, accumulate=True, select=True, keep_residual=False):
    """One row-wise proxy update: accumulate, then select/requantize/clear
    (C-11) or keep the residual (C-14)."""
    Pn = proxy_accumulate(P, dB_inc, A) if accumulate else np.array(P, dtype=np.float32, copy=True)
    if not select:
        return np.array(wq, dtype=np.uint8, copy=True), Pn, None, 0
    return proxy_select_residual(wq, s_w, Pn) if keep_residual else proxy_select(wq, s_w, Pn)


# ------------------------------------------------------------------ C-17
def matmul_f64(a, b, b_nk: bool) -> np.ndarray:
    """float64 sum in index order of a[m,k] * b(k,n); b is [N, K] when b_nk,
    else [K, N]."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    M, K = a.shape
    N = b.shape[0] if b_nk else b.shape[1]
    assert (b.shape[1] if b_nk else b.shape[0]) == K
    out = np.empty((M, N), dtype=np.float64)
    lib().fo_matmul_f64(_ptr(a), _ptr(b), M, N, K, int(bool(b_nk)), _ptr(out))
    return out


from .tolerance import within_tolerance, tolerance_report  # noqa: E402,F401
from .step import layer_step  # noqa: E402,F401

