"""C-17: LoRA kept as a separate path beside the FP8 backbone, in bfloat16 or
with every adapter operand quantized to E4M3 per product (test
infrastructure: the comparison the pages measure, for the rank sweep).

Every product is a float64 sum (C-5 for code operands, ``matmul_f64`` for
decoded values) rounded once to bfloat16; the adapter branch and the backbone
branch are added as bfloat16 tensors are (float32 add, one bfloat16
rounding).  ``rnd=False`` keeps every intermediate in float64 and skips the
roundings (the pin against automatic differentiation uses it).
"""

from __future__ import annotations

import numpy as np

from . import bf16_round, bf16_to_f64, e4m3_decode_table, linear_dx, linear_fwd, matmul_f64, quantize

_DEC = None


def _dec(codes):
    global _DEC
    if _DEC is None:
        _DEC = e4m3_decode_table()
    return _DEC[np.asarray(codes, dtype=np.uint8)]


def _r16(v, rnd):
    """bfloat16 rounding of a float64 array as its float64 values."""
    return bf16_to_f64(bf16_round(v)) if rnd else np.asarray(v, dtype=np.float64)


def _add16(a, b, rnd):
    """a + b as bfloat16 tensors add: float32 sum of the two, one bfloat16 rounding."""
    if not rnd:
        return a + b
    s = (np.asarray(a, dtype=np.float32) + np.asarray(b, dtype=np.float32)).astype(np.float64)
    return bf16_to_f64(bf16_round(s))


def _q(v64):
    """Per-tensor E4M3 quantization (C-2, C-3) of a float64 tensor of bfloat16
    values: (codes, scale)."""
    codes, s, _, _ = quantize(bf16_round(v64))
    return codes, s


def separate_fwd(X, A, B, xq, s_x, wq, s_w, precision, S_given=None, rnd=True):
    """Forward of the separate path.  X, A, B: bfloat16 bits; xq, s_x: the
    backbone's codes of X; precision "bf16" or "fp8".  S_given (float64
    values of bfloat16) replaces S in the second product (to check it given
    another implementation's S).  Returns a dict of float64 arrays."""
    out = {"Ybb": _r16(linear_fwd(xq, s_x, wq, s_w), rnd)}
    if precision == "bf16":
        out["S"] = _r16(matmul_f64(bf16_to_f64(X), bf16_to_f64(A), True), rnd)
        S = out["S"] if S_given is None else np.asarray(S_given, dtype=np.float64)
        out["Ylora"] = _r16(matmul_f64(S, bf16_to_f64(B), True), rnd)
    elif precision == "fp8":
        aq, s_a, _, _ = quantize(np.ascontiguousarray(A, dtype=np.uint16))
        bq, s_b, _, _ = quantize(np.ascontiguousarray(B, dtype=np.uint16))
        out.update(aq=aq, s_a=s_a, bq=bq, s_b=s_b)
        out["S"] = _r16(linear_fwd(xq, s_x, aq, s_a), rnd)
        S = out["S"] if S_given is None else np.asarray(S_given, dtype=np.float64)
        sq, s_s = _q(S)
        out.update(sq=sq, s_s=s_s)
        out["Ylora"] = _r16(linear_fwd(sq, s_s, bq, s_b), rnd)
    else:
        raise ValueError("precision must be 'bf16' or 'fp8'")
    out["Y"] = _add16(out["Ybb"], out["Ylora"], rnd)
    return out


def separate_bwd(X, dY, A, B, S, xq, s_x, dyq, s_dy, wq, s_w, precision, G_given=None, rnd=True):
    """Backward of the separate path.  S: the forward's S (float64 values of
    bfloat16); dY: bfloat16 bits; dyq, s_dy: the backbone's codes of dY.
    G_given replaces G in the products that read it.  Returns a dict of
    float64 arrays (dXbb, G, dXlora, dX, dB, dA, and the codes used)."""
    S = np.asarray(S, dtype=np.float64)
    out = {"dXbb": _r16(linear_dx(dyq, s_dy, wq, s_w), rnd)}
    if precision == "bf16":
        Xf, dYf, Af, Bf = bf16_to_f64(X), bf16_to_f64(dY), bf16_to_f64(A), bf16_to_f64(B)
        out["G"] = _r16(matmul_f64(dYf, Bf, False), rnd)
        G = out["G"] if G_given is None else np.asarray(G_given, dtype=np.float64)
        out["dXlora"] = _r16(matmul_f64(G, Af, False), rnd)
        out["dB"] = _r16(matmul_f64(np.ascontiguousarray(dYf.T), S, False), rnd)
        out["dA"] = _r16(matmul_f64(np.ascontiguousarray(G.T), Xf, False), rnd)
    elif precision == "fp8":
        aq, s_a, _, _ = quantize(np.ascontiguousarray(A, dtype=np.uint16))
        bq, s_b, _, _ = quantize(np.ascontiguousarray(B, dtype=np.uint16))
        sq, s_s = _q(S)
        out["G"] = _r16(linear_dx(dyq, s_dy, bq, s_b), rnd)
        G = out["G"] if G_given is None else np.asarray(G_given, dtype=np.float64)
        gq, s_g = _q(G)
        out.update(aq=aq, s_a=s_a, bq=bq, s_b=s_b, sq=sq, s_s=s_s, gq=gq, s_g=s_g)
        out["dXlora"] = _r16(linear_dx(gq, s_g, aq, s_a), rnd)
        # dB[n,i] = sum_m dec(dYq[m,n]) dec(Sq[m,i]) / (s_dY s_S): C-5 on the transposed codes
        out["dB"] = _r16(linear_fwd(np.ascontiguousarray(dyq.T), s_dy, np.ascontiguousarray(sq.T), s_s), rnd)
        out["dA"] = _r16(linear_fwd(np.ascontiguousarray(gq.T), s_g, np.ascontiguousarray(xq.T), s_x), rnd)
    else:
        raise ValueError("precision must be 'bf16' or 'fp8'")
    out["dX"] = _add16(out["dXbb"], out["dXlora"], rnd)
    return out
