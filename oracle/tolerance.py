"""Floating-point acceptance rule for Y, dX, dB and dA (test infrastructure).

The requirement is "max relative error 8e-3 and within 1 bf16 ulp of the
fp64 result rounded to bf16".  Both halves are undefined near zero, where
any float32-accumulated result differs from a tiny exact value by more than
one of that value's ulps; so both are measured against a floor
tau = 2^-8 * max|R| taken over the whole tensor:

    |G - bf16(R)| <= ulp_bf16(max(|bf16(R)|, tau))   and
    |G - R|       <= 8e-3 * max(|R|, tau)

with ulp_bf16(x) = 2^(floor(log2 x) - 7) (bfloat16 has 8 significant bits),
and never below the smallest bfloat16 subnormal 2^-133.  An all-zero R
(tau = 0) therefore demands G == 0 exactly.  8e-3 is about 2^-7, one
bfloat16 ulp at the bottom of a binade, so away from zero the two criteria
agree.
"""

from __future__ import annotations

import numpy as np

REL_TOL = 8e-3
TAU_FRACTION = 2.0 ** -8
_MIN_ULP = 2.0 ** -133


def _bf16_to_f64(bits):
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    x = np.abs(np.asarray(x, dtype=np.float64))
    out = np.full(x.shape, _MIN_ULP)
    pos = x > 0
    e = np.floor(np.log2(x[pos]))
    out[pos] = np.maximum(np.exp2(e - 7.0), _MIN_ULP)
    return out


def tolerance_report(G, R, Rb=None) -> dict:
    """Compares G (float values, or bfloat16 bits as uint16) with the float64 oracle R."""
    G = _bf16_to_f64(G) if np.asarray(G).dtype == np.uint16 else np.asarray(G, dtype=np.float64)
    R = np.asarray(R, dtype=np.float64)
    if Rb is None:
        from . import bf16_round
        Rb = bf16_round(R)
    Rb = _bf16_to_f64(Rb)
    tau = TAU_FRACTION * (np.max(np.abs(R)) if R.size else 0.0)
    if tau == 0.0:
        ok = G == 0.0
        return {"ok": bool(np.all(ok)), "n_bad": int(np.sum(~ok)), "tau": 0.0,
                "max_ulp_err": float(np.max(np.abs(G))) if G.size else 0.0, "max_rel_err": 0.0}
    ulp = ulp_bf16(np.maximum(np.abs(Rb), tau))
    c1 = np.abs(G - Rb) <= ulp
    c2 = np.abs(G - R) <= REL_TOL * np.maximum(np.abs(R), tau)
    ok = c1 & c2
    return {
        "ok": bool(np.all(ok)),
        "n_bad": int(np.sum(~ok)),
        "tau": float(tau),
        "max_ulp_err": float(np.max(np.abs(G - Rb) / ulp)) if G.size else 0.0,
        "max_rel_err": float(np.max(np.abs(G - R) / np.maximum(np.abs(R), tau))) if G.size else 0.0,
        "first_bad": None if np.all(ok) else int(np.flatnonzero(~ok.ravel())[0]),
    }


def within_tolerance(G, R, Rb=None) -> bool:
    return tolerance_report(G, R, Rb)["ok"]


def branch_sum_report(G, Y, branches) -> dict:
    """Acceptance for a sum of bf16 branches (C-17: the backbone output plus
    the separate adapter branch, each rounded to bf16 before the bf16 add).
    Y: the oracle's result (float64 values of bf16); branches: the oracle's
    rounded branch values.  Each branch of the implementation may differ
    from the oracle's by one bf16 unit (its float32 accumulation against the
    oracle's float64), and the sum is rounded once more:

        |G - Y| <= ulp(max(|Y|, tau)) + sum_b ulp(max(|b|, tau_b)),

    every tau being 2^-8 of the tensor's largest magnitude."""
    G = _bf16_to_f64(G) if np.asarray(G).dtype == np.uint16 else np.asarray(G, dtype=np.float64)
    Y = np.asarray(Y, dtype=np.float64)

    def unit(v):
        v = np.asarray(v, dtype=np.float64)
        t = TAU_FRACTION * (np.max(np.abs(v)) if v.size else 0.0)
        return ulp_bf16(np.maximum(np.abs(v), t)) if t > 0 else np.zeros(v.shape)
    bound = unit(Y) + sum(unit(b) for b in branches)
    err = np.abs(G - Y)
    ok = err <= bound
    return {"ok": bool(np.all(ok)), "n_bad": int(np.sum(~ok)),
            "max_err_over_bound": float(np.max(err / np.maximum(bound, _MIN_ULP))) if G.size else 0.0,
            "first_bad": None if np.all(ok) else int(np.flatnonzero(~ok.ravel())[0])}
