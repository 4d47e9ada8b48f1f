"""One melded FP8 linear training step composed from the oracle's parts.

Order (FALQON, [intro] and [R4-Q1]): quantize X, forward on the backbone,
quantize dY, dX on the backbone, T = Xq A^T, dB = dYq^T T, optionally
U = dYq B and dA = U^T Xq (T and U exact, float64), then the row-wise proxy
update with the adapter increment dB_inc.  Test infrastructure only.
"""

from __future__ import annotations

import numpy as np

from . import (adapter_da, adapter_db, adapter_t, adapter_u, bf16_round, linear_dx, linear_fwd,
               proxy_update, quantize)


def layer_step(X, wq, s_w, A, B, dY, P, dB_inc=None, lr=None, want_da=True, rows=None):
    """Returns a dict with every intermediate of one step.

    dB_inc: bfloat16 bits of the increment to fold into the proxy; when None
    and ``lr`` is given, it is bf16(-lr * bf16(dB)) (plain SGD).
    rows: optional (m0, m1) to compute Y and dX on a row range only.
    """
    out = {}
    xq, s_x, amax_x, st_x = quantize(X)
    dyq, s_dy, amax_dy, st_dy = quantize(dY)
    out.update(xq=xq, s_x=s_x, amax_x=amax_x, dyq=dyq, s_dy=s_dy, amax_dy=amax_dy,
               status=st_x | st_dy)
    out["y"] = linear_fwd(xq, s_x, wq, s_w, rows=rows)
    out["dx"] = linear_dx(dyq, s_dy, wq, s_w, rows=rows)
    t64, _ = adapter_t(xq, s_x, A)
    out["t64"] = t64
    out["db"] = adapter_db(dyq, s_dy, t64=t64)
    if want_da:
        u64, _ = adapter_u(dyq, s_dy, B)
        out["u64"] = u64
        out["da"] = adapter_da(xq, s_x, u64=u64)
    if dB_inc is None and lr is not None:
        db16 = bf16_round(out["db"])
        db_f = (db16.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        dB_inc = bf16_round(-float(lr) * db_f)
    if dB_inc is not None:
        wq2, P2, mask, cnt = proxy_update(wq, s_w, P, dB_inc, A)
        out.update(dB_inc=dB_inc, wq_new=wq2, P_new=P2, mask=mask, n_selected=cnt)
    return out
