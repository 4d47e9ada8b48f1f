"""B200 (sm_100a) hot path of FALQON's melded FP8 linear layer.

A thin ctypes binding over ``libfalqon.so`` (C ABI declared in
``include/falqon.h``).  Each Python function has the name of the C entry
point it marshals to and only turns torch tensors into device pointers and
the current CUDA stream into a ``void*``; all computation runs in the
library's CUDA kernels.  There is no CPU path: importing this package without
the built library raises.
"""

from __future__ import annotations

import ctypes as C
import os

import torch

__all__ = [
    "FalqonError", "lib", "falqon_quantize", "falqon_linear_fwd", "falqon_linear_bwd",
    "falqon_proxy_update", "falqon_workspace_size", "falqon_status_string", "falqon_version",
    "falqon_linear_bwd_noalloc", "falqon_proxy_update_topk", "falqon_linear_fwd_folded",
    "falqon_linear_bwd_folded", "folded_t_planes", "falqon_selftest_bounded_waits", "falqon_workspace_init",
    "workspace", "falqon_lora_separate_fwd", "falqon_lora_separate_bwd", "separate_saved_views",
    "separate_bwd_views", "falqon_linear_fwd_grouped",
    "SEPARATE_BF16", "SEPARATE_FP8", "OP_QUANTIZE",
    "OP_LINEAR_FWD",
    "OP_LINEAR_BWD", "OP_PROXY_UPDATE", "OP_PROXY_UPDATE_TOPK", "OP_FOLDED_T", "OP_LINEAR_BWD_FOLDED",
    "PROXY_ACCUMULATE", "PROXY_SELECT", "PROXY_KEEP_RESIDUAL", "PROXY_STRICT", "PROXY_TENSOR", "PROXY_DEFER_CLEAR", "DEV_NONFINITE", "DEV_SCALE_OVERFLOW", "DEV_TIMEOUT",
    "LIB_PATH", "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfalqon.so")

OP_QUANTIZE, OP_LINEAR_FWD, OP_LINEAR_BWD, OP_PROXY_UPDATE, OP_PROXY_UPDATE_TOPK = 0, 1, 2, 3, 4
OP_FOLDED_T, OP_LINEAR_BWD_FOLDED = 5, 6
OP_SEPARATE_SAVED_BF16, OP_SEPARATE_SAVED_FP8, OP_SEPARATE_FWD_FP8 = 7, 8, 9
OP_SEPARATE_BWD_BF16, OP_SEPARATE_BWD_FP8 = 10, 11
SEPARATE_BF16, SEPARATE_FP8 = 0, 1
DTYPE_BF16, DTYPE_F32 = 0, 1
PROXY_ACCUMULATE, PROXY_SELECT, PROXY_KEEP_RESIDUAL, PROXY_STRICT, PROXY_TENSOR = 1, 2, 4, 8, 16
PROXY_DEFER_CLEAR = 32  # with ACCUMULATE | SELECT: row_mask carries the clear to the next call
DEV_NONFINITE, DEV_SCALE_OVERFLOW, DEV_TIMEOUT = 1, 2, 4
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA"}

EXPORTED_SYMBOLS = (
    "falqon_quantize", "falqon_linear_fwd", "falqon_linear_bwd", "falqon_proxy_update",
    "falqon_workspace_size", "falqon_status_string", "falqon_version",
    "falqon_linear_bwd_noalloc", "falqon_proxy_update_topk", "falqon_quantize_e5m2",
    "falqon_linear_bwd_e5m2", "falqon_linear_fwd_folded", "falqon_linear_bwd_folded",
    "falqon_selftest_bounded_waits", "falqon_workspace_init", "falqon_lora_separate_fwd",
    "falqon_lora_separate_bwd", "falqon_linear_fwd_grouped",
)


class FalqonError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} "
                         f"({falqon_status_string(self.status)})")


_LIB = None


def lib():
    """The loaded C library (ctypes), with argument types declared."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m fp8_quantized_lora_b200.build` "
            "(there is no CPU fallback)")
    L = C.CDLL(LIB_PATH)
    p, i64, u32, sz = C.c_void_p, C.c_int64, C.c_uint32, C.c_size_t
    L.falqon_quantize.argtypes = [p, C.c_int, i64, i64, p, p, p, p, p, p, sz, p]
    L.falqon_quantize_e5m2.argtypes = [p, C.c_int, i64, i64, p, p, p, p, p, sz, p]
    L.falqon_linear_fwd.argtypes = [p, p, p, p, i64, i64, i64, p, p, p, sz, p]
    L.falqon_linear_bwd.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, p, p, p, p, p, sz, p]
    L.falqon_linear_bwd_e5m2.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, p, p, p, p, p, sz, p]
    L.falqon_proxy_update.argtypes = [p, p, p, p, p, i64, i64, i64, u32, p, p, p, p, sz, p]
    L.falqon_proxy_update_topk.argtypes = [p, p, p, p, p, i64, i64, i64, i64, u32, p, p, p, p, sz, p]
    L.falqon_linear_bwd_noalloc.argtypes = [p, p, p, p, p, p, p, p, i64, i64, i64, i64, p, p, p, p, p]
    L.falqon_linear_fwd_folded.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p, p, sz, p, p]
    L.falqon_selftest_bounded_waits.argtypes = [p, p, p, p]
    L.falqon_linear_bwd_folded.argtypes = [p, p, p, p, p, p, p, p, p, sz, i64, i64, i64, i64, p, p, p, p, p,
                                           sz, p]
    for f in ("falqon_quantize", "falqon_linear_fwd", "falqon_linear_bwd", "falqon_proxy_update",
              "falqon_linear_bwd_noalloc"):
        getattr(L, f).restype = C.c_int
    L.falqon_lora_separate_fwd.argtypes = [C.c_int, p, p, p, p, p, p, p, i64, i64, i64, i64, p, p, sz, p, p, sz, p]
    L.falqon_lora_separate_bwd.argtypes = [C.c_int, p, p, p, p, p, p, p, p, p, p, p, sz, i64, i64, i64, i64, p, p,
                                           p, p, p, sz, p]
    L.falqon_linear_fwd_grouped.argtypes = [p, p, C.c_int, p, p, p, p, i64, i64, p, p]
    L.falqon_linear_fwd_grouped.restype = C.c_int
    L.falqon_workspace_init.argtypes = [p, sz, p]
    L.falqon_workspace_init.restype = C.c_int
    L.falqon_workspace_size.argtypes = [C.c_int, i64, i64, i64, i64]
    L.falqon_workspace_size.restype = sz
    L.falqon_status_string.argtypes = [C.c_int]
    L.falqon_status_string.restype = C.c_char_p
    L.falqon_version.restype = C.c_char_p
    _LIB = L
    return L


def falqon_status_string(status: int) -> str:
    return lib().falqon_status_string(int(status)).decode()


def falqon_version() -> str:
    return lib().falqon_version().decode()


def falqon_workspace_size(op: int, M: int = 0, N: int = 0, K: int = 0, r: int = 0) -> int:
    return int(lib().falqon_workspace_size(int(op), int(M), int(N), int(K), int(r)))


# ------------------------------------------------------------------ marshalling helpers
def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("falqon tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("falqon tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise FalqonError(status, where)


def falqon_workspace_init(workspace, stream=None):
    """Zero-fills a workspace (uint8 tensor, 256-byte aligned) on the stream:
    required once for a quantize workspace before its first use."""
    st = lib().falqon_workspace_init(_ptr(workspace), workspace.numel(), _stream(stream, workspace.device))
    _check(st, "falqon_workspace_init")
    return workspace


def workspace(op, M=0, N=0, K=0, r=0, device="cuda", stream=None):
    """A 256-byte-aligned workspace for `op` at these sizes, initialised
    (falqon_workspace_init), or None when the op needs none."""
    need = falqon_workspace_size(op, M, N, K, r)
    if need == 0:
        return None
    raw = torch.empty(need + 256, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 256
    return falqon_workspace_init(raw[off:off + need], stream)


def _workspace(op, M, N, K, r, device, workspace):
    need = falqon_workspace_size(op, M, N, K, r)
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = globals()["workspace"](op, M, N, K, r, device)
    return workspace, workspace.numel()


def _u8(t):
    return t.view(torch.uint8) if t.dtype != torch.uint8 else t


# ------------------------------------------------------------------ entry points
def falqon_quantize(x, codes=None, scale=None, amax=None, residual=None, dev_status=None,
                    workspace=None, stream=None, fmt="e4m3"):
    """Per-tensor FP8 quantization of a 2-D bf16/fp32 tensor (E4M3, or E5M2
    for gradients: fmt="e5m2", no residual); returns (codes, scale, amax)."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    rows, cols = x.shape
    dt = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(x.dtype)
    if dt is None:
        raise ValueError("x must be bfloat16 or float32")
    dev = x.device
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=dev) if codes is None else codes
    scale = torch.empty(1, dtype=torch.float32, device=dev) if scale is None else scale
    amax = torch.empty(1, dtype=torch.float32, device=dev) if amax is None else amax
    ws, wsb = _workspace(OP_QUANTIZE, rows, cols, 0, 0, dev, workspace)
    if fmt == "e5m2":
        if residual is not None:
            raise ValueError("the residual is defined for E4M3 only")
        st = lib().falqon_quantize_e5m2(_ptr(x), dt, rows, cols, _ptr(_u8(codes)), _ptr(scale), _ptr(amax),
                                        _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
        _check(st, "falqon_quantize_e5m2")
        return codes, scale, amax
    if fmt != "e4m3":
        raise ValueError("fmt must be 'e4m3' or 'e5m2'")
    st = lib().falqon_quantize(_ptr(x), dt, rows, cols, _ptr(_u8(codes)), _ptr(scale), _ptr(amax),
                               _ptr(residual), _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
    _check(st, "falqon_quantize")
    return codes, scale, amax


def falqon_linear_fwd(xq, s_x, wq, s_w, y=None, dev_status=None, stream=None):
    """Y = Xq . Wq^T / (s_x s_w) in bf16."""
    M, K = xq.shape
    N = wq.shape[0]
    dev = xq.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    st = lib().falqon_linear_fwd(_ptr(_u8(xq)), _ptr(s_x), _ptr(_u8(wq)), _ptr(s_w), M, N, K,
                                 _ptr(y), _ptr(dev_status), None, 0, _stream(stream, dev))
    _check(st, "falqon_linear_fwd")
    return y


def falqon_linear_fwd_grouped(xq, s_x, wqs, s_ws, ys=None, dev_status=None, stream=None):
    """Y_s = Xq . Wq_s^T / (s_x s_w_s) for up to three backbones that read the
    same Xq, in one launch; returns the list of outputs."""
    M, K = xq.shape
    n = len(wqs)
    dev = xq.device
    if ys is None:
        ys = [torch.empty((M, w.shape[0]), dtype=torch.bfloat16, device=dev) for w in wqs]
    wp = (C.c_void_p * n)(*[_ptr(_u8(w)) for w in wqs])
    sp = (C.c_void_p * n)(*[_ptr(sw) for sw in s_ws])
    yp = (C.c_void_p * n)(*[_ptr(y) for y in ys])
    Ns = (C.c_int64 * n)(*[int(w.shape[0]) for w in wqs])
    st = lib().falqon_linear_fwd_grouped(_ptr(_u8(xq)), _ptr(s_x), n, wp, sp, Ns, yp, M, K, _ptr(dev_status),
                                         _stream(stream, dev))
    _check(st, "falqon_linear_fwd_grouped")
    return ys


def falqon_linear_bwd(dyq, s_dy, wq, s_w, xq, s_x, A, B, dx=True, dA=True, dB=True,
                      dev_status=None, workspace=None, stream=None, dy_fmt="e4m3"):
    """Backward of the melded layer; each output may be True (allocate), a tensor, or None.
    dy_fmt="e5m2": dyq holds E5M2 codes (falqon_quantize(..., fmt="e5m2"))."""
    M, N = dyq.shape
    K = wq.shape[1] if wq is not None else xq.shape[1]
    r = A.shape[0] if A is not None else 0
    dev = dyq.device

    def out(v, shape):
        if v is True:
            return torch.empty(shape, dtype=torch.bfloat16, device=dev)
        return v if v is not None and v is not False else None

    dx_t, dA_t, dB_t = out(dx, (M, K)), out(dA, (r, K)), out(dB, (N, r))
    ws, wsb = (None, 0)
    if dA_t is not None or dB_t is not None:
        ws, wsb = _workspace(OP_LINEAR_BWD, M, N, K, r, dev, workspace)
    if dy_fmt not in ("e4m3", "e5m2"):
        raise ValueError("dy_fmt must be 'e4m3' or 'e5m2'")
    fn = lib().falqon_linear_bwd_e5m2 if dy_fmt == "e5m2" else lib().falqon_linear_bwd
    st = fn(_ptr(_u8(dyq)), _ptr(s_dy), _ptr(None if wq is None else _u8(wq)),
            _ptr(s_w), _ptr(None if xq is None else _u8(xq)), _ptr(s_x),
            _ptr(A), _ptr(B), M, N, K, r, _ptr(dx_t), _ptr(dA_t), _ptr(dB_t),
            _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
    _check(st, "falqon_linear_bwd_e5m2" if dy_fmt == "e5m2" else "falqon_linear_bwd")
    return dx_t, dA_t, dB_t


def falqon_proxy_update(wq, s_w, proxy, dB_inc, A, flags=PROXY_ACCUMULATE | PROXY_SELECT,
                        row_mask=None, n_selected=None, dev_status=None, workspace=None,
                        stream=None):
    """Row-wise proxy update in place on (wq, proxy); returns (row_mask, n_selected).
    With PROXY_DEFER_CLEAR, row_mask is the caller's: zeros before the first
    call, then the previous call's output (rows it marks read as +0)."""
    N, K = proxy.shape
    r = A.shape[0] if A is not None else 0
    dev = proxy.device
    if flags & PROXY_DEFER_CLEAR and row_mask is None:
        raise ValueError("PROXY_DEFER_CLEAR reads the previous selection: pass row_mask")
    if flags & PROXY_SELECT:
        row_mask = torch.empty(N, dtype=torch.uint8, device=dev) if row_mask is None else row_mask
        n_selected = torch.empty(1, dtype=torch.int32, device=dev) if n_selected is None else n_selected
    ws, wsb = _workspace(OP_PROXY_UPDATE, 0, N, K, r, dev, workspace)
    st = lib().falqon_proxy_update(_ptr(None if wq is None else _u8(wq)), _ptr(s_w), _ptr(proxy),
                                   _ptr(dB_inc), _ptr(A), N, K, r, int(flags), _ptr(row_mask),
                                   _ptr(n_selected), _ptr(dev_status), _ptr(ws), wsb,
                                   _stream(stream, dev))
    _check(st, "falqon_proxy_update")
    return row_mask, n_selected


def falqon_proxy_update_topk(wq, s_w, proxy_q, dB_inc, A, k, flags=PROXY_ACCUMULATE | PROXY_SELECT,
                             comp_mask=None, n_selected=None, dev_status=None, workspace=None, stream=None):
    """Top-k proxy update over the r rank components, in place on (wq, proxy_q);
    proxy_q is float32 [r, N].  Returns (comp_mask, n_selected) (None, None
    without PROXY_SELECT)."""
    r, N = proxy_q.shape
    K = wq.shape[1] if wq is not None else (A.shape[1] if A is not None else 0)
    dev = proxy_q.device
    ws, wsb = (None, 0)
    if flags & PROXY_SELECT:
        comp_mask = torch.empty(r, dtype=torch.uint8, device=dev) if comp_mask is None else comp_mask
        n_selected = torch.empty(1, dtype=torch.int32, device=dev) if n_selected is None else n_selected
        ws, wsb = _workspace(OP_PROXY_UPDATE_TOPK, 0, N, K, r, dev, workspace)
    st = lib().falqon_proxy_update_topk(_ptr(None if wq is None else _u8(wq)), _ptr(s_w), _ptr(proxy_q),
                                        _ptr(dB_inc), _ptr(A), N, K, r, int(k), int(flags), _ptr(comp_mask),
                                        _ptr(n_selected), _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
    _check(st, "falqon_proxy_update_topk")
    return comp_mask, n_selected


def falqon_linear_bwd_noalloc(dyq, s_dy, wq, s_w, xq, s_x, A, B, dx=True, dA=True, dB=True,
                              dev_status=None, stream=None):
    """falqon_linear_bwd without a workspace: the library's built-in scratch
    array holds the intermediates (for callers that cannot allocate device
    memory).  Outputs follow falqon_linear_bwd; only the outputs themselves
    are allocated here when passed as True."""
    M, N = dyq.shape
    K = wq.shape[1] if wq is not None else xq.shape[1]
    r = A.shape[0] if A is not None else 0
    dev = dyq.device

    def out(v, shape):
        if v is True:
            return torch.empty(shape, dtype=torch.bfloat16, device=dev)
        return v if v is not None and v is not False else None

    dx_t, dA_t, dB_t = out(dx, (M, K)), out(dA, (r, K)), out(dB, (N, r))
    st = lib().falqon_linear_bwd_noalloc(
        _ptr(_u8(dyq)), _ptr(s_dy), _ptr(None if wq is None else _u8(wq)), _ptr(s_w),
        _ptr(None if xq is None else _u8(xq)), _ptr(s_x), _ptr(A), _ptr(B), M, N, K, r,
        _ptr(dx_t), _ptr(dA_t), _ptr(dB_t), _ptr(dev_status), _stream(stream, dev))
    _check(st, "falqon_linear_bwd_noalloc")
    return dx_t, dA_t, dB_t


def falqon_linear_fwd_folded(xq, s_x, wq, s_w, aq, s_a, y=None, t_saved=None, dev_status=None, stream=None):
    """[Y | T] = Xq . [Wq ; A~q]^T in one GEMM (quantized adapter folded into
    the backbone); returns (y, t_saved), t_saved being the uint8 buffer that
    holds T for falqon_linear_bwd_folded (see folded_t_planes)."""
    M, K = xq.shape
    N = wq.shape[0]
    r = aq.shape[0]
    dev = xq.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    if t_saved is None:
        t_saved, _ = _workspace(OP_FOLDED_T, M, 0, 0, r, dev, None)
    st = lib().falqon_linear_fwd_folded(_ptr(_u8(xq)), _ptr(s_x), _ptr(_u8(wq)), _ptr(s_w), _ptr(_u8(aq)),
                                        _ptr(s_a), M, N, K, r, _ptr(y), _ptr(t_saved), t_saved.numel(),
                                        _ptr(dev_status), _stream(stream, dev))
    _check(st, "falqon_linear_fwd_folded")
    return y, t_saved


def folded_t_planes(t_saved, M, r):
    """(hi, lo) bfloat16 views [r, ld] of a folded T (or U) buffer: T[m, i] = hi[i, m] + lo[i, m]."""
    ld = (M + 7) // 8 * 8
    plane = (ld * r * 2 + 255) // 256 * 256
    hi = t_saved[:ld * r * 2].view(torch.bfloat16).view(r, ld)
    lo = t_saved[plane:plane + ld * r * 2].view(torch.bfloat16).view(r, ld)
    return hi, lo


def falqon_linear_bwd_folded(dyq, s_dy, wq, s_w, bq, s_b, xq, s_x, t_saved, r, dx=True, dA=True, dB=True,
                             dev_status=None, workspace=None, stream=None):
    """[dX | U] = dYq . [Wq | B~q] in one GEMM, then dB from the forward's T
    and dA from U in one launch; each output may be True (allocate), a
    tensor, or None.  Returns (dx, dA, dB)."""
    M, N = dyq.shape
    K = wq.shape[1] if wq is not None else xq.shape[1]
    dev = dyq.device

    def out(v, shape):
        if v is True:
            return torch.empty(shape, dtype=torch.bfloat16, device=dev)
        return v if v is not None and v is not False else None

    dx_t, dA_t, dB_t = out(dx, (M, K)), out(dA, (r, K)), out(dB, (N, r))
    ws, wsb = (None, 0)
    if dA_t is not None:
        ws, wsb = _workspace(OP_LINEAR_BWD_FOLDED, M, N, K, r, dev, workspace)
    st = lib().falqon_linear_bwd_folded(
        _ptr(_u8(dyq)), _ptr(s_dy), _ptr(None if wq is None else _u8(wq)), _ptr(s_w),
        _ptr(None if bq is None else _u8(bq)), _ptr(s_b), _ptr(None if xq is None else _u8(xq)), _ptr(s_x),
        _ptr(t_saved), 0 if t_saved is None else t_saved.numel(), M, N, K, r, _ptr(dx_t), _ptr(dA_t),
        _ptr(dB_t), _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
    _check(st, "falqon_linear_bwd_folded")
    return dx_t, dA_t, dB_t


def falqon_selftest_bounded_waits(flag, dev_status, which, stream=None):
    """Launches the library's self-test of its bounded waits (about one
    second): see include/falqon.h."""
    st = lib().falqon_selftest_bounded_waits(_ptr(flag), _ptr(dev_status), _ptr(which),
                                             _stream(stream, flag.device))
    _check(st, "falqon_selftest_bounded_waits")


# ------------------------------------------------------------------ separate LoRA paths (the comparison)
def _a256(v):
    return (v + 255) // 256 * 256


def separate_saved_views(saved, precision, M, N, K, r):
    """Views of the forward's saved buffer: {"S": bf16 [M, r]} and, for the
    FP8 path, "sq" [M, r], "aq" [r, K], "bq" [N, r] codes and "scales" (s_S,
    s_A, s_B) as float32 [3]."""
    o = 0
    v = {"S": saved[o:o + M * r * 2].view(torch.bfloat16).view(M, r)}
    o += _a256(M * r * 2)
    if precision == SEPARATE_FP8:
        v["sq"] = saved[o:o + M * r].view(M, r)
        o += _a256(M * r)
        v["aq"] = saved[o:o + r * K].view(r, K)
        o += _a256(r * K)
        v["bq"] = saved[o:o + N * r].view(N, r)
        o += _a256(N * r)
        v["scales"] = saved[o:o + 12].view(torch.float32)
    return v


def separate_bwd_views(workspace, precision, M, N, r, quantize_ws_bytes):
    """Views of the backward's workspace: "G" bf16 [M, r] and, for the FP8
    path, "gq" [M, r] codes and "s_g" float32 [1]."""
    o = _a256(quantize_ws_bytes)
    v = {"G": workspace[o:o + M * r * 2].view(torch.bfloat16).view(M, r)}
    o += _a256(M * r * 2)
    if precision == SEPARATE_FP8:
        v["gq"] = workspace[o:o + M * r].view(M, r)
        o += _a256(M * r)
    ldt = (M + 15) // 16 * 16
    o += 2 * _a256(ldt * r * (1 if precision == SEPARATE_FP8 else 2)) + _a256(N * r * 2)
    v["s_g"] = workspace[o:o + 4].view(torch.float32)
    return v


def falqon_lora_separate_fwd(precision, xq, s_x, x, wq, s_w, A, B, y=None, saved=None, dev_status=None,
                             workspace=None, stream=None):
    """Separate LoRA path forward (bf16 or FP8 adapter products beside the FP8
    backbone); returns (y, saved)."""
    M, K = xq.shape
    N = wq.shape[0]
    r = A.shape[0]
    dev = xq.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    sop = OP_SEPARATE_SAVED_FP8 if precision == SEPARATE_FP8 else OP_SEPARATE_SAVED_BF16
    if saved is None:
        saved, _ = _workspace(sop, M, N, K, r, dev, None)
    ws, wsb = (None, 0)
    if precision == SEPARATE_FP8:
        ws, wsb = _workspace(OP_SEPARATE_FWD_FP8, M, N, K, r, dev, workspace)
    st = lib().falqon_lora_separate_fwd(int(precision), _ptr(_u8(xq)), _ptr(s_x), _ptr(x), _ptr(_u8(wq)), _ptr(s_w),
                                        _ptr(A), _ptr(B), M, N, K, r, _ptr(y), _ptr(saved), saved.numel(),
                                        _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
    _check(st, "falqon_lora_separate_fwd")
    return y, saved


def falqon_lora_separate_bwd(precision, dyq, s_dy, dy, wq, s_w, xq, s_x, x, A, B, saved, dx=True, dA=True, dB=True,
                             dev_status=None, workspace=None, stream=None):
    """Separate LoRA path backward; each output may be True (allocate), a
    tensor, or None.  Returns (dx, dA, dB)."""
    M, N = dyq.shape
    r, K = A.shape
    dev = dyq.device

    def out(v, shape):
        if v is True:
            return torch.empty(shape, dtype=torch.bfloat16, device=dev)
        return v if v is not None and v is not False else None

    dx_t, dA_t, dB_t = out(dx, (M, K)), out(dA, (r, K)), out(dB, (N, r))
    bop = OP_SEPARATE_BWD_FP8 if precision == SEPARATE_FP8 else OP_SEPARATE_BWD_BF16
    ws, wsb = _workspace(bop, M, N, K, r, dev, workspace)
    st = lib().falqon_lora_separate_bwd(
        int(precision), _ptr(_u8(dyq)), _ptr(s_dy), _ptr(dy), _ptr(None if wq is None else _u8(wq)), _ptr(s_w),
        _ptr(None if xq is None else _u8(xq)), _ptr(s_x), _ptr(x), _ptr(A), _ptr(B), _ptr(saved), saved.numel(),
        M, N, K, r, _ptr(dx_t), _ptr(dA_t), _ptr(dB_t), _ptr(dev_status), _ptr(ws), wsb, _stream(stream, dev))
    _check(st, "falqon_lora_separate_bwd")
    return dx_t, dA_t, dB_t
