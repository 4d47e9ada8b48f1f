"""CPU checks of the C ABI: the library loads, exports what include/falqon.h
declares, and rejects bad arguments before touching a GPU."""

import ctypes as C
import os
import re
import subprocess

import pytest

import fp8_quantized_lora_b200 as F

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "falqon.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FALQON_API\s+[\w\s\*]+?\b(falqon_\w+)\s*\(", text)))


def test_header_declares_the_four_calls_and_helpers():
    names = _declared()
    for n in ("falqon_quantize", "falqon_linear_fwd", "falqon_linear_bwd", "falqon_proxy_update",
              "falqon_workspace_size", "falqon_status_string", "falqon_version"):
        assert n in names
    assert set(names) == set(F.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    L = F.lib()
    for n in _declared():
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", F.LIB_PATH], capture_output=True, text=True)
    if out.returncode == 0:
        exported = {line.split()[-1] for line in out.stdout.splitlines() if " T " in line}
        assert set(_declared()) <= exported
        assert not [s for s in exported if s.startswith("_ZN6falqon")], "internal symbols leaked"


def test_status_strings_and_version():
    assert F.falqon_status_string(0) == "ok"
    assert "workspace" in F.falqon_status_string(3)
    assert "sm_100a" in F.falqon_version()


def test_workspace_sizes_are_positive_and_aligned():
    assert F.falqon_workspace_size(F.OP_LINEAR_FWD, 4096, 4096, 4096, 64) == 0
    for op in (F.OP_QUANTIZE, F.OP_LINEAR_BWD, F.OP_PROXY_UPDATE, F.OP_PROXY_UPDATE_TOPK):
        n = F.falqon_workspace_size(op, 4096, 4096, 4096, 64)
        assert n > 0 and n % 256 == 0


# Fake, 256-byte aligned addresses: validation must reject the call before any
# pointer is dereferenced or any CUDA call is made.
P = C.c_void_p(1 << 20)
P8 = C.c_void_p((1 << 20) + 8)


def test_quantize_argument_errors():
    L = F.lib()
    assert L.falqon_quantize(None, 0, 4, 16, P, P, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_quantize(P, 0, 0, 16, P, P, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_quantize(P, 7, 4, 16, P, P, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_quantize(P, 0, 4, 24, P, P, None, None, None, P, 1 << 20, None) == 2
    assert L.falqon_quantize(P8, 0, 4, 16, P, P, None, None, None, P, 1 << 20, None) == 2
    assert L.falqon_quantize(P, 0, 4, 16, P, P, None, None, None, None, 0, None) == 3
    assert L.falqon_quantize(P, 0, 4, 16, P, P, None, None, None, P, 8, None) == 3


def test_linear_argument_errors():
    L = F.lib()
    assert L.falqon_linear_fwd(None, P, P, P, 4, 16, 16, P, None, None, 0, None) == 1
    assert L.falqon_linear_fwd(P, P, P, P, 4, 24, 16, P, None, None, 0, None) == 2
    assert L.falqon_linear_fwd(P, P, P, P, 4, 16, 40, P, None, None, 0, None) == 2
    assert L.falqon_linear_fwd(P, P, P, P, -1, 16, 16, P, None, None, 0, None) == 1
    # no output requested
    assert L.falqon_linear_bwd(P, P, P, P, P, P, P, P, 4, 16, 16, 16, None, None, None,
                               None, P, 1 << 20, None) == 1
    # dA requested without B
    assert L.falqon_linear_bwd(P, P, P, P, P, P, P, None, 4, 16, 16, 16, None, P, None,
                               None, P, 1 << 20, None) == 1
    # r not a multiple of 16
    assert L.falqon_linear_bwd(P, P, P, P, P, P, P, P, 4, 16, 16, 8, None, None, P,
                               None, P, 1 << 20, None) == 2
    # workspace too small
    assert L.falqon_linear_bwd(P, P, P, P, P, P, P, P, 4, 16, 16, 16, None, None, P,
                               None, P, 64, None) == 3


def test_proxy_argument_errors():
    L = F.lib()
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 0, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 8, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_proxy_update(P, P, P, None, P, 4, 16, 2, 1, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 20, 2, 3, None, None, None, P, 1 << 20, None) == 2
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 3, None, None, None, None, 0, None) == 3
    # KEEP_RESIDUAL only together with SELECT
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 5, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 4, None, None, None, P, 1 << 20, None) == 1
    # STRICT is accepted with any valid combination (the K % 16 check fires next) ...
    for flags in (1 | 8, 3 | 8, 7 | 8):
        assert L.falqon_proxy_update(P, P, P, P, P, 4, 20, 2, flags, None, None, None, P, 1 << 20, None) == 2
    # ... but not alone, and unknown bits are still rejected
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 8, None, None, None, P, 1 << 20, None) == 1
    assert L.falqon_proxy_update(P, P, P, P, P, 4, 16, 2, 3 | 64, None, None, None, P, 1 << 20, None) == 1


def test_proxy_defer_clear_argument_errors():
    """DEFER_CLEAR (32) goes with ACCUMULATE and SELECT both, never with
    KEEP_RESIDUAL or TENSOR, and needs the row mask it reads and writes; a
    valid combination gets as far as the shape check (K % 16 -> UNSUPPORTED)."""
    L = F.lib()
    D = 32
    f = L.falqon_proxy_update
    assert f(P, P, P, P, P, 4, 20, 2, 3 | D, P, None, None, P, 1 << 20, None) == 2
    assert f(P, P, P, P, P, 4, 20, 2, 3 | 8 | D, P, None, None, P, 1 << 20, None) == 2  # with STRICT
    assert f(P, P, P, P, P, 4, 16, 2, 3 | D, None, None, None, P, 1 << 20, None) == 1   # no row mask
    assert f(P, P, P, P, P, 4, 16, 2, 2 | D, P, None, None, P, 1 << 20, None) == 1      # SELECT alone
    assert f(P, P, P, P, P, 4, 16, 2, 1 | D, P, None, None, P, 1 << 20, None) == 1      # ACCUMULATE alone
    assert f(P, P, P, P, P, 4, 16, 2, 7 | D, P, None, None, P, 1 << 20, None) == 1      # KEEP_RESIDUAL
    assert f(P, P, P, P, P, 4, 16, 2, 3 | 16 | D, P, None, None, P, 1 << 20, None) == 1  # TENSOR


def test_proxy_topk_argument_errors():
    L = F.lib()
    ws = F.falqon_workspace_size(F.OP_PROXY_UPDATE_TOPK, 0, 4, 16, 2)
    assert ws >= 256 and ws % 256 == 0
    assert F.falqon_workspace_size(F.OP_PROXY_UPDATE_TOPK, 0, 4, 16, 0) == 0
    f = L.falqon_proxy_update_topk
    AS = 1 | 2  # ACCUMULATE | SELECT
    assert f(None, P, P, P, P, 4, 16, 2, 1, AS, None, None, None, P, ws, None) == 1  # no codes
    assert f(P, P, P, None, P, 4, 16, 2, 1, AS, None, None, None, P, ws, None) == 1  # no increment
    assert f(P, P, P, P, None, 4, 16, 2, 1, AS, None, None, None, P, ws, None) == 1  # no A
    assert f(P, P, None, P, P, 4, 16, 2, 1, AS, None, None, None, P, ws, None) == 1  # no proxy
    assert f(P, P, P, P, P, 4, 16, 0, 1, AS, None, None, None, P, ws, None) == 1     # r = 0
    assert f(P, P, P, P, P, 4, 16, 2, -1, AS, None, None, None, P, ws, None) == 1    # k < 0
    assert f(P, P, P, P, P, 4, 16, 2, 1, 0, None, None, None, P, ws, None) == 1      # neither step
    assert f(P, P, P, P, P, 4, 16, 2, 1, AS | 4, None, None, None, P, ws, None) == 1  # no residual form
    assert f(P, P, P, P, P, 4, 16, 2, 1, AS | 16, None, None, None, P, ws, None) == 1  # unknown flag
    assert f(P, P, P, P, P, 0, 16, 2, 1, AS, None, None, None, P, ws, None) == 1     # N = 0
    assert f(P, P, P, P, P, 4, 20, 2, 1, AS, None, None, None, P, ws, None) == 2     # K % 16
    assert f(P, P, P, P, P, 4, 20, 2, 1, AS | 8, None, None, None, P, ws, None) == 2  # STRICT accepted
    assert f(P, P, P, P, P, 4, 16, 16385, 1, AS, None, None, None, P, 1 << 30, None) == 2  # r too large
    assert f(P8, P, P, P, P, 4, 16, 2, 1, AS, None, None, None, P, ws, None) == 2    # unaligned codes
    assert f(P, P, P, P, P, 4, 16, 2, 1, AS, None, None, None, P, ws - 256, None) == 3  # workspace
    assert f(P, P, P, P, P, 4, 16, 2, 1, AS, None, None, None, P8, ws, None) == 3   # misaligned workspace


def test_folded_argument_errors():
    L = F.lib()
    M, N, K, r = 64, 32, 48, 16
    tb = F.falqon_workspace_size(F.OP_FOLDED_T, M, 0, 0, r)
    assert tb == F.falqon_workspace_size(F.OP_LINEAR_BWD_FOLDED, M, N, K, r)
    assert tb >= 2 * 64 * 16 * 2 and tb % 256 == 0  # two bf16 planes [r][M]
    fwd = L.falqon_linear_fwd_folded
    assert fwd(P, P, P, P, None, P, M, N, K, r, P, P, tb, None, None) == 1       # no A~q
    assert fwd(P, P, P, P, P, P, M, N, K, 0, P, P, tb, None, None) == 1          # r = 0
    assert fwd(P, P, P, P, P, P, M, N, K, 24, P, P, tb, None, None) == 2         # r % 16
    assert fwd(P, P, P, P, P, P, M, N, 40, r, P, P, tb, None, None) == 2         # K % 16
    assert fwd(P, P, P, P, P8, P, M, N, K, r, P, P, tb, None, None) == 2         # unaligned A~q
    assert fwd(P, P, P, P, P, P, M, N, K, r, P, P, tb - 256, None, None) == 3    # T buffer too small
    assert fwd(P, P, P, P, P, P, M, N, K, r, P, P8, tb, None, None) == 3         # T buffer misaligned
    bwd = L.falqon_linear_bwd_folded
    args = dict(dyq=P, s_dy=P, wq=P, s_w=P, bq=P, s_b=P, xq=P, s_x=P, t=P, tb=tb, dx=P, dA=P, dB=P, ws=P, wsb=tb)

    def call(**kw):
        a = dict(args, **kw)
        return bwd(a["dyq"], a["s_dy"], a["wq"], a["s_w"], a["bq"], a["s_b"], a["xq"], a["s_x"], a["t"], a["tb"],
                   M, N, K, r, a["dx"], a["dA"], a["dB"], None, a["ws"], a["wsb"], None)
    assert call(dx=None, dA=None, dB=None) == 1   # nothing to compute
    assert call(bq=None) == 1                     # dA needs B~q
    assert call(t=None) == 1                      # dB needs the forward's T
    assert call(tb=tb - 256) == 3                 # T buffer too small
    assert call(ws=None, wsb=0) == 3              # dA needs U's workspace
    assert call(dA=P8) == 2                       # unaligned output


def test_selftest_argument_errors():
    L = F.lib()
    f = L.falqon_selftest_bounded_waits
    assert f(None, P, P, None) == 1
    assert f(P, None, P, None) == 1
    assert f(P, P, None, None) == 1


@pytest.mark.parametrize("name", ["falqon_quantize", "falqon_linear_fwd"])
def test_binding_refuses_cpu_tensors(name):
    import torch

    x = torch.zeros(4, 16)
    with pytest.raises(ValueError):
        if name == "falqon_quantize":
            F.falqon_quantize(x)
        else:
            F.falqon_linear_fwd(x.to(torch.uint8), torch.ones(1), x.to(torch.uint8), torch.ones(1))


def test_noalloc_reports_argument_errors_like_the_workspace_call():
    """The no-allocation backward runs falqon_linear_bwd's argument checks
    before its own scratch-size check: the same bad arguments give the same
    status, even on a problem too large for its scratch."""
    L = F.lib()
    bwd, na = L.falqon_linear_bwd, L.falqon_linear_bwd_noalloc
    big = 1 << 40  # a workspace size that never limits falqon_linear_bwd's checks

    def both(M, N, K, r, dx=P, dA=P, dB=P, A=P, dyq=P):
        s1 = bwd(dyq, P, P, P, P, P, A, P, M, N, K, r, dx, dA, dB, None, P, big, None)
        s2 = na(dyq, P, P, P, P, P, A, P, M, N, K, r, dx, dA, dB, None, None)
        return s1, s2
    M = 32768  # with r = 256 the intermediates need 64 MiB, beyond the 16 MiB scratch
    assert both(M, 256, 256, 24) == (2, 2)            # r % 16: UNSUPPORTED first
    assert both(M, 256, 256, 256, A=None) == (1, 1)   # no A: INVALID_ARG first
    assert both(M, 250, 256, 256) == (2, 2)           # N % 16
    assert both(M, 256, 256, 256, dyq=P8) == (2, 2)   # unaligned codes
    assert both(M, 256, 256, 256, dx=None, dA=None, dB=None) == (1, 1)
    assert na(P, P, P, P, P, P, P, P, M, 256, 256, 256, P, P, P, None, None) == 3  # then the scratch limit


def test_workspace_init_argument_errors():
    L = F.lib()
    assert L.falqon_workspace_init(None, 256, None) == 1   # no workspace
    assert L.falqon_workspace_init(P, 0, None) == 1        # no bytes
    assert L.falqon_workspace_init(P8, 256, None) == 3     # not 256-byte aligned


def test_separate_path_argument_errors():
    L = F.lib()
    M, N, K, r = 64, 32, 48, 16
    sb = F.falqon_workspace_size(F.OP_SEPARATE_SAVED_FP8, M, N, K, r)
    wf = F.falqon_workspace_size(F.OP_SEPARATE_FWD_FP8, M, N, K, r)
    wb = F.falqon_workspace_size(F.OP_SEPARATE_BWD_FP8, M, N, K, r)
    assert sb % 256 == 0 and wf % 256 == 0 and wb % 256 == 0
    assert F.falqon_workspace_size(F.OP_SEPARATE_SAVED_BF16, M, N, K, r) < sb
    fwd, bwd = L.falqon_lora_separate_fwd, L.falqon_lora_separate_bwd

    def f(prec=1, x=P, A=P, y=P, r_=r, K_=K, saved=P, sbytes=sb, ws=P, wsb=wf):
        return fwd(prec, P, P, x, P, P, A, P, M, N, K_, r_, y, saved, sbytes, None, ws, wsb, None)
    assert f(prec=2) == 1                 # unknown precision
    assert f(A=None) == 1                 # no A
    assert f(prec=0, x=None) == 1         # the bf16 path reads X
    assert f(r_=24) == 2                  # r % 16
    assert f(K_=40) == 2                  # K % 16
    assert f(y=P8) == 2                   # unaligned output
    assert f(sbytes=sb - 256) == 3        # saved buffer too small
    assert f(ws=None, wsb=0) == 3         # the FP8 forward needs its quantize workspace

    def b(prec=1, dx=P, dA=P, dB=P, xq=P, x=P, dy=P, ws=P, wsb=wb):
        return bwd(prec, P, P, dy, P, P, xq, P, x, P, P, P, sb, M, N, K, r, dx, dA, dB, None, ws, wsb, None)
    assert b(dx=None, dA=None, dB=None) == 1  # nothing to compute
    assert b(xq=None) == 1                    # FP8 dA reads the codes of X
    assert b(prec=0, dy=None) == 1            # the bf16 path reads dY
    assert b(wsb=wb - 256) == 3               # workspace too small


def test_proxy_tensor_flag_errors():
    L = F.lib()
    f = L.falqon_proxy_update
    ws = 1 << 20
    assert f(P, P, P, P, P, 4, 16, 16, 2 | 16, None, None, None, P, ws, None) == 1       # TENSOR without ACCUMULATE
    assert f(P, P, P, P, P, 4, 16, 16, 1 | 8 | 16, None, None, None, P, ws, None) == 1   # TENSOR with STRICT
    assert f(P, P, P, P, P, 4, 16, 12, 1 | 16, None, None, None, P, ws, None) == 2       # r % 8
    assert f(P, P, P, P8, P, 4, 16, 16, 1 | 16, None, None, None, P, ws, None) == 2      # unaligned dB_inc


def test_grouped_forward_argument_errors():
    L = F.lib()
    f = L.falqon_linear_fwd_grouped
    arr = lambda *v: (C.c_void_p * len(v))(*v)
    n = lambda *v: (C.c_int64 * len(v))(*v)
    assert f(P, P, 0, arr(P), arr(P), n(16), arr(P), 64, 32, None, None) == 1        # no segment
    assert f(P, P, 4, arr(P, P, P, P), arr(P, P, P, P), n(16, 16, 16, 16), arr(P, P, P, P), 64, 32, None, None) == 1
    assert f(P, P, 2, arr(P, None), arr(P, P), n(16, 16), arr(P, P), 64, 32, None, None) == 1  # a missing backbone
    assert f(P, P, 2, arr(P, P), arr(P, P), n(16, 24), arr(P, P), 64, 32, None, None) == 2     # N % 16
    assert f(P, P, 1, arr(P), arr(P), n(16), arr(P8), 64, 32, None, None) == 2                # unaligned output
    assert f(P, P, 1, arr(P), arr(P), n(16), arr(P), 64, 40, None, None) == 2                 # K % 16


C_CALLER = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "falqon.h"

/* A C99 caller of the library: host-side queries and argument checks only
   (fake device addresses, rejected before any CUDA call). */
int main(void) {
  void* p = (void*)(uintptr_t)(1u << 20);
  uint8_t* p8 = (uint8_t*)p;
  float* pf = (float*)p;
  size_t q = falqon_workspace_size(FALQON_OP_QUANTIZE, 4096, 4096, 0, 0);
  size_t pu = falqon_workspace_size(FALQON_OP_PROXY_UPDATE, 0, 4096, 4096, 64);
  printf("version %s\n", falqon_version());
  printf("ok %s\n", falqon_status_string(FALQON_OK));
  printf("sizes %d %d\n", q > 0 && q % 256 == 0, pu > 0 && pu % 256 == 0);
  printf("init %d\n", (int)falqon_workspace_init(NULL, 256, NULL));
  printf("quantize %d %d %d\n",
         (int)falqon_quantize(NULL, FALQON_DTYPE_BF16, 4, 16, p8, pf, NULL, NULL, NULL, p, q, NULL),
         (int)falqon_quantize(p, FALQON_DTYPE_BF16, 4, 24, p8, pf, NULL, NULL, NULL, p, q, NULL),
         (int)falqon_quantize(p, FALQON_DTYPE_BF16, 4, 16, p8, pf, NULL, NULL, NULL, p, 8, NULL));
  printf("proxy %d\n", (int)falqon_proxy_update(p8, pf, pf, p, p, 4, 16, 2, 3u | FALQON_PROXY_DEFER_CLEAR,
                                                NULL, NULL, NULL, p, pu, NULL));
  return 0;
}
"""


def test_a_c99_program_builds_links_and_calls_the_library(tmp_path):
    """The boundary is a C ABI: a plain C99 program compiles against
    include/falqon.h (warnings are errors), links the shared library and gets
    the documented statuses for argument errors without a GPU."""
    import shutil

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    F.lib()  # the library is built
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(F.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(exe), "-L", libdir, "-lfalqon", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    got = dict(line.split(" ", 1) for line in out)
    assert "sm_100a" in got["version"]
    assert got["ok"] == "ok"
    assert got["sizes"] == "1 1"
    assert got["init"] == "1"                  # no workspace
    assert got["quantize"] == "1 2 3"          # null x; cols not a multiple of 16; workspace too small
    assert got["proxy"] == "1"                 # DEFER_CLEAR without the row mask


def test_workspace_sizes_of_every_op_and_the_large_rank_path():
    """Every op's workspace size is a multiple of 256 bytes; the backward's
    grows with r, and from r = 512 (M % 8 == 0) it holds the codes of X and
    dY expanded to bf16 once (2 bytes per code), which the rank-on-M path
    never stores."""
    M, N, K = 4096, 4096, 4096
    for op in range(12):
        for r in (16, 64, 512):
            n = F.falqon_workspace_size(op, M, N, K, r)
            assert n % 256 == 0, (op, r, n)
    bwd = [F.falqon_workspace_size(F.OP_LINEAR_BWD, M, N, K, r) for r in (16, 64, 256, 512, 1024)]
    assert bwd == sorted(bwd) and bwd[0] > 0
    assert bwd[2] < 2 * M * (K + N) <= bwd[3]
    # M not a multiple of 8 keeps the rank-on-M path (no expanded codes)
    assert F.falqon_workspace_size(F.OP_LINEAR_BWD, M - 1, N, K, 512) < 2 * (M - 1) * (K + N)
