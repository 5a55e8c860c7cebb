"""The C-ABI library loads and exports every symbol include/lmhead.h declares;
host-side validation rejects bad arguments before anything is launched.

No test here launches a kernel or needs a GPU: every call below fails the
host checks (null pointer, bad size, bad dtype, misalignment) and returns
before touching the device.
"""
import ctypes
import os
import re
import subprocess

import pytest

from lm_head_fp32_b200 import lmhead

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lmhead.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*LMH_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_header_declares_the_five_calls():
    fns = declared_functions()
    for f in ("lmhead_fwd", "ce_fwd", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw",
              "lmhead_fwd_ce", "lmhead_fwd_ce_workspace_bytes", "lmh_status_string"):
        assert f in fns


def test_library_exports_every_declared_symbol():
    L = lmhead.lib()
    for f in declared_functions():
        assert hasattr(L, f), f"{f} declared in lmhead.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", lmhead.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared_functions()) <= exported


def test_header_compiles_as_plain_c():
    # the boundary carries no CUDA or torch types: the header builds with gcc alone
    r = subprocess.run(["gcc", "-std=c99", "-fsyntax-only", "-x", "c", HEADER],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_status_strings_and_version():
    assert lmhead.status_string(0) == "ok"
    assert "misaligned" in lmhead.status_string(2)
    assert lmhead.lib().lmh_version() == 20000      # 2.0.0


P = ctypes.c_void_p
NULL = None
A = P(0x10000)     # never dereferenced: each call below fails validation first
UNALIGNED = P(0x10008)


@pytest.mark.parametrize("fn", ["lmhead_fwd", "lmhead_bwd_dx", "lmhead_bwd_dw"])
def test_gemm_validation(fn):
    f = getattr(lmhead.lib(), fn)
    assert f(NULL, A, A, 0, 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, 0, 0, 64, 64, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, 0, 16, 64, 1 << 31, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, lmhead.F16, 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_UNSUPPORTED
    assert f(A, A, A, 7, 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_UNSUPPORTED
    assert f(A, A, A, 0, 16, 60, 64, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED      # K % 8
    assert f(UNALIGNED, A, A, 0, 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED
    assert f(A, A, P(0x10002), 0, 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED


@pytest.mark.parametrize("fn", ["lmhead_bwd_dx", "lmhead_bwd_dw"])
def test_grad_gemm_needs_v_multiple_of_8(fn):
    f = getattr(lmhead.lib(), fn)
    assert f(A, A, A, 0, 16, 64, 100, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED


def test_ce_validation():
    L = lmhead.lib()
    assert L.ce_fwd(NULL, A, A, 4, 10, -100, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert L.ce_fwd(A, A, A, 0, 10, -100, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert L.ce_fwd(A, A, P(0x10004), 4, 10, -100, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED
    assert L.ce_bwd(A, A, A, A, 2, A, 0, 4, 10, -100, NULL, NULL) == lmhead.LMH_ERR_UNSUPPORTED
    assert L.ce_bwd(A, A, A, A, 0, A, lmhead.F16, 4, 10, -100, NULL, NULL) == \
        lmhead.LMH_ERR_UNSUPPORTED
    # an in-place BF16 gradient would overwrite FP32 logits with half-width data
    assert L.ce_bwd(A, A, A, A, 0, A, lmhead.BF16, 4, 10, -100, NULL, NULL) == \
        lmhead.LMH_ERR_UNSUPPORTED
    assert L.ce_bwd(A, A, A, NULL, 0, A, 0, 4, 10, -100, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG


def test_binding_rejects_fp16_like_the_flag():
    import torch
    # the logit dtype option accepts only bf16 and fp32 and rejects fp16
    assert lmhead._dtype_code(torch.float16) == lmhead.F16
    with pytest.raises(TypeError):
        lmhead._dtype_code(torch.int8)


def test_watchdog_selftest_validation():
    L = lmhead.lib()
    assert L.lmh_watchdog_selftest(NULL, 1000, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert L.lmh_watchdog_selftest(A, 0, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert L.lmh_watchdog_selftest(A, 2000000, NULL) == lmhead.LMH_ERR_INVALID_ARG


def test_gemm_watchdog_selftest_validation():
    f = lmhead.lib().lmh_gemm_watchdog_selftest
    assert f(A, A, A, 16, 64, 64, 1, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG   # no status
    assert f(A, A, A, 16, 64, 64, 0, A, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, 16, 64, 64, 2000000000, A, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(NULL, A, A, 16, 64, 64, 1, A, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, 16, 60, 64, 1, A, NULL) == lmhead.LMH_ERR_MISALIGNED       # K % 8


def test_fused_ce_workspace_size_and_validation():
    L = lmhead.lib()
    # two 128-wide vocabulary blocks per 256 columns, one (max, sum-exp) pair each per token
    assert lmhead.lmhead_fwd_ce_workspace_bytes(1024, 32768) == 2 * 128 * 1024 * 8
    assert lmhead.lmhead_fwd_ce_workspace_bytes(16, 1) == 2 * 1 * 16 * 8
    assert lmhead.lmhead_fwd_ce_workspace_bytes(0, 10) == -1
    f = L.lmhead_fwd_ce
    need = lmhead.lmhead_fwd_ce_workspace_bytes(16, 64)
    assert f(NULL, A, A, A, A, A, need, 16, 64, 64, -100, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, A, A, A, need, 16, 60, 64, -100, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED
    assert f(A, A, A, A, P(0x10008), A, need, 16, 64, 64, -100, NULL, NULL) == \
        lmhead.LMH_ERR_MISALIGNED                     # stats not 16-byte aligned
    # the fused path needs the workspace (V % 4 == 0, aligned logits)
    assert f(A, A, A, A, A, NULL, need, 16, 64, 64, -100, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, A, A, A, need - 8, 16, 64, 64, -100, NULL, NULL) == \
        lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, A, A, P(0x10008), need, 16, 64, 64, -100, NULL, NULL) == \
        lmhead.LMH_ERR_MISALIGNED


def test_dw_accumulate_validation():
    f = lmhead.lib().lmhead_bwd_dw_acc
    assert f(NULL, A, A, 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_INVALID_ARG
    assert f(A, A, A, 16, 60, 64, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED
    assert f(A, A, A, 16, 64, 60, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED
    assert f(A, A, P(0x10002), 16, 64, 64, NULL, NULL) == lmhead.LMH_ERR_MISALIGNED
