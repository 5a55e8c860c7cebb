"""FP64 CPU oracle for the LM-head loss path (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product library never imports this package, and this package
never imports the product.  It shares no code with the CUDA path; the seeded
input generators (``lm_head_fp32_b200.synth``) are the only thing both sides
consume, and they hold none of the method's arithmetic.

Sources (page title, section):
  * Megatron-LM PR #6252 "Add mixed-precision (FP32) LM output logits",
    "What does this PR do?", "Tests", "Integer bitwise exactness results".
  * TransformerEngine #2325 "[Pytorch] change fused cross entropy backward
    grad to fp32 and reduce one read", "Description", "Changes", discussion.

Every array function takes numpy arrays (bf16 passed as uint16 bit patterns)
and returns FP64 results; rounding to the dtype under test is separate
(``round_f32``, ``round_bf16``) so that it happens exactly once.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ROW_VALID = 0
ROW_IGNORED = 1
ROW_BAD_TARGET = 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain C, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f64.restype = ctypes.c_double
        L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.oracle_logits.argtypes = [P, P, I64, I64, I64, P, I64, P]
        L.oracle_ce_fwd.argtypes = [P, P, I64, I64, I64, P, I64, P, P]
        L.oracle_ce_bwd.argtypes = [P, P, P, I64, I64, I64, I64, P, I64, P]
        L.oracle_dx.argtypes = [P, P, I64, I64, I64, P, I64, P]
        L.oracle_dw.argtypes = [P, P, I64, I64, I64, P, I64, P]
        L.oracle_round_f32.argtypes = [P, I64, P]
        L.oracle_round_bf16.argtypes = [P, I64, P]
        L.oracle_num_threads.restype = ctypes.c_int
        for f in ("oracle_logits", "oracle_ce_fwd", "oracle_ce_bwd", "oracle_dx", "oracle_dw",
                  "oracle_round_f32", "oracle_round_bf16"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 operands are passed as uint16 bit patterns")
    return a


def _rows(rows, n):
    if rows is None:
        return None, n
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.shape[0]


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def bf16_to_f64(bits: int) -> float:
    return float(lib().oracle_bf16_to_f64(int(bits)))


def f64_to_bf16(v: float) -> int:
    return int(lib().oracle_f64_to_bf16(float(v)))


def logits(X, W, rows=None) -> np.ndarray:
    """FP64 logits[r, v] = sum_k X[i,k] W[v,k] for i = rows[r] (all rows if None)."""
    X, W = _u16(X), _u16(W)
    M, K = X.shape
    V, K2 = W.shape
    assert K == K2
    r, n = _rows(rows, M)
    out = np.empty((n, V), dtype=np.float64)
    lib().oracle_logits(_p(X), _p(W), M, K, V, None if r is None else _p(r), n, _p(out))
    return out


def ce_fwd(logits_f32, target, ignore_index=-100, rows=None):
    """Per-row FP64 stats {m, d, x_y, loss} and the row code (valid/ignored/bad target)."""
    x = np.ascontiguousarray(logits_f32, dtype=np.float32)
    t = np.ascontiguousarray(target, dtype=np.int64)
    M, V = x.shape
    r, n = _rows(rows, M)
    stats = np.empty((n, 4), dtype=np.float64)
    code = np.empty((n,), dtype=np.int32)
    lib().oracle_ce_fwd(_p(x), _p(t), M, V, int(ignore_index), None if r is None else _p(r), n,
                        _p(stats), _p(code))
    return stats, code


def ce_bwd(logits_f32, target, grad_loss, ignore_index=-100, rows=None):
    """FP64 dlogits = (softmax - onehot) * g; grad_loss is a scalar or a per-row array."""
    x = np.ascontiguousarray(logits_f32, dtype=np.float32)
    t = np.ascontiguousarray(target, dtype=np.int64)
    M, V = x.shape
    g = np.ascontiguousarray(np.atleast_1d(np.asarray(grad_loss, dtype=np.float32)))
    stride = 0 if g.shape[0] == 1 else 1
    if stride == 1:
        assert g.shape[0] == M
    r, n = _rows(rows, M)
    out = np.empty((n, V), dtype=np.float64)
    lib().oracle_ce_bwd(_p(x), _p(t), _p(g), stride, M, V, int(ignore_index),
                        None if r is None else _p(r), n, _p(out))
    return out


def dx(dl_bf16, W, rows=None) -> np.ndarray:
    """FP64 dX[r, k] = sum_v dl[i,v] W[v,k]."""
    dl, W = _u16(dl_bf16), _u16(W)
    M, V = dl.shape
    V2, K = W.shape
    assert V == V2
    r, n = _rows(rows, M)
    out = np.empty((n, K), dtype=np.float64)
    lib().oracle_dx(_p(dl), _p(W), M, K, V, None if r is None else _p(r), n, _p(out))
    return out


def dw(dl_bf16, X, vrows=None) -> np.ndarray:
    """FP64 dW[r, k] = sum_i dl[i,v] X[i,k] for v = vrows[r]."""
    dl, X = _u16(dl_bf16), _u16(X)
    M, V = dl.shape
    M2, K = X.shape
    assert M == M2
    r, n = _rows(vrows, V)
    out = np.empty((n, K), dtype=np.float64)
    lib().oracle_dw(_p(dl), _p(X), M, K, V, None if r is None else _p(r), n, _p(out))
    return out


def round_f32(a) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.float32)
    lib().oracle_round_f32(_p(a), a.size, _p(out))
    return out


def round_bf16(a) -> np.ndarray:
    """RNE to bfloat16 directly from FP64; returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_round_bf16(_p(a), a.size, _p(out))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
