"""ctypes binding of liblmhead.so: the five calls of include/lmhead.h.

Argument marshalling only: shapes, dtypes and device pointers are read off
torch tensors and passed to the C ABI on the caller's current CUDA stream.
All arithmetic happens in the library's kernels.  If the library is missing
or cannot be loaded, every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblmhead.so")

LMH_OK, LMH_ERR_INVALID_ARG, LMH_ERR_MISALIGNED, LMH_ERR_UNSUPPORTED, LMH_ERR_CUDA = range(5)
F32, BF16, F16 = 0, 1, 2
DEV_BAD_TARGET = 0x1
DEV_PIPE_TIMEOUT = 0x2
IGNORE_INDEX = -100

EXPORTS = ("lmhead_fwd", "ce_fwd", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw",
           "lmhead_fwd_ce", "lmhead_fwd_ce_workspace_bytes", "lmhead_fwd_ce_noalloc",
           "lmhead_bwd_dw_acc", "ce_fwd_shard", "ce_merge_shards", "ce_bwd_shard",
           "lmh_status_string", "lmh_version", "lmh_watchdog_selftest",
           "lmh_gemm_watchdog_selftest")

_lib = None


class LmhError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def lib() -> ctypes.CDLL:
    """Load liblmhead.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"liblmhead.so not found at {LIB_PATH}; build it with "
                               "`python -m lm_head_fp32_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.lmhead_fwd.argtypes = [P, P, P, I32, I64, I64, I64, P, P]
        L.ce_fwd.argtypes = [P, P, P, I64, I64, I64, P, P]
        L.ce_bwd.argtypes = [P, P, P, P, I64, P, I32, I64, I64, I64, P, P]
        L.lmhead_bwd_dx.argtypes = [P, P, P, I32, I64, I64, I64, P, P]
        L.lmhead_bwd_dw.argtypes = [P, P, P, I32, I64, I64, I64, P, P]
        for f in ("lmhead_fwd", "ce_fwd", "ce_bwd", "lmhead_bwd_dx", "lmhead_bwd_dw"):
            getattr(L, f).restype = ctypes.c_int
        L.lmh_status_string.argtypes = [ctypes.c_int]
        L.lmh_status_string.restype = ctypes.c_char_p
        L.lmh_version.restype = ctypes.c_int32
        L.lmhead_fwd_ce.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64, I64, P, P]
        L.lmhead_fwd_ce.restype = ctypes.c_int
        L.ce_fwd_shard.argtypes = [P, P, P, I64, I64, I64, I64, I64, P, P]
        L.ce_merge_shards.argtypes = [P, I64, P, P, I64, I64, I64, P, P]
        L.ce_bwd_shard.argtypes = [P, P, P, P, I64, P, I32, I64, I64, I64, I64, I64, P, P]
        for f in ("ce_fwd_shard", "ce_merge_shards", "ce_bwd_shard"):
            getattr(L, f).restype = ctypes.c_int
        L.lmhead_bwd_dw_acc.argtypes = [P, P, P, I64, I64, I64, P, P]
        L.lmhead_bwd_dw_acc.restype = ctypes.c_int
        L.lmhead_fwd_ce_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, P]
        L.lmhead_fwd_ce_noalloc.restype = ctypes.c_int
        L.lmhead_fwd_ce_workspace_bytes.argtypes = [I64, I64]
        L.lmhead_fwd_ce_workspace_bytes.restype = I64
        L.lmh_watchdog_selftest.argtypes = [P, I64, P]
        L.lmh_watchdog_selftest.restype = ctypes.c_int
        L.lmh_gemm_watchdog_selftest.argtypes = [P, P, P, I64, I64, I64, I64, P, P]
        L.lmh_gemm_watchdog_selftest.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().lmh_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float16:
        return F16          # passed through so that the library rejects it
    raise TypeError(f"unsupported dtype {dt}")


def _check(code: int, where: str):
    if code != LMH_OK:
        raise LmhError(code, where)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major)")


def lmhead_fwd(X: torch.Tensor, W: torch.Tensor, logits: torch.Tensor,
               status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """logits[M,V] (FP32 or BF16) = X[M,K] . W[V,K]^T."""
    _contig(X, W, logits)
    M, K = X.shape
    V = W.shape[0]
    assert W.shape[1] == K and tuple(logits.shape) == (M, V)
    _check(lib().lmhead_fwd(_ptr(X), _ptr(W), _ptr(logits), _dtype_code(logits.dtype),
                            M, K, V, _ptr(status), _stream(stream)), "lmhead_fwd")
    return logits


def ce_fwd(logits: torch.Tensor, target: torch.Tensor, stats: torch.Tensor,
           ignore_index: int = IGNORE_INDEX, status: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """stats[M,4] = {m, d, x_y, loss} per row of FP32 logits."""
    _contig(logits, target, stats)
    M, V = logits.shape
    assert tuple(stats.shape) == (M, 4) and target.shape[0] == M
    _check(lib().ce_fwd(_ptr(logits), _ptr(target), _ptr(stats), M, V, int(ignore_index),
                        _ptr(status), _stream(stream)), "ce_fwd")
    return stats


def ce_bwd(logits: torch.Tensor, target: torch.Tensor, stats: torch.Tensor,
           grad_loss: torch.Tensor, dlogits: torch.Tensor, ignore_index: int = IGNORE_INDEX,
           status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dlogits = (softmax - onehot) * grad_loss in FP32, stored FP32 or BF16.
    grad_loss: one element (broadcast to every row) or M elements."""
    _contig(logits, target, stats, grad_loss, dlogits)
    M, V = logits.shape
    assert tuple(dlogits.shape) == (M, V)
    stride = 0 if grad_loss.numel() == 1 else 1
    if stride == 1:
        assert grad_loss.numel() == M
    _check(lib().ce_bwd(_ptr(logits), _ptr(target), _ptr(stats), _ptr(grad_loss), stride,
                        _ptr(dlogits), _dtype_code(dlogits.dtype), M, V, int(ignore_index),
                        _ptr(status), _stream(stream)), "ce_bwd")
    return dlogits


def lmhead_fwd_ce_workspace_bytes(M: int, V: int) -> int:
    """Scratch bytes lmhead_fwd_ce needs for M tokens and a vocabulary of V."""
    return int(lib().lmhead_fwd_ce_workspace_bytes(int(M), int(V)))


def lmhead_fwd_ce(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor, logits: torch.Tensor,
                  stats: torch.Tensor, workspace: torch.Tensor,
                  ignore_index: int = IGNORE_INDEX, status: Optional[torch.Tensor] = None,
                  stream=None):
    """FP32 logits = X . W^T and stats[M,4] = {m, d, x_y, loss} in one pass over
    the logits; `workspace` is caller-owned scratch (uint8, see
    lmhead_fwd_ce_workspace_bytes)."""
    _contig(X, W, target, logits, stats, workspace)
    M, K = X.shape
    V = W.shape[0]
    assert W.shape[1] == K and tuple(logits.shape) == (M, V) and tuple(stats.shape) == (M, 4)
    assert logits.dtype == torch.float32
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().lmhead_fwd_ce(_ptr(X), _ptr(W), _ptr(target), _ptr(logits), _ptr(stats),
                               _ptr(workspace), nbytes, M, K, V, int(ignore_index), _ptr(status),
                               _stream(stream)), "lmhead_fwd_ce")
    return logits, stats


def lmhead_fwd_ce_noalloc(X: torch.Tensor, W: torch.Tensor, target: torch.Tensor,
                          logits: torch.Tensor, stats: torch.Tensor,
                          ignore_index: int = IGNORE_INDEX, status: Optional[torch.Tensor] = None,
                          stream=None):
    """lmhead_fwd_ce without a workspace, for callers that cannot allocate
    device memory: the partial statistics live in a fixed 8 MiB array inside
    the library (M * 2 * ceil(V/256) <= 1048576).  Calls that overlap on the
    GPU share that array and race."""
    _contig(X, W, target, logits, stats)
    M, K = X.shape
    V = W.shape[0]
    assert W.shape[1] == K and tuple(logits.shape) == (M, V) and tuple(stats.shape) == (M, 4)
    assert logits.dtype == torch.float32
    _check(lib().lmhead_fwd_ce_noalloc(_ptr(X), _ptr(W), _ptr(target), _ptr(logits), _ptr(stats),
                                       M, K, V, int(ignore_index), _ptr(status), _stream(stream)),
           "lmhead_fwd_ce_noalloc")
    return logits, stats


def lmhead_bwd_dx(dlogits: torch.Tensor, W: torch.Tensor, dX: torch.Tensor,
                  status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dX[M,K] = dlogits[M,V] . W[V,K]."""
    _contig(dlogits, W, dX)
    M, V = dlogits.shape
    K = W.shape[1]
    assert W.shape[0] == V and tuple(dX.shape) == (M, K)
    _check(lib().lmhead_bwd_dx(_ptr(dlogits), _ptr(W), _ptr(dX), _dtype_code(dX.dtype),
                               M, K, V, _ptr(status), _stream(stream)), "lmhead_bwd_dx")
    return dX


def lmhead_bwd_dw(dlogits: torch.Tensor, X: torch.Tensor, dW: torch.Tensor,
                  status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dW[V,K] = dlogits[M,V]^T . X[M,K]."""
    _contig(dlogits, X, dW)
    M, V = dlogits.shape
    K = X.shape[1]
    assert X.shape[0] == M and tuple(dW.shape) == (V, K)
    _check(lib().lmhead_bwd_dw(_ptr(dlogits), _ptr(X), _ptr(dW), _dtype_code(dW.dtype),
                               M, K, V, _ptr(status), _stream(stream)), "lmhead_bwd_dw")
    return dW


def watchdog_selftest(status: torch.Tensor, limit_us: int = 1000, stream=None) -> None:
    """Make one bounded pipeline wait run out on purpose; sets DEV_PIPE_TIMEOUT."""
    _check(lib().lmh_watchdog_selftest(_ptr(status), int(limit_us), _stream(stream)),
           "lmh_watchdog_selftest")


def gemm_watchdog_selftest(X: torch.Tensor, W: torch.Tensor, logits: torch.Tensor,
                           status: torch.Tensor, limit_ns: int = 1, stream=None) -> None:
    """lmhead_fwd (FP32 logits) with every pipeline wait limited to limit_ns:
    the GEMM's own timeout path, which sets DEV_PIPE_TIMEOUT."""
    _contig(X, W, logits)
    M, K = X.shape
    V = W.shape[0]
    assert W.shape[1] == K and tuple(logits.shape) == (M, V) and logits.dtype == torch.float32
    _check(lib().lmh_gemm_watchdog_selftest(_ptr(X), _ptr(W), _ptr(logits), M, K, V,
                                            int(limit_ns), _ptr(status), _stream(stream)),
           "lmh_gemm_watchdog_selftest")


def lmhead_bwd_dw_acc(dlogits: torch.Tensor, X: torch.Tensor, dW: torch.Tensor,
                      status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dW[V,K] (FP32) += dlogits[M,V]^T . X[M,K]."""
    _contig(dlogits, X, dW)
    M, V = dlogits.shape
    K = X.shape[1]
    assert X.shape[0] == M and tuple(dW.shape) == (V, K) and dW.dtype == torch.float32
    _check(lib().lmhead_bwd_dw_acc(_ptr(dlogits), _ptr(X), _ptr(dW), M, K, V, _ptr(status),
                                   _stream(stream)), "lmhead_bwd_dw_acc")
    return dW


def ce_fwd_shard(logits: torch.Tensor, target: torch.Tensor, shard_stats: torch.Tensor,
                 vocab_offset: int, vocab_total: int, ignore_index: int = IGNORE_INDEX,
                 status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """shard_stats[M,4] = {m_r, d_r, x_y or 0, owner flag} of one vocabulary shard."""
    _contig(logits, target, shard_stats)
    M, V = logits.shape
    assert tuple(shard_stats.shape) == (M, 4)
    _check(lib().ce_fwd_shard(_ptr(logits), _ptr(target), _ptr(shard_stats), M, V,
                              int(vocab_offset), int(vocab_total), int(ignore_index),
                              _ptr(status), _stream(stream)), "ce_fwd_shard")
    return shard_stats


def ce_merge_shards(shard_stats: torch.Tensor, target: torch.Tensor, stats: torch.Tensor,
                    vocab_total: int, ignore_index: int = IGNORE_INDEX,
                    status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """stats[M,4] = {m, d, x_y, loss} from shard_stats[R,M,4] (shard-major)."""
    _contig(shard_stats, target, stats)
    R, M, four = shard_stats.shape
    assert four == 4 and tuple(stats.shape) == (M, 4)
    _check(lib().ce_merge_shards(_ptr(shard_stats), R, _ptr(target), _ptr(stats), M,
                                 int(vocab_total), int(ignore_index), _ptr(status),
                                 _stream(stream)), "ce_merge_shards")
    return stats


def ce_bwd_shard(logits: torch.Tensor, target: torch.Tensor, stats: torch.Tensor,
                 grad_loss: torch.Tensor, dlogits: torch.Tensor, vocab_offset: int,
                 vocab_total: int, ignore_index: int = IGNORE_INDEX,
                 status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """ce_bwd on one vocabulary shard with the merged statistics."""
    _contig(logits, target, stats, grad_loss, dlogits)
    M, V = logits.shape
    stride = 0 if grad_loss.numel() == 1 else 1
    _check(lib().ce_bwd_shard(_ptr(logits), _ptr(target), _ptr(stats), _ptr(grad_loss), stride,
                              _ptr(dlogits), _dtype_code(dlogits.dtype), M, V, int(vocab_offset),
                              int(vocab_total), int(ignore_index), _ptr(status), _stream(stream)),
           "ce_bwd_shard")
    return dlogits
