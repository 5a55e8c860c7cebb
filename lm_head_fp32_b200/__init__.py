"""B200-native LM-head loss path: FP32-output vocabulary GEMM, fused FP32
cross-entropy forward/backward and the two gradient GEMMs, as a C-ABI CUDA
library (``liblmhead.so``) with a thin ctypes binding.

The binding (``lm_head_fp32_b200.lmhead``) loads the library on first use and
raises if it is missing: there is no CPU fallback.  ``lm_head_fp32_b200.loss``
wraps the five calls as a PyTorch autograd function (per-token loss forward,
dX and dW backward).
"""
__all__ = ["lmhead", "loss", "synth"]
