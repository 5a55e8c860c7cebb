// softmax_merge.cuh -- the associative (max, sum-exp) pair of the online
// softmax, shared by the cross-entropy kernels and the fused statistics in
// the vocabulary GEMM's epilogue.
//
// TransformerEngine #2325 "[Pytorch] change fused cross entropy backward grad
// to fp32 and reduce one read", review discussion: the forward keeps per row
// the maximum m and the sum d of exp(x - m) (with the target logit), from
// which the loss and, later, the gradient are recomputed.
#pragma once
#include <cmath>

namespace lmh {

constexpr float kLog2e = 1.4426950408889634f;  // 1 / ln 2

struct MaxSum {
    float m;  // running maximum
    float d;  // sum of exp(x - m)
};

// exp(t) for t <= 0, via the hardware base-2 exponential.
__device__ __forceinline__ float exp_neg(float t) { return exp2f(t * kLog2e); }

// exp(t) for t <= 0 through the approximate base-2 exponential with results
// below the smallest normal float flushed to zero (PTX ex2.approx.ftz.f32):
// fewer instructions than exp_neg where they share the SMs with the tensor
// pipe.  A flushed term is below 2^-126, and every sum it enters holds a term
// exp(0) = 1, so flushing moves no such sum.
__device__ __forceinline__ float exp_neg_ftz(float t)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(t * kLog2e));
    return y;
}

// Merge two (max, sum-exp) pairs: the associative step of the online softmax.
__device__ __forceinline__ MaxSum merge(MaxSum a, MaxSum b)
{
    if (a.m < b.m) {
        MaxSum t = a;
        a = b;
        b = t;
    }
    // a.m >= b.m; b.m == -inf means b holds nothing
    if (b.m == -INFINITY)
        return a;
    return MaxSum{a.m, a.d + b.d * exp_neg(b.m - a.m)};
}

}  // namespace lmh
