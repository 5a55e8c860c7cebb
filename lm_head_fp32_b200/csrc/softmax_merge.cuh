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
