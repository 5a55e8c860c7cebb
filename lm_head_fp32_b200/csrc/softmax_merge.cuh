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
// pipe.  A flushed term is below 2^-126: it moves no sum that holds the term
// exp(0) = 1 of its block's maximum, and in the one block per row whose sum
// leaves out the target's term it can only move losses below ~1e-35.
__device__ __forceinline__ float exp_neg_ftz(float t)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(t * kLog2e));
    return y;
}

// Per-row loss -log softmax_y from the row maximum m, the sum dx of
// exp(x_j - m) over every column but the target, and the target logit x_y:
// log((dx + e) / e) with e = exp(x_y - m), i.e. log1p(dx * exp(m - x_y)).
// Kept apart from the target's own term, dx is not rounded away when the
// target holds nearly all of the row's mass (e = 1, dx tiny), where
// m + log(d) - x_y would return 0.  Where exp(m - x_y) would overflow the
// target lies far below the maximum, so dx >= 1 and (m - x_y) + log(dx) is
// the loss to rounding.
__device__ __forceinline__ float ce_loss(float m, float dx, float xy)
{
    const float t = m - xy;  // >= 0
    return t < 64.f ? log1pf(dx * expf(t)) : t + logf(dx);
}

// The row's full sum d = dx + exp(x_y - m) for the saved statistics.
__device__ __forceinline__ float ce_full_sum(float m, float dx, float xy) { return dx + exp_neg(xy - m); }

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
