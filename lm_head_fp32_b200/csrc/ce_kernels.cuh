// ce_kernels.cuh -- cross-entropy forward statistics and FP32 backward.
//
// TransformerEngine #2325 "[Pytorch] change fused cross entropy backward grad
// to fp32 and reduce one read": the forward makes one pass over each row of
// FP32 logits and saves only the target and m_d_X_y (n_rows x 4) instead of
// writing gradients; the backward recomputes softmax from the saved (m, d) in
// FP32 and writes the gradient, so each kernel reads the logits once.
//
// Both kernels are HBM-bound row sweeps: one CTA per row (the loops also
// stride over rows, so any grid works), 128-bit read-only streaming loads, an
// online (max, sum-exp) pair per thread merged by warp shuffles and then
// across warps in shared memory.
//
// The forward sums exp(x_j - m) over every column but the target (dx) and
// adds the target's term only at the end: the loss log1p(dx * exp(m - x_y))
// and, in the backward, the target's gradient (softmax_y - 1) g =
// expm1(-loss) g then keep their precision on rows whose target holds nearly
// all of the mass, where 1/d - 1 in FP32 would cancel to 0.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "softmax_merge.cuh"

namespace lmh {

// Fold a batch of N values into the running pair: one rescale per batch,
// and the batch's own exponentials are summed first (short partial sums).
template <int N>
__device__ __forceinline__ void fold(MaxSum &s, const float (&v)[N])
{
    float mx = v[0];
#pragma unroll
    for (int i = 1; i < N; ++i)
        mx = fmaxf(mx, v[i]);
    if (mx > s.m) {
        s.d = (s.m == -INFINITY) ? 0.f : s.d * exp_neg(s.m - mx);
        s.m = mx;
    }
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < N; ++i)
        part += exp_neg(v[i] - s.m);
    s.d += part;
}

__device__ __forceinline__ void fold1(MaxSum &s, float x)
{
    if (x > s.m) {
        s.d = (s.m == -INFINITY) ? 0.f : s.d * exp_neg(s.m - x);
        s.m = x;
    }
    s.d += exp_neg(x - s.m);
}

__device__ __forceinline__ float4 ldg_stream(const float4 *p)
{
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float ldg_stream1(const float *p)
{
    float v;
    asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Coherent streaming loads, for a buffer the same kernel also writes (in-place).
__device__ __forceinline__ float4 ld_cs(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ float ld_cs1(const float *p) { return __ldcs(p); }

template <bool ALIAS>
__device__ __forceinline__ float4 load4(const float4 *p) { return ALIAS ? ld_cs(p) : ldg_stream(p); }
template <bool ALIAS>
__device__ __forceinline__ float load1(const float *p) { return ALIAS ? ld_cs1(p) : ldg_stream1(p); }

// Block-wide merge of every thread's pair; the result is valid in all threads.
__device__ __forceinline__ MaxSum block_merge(MaxSum s, MaxSum *red /* [32] */)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        MaxSum t{__shfl_xor_sync(0xffffffffu, s.m, o), __shfl_xor_sync(0xffffffffu, s.d, o)};
        s = merge(s, t);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        red[warp] = s;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        s = lane < nw ? red[lane] : MaxSum{-INFINITY, 0.f};
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            MaxSum t{__shfl_xor_sync(0xffffffffu, s.m, o), __shfl_xor_sync(0xffffffffu, s.d, o)};
            s = merge(s, t);
        }
        if (lane == 0)
            red[0] = s;
    }
    __syncthreads();
    s = red[0];
    __syncthreads();  // red[] may be reused by the next row
    return s;
}

// Row classification shared by both kernels: 0 valid, 1 ignored, 2 bad target.
__device__ __forceinline__ int row_kind(int64_t y, int64_t V, int64_t ignore_index)
{
    if (y == ignore_index)
        return 1;
    if (y < 0 || y >= V)
        return 2;
    return 0;
}

// Component c of a loaded float4 replaced by -inf (the target's column, left
// out of the running pair).
__device__ __forceinline__ void mask_lane(float4 &a, int c)
{
    a.x = c == 0 ? -INFINITY : a.x;
    a.y = c == 1 ? -INFINITY : a.y;
    a.z = c == 2 ? -INFINITY : a.z;
    a.w = c == 3 ? -INFINITY : a.w;
}

// stats[row] = {m, d, x_y, loss}.  VEC: V % 4 == 0 and logits 16-byte aligned.
// The rows hold vocabulary entries [voff, voff + V) of a vocabulary of Vtot
// (voff = 0, Vtot = V for a whole row); targets are global ids.  SHARD: the
// rows are one shard of a vocabulary split across devices, and the record is
// {m, d, x_y or 0, 1 if the target lies in this shard else 0} for
// ce_merge_shards_kernel to combine, where the shard that owns the target
// leaves the target's term out of d (and still counts x_y in m).
template <bool VEC, int THREADS = 512, bool SHARD = false>
__global__ void __launch_bounds__(THREADS, 2048 / THREADS) ce_fwd_kernel(const float *__restrict__ logits,
                                                            const int64_t *__restrict__ target,
                                                            float4 *__restrict__ stats, int64_t M,
                                                            int64_t V, int64_t ignore_index,
                                                            int32_t *status, int64_t voff,
                                                            int64_t Vtot)
{
    __shared__ MaxSum red[32];
    pdl_wait();  // the logits may come from the kernel just before this one
    pdl_launch_dependents();
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
        const int64_t y = target[row];
        const int kind = row_kind(y, Vtot, ignore_index);
        if (kind != 0) {
            if (threadIdx.x == 0) {
                stats[row] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (kind == 2 && status)
                    atomicOr(status, 1);
            }
            continue;  // uniform across the block: no barrier skipped unevenly
        }
        const float *x = logits + row * V;
        // the target logit is fetched up front by the thread that reports the
        // row, so its latency hides behind the row's stream
        const int64_t yl = y - voff;  // local column (may lie outside [0, V) for a shard)
        const bool owner = yl >= 0 && yl < V;
        float xy = 0.f;
        if (threadIdx.x == 0 && owner)
            xy = x[yl];
        MaxSum s{-INFINITY, 0.f};
        if (VEC) {
            const float4 *x4 = reinterpret_cast<const float4 *>(x);
            const int64_t n4 = V >> 2;
            int64_t i = threadIdx.x;
            // the one thread whose vectors include the target's leaves it out
            const int64_t iy = owner ? (yl >> 2) : -1;
            const bool has_y = owner && (iy % THREADS) == threadIdx.x;
            const int cy = static_cast<int>(yl & 3);
            // four independent 128-bit loads in flight per thread per step
            for (; i + 3 * THREADS < n4; i += 4 * THREADS) {
                float4 a = ldg_stream(x4 + i), b = ldg_stream(x4 + i + THREADS),
                       c = ldg_stream(x4 + i + 2 * THREADS),
                       e = ldg_stream(x4 + i + 3 * THREADS);
                if (has_y) {
                    if (i == iy) mask_lane(a, cy);
                    if (i + THREADS == iy) mask_lane(b, cy);
                    if (i + 2 * THREADS == iy) mask_lane(c, cy);
                    if (i + 3 * THREADS == iy) mask_lane(e, cy);
                }
                const float v[16] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w,
                                     c.x, c.y, c.z, c.w, e.x, e.y, e.z, e.w};
                fold<16>(s, v);
            }
            for (; i < n4; i += THREADS) {
                float4 a = ldg_stream(x4 + i);
                if (has_y && i == iy)
                    mask_lane(a, cy);
                const float v[4] = {a.x, a.y, a.z, a.w};
                fold<4>(s, v);
            }
        } else {
            for (int64_t j = threadIdx.x; j < V; j += THREADS)
                if (j != yl)
                    fold1(s, ldg_stream1(x + j));
        }
        s = block_merge(s, red);
        if (threadIdx.x == 0) {
            // (m, dx) over every column but the target; the target joins the
            // maximum here
            float m = s.m, dx = s.d;
            if (owner && xy > m) {
                dx = m == -INFINITY ? 0.f : dx * exp_neg(m - xy);
                m = xy;
            }
            if (SHARD)
                stats[row] = make_float4(m, dx, xy, owner ? 1.f : 0.f);
            else
                stats[row] = make_float4(m, ce_full_sum(m, dx, xy), xy, ce_loss(m, dx, xy));
        }
    }
}

template <typename OutT>
__device__ __forceinline__ void store4(OutT *p, float a, float b, float c, float d);

template <>
__device__ __forceinline__ void store4<float>(float *p, float a, float b, float c, float d)
{
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}

template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, float a, float b, float c,
                                                      float d)
{
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
}

__device__ __forceinline__ void store1(float *p, float a) { *p = a; }
__device__ __forceinline__ void store1(__nv_bfloat16 *p, float a) { *p = __float2bfloat16_rn(a); }

// dl[row, j] = (exp(x - m) / d - [j == y]) * g, FP32 arithmetic, rounded to
// OutT only at the store; at the target, softmax_y - 1 = exp(-loss) - 1 is
// taken as expm1(-loss) from the saved loss, so that it does not cancel when
// softmax_y is close to 1 (the thread that stored the target's entry with the
// rest of its vector overwrites it).  Ignored / bad-target rows are written
// as zeros.
// VEC: V % 4 == 0, logits 16-byte and dl (4 * sizeof(OutT))-byte aligned.
// Each element is read before it is written, by the same thread, so dl may
// alias logits when OutT is float (ALIAS: coherent loads instead of the
// read-only path).
// The rows hold vocabulary entries [voff, voff + V) of a vocabulary of Vtot
// (a shard when voff > 0 or V < Vtot): the one-hot is at the global target.
template <typename OutT, bool VEC, bool ALIAS, int THREADS = 512>
__global__ void __launch_bounds__(THREADS, 2048 / THREADS) ce_bwd_kernel(
    const float *logits, const int64_t *__restrict__ target, const float4 *__restrict__ stats,
    const float *__restrict__ grad_loss, int64_t grad_stride, OutT *dl, int64_t M, int64_t V,
    int64_t ignore_index, int32_t *status, int64_t voff, int64_t Vtot)
{
    pdl_wait();
    pdl_launch_dependents();
    // rows in the opposite order to ce_fwd: the rows it read last are the
    // ones most likely still in L2
    for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
        const int64_t row = M - 1 - r;
        const int64_t yg = target[row];
        const int kind = row_kind(yg, Vtot, ignore_index);
        const int64_t y = yg - voff;  // local column of the target (may lie outside [0, V))
        const float *x = logits + row * V;
        OutT *o = dl + row * V;
        // issued before the branch so that their latency overlaps the target's
        const float4 st = stats[row];
        const float g = grad_loss[row * grad_stride];
        if (kind != 0) {
            if (kind == 2 && status && threadIdx.x == 0)
                atomicOr(status, 1);
            if (VEC) {
                for (int64_t i = threadIdx.x; i < (V >> 2); i += THREADS)
                    store4<OutT>(o + 4 * i, 0.f, 0.f, 0.f, 0.f);
            } else {
                for (int64_t j = threadIdx.x; j < V; j += THREADS)
                    store1(o + j, 0.f);
            }
            continue;
        }
        const float m = st.x;
        const float gd = g / st.y;  // g / d: softmax_j g = exp(x_j - m) gd
        // the thread that stores the target's entry with the rest of its vector
        const bool own_y = y >= 0 && y < V && ((VEC ? (y >> 2) : y) % THREADS) == threadIdx.x;
        const float gy = own_y ? expm1f(-st.w) * g : 0.f;
        if (VEC) {
            const float4 *x4 = reinterpret_cast<const float4 *>(x);
            const int64_t n4 = V >> 2;
            int64_t i = threadIdx.x;
            // four independent 128-bit loads in flight per thread per step
            for (; i + 3 * THREADS < n4; i += 4 * THREADS) {
                float4 a[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    a[u] = load4<ALIAS>(x4 + i + u * THREADS);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    store4<OutT>(o + 4 * (i + u * THREADS), exp_neg(a[u].x - m) * gd,
                                 exp_neg(a[u].y - m) * gd, exp_neg(a[u].z - m) * gd,
                                 exp_neg(a[u].w - m) * gd);
            }
            for (; i < n4; i += THREADS) {
                const float4 a = load4<ALIAS>(x4 + i);
                store4<OutT>(o + 4 * i, exp_neg(a.x - m) * gd, exp_neg(a.y - m) * gd,
                             exp_neg(a.z - m) * gd, exp_neg(a.w - m) * gd);
            }
        } else {
            for (int64_t j = threadIdx.x; j < V; j += THREADS)
                store1(o + j, exp_neg(load1<ALIAS>(x + j) - m) * gd);
        }
        // the target's entry, over the one stored above (program order)
        if (own_y)
            store1(o + y, gy);
    }
}

// stats[i] = {m, d, x_y, loss} from R shard records (ce_fwd_kernel with
// SHARD) laid out shard-major, shard_stats[r * M + i]: the pairs are merged
// in shard order (their sums leave out the target's term, which the owning
// shard dropped) and x_y comes from the shard that owns the target.
__global__ void __launch_bounds__(256)
    ce_merge_shards_kernel(const float4 *__restrict__ shard_stats, int64_t R,
                           const int64_t *__restrict__ target, float4 *__restrict__ stats, int64_t M,
                           int64_t Vtot, int64_t ignore_index, int32_t *status)
{
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < M;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int kind = row_kind(target[i], Vtot, ignore_index);
        if (kind != 0) {
            stats[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (kind == 2 && status)
                atomicOr(status, 1);
            continue;
        }
        MaxSum s{-INFINITY, 0.f};
        float xy = 0.f;
        for (int64_t r = 0; r < R; ++r) {
            const float4 q = shard_stats[r * M + i];
            s = merge(s, MaxSum{q.x, q.y});
            if (q.w != 0.f)
                xy = q.z;
        }
        stats[i] = make_float4(s.m, ce_full_sum(s.m, s.d, xy), xy, ce_loss(s.m, s.d, xy));
    }
}

// stats[i] = {m, d, x_y, loss} from the per-slice partials the fused
// vocabulary GEMM wrote (partial[s * M + i]; the target logit is already in
// stats[i].x_y).  One CTA per kFinalizeTokens = 8 tokens: lane = (slice
// offset 0..3) x (token 0..7), so a warp-wide load reads four 64-byte runs of
// eight consecutive tokens; warp w takes slice groups w, w + WARPS, ...
// (eight loads in flight per lane).  The four lanes of a token are merged by
// shuffles and the warps by warp 0 in a fixed order, so the result does not
// depend on scheduling.
constexpr int kFinalizeTokens = 8;

template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    ce_finalize_kernel(const float2 *__restrict__ partial, int64_t nslices,
                       const int64_t *__restrict__ target, float4 *stats, int64_t M, int64_t V,
                       int64_t ignore_index, int32_t *status)
{
    constexpr int T = kFinalizeTokens;
    constexpr int SL = 32 / T;  // slices per warp-wide load
    __shared__ MaxSum red[WARPS][T];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tok = static_cast<int64_t>(blockIdx.x) * T + (lane % T);
    const int64_t sl0 = lane / T;
    MaxSum s{-INFINITY, 0.f};
    if (tok < M) {
        int64_t g = warp;  // slice group: slices g * SL + sl0
        for (; (g + 7 * WARPS) * SL < nslices; g += 8 * WARPS) {
            float2 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t sl = (g + u * WARPS) * SL + sl0;
                v[u] = sl < nslices ? partial[sl * M + tok] : make_float2(-INFINITY, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                s = merge(s, MaxSum{v[u].x, v[u].y});
        }
        for (; g * SL < nslices; g += WARPS) {
            const int64_t sl = g * SL + sl0;
            if (sl < nslices) {
                const float2 v = partial[sl * M + tok];
                s = merge(s, MaxSum{v.x, v.y});
            }
        }
    }
#pragma unroll
    for (int off = T; off < 32; off <<= 1) {
        const MaxSum o{__shfl_xor_sync(0xffffffffu, s.m, off), __shfl_xor_sync(0xffffffffu, s.d, off)};
        s = merge(s, o);
    }
    if (lane < T)
        red[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && lane < T && tok < M) {
        MaxSum r = red[0][lane];
#pragma unroll
        for (int w = 1; w < WARPS; ++w)
            r = merge(r, red[w][lane]);
        const int64_t y = target[tok];
        const int kind = row_kind(y, V, ignore_index);
        if (kind != 0) {
            stats[tok] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (kind == 2 && status)
                atomicOr(status, 1);
        } else {
            // the partials leave out the target's term (see ce_subtile_stats)
            const float xy = reinterpret_cast<const float *>(stats)[tok * 4 + 2];
            stats[tok] = make_float4(r.m, ce_full_sum(r.m, r.d, xy), xy, ce_loss(r.m, r.d, xy));
        }
    }
}

}  // namespace lmh
