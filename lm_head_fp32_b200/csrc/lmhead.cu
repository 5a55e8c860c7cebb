// lmhead.cu -- C ABI of the LM-head loss path (declared in include/lmhead.h):
// host-side argument validation, TMA descriptor encoding, kernel selection and
// launch.  Every call only enqueues work on the caller's stream.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "lmhead.h"
#include "ce_kernels.cuh"
#include "gemm_tc.cuh"

namespace {

using lmh::GemmCfg;
using lmh::GemmParams;

constexpr int64_t kMaxDim = 0x7fffffff;
constexpr int64_t kMaxSplitRounds = 8;  // short parts per idle unit in a split last wave
constexpr int kMaxDevices = 64;
constexpr int kCeThreads = 1024;  // threads per cross-entropy CTA; one CTA per row


bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms()
{
    // per device, filled on first use; host threads may race to fill it, with the same value
    static std::atomic<int> cached[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// cuTensorMapEncodeTiled, resolved once through the runtime (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D BF16 tensor [outer, inner] (inner contiguous), 128-byte swizzled boxes
// of box_inner x box_outer elements; out-of-range elements read as zero.
bool make_map(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output tensor map for the TMA-store epilogue: [outer rows][row stride ld]
// of FP32 or BF16, box {32, box_rows}, no swizzle.  False when the layout
// cannot be described (base not 16-byte aligned, row stride not a multiple
// of 16 bytes); the caller then uses the direct-store epilogue.
bool make_out_map(CUtensorMap *map, void *base, bool bf16, uint64_t inner, uint64_t outer,
                  uint64_t ld, uint32_t box_rows)
{
    const uint64_t esize = bf16 ? 2 : 4;
    if (!aligned(base, 16) || (ld * esize) % 16 != 0)
        return false;
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld * esize};
    const cuuint32_t box[2] = {32, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base,
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

lmh_status_t last_cuda_error()
{
    return cudaGetLastError() == cudaSuccess ? LMH_OK : LMH_ERR_CUDA;
}

// Programmatic dependent launch is on unless the library is built with
// -DLMH_NO_PDL (a build-time switch for measurements; nothing in the
// environment changes the kernels a call launches).
constexpr bool pdl_enabled()
{
#ifdef LMH_NO_PDL
    return false;
#else
    return true;
#endif
}

// Launch with programmatic stream serialisation allowed (the kernel waits in
// pdl_wait before touching memory the previous kernel may still write) and,
// for cluster_x > 1, thread-block clusters of cluster_x CTAs.
template <typename... KArgs, typename... Args>
lmh_status_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, unsigned cluster_x, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess)
        return LMH_ERR_CUDA;
    return last_cuda_error();
}

// A GEMM operand as a 2-D BF16 tensor [outer][inner] (inner contiguous).
// mn_major: the inner dimension is the operand's m (or n) dimension and the
// outer one its reduction dimension; otherwise the reverse.
struct Operand {
    const void *base;
    uint64_t inner, outer;
    bool mn_major;
};

// Tensor map of an operand for tiles of `rows` m/n rows x 64 k: K-major
// operands are one box {64, rows}, MN-major ones boxes {64, 64}.
bool make_operand_map(CUtensorMap *map, const Operand &op, uint32_t rows)
{
    return op.mn_major ? make_map(map, op.base, op.inner, op.outer, 64, lmh::kBlockK)
                       : make_map(map, op.base, op.inner, op.outer, lmh::kBlockK, rows);
}

// One GEMM launch: D[m,n] = sum_k A[m,k] B[n,k] -> out[n*ldo + m].
template <int BN, bool A_MN, bool B_MN, typename OutT, bool TMA_STORE, bool PAIR, bool CE = false,
          bool ACC = false, int RES = 1, int EW = lmh::epi_warps(A_MN, B_MN, CE, ACC)>
lmh_status_t launch_gemm_impl(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc,
                              GemmParams p, cudaStream_t stream)
{
    using C = GemmCfg<BN, A_MN, B_MN, PAIR, RES, EW, CE>;
    auto kern = lmh::gemm_tc_kernel<BN, A_MN, B_MN, OutT, TMA_STORE, PAIR, CE, ACC, RES, EW>;
    // set once per process and device; the attribute is per function
    static std::atomic<uint64_t> attr_set{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
            cudaSuccess)
            return LMH_ERR_CUDA;
        // several CTAs per SM need the whole unified memory as shared memory
        if (RES > 1 && cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                            100) != cudaSuccess)
            return LMH_ERR_CUDA;
        attr_set.fetch_or(bit);
    }
    if (p.wait_limit_ns == 0)
        p.wait_limit_ns = lmh::kWaitLimitNs;
    p.num_m_tiles = static_cast<int32_t>((p.Mdim + C::TILE_M - 1) / C::TILE_M);
    p.num_n_tiles = static_cast<int32_t>((p.Ndim + BN - 1) / BN);
    const int64_t tiles = static_cast<int64_t>(p.num_m_tiles) * p.num_n_tiles;
    if (tiles > kMaxDim)
        return LMH_ERR_INVALID_ARG;
    // persistent: one CTA (or CTA pair) per SM (pair); several resident per SM: one per tile
    const int64_t units = RES == 1 ? num_sms() / C::CTAS : tiles;
    p.split_tiles = 0;
    p.split_kb = 0;
    p.split_rounds = 0;
    int64_t items = tiles;
    if constexpr (sizeof(OutT) == 4 && !CE && !ACC && RES == 1) {
        // A last (or only) wave of rem tiles leaves units - rem units idle.
        // Split each of its tiles into a long part [0, B) for the unit that
        // would have run it and a short part [B, num_kb) for an idle unit,
        // each idle unit taking k short parts: B = ceil(num_kb k / (k + 1))
        // makes the k short parts no longer than the long one.  Both parts
        // add into zeroed output (TMA reduce-add, or per-element atomic adds
        // on the direct-store path; deterministic: two addends, so both
        // epilogue paths give the same bits).  The split tiles come last in
        // the tile order, and whole output rows are contiguous, so one memset
        // zeroes them.  Taken when the last round shortens by a tenth or more,
        // and with several short parts per unit (k > 1) only after a full
        // wave: measured at 2048 x 4096 x 32768 (one full wave, then 54 tiles
        // on 74 pairs, k = 3) 360 against 382 us; in a single wave of 64 tiles
        // (1024 tokens, k = 7) 192 against 190.5 us, where the tiles running
        // in step share their operand reads and the extra units add nothing.
        const int64_t rem = tiles % units;
        const int64_t num_kb = (p.Kdim + lmh::kBlockK - 1) / lmh::kBlockK;
        if (p.allow_split && p.m_fastest && num_kb >= 2 && rem > 0) {
            const int64_t spare = units - rem;
            const int64_t k = (rem + spare - 1) / spare;
            const int64_t B = (num_kb * k + k) / (k + 1);  // ceil(num_kb k / (k + 1))
            const int64_t span = B > k * (num_kb - B) ? B : k * (num_kb - B);
            if ((k == 1 || tiles > units) && k <= kMaxSplitRounds && B < num_kb &&
                10 * span <= 9 * num_kb) {
                p.split_tiles = static_cast<int32_t>(rem);
                p.split_kb = static_cast<int32_t>(B);
                p.split_rounds = static_cast<int32_t>(k);
                items = tiles - rem + units * k;
            }
        }
        if (p.split_tiles > 0) {
            // zero every output row from the lowest n-row any split tile
            // covers (rows below it are all stored, not added)
            int nt_min = p.num_n_tiles;
            for (int64_t t = tiles - p.split_tiles; t < tiles; ++t) {
                int mt = 0, nt = 0;
                lmh::tile_coords(static_cast<int>(t), p, mt, nt);
                nt_min = nt < nt_min ? nt : nt_min;
            }
            const int64_t row0 = static_cast<int64_t>(nt_min) * BN;
            const size_t bytes = static_cast<size_t>(p.Ndim - row0) * p.ldo * sizeof(float);
            if (cudaMemsetAsync(static_cast<float *>(p.out) + row0 * p.ldo, 0, bytes, stream) !=
                cudaSuccess)
                return LMH_ERR_CUDA;
        }
    }
    const int grid = static_cast<int>((items < units ? items : units) * C::CTAS);
    return launch_ex(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream,
                     PAIR ? 2u : 1u, ta, tb, tc, p);
}

template <int BN, bool A_MN, bool B_MN, typename OutT, bool PAIR, int RES = 1>
lmh_status_t launch_gemm(const Operand &a, const Operand &b, GemmParams p, cudaStream_t stream)
{
    using C = GemmCfg<BN, A_MN, B_MN, PAIR, RES>;
    CUtensorMap ta, tb, tc;
    if (!make_operand_map(&ta, a, lmh::kBlockM) || !make_operand_map(&tb, b, C::BN_CTA))
        return LMH_ERR_CUDA;
    if (make_out_map(&tc, p.out, sizeof(OutT) == 2, static_cast<uint64_t>(p.Mdim),
                     static_cast<uint64_t>(p.Ndim), static_cast<uint64_t>(p.ldo), C::EPI_CHUNK))
        return launch_gemm_impl<BN, A_MN, B_MN, OutT, true, PAIR, false, false, RES>(ta, tb, tc, p,
                                                                                   stream);
    std::memset(&tc, 0, sizeof tc);
    return launch_gemm_impl<BN, A_MN, B_MN, OutT, false, PAIR, false, false, RES>(ta, tb, tc, p,
                                                                                stream);
}

// dW += dlogits^T . X (FP32): the dW GEMM with an accumulating epilogue.
template <int BN, bool PAIR>
lmh_status_t launch_dw_acc(const Operand &a, const Operand &b, GemmParams p, cudaStream_t stream)
{
    using C = GemmCfg<BN, true, true, PAIR>;
    CUtensorMap ta, tb, tc;
    if (!make_operand_map(&ta, a, lmh::kBlockM) || !make_operand_map(&tb, b, C::BN_CTA))
        return LMH_ERR_CUDA;
    if (make_out_map(&tc, p.out, false, static_cast<uint64_t>(p.Mdim),
                     static_cast<uint64_t>(p.Ndim), static_cast<uint64_t>(p.ldo), C::EPI_CHUNK))
        return launch_gemm_impl<BN, true, true, float, true, PAIR, false, true>(ta, tb, tc, p, stream);
    std::memset(&tc, 0, sizeof tc);
    return launch_gemm_impl<BN, true, true, float, false, PAIR, false, true>(ta, tb, tc, p, stream);
}

// Token-dimension tile width for the vocabulary GEMM and dX: the smallest
// supported MMA N that covers M, capped at 256.
int pick_bn_tokens(int64_t M)
{
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

// L2 policy of the logits the vocabulary GEMM stores.  Evict first: while the
// tensor-bound GEMM still streams W through L2, its logit lines are the first
// to be written back, so the kernel that reads them next does not inherit a
// cache full of dirty lines to write back under its own reads.
#ifndef LMH_LOGITS_L2_POLICY
#define LMH_LOGITS_L2_POLICY 1
#endif
constexpr int kLogitsL2Policy = LMH_LOGITS_L2_POLICY;

// L2 policy of W in the vocabulary GEMM: streamed once (evict first) when a
// single token tile reads each W panel, normal when several token tiles reuse
// it (measured: +13 % for M <= 128, -7 % at M = 1024 with evict first).
int w_policy(int64_t M, int bn) { return M <= bn ? 1 : 0; }

// CTA-pair tiles (256 x 256) are used when the n extent fills a 256-wide
// tile.  Building with -DLMH_GEMM_PAIR=0 or =1 forces single-CTA or pair tiles
// where both are possible (a build-time switch for measurements).
constexpr int pair_override()
{
#ifdef LMH_GEMM_PAIR
    return LMH_GEMM_PAIR ? 1 : 0;
#else
    return -1;
#endif
}

bool use_pair(int bn, int64_t Mdim)
{
    if (bn != 256 || Mdim < 256)
        return false;
    const int o = pair_override();
    return o < 0 ? true : o == 1;
}

// The single-token-tile vocabulary GEMM (two CTAs per SM) in CTA pairs: each
// CTA stages half of X, so X crosses L2 -> SM once per pair instead of once
// per CTA.  It pays only when X is large (measured at V = 32768: 128 tokens,
// K = 16384: 204.8 -> 190.5 us; K = 4096: 61.5 -> 63.5 us; 64 tokens: no
// gain at any K).
bool use_pair_small(int bn, int64_t Mdim, int64_t Kdim)
{
    if (bn != 128 || Kdim < 16384 || Mdim < 256)
        return false;
    const int o = pair_override();
    return o < 0 ? true : o == 1;
}

// Vocabulary GEMM with the fused cross-entropy statistics (FP32 logits through
// the TMA-store epilogue; the caller has checked that a tensor map can describe
// them).  *nslices receives the number of 128-wide vocabulary blocks written.
template <int BN, bool PAIR, int RES = 1>
lmh_status_t launch_gemm_ce(const Operand &a, const Operand &b, GemmParams p, int64_t *nslices,
                            cudaStream_t stream)
{
    using C = GemmCfg<BN, false, false, PAIR, RES>;
    CUtensorMap ta, tb, tc;
    if (!make_operand_map(&ta, a, lmh::kBlockM) || !make_operand_map(&tb, b, C::BN_CTA) ||
        !make_out_map(&tc, p.out, false, static_cast<uint64_t>(p.Mdim),
                      static_cast<uint64_t>(p.Ndim), static_cast<uint64_t>(p.ldo), C::EPI_CHUNK))
        return LMH_ERR_CUDA;
    *nslices = static_cast<int64_t>(C::CTAS) * ((p.Mdim + C::TILE_M - 1) / C::TILE_M);
    return launch_gemm_impl<BN, false, false, float, true, PAIR, true, false, RES>(ta, tb, tc, p,
                                                                                 stream);
}

lmh_status_t dispatch_ce(int bn, const Operand &a, const Operand &b, GemmParams p, int64_t *nslices,
                         cudaStream_t s)
{
    // one token tile (bn covers every token): HBM-bound, two CTAs resident per SM
    switch (bn) {
    case 16: return launch_gemm_ce<16, false, 2>(a, b, p, nslices, s);
    case 32: return launch_gemm_ce<32, false, 2>(a, b, p, nslices, s);
    case 64: return launch_gemm_ce<64, false, 2>(a, b, p, nslices, s);
    case 128:
        return use_pair_small(bn, p.Mdim, p.Kdim) ? launch_gemm_ce<128, true, 2>(a, b, p, nslices, s)
                                                  : launch_gemm_ce<128, false, 2>(a, b, p, nslices, s);
    case 256:
        return use_pair(bn, p.Mdim) ? launch_gemm_ce<256, true>(a, b, p, nslices, s)
                                    : launch_gemm_ce<256, false>(a, b, p, nslices, s);
    default: return LMH_ERR_UNSUPPORTED;
    }
}

// Blocks of partial statistics the fused GEMM may write for a vocabulary of V
// (one per CTA's 128 rows of a tile; both tile modes fit: 2 per 256
// vocabulary columns).
int64_t ce_slices(int64_t V) { return 2 * ((V + 255) / 256); }

template <bool A_MN, bool B_MN, typename OutT>
lmh_status_t dispatch_bn(int bn, const Operand &a, const Operand &b, GemmParams p, cudaStream_t s)
{
    if constexpr (!A_MN && !B_MN) {
        // vocabulary GEMM with one token tile (bn covers every token): HBM-bound
        // on W, so two CTAs resident per SM with one CTA per tile
        switch (bn) {
        case 16: return launch_gemm<16, A_MN, B_MN, OutT, false, 2>(a, b, p, s);
        case 32: return launch_gemm<32, A_MN, B_MN, OutT, false, 2>(a, b, p, s);
        case 64: return launch_gemm<64, A_MN, B_MN, OutT, false, 2>(a, b, p, s);
        case 128:
            return use_pair_small(bn, p.Mdim, p.Kdim)
                       ? launch_gemm<128, A_MN, B_MN, OutT, true, 2>(a, b, p, s)
                       : launch_gemm<128, A_MN, B_MN, OutT, false, 2>(a, b, p, s);
        default: break;
        }
    }
    if constexpr (!B_MN) {
        switch (bn) {
        case 16: return launch_gemm<16, A_MN, B_MN, OutT, false>(a, b, p, s);
        case 32: return launch_gemm<32, A_MN, B_MN, OutT, false>(a, b, p, s);
        default: break;
        }
    }
    switch (bn) {
    case 64: return launch_gemm<64, A_MN, B_MN, OutT, false>(a, b, p, s);
    case 128: return launch_gemm<128, A_MN, B_MN, OutT, false>(a, b, p, s);
    case 256:
        return use_pair(bn, p.Mdim) ? launch_gemm<256, A_MN, B_MN, OutT, true>(a, b, p, s)
                                    : launch_gemm<256, A_MN, B_MN, OutT, false>(a, b, p, s);
    default: return LMH_ERR_UNSUPPORTED;
    }
}

bool bad_dtype(int32_t t) { return t != LMH_F32 && t != LMH_BF16; }

// One thread waits on a barrier that expects an arrival nobody makes.
__global__ void watchdog_selftest_kernel(int32_t *status, uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        lmh::mbar_init(&bar, 1);
        abort_flag = 0;
        lmh::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!lmh::mbar_wait(&bar, 0, &abort_flag, limit_ns))
            atomicOr(status, LMH_DEV_PIPE_TIMEOUT);
    }
}

bool dims_ok(int64_t a, int64_t b, int64_t c)
{
    return a >= 1 && b >= 1 && c >= 1 && a <= kMaxDim && b <= kMaxDim && c <= kMaxDim;
}

// lmhead_fwd with a given pipeline wait limit (0: the default limit).
lmh_status_t fwd_impl(const void *X, const void *W, void *logits, int32_t out_dtype, int64_t M,
                      int64_t K, int64_t V, int32_t *status, lmh_stream_t stream,
                      uint64_t wait_limit_ns)
{
    if (!X || !W || !logits || !dims_ok(M, K, V))
        return LMH_ERR_INVALID_ARG;
    if (bad_dtype(out_dtype))
        return LMH_ERR_UNSUPPORTED;
    if (K % 8 || !aligned(X, 16) || !aligned(W, 16) ||
        !aligned(logits, out_dtype == LMH_F32 ? 4 : 2))
        return LMH_ERR_MISALIGNED;
    const int bn = pick_bn_tokens(M);
    const Operand a{W, static_cast<uint64_t>(K), static_cast<uint64_t>(V), false};  // A = W
    const Operand b{X, static_cast<uint64_t>(K), static_cast<uint64_t>(M), false};  // B = X
    GemmParams p{};
    p.out = logits;
    p.ldo = V;
    p.Mdim = static_cast<int32_t>(V);
    p.Ndim = static_cast<int32_t>(M);
    p.Kdim = static_cast<int32_t>(K);
    p.m_fastest = 0;  // consecutive tiles share one W panel
    p.l2_a = w_policy(M, bn);
    p.l2_b = 2;  // X is reread by every tile
    p.l2_out = kLogitsL2Policy;
    p.status = status;
    p.wait_limit_ns = wait_limit_ns;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return out_dtype == LMH_F32 ? dispatch_bn<false, false, float>(bn, a, b, p, s)
                                : dispatch_bn<false, false, __nv_bfloat16>(bn, a, b, p, s);
}

}  // namespace

extern "C" {

const char *lmh_status_string(lmh_status_t s)
{
    switch (s) {
    case LMH_OK: return "ok";
    case LMH_ERR_INVALID_ARG: return "invalid argument (null pointer or size out of range)";
    case LMH_ERR_MISALIGNED: return "misaligned pointer or row stride";
    case LMH_ERR_UNSUPPORTED: return "unsupported dtype or stride";
    case LMH_ERR_CUDA: return "CUDA runtime error";
    }
    return "unknown status";
}

int32_t lmh_version(void) { return 20000; }

lmh_status_t lmh_watchdog_selftest(int32_t *status, int64_t limit_us, lmh_stream_t stream)
{
    if (!status || limit_us < 1 || limit_us > 1000000)
        return LMH_ERR_INVALID_ARG;
    watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        status, static_cast<uint64_t>(limit_us) * 1000ull);
    return last_cuda_error();
}

lmh_status_t lmhead_fwd(const void *X, const void *W, void *logits, int32_t out_dtype, int64_t M,
                        int64_t K, int64_t V, int32_t *status, lmh_stream_t stream)
{
    return fwd_impl(X, W, logits, out_dtype, M, K, V, status, stream, 0);
}

lmh_status_t lmh_gemm_watchdog_selftest(const void *X, const void *W, float *logits, int64_t M,
                                        int64_t K, int64_t V, int64_t limit_ns, int32_t *status,
                                        lmh_stream_t stream)
{
    if (!status || limit_ns < 1 || limit_ns > 1000000000)
        return LMH_ERR_INVALID_ARG;
    return fwd_impl(X, W, logits, LMH_F32, M, K, V, status, stream,
                    static_cast<uint64_t>(limit_ns));
}

lmh_status_t lmhead_bwd_dx(const void *dlogits, const void *W, void *dX, int32_t out_dtype,
                           int64_t M, int64_t K, int64_t V, int32_t *status, lmh_stream_t stream)
{
    if (!dlogits || !W || !dX || !dims_ok(M, K, V))
        return LMH_ERR_INVALID_ARG;
    if (bad_dtype(out_dtype))
        return LMH_ERR_UNSUPPORTED;
    if (K % 8 || V % 8 || !aligned(dlogits, 16) || !aligned(W, 16) ||
        !aligned(dX, out_dtype == LMH_F32 ? 4 : 2))
        return LMH_ERR_MISALIGNED;
    const int bn = pick_bn_tokens(M);
    // A = W^T (m = k_out contiguous, k = v), B = dl (n = token, k = v contiguous)
    const Operand a{W, static_cast<uint64_t>(K), static_cast<uint64_t>(V), true};
    const Operand b{dlogits, static_cast<uint64_t>(V), static_cast<uint64_t>(M), false};
    GemmParams p{};
    p.out = dX;
    p.ldo = K;
    p.Mdim = static_cast<int32_t>(K);
    p.Ndim = static_cast<int32_t>(M);
    p.Kdim = static_cast<int32_t>(V);
    p.m_fastest = 1;
    // every W and dlogits chunk is read by several of the tiles running at
    // once: both kept evict-last (measured against the default policy, same
    // box: 2.86 against 2.90 ms at 4096 x 4096 x 128256, 351 against 357 us at
    // 2048 tokens, 187 against 189 us at 1024; evict-first on either operand
    // read 11-13 GB from DRAM instead of 8.8 and ran 4-7 % slower)
    p.l2_a = 2;
    p.l2_b = 2;
    p.status = status;
    p.allow_split = 1;  // few output tiles, each with a long reduction over V
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return out_dtype == LMH_F32 ? dispatch_bn<true, false, float>(bn, a, b, p, s)
                                : dispatch_bn<true, false, __nv_bfloat16>(bn, a, b, p, s);
}

lmh_status_t lmhead_bwd_dw(const void *dlogits, const void *X, void *dW, int32_t out_dtype,
                           int64_t M, int64_t K, int64_t V, int32_t *status, lmh_stream_t stream)
{
    if (!dlogits || !X || !dW || !dims_ok(M, K, V))
        return LMH_ERR_INVALID_ARG;
    if (bad_dtype(out_dtype))
        return LMH_ERR_UNSUPPORTED;
    if (K % 8 || V % 8 || !aligned(dlogits, 16) || !aligned(X, 16) ||
        !aligned(dW, out_dtype == LMH_F32 ? 4 : 2))
        return LMH_ERR_MISALIGNED;
    const int bn = V <= 64 ? 64 : V <= 128 ? 128 : 256;
    // A = X^T (m = k_out contiguous, k = token), B = dl^T (n = v contiguous, k = token)
    const Operand a{X, static_cast<uint64_t>(K), static_cast<uint64_t>(M), true};
    const Operand b{dlogits, static_cast<uint64_t>(V), static_cast<uint64_t>(M), true};
    GemmParams p{};
    p.out = dW;
    p.ldo = K;
    p.Mdim = static_cast<int32_t>(K);
    p.Ndim = static_cast<int32_t>(V);
    p.Kdim = static_cast<int32_t>(M);
    p.m_fastest = 1;  // consecutive tiles share one dlogits panel
    p.l2_a = 2;       // X is reread by every tile
    p.l2_b = 0;
    p.status = status;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return out_dtype == LMH_F32 ? dispatch_bn<true, true, float>(bn, a, b, p, s)
                                : dispatch_bn<true, true, __nv_bfloat16>(bn, a, b, p, s);
}

lmh_status_t lmhead_bwd_dw_acc(const void *dlogits, const void *X, float *dW, int64_t M, int64_t K,
                               int64_t V, int32_t *status, lmh_stream_t stream)
{
    if (!dlogits || !X || !dW || !dims_ok(M, K, V))
        return LMH_ERR_INVALID_ARG;
    if (K % 8 || V % 8 || !aligned(dlogits, 16) || !aligned(X, 16) || !aligned(dW, 4))
        return LMH_ERR_MISALIGNED;
    const int bn = V <= 64 ? 64 : V <= 128 ? 128 : 256;
    const Operand a{X, static_cast<uint64_t>(K), static_cast<uint64_t>(M), true};
    const Operand b{dlogits, static_cast<uint64_t>(V), static_cast<uint64_t>(M), true};
    GemmParams p{};
    p.out = dW;
    p.ldo = K;
    p.Mdim = static_cast<int32_t>(K);
    p.Ndim = static_cast<int32_t>(V);
    p.Kdim = static_cast<int32_t>(M);
    p.m_fastest = 1;
    p.l2_a = 2;
    p.l2_b = 0;
    p.status = status;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (bn) {
    case 64: return launch_dw_acc<64, false>(a, b, p, s);
    case 128: return launch_dw_acc<128, false>(a, b, p, s);
    default:
        return use_pair(bn, p.Mdim) ? launch_dw_acc<256, true>(a, b, p, s)
                                    : launch_dw_acc<256, false>(a, b, p, s);
    }
}

int64_t lmhead_fwd_ce_workspace_bytes(int64_t M, int64_t V)
{
    if (M < 1 || V < 1 || M > kMaxDim || V > kMaxDim)
        return -1;
    return ce_slices(V) * M * static_cast<int64_t>(sizeof(float2));
}

lmh_status_t lmhead_fwd_ce(const void *X, const void *W, const int64_t *target, float *logits,
                           float *stats, void *workspace, int64_t workspace_bytes, int64_t M,
                           int64_t K, int64_t V, int64_t ignore_index, int32_t *status,
                           lmh_stream_t stream)
{
    if (!X || !W || !target || !logits || !stats || !dims_ok(M, K, V))
        return LMH_ERR_INVALID_ARG;
    if (K % 8 || !aligned(X, 16) || !aligned(W, 16) || !aligned(logits, 4) || !aligned(target, 8) ||
        !aligned(stats, 16))
        return LMH_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (V % 4 != 0 || !aligned(logits, 16)) {
        // logits a tensor map cannot describe: the two separate passes
        const lmh_status_t r = lmhead_fwd(X, W, logits, LMH_F32, M, K, V, status, stream);
        return r != LMH_OK ? r : ce_fwd(logits, target, stats, M, V, ignore_index, status, stream);
    }
    if (!workspace || workspace_bytes < lmhead_fwd_ce_workspace_bytes(M, V))
        return LMH_ERR_INVALID_ARG;
    if (!aligned(workspace, 16))
        return LMH_ERR_MISALIGNED;
    const int bn = pick_bn_tokens(M);
    const Operand a{W, static_cast<uint64_t>(K), static_cast<uint64_t>(V), false};
    const Operand b{X, static_cast<uint64_t>(K), static_cast<uint64_t>(M), false};
    GemmParams p{};
    p.out = logits;
    p.ldo = V;
    p.Mdim = static_cast<int32_t>(V);
    p.Ndim = static_cast<int32_t>(M);
    p.Kdim = static_cast<int32_t>(K);
    p.m_fastest = 0;
    p.l2_a = w_policy(M, bn);
    p.l2_b = 2;
    p.l2_out = kLogitsL2Policy;
    p.status = status;
    p.ce_partial = static_cast<float2 *>(workspace);
    p.ce_target = target;
    p.ce_stats = stats;
    int64_t nslices = 0;
    const lmh_status_t r = dispatch_ce(bn, a, b, p, &nslices, s);
    if (r != LMH_OK)
        return r;
    constexpr int kFinalizeWarps = 32;  // kFinalizeTokens tokens per CTA, slices split over the warps
    const int64_t grid = (M + lmh::kFinalizeTokens - 1) / lmh::kFinalizeTokens;
    return launch_ex(lmh::ce_finalize_kernel<kFinalizeWarps>, dim3(static_cast<unsigned>(grid)),
                     dim3(kFinalizeWarps * 32), 0, s, 1u, static_cast<const float2 *>(workspace),
                     nslices, target, reinterpret_cast<float4 *>(stats), M, V, ignore_index, status);
}

lmh_status_t ce_fwd(const float *logits, const int64_t *target, float *stats, int64_t M, int64_t V,
                    int64_t ignore_index, int32_t *status, lmh_stream_t stream)
{
    if (!logits || !target || !stats || M < 1 || V < 1 || M > kMaxDim || V > kMaxDim)
        return LMH_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(target, 8) || !aligned(stats, 16))
        return LMH_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one CTA per row: the block scheduler balances rows across SMs
    const int grid = static_cast<int>(M);
    const bool vec = (V % 4 == 0) && aligned(logits, 16);
    float4 *st4 = reinterpret_cast<float4 *>(stats);
    if (vec)
        return launch_ex(lmh::ce_fwd_kernel<true, kCeThreads>, dim3(grid), dim3(kCeThreads), 0, s, 1u,
                         logits, target, st4, M, V, ignore_index, status, int64_t{0}, V);
    return launch_ex(lmh::ce_fwd_kernel<false, kCeThreads>, dim3(grid), dim3(kCeThreads), 0, s, 1u,
                     logits, target, st4, M, V, ignore_index, status, int64_t{0}, V);
}

}  // extern "C"

namespace {

// ce_bwd over vocabulary entries [voff, voff + V) of a vocabulary of Vtot.
lmh_status_t ce_bwd_range(const float *logits, const int64_t *target, const float *stats,
                          const float *grad_loss, int64_t grad_loss_stride, void *dlogits,
                          int32_t dl_dtype, int64_t M, int64_t V, int64_t voff, int64_t Vtot,
                          int64_t ignore_index, int32_t *status, lmh_stream_t stream)
{
    if (!logits || !target || !stats || !grad_loss || !dlogits || M < 1 || V < 1 ||
        M > kMaxDim || V > kMaxDim)
        return LMH_ERR_INVALID_ARG;
    if (bad_dtype(dl_dtype) || (grad_loss_stride != 0 && grad_loss_stride != 1))
        return LMH_ERR_UNSUPPORTED;
    if (dl_dtype == LMH_BF16 && static_cast<const void *>(logits) == dlogits)
        return LMH_ERR_UNSUPPORTED;  // in-place only for an FP32 gradient
    if (!aligned(logits, 4) || !aligned(target, 8) || !aligned(stats, 16) || !aligned(grad_loss, 4) ||
        !aligned(dlogits, dl_dtype == LMH_F32 ? 4 : 2))
        return LMH_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one CTA per row: the block scheduler balances rows across SMs
    const int grid = static_cast<int>(M);
    const float4 *st4 = reinterpret_cast<const float4 *>(stats);
    if (dl_dtype == LMH_F32) {
        float *o = static_cast<float *>(dlogits);
        const bool vec = (V % 4 == 0) && aligned(logits, 16) && aligned(o, 16);
        const bool alias = static_cast<const void *>(logits) == dlogits;
        auto k = vec ? (alias ? lmh::ce_bwd_kernel<float, true, true, kCeThreads>
                              : lmh::ce_bwd_kernel<float, true, false, kCeThreads>)
                     : (alias ? lmh::ce_bwd_kernel<float, false, true, kCeThreads>
                              : lmh::ce_bwd_kernel<float, false, false, kCeThreads>);
        return launch_ex(k, dim3(grid), dim3(kCeThreads), 0, s, 1u, logits, target, st4, grad_loss,
                         grad_loss_stride, o, M, V, ignore_index, status, voff, Vtot);
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(dlogits);
    const bool vec = (V % 4 == 0) && aligned(logits, 16) && aligned(o, 8);
    auto k = vec ? lmh::ce_bwd_kernel<__nv_bfloat16, true, false, kCeThreads>
                 : lmh::ce_bwd_kernel<__nv_bfloat16, false, false, kCeThreads>;
    return launch_ex(k, dim3(grid), dim3(kCeThreads), 0, s, 1u, logits, target, st4, grad_loss,
                     grad_loss_stride, o, M, V, ignore_index, status, voff, Vtot);
}

}  // namespace

extern "C" {

lmh_status_t ce_bwd(const float *logits, const int64_t *target, const float *stats,
                    const float *grad_loss, int64_t grad_loss_stride, void *dlogits,
                    int32_t dl_dtype, int64_t M, int64_t V, int64_t ignore_index,
                    int32_t *status, lmh_stream_t stream)
{
    return ce_bwd_range(logits, target, stats, grad_loss, grad_loss_stride, dlogits, dl_dtype, M, V,
                        0, V, ignore_index, status, stream);
}

lmh_status_t ce_fwd_shard(const float *logits, const int64_t *target, float *shard_stats,
                          int64_t M, int64_t V, int64_t vocab_offset, int64_t vocab_total,
                          int64_t ignore_index, int32_t *status, lmh_stream_t stream)
{
    if (!logits || !target || !shard_stats || M < 1 || V < 1 || M > kMaxDim || V > kMaxDim ||
        vocab_offset < 0 || vocab_total > kMaxDim || vocab_offset + V > vocab_total)
        return LMH_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(target, 8) || !aligned(shard_stats, 16))
        return LMH_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int grid = static_cast<int>(M);
    float4 *st4 = reinterpret_cast<float4 *>(shard_stats);
    if ((V % 4 == 0) && aligned(logits, 16))
        return launch_ex(lmh::ce_fwd_kernel<true, kCeThreads, true>, dim3(grid), dim3(kCeThreads), 0,
                         s, 1u, logits, target, st4, M, V, ignore_index, status, vocab_offset,
                         vocab_total);
    return launch_ex(lmh::ce_fwd_kernel<false, kCeThreads, true>, dim3(grid), dim3(kCeThreads), 0, s,
                     1u, logits, target, st4, M, V, ignore_index, status, vocab_offset, vocab_total);
}

lmh_status_t ce_merge_shards(const float *shard_stats, int64_t num_shards, const int64_t *target,
                             float *stats, int64_t M, int64_t vocab_total, int64_t ignore_index,
                             int32_t *status, lmh_stream_t stream)
{
    if (!shard_stats || !target || !stats || num_shards < 1 || num_shards > 65536 || M < 1 ||
        M > kMaxDim || vocab_total < 1 || vocab_total > kMaxDim)
        return LMH_ERR_INVALID_ARG;
    if (!aligned(shard_stats, 16) || !aligned(target, 8) || !aligned(stats, 16))
        return LMH_ERR_MISALIGNED;
    const int64_t blocks = (M + 255) / 256;
    return launch_ex(lmh::ce_merge_shards_kernel, dim3(static_cast<unsigned>(blocks < 65535 ? blocks : 65535)),
                     dim3(256), 0, reinterpret_cast<cudaStream_t>(stream), 1u,
                     reinterpret_cast<const float4 *>(shard_stats), num_shards, target,
                     reinterpret_cast<float4 *>(stats), M, vocab_total, ignore_index, status);
}

lmh_status_t ce_bwd_shard(const float *logits, const int64_t *target, const float *stats,
                          const float *grad_loss, int64_t grad_loss_stride, void *dlogits,
                          int32_t dl_dtype, int64_t M, int64_t V, int64_t vocab_offset,
                          int64_t vocab_total, int64_t ignore_index, int32_t *status,
                          lmh_stream_t stream)
{
    if (vocab_offset < 0 || vocab_total > kMaxDim || V < 1 || vocab_offset + V > vocab_total)
        return LMH_ERR_INVALID_ARG;
    return ce_bwd_range(logits, target, stats, grad_loss, grad_loss_stride, dlogits, dl_dtype, M, V,
                        vocab_offset, vocab_total, ignore_index, status, stream);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// lmhead_fwd_ce_noalloc: lmhead_fwd_ce for callers that cannot allocate.
//
// Some callers cannot hand this library a scratch buffer: plug-ins whose host
// framework owns all device memory and gives them no allocator, and code on
// paths where calling cudaMalloc (which may synchronise the device) is not
// allowed.  For them the partial statistics live in one fixed array below,
// part of the library image: every GPU that loads the library holds these
// 8 MiB until the process exits.  The caller still passes every input and
// output.  This call allocates nothing and calls no allocating routine.
//
// In host code `g_fwd_ce_scratch` only names a host-side stand-in for the
// array; handing it to a kernel would fault, or on systems where the GPU can
// reach host memory silently use the wrong memory.  The device address is
// therefore looked up with cudaGetSymbolAddress, once per device, with that
// device current, the first time the call runs on it; make that first call
// before any stream capture.
// ----------------------------------------------------------------------------

namespace {

constexpr int64_t kNoAllocScratchBytes = 8ll << 20;  // 8 MiB of partial statistics
static __device__ __align__(256) float2 g_fwd_ce_scratch[kNoAllocScratchBytes / sizeof(float2)];

// Device address of g_fwd_ce_scratch on the current device (nullptr on error).
float2 *noalloc_scratch()
{
    static std::mutex mu;
    static float2 *addr[kMaxDevices] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fwd_ce_scratch) != cudaSuccess)
            return nullptr;
        addr[dev] = static_cast<float2 *>(p);
    }
    return addr[dev];
}

}  // namespace

extern "C" lmh_status_t lmhead_fwd_ce_noalloc(const void *X, const void *W, const int64_t *target,
                                              float *logits, float *stats, int64_t M, int64_t K,
                                              int64_t V, int64_t ignore_index, int32_t *status,
                                              lmh_stream_t stream)
{
    if (!X || !W || !target || !logits || !stats || !dims_ok(M, K, V))
        return LMH_ERR_INVALID_ARG;
    if (K % 8 || !aligned(X, 16) || !aligned(W, 16) || !aligned(logits, 4) || !aligned(target, 8) ||
        !aligned(stats, 16))
        return LMH_ERR_MISALIGNED;
    if (V % 4 != 0 || !aligned(logits, 16))  // the two separate passes need no scratch
        return lmhead_fwd_ce(X, W, target, logits, stats, nullptr, 0, M, K, V, ignore_index, status,
                             stream);
    // larger problems are rejected before anything is launched
    if (ce_slices(V) > kNoAllocScratchBytes / static_cast<int64_t>(sizeof(float2)) / M)
        return LMH_ERR_INVALID_ARG;
    float2 *scratch = noalloc_scratch();
    if (!scratch)
        return LMH_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int bn = pick_bn_tokens(M);
    const Operand a{W, static_cast<uint64_t>(K), static_cast<uint64_t>(V), false};
    const Operand b{X, static_cast<uint64_t>(K), static_cast<uint64_t>(M), false};
    GemmParams p{};
    p.out = logits;
    p.ldo = V;
    p.Mdim = static_cast<int32_t>(V);
    p.Ndim = static_cast<int32_t>(M);
    p.Kdim = static_cast<int32_t>(K);
    p.m_fastest = 0;
    p.l2_a = w_policy(M, bn);
    p.l2_b = 2;
    p.l2_out = kLogitsL2Policy;
    p.status = status;
    p.ce_partial = scratch;
    p.ce_target = target;
    p.ce_stats = stats;
    int64_t nslices = 0;
    const lmh_status_t r = dispatch_ce(bn, a, b, p, &nslices, s);
    if (r != LMH_OK)
        return r;
    constexpr int kFinalizeWarps = 32;
    const int64_t grid = (M + lmh::kFinalizeTokens - 1) / lmh::kFinalizeTokens;
    return launch_ex(lmh::ce_finalize_kernel<kFinalizeWarps>, dim3(static_cast<unsigned>(grid)),
                     dim3(kFinalizeWarps * 32), 0, s, 1u, static_cast<const float2 *>(scratch), nslices,
                     target, reinterpret_cast<float4 *>(stats), M, V, ignore_index, status);
}
