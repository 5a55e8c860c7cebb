// gemm_tc.cuh -- persistent tcgen05 GEMM for sm_100a with a direct FP32 (or
// BF16) epilogue, used for the three contractions of the LM head:
//
//   logits[i, v] = sum_k X[i,k] W[v,k]        (A = W,   B = X,    both K-major)
//   dX[i, k]     = sum_v dl[i,v] W[v,k]       (A = W^T  MN-major, B = dl K-major)
//   dW[v, k]     = sum_i dl[i,v] X[i,k]       (A = X^T  MN-major, B = dl^T MN-major)
//
// Megatron-LM PR #6252 "Add mixed-precision (FP32) LM output logits", "What
// does this PR do?": the vocabulary GEMM keeps its FP32 accumulator as the
// output instead of rounding every logit to BF16.  Here the accumulator lives
// in tensor memory and the epilogue stores it unrounded.
//
// Generic form: D[m, n] = sum_k A[m, k] B[n, k], stored at out[n * ldo + m].
// The MMA's M dimension (128 lanes of tensor memory) is always the output's
// contiguous dimension, so each epilogue warp stores 32 consecutive elements
// (one 128-byte line for FP32) per instruction straight from registers.
//
// CTA roles (64 + 32 EW threads, one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: fills a STAGES-deep ring of A/B k-blocks
//   warp 1      tensor-memory owner and MMA issuer (one elected thread)
//   warps 2..   EW = 4 or 8 epilogue warps: tensor memory -> registers ->
//               shared memory -> TMA bulk tensor store (or, for outputs a
//               tensor map cannot describe, registers -> global stores).  A
//               warp may only read its own quarter (warp % 4) of the 128
//               tensor-memory lanes; with eight, two warps share each quarter
//               and take alternate sub-tiles.
// Two accumulators of BN columns let the epilogue of tile t overlap the MMAs
// of tile t+1.  With the TMA-store epilogue the warps stage 32 x 32 sub-tiles
// in eight shared-memory slots (two per warp, or one) and hand them to the TMA
// engine, so tensor memory is released as soon as its values are in shared
// memory instead of after 128 KB of global stores have drained.  Eight warps
// halve the epilogue of a tile, which matters where no MMA hides it: the last
// tile of each CTA when the fused cross-entropy statistics lengthen it.
// Every wait is bounded (see mbar_wait); on a timeout the CTA drains its own
// copies and MMAs, frees tensor memory, sets a status bit and returns.  A CTA
// pair first settles, through distributed shared memory, which operand copies
// either CTA has issued, completes the set, and waits for all of them to land
// before either CTA leaves (see the end of the kernel).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "softmax_merge.cuh"

namespace lmh {

constexpr int kBlockM = 128;  // MMA M: tensor-memory lanes
constexpr int kBlockK = 64;   // one 128-byte swizzle row of BF16
constexpr int kUmmaK = 16;    // K of one kind::f16 MMA

struct GemmParams {
    void *out;
    int64_t ldo;        // elements between consecutive n of the output
    int32_t Mdim;       // extent of m (output contiguous dim)
    int32_t Ndim;       // extent of n
    int32_t Kdim;       // reduction length
    int32_t num_m_tiles;
    int32_t num_n_tiles;
    int32_t m_fastest;  // tile order: 1 = consecutive tiles share n (B panel)
    int32_t l2_a;       // L2 policy of A / B loads: 0 normal, 1 evict first, 2 evict last
    int32_t l2_b;
    int32_t l2_out;     // L2 policy of the output stores (TMA store epilogue): 0 none, 1 evict first
    int32_t *status;
    uint64_t wait_limit_ns;  // limit of every pipeline wait (the host sets kWaitLimitNs)
    // The last split_tiles tiles of the tile order (the last wave, which
    // would leave units idle) are each computed as two work items: a long part,
    // k-blocks [0, split_kb), on the unit that would have run the tile, and a
    // short part, [split_kb, num_kb), on one of the units the wave leaves
    // idle, each of which runs split_rounds short parts in turn.  Both parts'
    // FP32 sums are added (TMA reduce-add, or atomic adds on the direct-store
    // path) into output the host has zeroed: fl(0 + a) = a and fl(a + b) =
    // fl(b + a), so the result does not depend on which part lands first.
    // 0 = no split; the tiles before the split ones fill whole waves.
    int32_t split_tiles;
    int32_t split_kb;
    int32_t split_rounds;
    int32_t allow_split;  // host side: the call may split its last wave (FP32 output)
    // fused cross-entropy statistics (vocabulary GEMM only): per 128-wide
    // vocabulary block s (one CTA's rows of a tile) and token i,
    // ce_partial[s * Ndim + i] = (max, sum-exp) of the block (a warp stores
    // 32 consecutive tokens of one block); the target logit goes to
    // ce_stats[4 i + 2].
    float2 *ce_partial;
    const int64_t *ce_target;
    float *ce_stats;
};

constexpr int kEpiSlots = 8;  // 32 x EPI_CHUNK staging slots shared by the epilogue warps
#ifndef LMH_DW_STORE_PACE_NS
#define LMH_DW_STORE_PACE_NS 200
#endif
constexpr unsigned kDwStorePaceNs = LMH_DW_STORE_PACE_NS;  // pause after each dW sub-tile store

// Epilogue warps of each GEMM.  Measured at 1024 x 4096 x 32768 (L2 flushed,
// medians): eight take the fused cross-entropy GEMM from 195.6 to 187.4 us,
// where the statistics make the last tile's epilogue long; four are better
// for the plain GEMMs (forward 170.0 against 172.1 us, dW 214.5 against
// 223.3 us, dX equal), whose epilogue is short and whose extra store bursts
// compete with the operand loads.
constexpr int epi_warps(bool /*a_mn*/, bool /*b_mn*/, bool ce, bool /*acc*/) { return ce ? 8 : 4; }
constexpr int kSmemLimit = 232448;  // 227 KB of dynamic shared memory per CTA
constexpr int kSmemPerSm = 233472;  // 228 KB per SM, of which 1 KB is reserved per CTA

// RES: CTAs meant to be resident per SM.  1 (persistent, deepest ring) for
// the tensor-bound shapes; 2 for HBM-bound single-token-tile shapes, whose
// tiles are then all in flight at once instead of running in waves.
template <int BN, bool A_MN, bool B_MN, bool PAIR, int RES = 1, int EW = 4, bool CE = false>
struct GemmCfg {
    static_assert(EW == 4 || EW == 8, "epilogue warps");
    static_assert(!CE || EW == 8, "the statistics exchange is laid out for eight epilogue warps");
    static constexpr int THREADS = 64 + 32 * EW;
    static constexpr int NSLOT = kEpiSlots / EW;  // staging slots per epilogue warp
    static constexpr int CTAS = PAIR ? 2 : 1;
    static constexpr int TILE_M = kBlockM * CTAS;  // m extent of one (pair) tile
    static constexpr int BN_CTA = BN / CTAS;       // n rows of B held by each CTA
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(!PAIR || BN % 32 == 0, "pair MMA N");
    static_assert(!B_MN || BN_CTA % 64 == 0, "MN-major B is loaded in 64-wide boxes");
    static constexpr int A_BYTES = kBlockM * kBlockK * 2;  // 16 KB
    static constexpr int B_BYTES = BN_CTA * kBlockK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
    static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
    static constexpr int EPI_CHUNK = BN < 32 ? BN : 32;  // accumulator columns per sub-tile
    // staging slots of 32 lanes x EPI_CHUNK columns, sized for FP32 (a BF16
    // output uses half of each)
    static constexpr int EPI_SLOT_BYTES = 32 * EPI_CHUNK * 4;
    static constexpr int EPI_BYTES = kEpiSlots * EPI_SLOT_BYTES;
    // CE: per half of the epilogue warps, the (max, sum-exp) pairs of three
    // lane quarters for the fourth to merge, and a full / free barrier pair
    static constexpr int XCH_BYTES = CE ? 2 * 3 * 32 * 8 + 4 * 8 : 0;
    // 1024 bytes of alignment slack, the ring (each stage with its full and
    // empty barrier), the staging slots, acc_full[2], acc_empty[2], drain,
    // the tensor-memory address, abort flag and issued k-block count (16),
    // the CE exchange
    static constexpr int BUDGET = RES == 1 ? kSmemLimit : kSmemPerSm / RES - 1024;
    static constexpr int STAGES_RAW =
        (BUDGET - 1024 - EPI_BYTES - 5 * 8 - 16 - XCH_BYTES) / (STAGE_BYTES + 16);
    static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
    static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8;
    static constexpr int SMEM_BYTES =
        1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 16 + XCH_BYTES;
    static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, BN, A_MN ? 1u : 0u, B_MN ? 1u : 0u);
    static_assert(STAGES >= 2, "pipeline depth");
    static_assert(SMEM_BYTES <= BUDGET, "shared memory");
    static_assert(RES * TMEM_COLS <= 512, "tensor memory of the resident CTAs");
};

template <int N>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, uint32_t (&r)[32]);

template <>
__device__ __forceinline__ void tmem_ld_chunk<32>(uint32_t taddr, uint32_t (&r)[32])
{
    tmem_ld32(taddr, r);
}

template <>
__device__ __forceinline__ void tmem_ld_chunk<16>(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void store_out(float *p, uint32_t bits) { *p = __uint_as_float(bits); }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, uint32_t bits)
{
    *p = __float2bfloat16_rn(__uint_as_float(bits));
}
__device__ __forceinline__ void stage_out(float *p, uint32_t bits) { *p = __uint_as_float(bits); }
__device__ __forceinline__ void stage_out(__nv_bfloat16 *p, uint32_t bits)
{
    *p = __float2bfloat16_rn(__uint_as_float(bits));
}

__host__ __device__ inline void tile_coords(int t, const GemmParams &p, int &mt, int &nt)
{
    if (p.m_fastest) {
        mt = t % p.num_m_tiles;
        nt = t / p.num_m_tiles;
    } else {
        nt = t % p.num_n_tiles;
        mt = t / p.num_n_tiles;
    }
}

// Partial cross-entropy statistics of one staged sub-tile (FP32 logits):
// lane l takes token row l of the 32 x 32 box in shared memory (32 vocabulary
// columns starting at vbase; columns at or past V excluded) and returns its
// (max, sum of exp(x - max)), the sum over every column but the token's
// target (which counts in the max; the finalize adds its term, so that the
// loss keeps its precision when the target holds nearly all of the mass);
// the lane whose row holds its token's target column also records the target
// logit.  Lanes without a token return the empty pair.  The row is read as
// eight 16-byte chunks, lane l starting at chunk l mod 8, so the eight lanes
// of each quarter-warp read eight different bank groups; max and sum do not
// depend on the order the values are held in.
__device__ __forceinline__ MaxSum ce_subtile_stats(const float *buf, int lane, int rows, int vbase,
                                                   int V, int tok, int ntok, const GemmParams &p)
{
    if (lane >= rows || tok >= ntok)
        return MaxSum{-INFINITY, 0.f};
    const int64_t y = p.ce_target[tok];
    const int yc = (y >= vbase && y < vbase + 32 && y < V) ? static_cast<int>(y - vbase) : -1;
    const float *rowp = buf + lane * 32;
    const float4 *row4 = reinterpret_cast<const float4 *>(rowp);
    const int nvalid = V - vbase;  // may be <= 0 (a slice past the vocabulary) or > 32
    float v[32];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const float4 q = row4[(kk + lane) & 7];
        v[4 * kk + 0] = q.x;
        v[4 * kk + 1] = q.y;
        v[4 * kk + 2] = q.z;
        v[4 * kk + 3] = q.w;
    }
    if (nvalid < 32) {
        // the vocabulary ends inside this block (the same for the whole warp)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c = (kk + lane) & 7;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (4 * c + e >= nvalid)
                    v[4 * kk + e] = -INFINITY;
        }
    }
    float vmax = v[0];
#pragma unroll
    for (int i = 1; i < 32; ++i)
        vmax = fmaxf(vmax, v[i]);
    float dsum = 0.f;
    if (vmax != -INFINITY) {
        if (yc < 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                dsum += exp_neg_ftz(v[i] - vmax);  // a masked column adds exp(-inf) = 0
        } else {
            // the block of this token's target (one in V / 32 of them)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c = (kk + lane) & 7;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * c + e != yc)
                        dsum += exp_neg_ftz(v[4 * kk + e] - vmax);
            }
        }
    }
    if (yc >= 0)
        p.ce_stats[static_cast<int64_t>(tok) * 4 + 2] = rowp[yc];
    return MaxSum{vmax, dsum};
}

// TMA_STORE: the output is written through tmC, a tensor map over
// out[Ndim][ldo] with box {32, EPI_CHUNK}; otherwise by direct global stores.
// PAIR: a cluster of two CTAs on one tile of 256 (m) x BN (n) with
// tcgen05.mma.cta_group::2 -- each CTA stages its own 128 rows of A and BN/2
// rows of B, the leader (rank 0) issues the MMAs, and each CTA's tensor
// memory receives its 128 rows of the accumulator.  B is read from L2 once
// per pair instead of once per SM.
// CE (vocabulary GEMM, FP32 output, TMA_STORE, eight epilogue warps): also
// emit the partial cross-entropy statistics of every CTA's 128-wide
// vocabulary block, so that the logits need not be read back.  Each warp
// reduces its lane quarter of a sub-tile (ce_subtile_stats); the four warps
// of a half hand their pairs to the one on quarter 0 through shared memory
// (two mbarriers, bounded waits), which merges them in quarter order and
// stores one pair per token.
// ACC (FP32 output): add the product to the output instead of overwriting it
// (TMA reduce-add, or one atomic add per element on the direct path).
template <int BN, bool A_MN, bool B_MN, typename OutT, bool TMA_STORE, bool PAIR, bool CE = false,
          bool ACC = false, int RES = 1, int EW = epi_warps(A_MN, B_MN, CE, ACC)>
__global__ void __launch_bounds__(64 + 32 * EW, RES)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const GemmParams p)
{
    using C = GemmCfg<BN, A_MN, B_MN, PAIR, RES, EW, CE>;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *tiles = smem;
    uint8_t *epi_smem = smem + S * C::STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(epi_smem + C::EPI_BYTES);
    uint64_t *full = bars;
    uint64_t *empty = bars + S;
    uint64_t *acc_full = bars + 2 * S;
    uint64_t *acc_empty = bars + 2 * S + 2;
    uint64_t *drain = bars + 2 * S + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile uint32_t *issued_sh = tmem_slot + 2;  // k-blocks whose copies this CTA issued
    // CE exchange: xch_full[2], xch_free[2], then xch[2][3][32] pairs
    uint64_t *xch_full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(bars) +
                                                      C::BAR_BYTES + 16);
    uint64_t *xch_free = xch_full + 2;
    MaxSum *xch = reinterpret_cast<MaxSum *>(xch_free + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int num_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int num_tiles = p.num_m_tiles * p.num_n_tiles;
    const int num_kb = (p.Kdim + kBlockK - 1) / kBlockK;
    const int split_first = num_tiles - p.split_tiles;  // a whole number of waves
    const int num_items = split_first + (p.split_tiles > 0 ? num_units * p.split_rounds : 0);
    // work item -> tile and k-block range [kb0, kb1): 0 a whole tile, 1 a part
    // of a split tile, -1 no work (every role skips the same items).  Past
    // split_first, item it belongs to unit (it - split_first) % num_units.
    auto item_of = [&](int it, int &t, int &kb0, int &kb1) -> int {
        if (it < split_first) {
            t = it;
            kb0 = 0;
            kb1 = num_kb;
            return 0;
        }
        const int j = it - split_first;
        const int r = j / num_units;       // round of the last wave
        const int u = j - r * num_units;   // the unit
        if (u < p.split_tiles) {
            // the long part of the tile this unit would have run
            if (r != 0)
                return -1;
            t = split_first + u;
            kb0 = 0;
            kb1 = p.split_kb;
            return 1;
        }
        // the units the wave leaves idle take the short parts, round by round
        const int idx = (u - p.split_tiles) + r * (num_units - p.split_tiles);
        if (idx >= p.split_tiles)
            return -1;
        t = split_first + idx;
        kb0 = p.split_kb;
        kb1 = num_kb;
        return 1;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], EW * C::CTAS);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        if (CE) {
            for (int h = 0; h < 2; ++h) {
                mbar_init(&xch_full[h], 3);  // the warps on lane quarters 1..3
                mbar_init(&xch_free[h], 1);  // the warp on quarter 0, once it has read them
            }
        }
        *abort_flag = 0;
        *issued_sh = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (TMA_STORE)
            tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        if (PAIR)
            tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        else
            tmem_alloc(tmem_slot, C::TMEM_COLS);
    }
    tc_fence_before();
    if (PAIR)
        cluster_sync();  // the peer signals the leader's barriers only after they exist
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // everything above overlaps the previous kernel's tail; inputs and
    // outputs are touched only after it has completed
    pdl_wait();
    pdl_launch_dependents();

    // Copies of one k-block into ring slot `stage`: this CTA's A rows from m0
    // and B rows from nb0 at reduction offset k0.  The full barrier (the
    // leader's, for a pair) counts the bytes of both CTAs; the leader arms it.
    const uint64_t pol_a = policy_of(p.l2_a);
    const uint64_t pol_b = policy_of(p.l2_b);
    auto issue_kblock = [&](uint32_t stage, int m0, int nb0, int k0) {
        uint8_t *sa = tiles + stage * C::STAGE_BYTES;
        uint8_t *sb = sa + C::A_BYTES;
        const uint32_t fb = PAIR ? mapa_shared(smem_u32(&full[stage]), 0) : 0u;
        if (leader)
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES * C::CTAS);
        if (A_MN) {
#pragma unroll
            for (int j = 0; j < kBlockM / 64; ++j) {
                if (PAIR)
                    tma_load_2d_pair(&tmA, fb, sa + j * 64 * kBlockK * 2, m0 + 64 * j, k0, pol_a);
                else
                    tma_load_2d(&tmA, &full[stage], sa + j * 64 * kBlockK * 2, m0 + 64 * j, k0, pol_a);
            }
        } else {
            if (PAIR)
                tma_load_2d_pair(&tmA, fb, sa, k0, m0, pol_a);
            else
                tma_load_2d(&tmA, &full[stage], sa, k0, m0, pol_a);
        }
        if (B_MN) {
#pragma unroll
            for (int j = 0; j < C::BN_CTA / 64; ++j) {
                if (PAIR)
                    tma_load_2d_pair(&tmB, fb, sb + j * 64 * kBlockK * 2, nb0 + 64 * j, k0, pol_b);
                else
                    tma_load_2d(&tmB, &full[stage], sb + j * 64 * kBlockK * 2, nb0 + 64 * j, k0, pol_b);
            }
        } else {
            if (PAIR)
                tma_load_2d_pair(&tmB, fb, sb, k0, nb0, pol_b);
            else
                tma_load_2d(&tmB, &full[stage], sb, k0, nb0, pol_b);
        }
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t issued = 0;
            bool ok = true;
            for (int it = unit; it < num_items && ok; it += num_units) {
                int t, kb0, kb1, mt, nt;
                if (item_of(it, t, kb0, kb1) < 0)
                    continue;
                tile_coords(t, p, mt, nt);
                const int m0 = mt * C::TILE_M + static_cast<int>(rank) * kBlockM;  // this CTA's A rows
                const int nb0 = nt * BN + static_cast<int>(rank) * C::BN_CTA;     // this CTA's B rows
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    issue_kblock(stage, m0, nb0, kb * kBlockK);
                    ++issued;
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            *issued_sh = issued;
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (pair: leader only)
        if (lane == 0 && leader) {
            uint32_t stage = 0, phase = 0;
            uint32_t acc = 0, acc_phase = 0;
            bool ok = true;
            for (int it = unit; it < num_items && ok; it += num_units) {
                int t, kb0, kb1;
                if (item_of(it, t, kb0, kb1) < 0)
                    continue;
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(tiles + stage * C::STAGE_BYTES);
                    const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < kBlockK / kUmmaK; ++k) {
                        // K-major: advance 32 bytes along the swizzled row.
                        // MN-major: advance 16 rows of 128 bytes.
                        const uint64_t da = A_MN ? smem_desc_sw128(sa + k * 2048, 64 * kBlockK * 2, 1024)
                                                 : smem_desc_sw128(sa + k * 32, 16, 1024);
                        const uint64_t db = B_MN ? smem_desc_sw128(sb + k * 2048, 64 * kBlockK * 2, 1024)
                                                 : smem_desc_sw128(sb + k * 32, 16, 1024);
                        const uint32_t accumulate = (kb != kb0 || k != 0) ? 1u : 0u;
                        if (PAIR)
                            mma_bf16_pair(d_tmem, da, db, C::IDESC, accumulate);
                        else
                            mma_bf16(d_tmem, da, db, C::IDESC, accumulate);
                    }
                    // frees the smem slot (of both CTAs) when these MMAs finish
                    if (PAIR)
                        mma_commit_pair(&empty[stage], 0x3);
                    else
                        mma_commit(&empty[stage]);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok)
                    break;
                // accumulator ready for the epilogue (of both CTAs)
                if (PAIR)
                    mma_commit_pair(&acc_full[acc], 0x3);
                else
                    mma_commit(&acc_full[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // wait until every MMA issued by this thread has completed
            if (PAIR)
                mma_commit_pair(drain, 0x1);
            else
                mma_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort, kDrainLimitNs);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2 .. 2 + EW - 1)
        const int q = warp & 3;            // tensor-memory lane quarter this warp may access
        const int half = (warp - 2) >> 2;  // EW = 8: which alternate sub-tiles of the quarter
        const int row = q * 32 + lane;
        OutT *out = static_cast<OutT *>(p.out);
        const uint64_t pol_out = policy_of(p.l2_out);
        OutT *slots = reinterpret_cast<OutT *>(epi_smem + (warp - 2) * C::NSLOT * C::EPI_SLOT_BYTES);
        constexpr int SLOT_ELEMS = C::EPI_SLOT_BYTES / static_cast<int>(sizeof(float));
        uint32_t slot = 0;
        uint32_t xch_phase = 0;
        // where this warp releases an accumulator: the leader's barrier
        const uint32_t empty_addr0 = PAIR ? mapa_shared(smem_u32(&acc_empty[0]), 0) : 0u;
        uint32_t acc = 0, acc_phase = 0;
        for (int it = unit; it < num_items; it += num_units) {
            int t, kb0, kb1, mt, nt;
            const int kind = item_of(it, t, kb0, kb1);
            if (kind < 0)
                continue;
            const bool part = kind == 1;  // one of two addends of a split tile
            // every lane waits, then the warp agrees, so the .sync.aligned
            // tensor-memory loads below always run with the full warp
            const bool ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok))
                break;
            tc_fence_after();
            tile_coords(t, p, mt, nt);
            const int mbase = mt * C::TILE_M + static_cast<int>(rank) * kBlockM;
            const int m = mbase + row;
            const int n0 = nt * BN;
            const bool m_ok = m < p.Mdim;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
#pragma unroll 1
            for (int c = half * C::EPI_CHUNK; c < BN; c += (EW / 4) * C::EPI_CHUNK) {
                if (TMA_STORE && n0 + c >= p.Ndim)
                    break;  // the rest of this tile lies beyond the output
                uint32_t r[32];
                tmem_ld_chunk<C::EPI_CHUNK>(taddr + c, r);
                tmem_ld_wait();
                if (TMA_STORE) {
                    // the slot is free once the store issued NSLOT sub-tiles
                    // ago has finished reading it
                    if (lane == 0)
                        bulk_wait_read<C::NSLOT - 1>();
                    __syncwarp();
                    OutT *buf = slots + slot * SLOT_ELEMS;
#pragma unroll
                    for (int j = 0; j < C::EPI_CHUNK; ++j)
                        stage_out(buf + j * 32 + lane, r[j]);  // box row j = output row n0+c+j
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (ACC || part)
                            tma_reduce_add_2d(&tmC, buf, mbase + q * 32, n0 + c);
                        else if (p.l2_out)
                            tma_store_2d_hint(&tmC, buf, mbase + q * 32, n0 + c, pol_out);
                        else
                            tma_store_2d(&tmC, buf, mbase + q * 32, n0 + c);
                        bulk_commit();
                    }
                    if constexpr (A_MN && B_MN && !ACC) {
                        // dW: a short reduction (the tokens) and a large FP32
                        // output; spacing the sub-tile stores keeps them from
                        // delaying the operand loads queued behind them
                        // (measured 214.0 -> 206.9 us at 1024 x 4096 x 32768)
                        if (kDwStorePaceNs > 0)
                            __nanosleep(kDwStorePaceNs);
                    }
                    if constexpr (CE) {
                        // the TMA store only reads the slot, so it can be read here too
                        const int tok = n0 + c + lane;
                        const MaxSum sv =
                            ce_subtile_stats(reinterpret_cast<const float *>(buf), lane,
                                             C::EPI_CHUNK, mbase + q * 32, p.Mdim, tok, p.Ndim, p);
                        MaxSum *xh = xch + half * 3 * 32;
                        if (q != 0) {
                            if (mbar_wait(&xch_free[half], xch_phase ^ 1, abort_flag, p.wait_limit_ns))
                                xh[(q - 1) * 32 + lane] = sv;
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive(&xch_full[half]);
                        } else {
                            const bool got =
                                mbar_wait(&xch_full[half], xch_phase, abort_flag, p.wait_limit_ns);
                            MaxSum r = sv;
                            if (got) {
#pragma unroll
                                for (int j = 0; j < 3; ++j)
                                    r = merge(r, xh[j * 32 + lane]);
                            }
                            __syncwarp();
                            if (lane == 0)
                                mbar_arrive(&xch_free[half]);
                            if (got && lane < C::EPI_CHUNK && tok < p.Ndim) {
                                const int64_t block = mt * C::CTAS + static_cast<int>(rank);
                                p.ce_partial[block * p.Ndim + tok] = make_float2(r.m, r.d);
                            }
                        }
                        xch_phase ^= 1;
                    }
                    slot = slot + 1 == C::NSLOT ? 0 : slot + 1;
                } else if (m_ok) {
                    OutT *o = out + static_cast<int64_t>(n0 + c) * p.ldo + m;
#pragma unroll
                    for (int j = 0; j < C::EPI_CHUNK; ++j)
                        if (n0 + c + j < p.Ndim) {
                            // FP32 only: an accumulating or half-tile store adds
                            if (sizeof(OutT) == 4 && (ACC || part))
                                atomicAdd(reinterpret_cast<float *>(o) + static_cast<int64_t>(j) * p.ldo,
                                          __uint_as_float(r[j]));
                            else
                                store_out(o + static_cast<int64_t>(j) * p.ldo, r[j]);
                        }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR)
                    mbar_arrive_cluster(empty_addr0 + acc * 8);
                else
                    mbar_arrive(&acc_empty[acc]);
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (TMA_STORE && lane == 0)
            bulk_wait_all();  // every output byte written before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) {
        // Every role of both CTAs has finished (the leader's MMAs are
        // drained); the abort flags and issued counts are final.
        cluster_sync();
        const uint32_t peer = rank ^ 1u;
        const int peer_abort = static_cast<int>(
            ld_shared_cluster_u32(mapa_shared(smem_u32(const_cast<int *>(abort_flag)), peer)));
        if (*abort_flag || peer_abort) {
            // After a timeout the two producers may have stopped at different
            // k-blocks, so the leader's full barriers may wait for bytes that
            // will never come, or copies may still be landing in either CTA.
            // A k-block issued by one CTA implies that the MMAs of the
            // k-block S earlier in its slot completed, hence that slot's
            // previous phase completed in both CTAs.  So the CTA that is
            // behind can issue (and the leader arm) the k-blocks it missed;
            // every issued copy then belongs to a phase that completes, and
            // the leader waits for the last phase of each slot.  The copied
            // data is not used.
            if (threadIdx.x == 0) {
                const uint32_t mine = *issued_sh;
                const uint32_t theirs = ld_shared_cluster_u32(
                    mapa_shared(smem_u32(const_cast<uint32_t *>(issued_sh)), peer));
                const uint32_t all = mine > theirs ? mine : theirs;
                for (uint32_t i = mine; i < all; ++i)
                    issue_kblock(i % S, static_cast<int>(rank) * kBlockM,
                                 static_cast<int>(rank) * C::BN_CTA, 0);
                if (leader) {
                    volatile int no_abort = 0;
                    for (uint32_t i = all > S ? all - S : 0; i < all; ++i)
                        mbar_wait(&full[i % S], (i / S) & 1u, &no_abort, kDrainLimitNs);
                }
            }
            cluster_sync();  // every copy into either CTA has landed
        }
        cluster_sync();  // neither CTA reads the other's shared memory any more
    } else {
        if (*abort_flag && threadIdx.x == 0) {
            // Copies issued but never consumed may still be landing: wait for
            // the last phase of each slot (older phases completed before
            // their slots were refilled).  The CTA stays resident meanwhile.
            const uint32_t all = *issued_sh;
            volatile int no_abort = 0;
            for (uint32_t i = all > S ? all - S : 0; i < all; ++i)
                mbar_wait(&full[i % S], (i / S) & 1u, &no_abort, kDrainLimitNs);
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
        else
            tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
    if (threadIdx.x == 0 && *abort_flag && p.status)
        atomicOr(p.status, 2);
}

}  // namespace lmh
