/*
 * lmhead.h -- C ABI of the B200 (sm_100a) LM-head loss path.
 *
 * The library computes, on one GPU:
 *   lmhead_fwd     logits[M,V] = X[M,K] . W[V,K]^T, FP32 accumulator stored
 *                  unrounded (or a BF16 copy of it, for comparison)
 *   ce_fwd         per-row cross-entropy statistics {m, d, x_y, loss}
 *   ce_bwd         dlogits = (softmax - onehot(target)) * grad_loss, in FP32,
 *                  rounded to the output dtype only at the store
 *   lmhead_bwd_dx  dX[M,K] = dlogits[M,V] . W[V,K]
 *   lmhead_bwd_dw  dW[V,K] = dlogits[M,V]^T . X[M,K]
 *
 * Sources (page title, section):
 *   [P1] Megatron-LM PR #6252 "Add mixed-precision (FP32) LM output logits":
 *        "What does this PR do?" (FP32 GEMM output instead of BF16-rounded
 *        logits; gradients cast back to BF16 under the GEMM contract),
 *        "Tests" (only bf16 and fp32 logit dtypes are accepted, fp16 is
 *        rejected), "Integer bitwise exactness results".
 *   [P2] TransformerEngine #2325 "[Pytorch] change fused cross entropy
 *        backward grad to fp32 and reduce one read": "Description" and
 *        "Changes" (backward computed in FP32, one fewer read of the logits)
 *        and the review discussion (the forward saves the target, n_rows x 1,
 *        and m_d_X_y, n_rows x 4).
 *
 * Conventions shared by every call
 *   - All array arguments are DEVICE pointers into row-major, contiguous
 *     buffers owned by the caller.  The library allocates nothing, keeps no
 *     per-call state and never synchronises: every call only enqueues work on
 *     `stream` (NULL = legacy default stream) and returns.
 *   - BF16 data is IEEE binary32's upper 16 bits; FP32 is IEEE binary32.
 *   - Errors are returned, never raised: arguments are validated on the host
 *     before anything is launched, and a failing launch maps to LMH_ERR_CUDA.
 *   - `status` (nullable) is a device int32 word that kernels OR condition
 *     bits into (LMH_DEV_*).  The caller zeroes it, and reads it after the
 *     stream has been synchronised.  Nothing is trapped on the device.
 *   - Sizes are int64; every size must be >= 1 unless stated otherwise.
 */
#ifndef LMHEAD_H_
#define LMHEAD_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported from liblmhead.so (everything else in the library is hidden). */
#if defined(__GNUC__)
#define LMH_API __attribute__((visibility("default")))
#else
#define LMH_API
#endif

/* Host-side result of a call. */
typedef enum {
    LMH_OK = 0,
    LMH_ERR_INVALID_ARG = 1,  /* null pointer, size < 1, size too large   */
    LMH_ERR_MISALIGNED = 2,   /* pointer or row stride breaks the layout  */
    LMH_ERR_UNSUPPORTED = 3,  /* dtype or stride value not supported      */
    LMH_ERR_CUDA = 4          /* the CUDA runtime reported an error       */
} lmh_status_t;

/* Element types.  As with the logit-dtype option of [P1] "Tests", only FP32
 * and BF16 are accepted; LMH_F16 (and any other value) is rejected with
 * LMH_ERR_UNSUPPORTED. */
typedef enum { LMH_F32 = 0, LMH_BF16 = 1, LMH_F16 = 2 } lmh_dtype_t;

/* Bits ORed into *status by the kernels. */
#define LMH_DEV_BAD_TARGET 0x1   /* a target neither ignore_index nor in [0,V);
                                    the row was treated as ignored          */
#define LMH_DEV_PIPE_TIMEOUT 0x2 /* a pipeline wait gave up (bounded spin);
                                    the output of that call is not valid    */

/* Same type as cudaStream_t. */
typedef struct CUstream_st *lmh_stream_t;

/* logits = X . W^T  ([P1] "What does this PR do?").
 *   X       [M,K] BF16, K contiguous.         W [V,K] BF16, K contiguous.
 *   logits  [M,V] FP32 (out_dtype LMH_F32: the accumulator, unrounded) or
 *           BF16 (LMH_BF16: the accumulator rounded to nearest even).
 *   Requirements: K % 8 == 0 (16-byte rows for the tensor-memory copies),
 *   X and W 16-byte aligned, logits 4-byte aligned; M, V, K <= 2^31 - 1.
 *   Accumulation is FP32 inside the tensor cores; when every partial sum is
 *   an exactly representable integer (BF16 integers in [-8,8] with
 *   K * 64 < 2^24, [P1] "Integer bitwise exactness results") the FP32 output
 *   is exact.  Deterministic: repeated calls give identical bits. */
LMH_API lmh_status_t lmhead_fwd(const void *X, const void *W, void *logits, int32_t out_dtype,
                        int64_t M, int64_t K, int64_t V, int32_t *status,
                        lmh_stream_t stream);

/* Cross-entropy forward statistics ([P2] discussion: target and m_d_X_y).
 *   logits  [M,V] FP32.   target [M] int64.
 *   stats   [M,4] FP32, per row {m, d, x_y, loss}:
 *             m = max_j x_j, d = sum_j exp(x_j - m), x_y = x[target],
 *             loss = -log softmax(x)_target = m + log(d) - x_y, computed as
 *             log1p(s exp(m - x_y)) with s = d - exp(x_y - m) summed over the
 *             other columns, so that it keeps its precision when the target
 *             holds nearly all of the row's mass.
 *   A row whose target equals ignore_index is not read and gets
 *   {0,0,0,0}.  A target outside [0,V) that is not ignore_index sets
 *   LMH_DEV_BAD_TARGET in *status and the row is treated as ignored.
 *   Any V >= 1; no alignment beyond the element size. */
LMH_API lmh_status_t ce_fwd(const float *logits, const int64_t *target, float *stats,
                    int64_t M, int64_t V, int64_t ignore_index, int32_t *status,
                    lmh_stream_t stream);

/* Cross-entropy backward in FP32 ([P2] "Description", "Changes"; the BF16
 * cast at the end is the one of [P1] "What does this PR do?").
 *   logits     [M,V] FP32, the same buffer ce_fwd read.
 *   target     [M] int64.   stats [M,4] FP32 from ce_fwd.
 *   grad_loss  FP32 upstream gradient of the per-row loss:
 *              grad_loss_stride 0 = one scalar for every row,
 *              1 = one value per row ([M]); anything else is unsupported.
 *   dlogits    [M,V], dl_dtype LMH_F32 or LMH_BF16 (round to nearest even):
 *              dl[i,j] = (exp(x_ij - m_i) / d_i - [j == target_i]) * g_i;
 *              at the target, softmax - 1 = exp(-loss_i) - 1 is taken as
 *              expm1(-loss_i) from the saved loss (no cancellation).
 *              Ignored and bad-target rows are written as zeros.
 *              With LMH_F32, dlogits may be the logits buffer itself
 *              (in-place; each element is read before it is overwritten).
 *   Any V >= 1. */
LMH_API lmh_status_t ce_bwd(const float *logits, const int64_t *target, const float *stats,
                    const float *grad_loss, int64_t grad_loss_stride, void *dlogits,
                    int32_t dl_dtype, int64_t M, int64_t V, int64_t ignore_index,
                    int32_t *status, lmh_stream_t stream);

/* logits = X . W^T (FP32) and the cross-entropy forward statistics of those
 * logits in one pass over them: the vocabulary GEMM's epilogue reduces every
 * 128-wide vocabulary block of each token row to a partial (max, sum-exp,
 * the sum leaving out the target's own term) in
 * `workspace` and records the target logit while the tile is still on chip,
 * and a second kernel merges each token's partials (in a fixed order) into
 * stats[M,4] = {m, d, x_y, loss}.  The logits are written but not read back
 * -- the "one fewer read of the logits" of [P2] "Changes", taken one step
 * further than a separate ce_fwd.
 *   Arguments and results as lmhead_fwd (out_dtype FP32) followed by ce_fwd
 *   (same tolerances; the statistics are merged in a different order, so they
 *   need not be bitwise equal to ce_fwd's).
 *   workspace: device scratch of at least lmhead_fwd_ce_workspace_bytes(M, V)
 *   bytes, 16-byte aligned, owned by the caller; its contents on entry do not
 *   matter and on return are unspecified.  When V % 4 != 0 or logits is not
 *   16-byte aligned the call runs lmhead_fwd then ce_fwd and does not touch
 *   the workspace (which may then be NULL). */
LMH_API lmh_status_t lmhead_fwd_ce(const void *X, const void *W, const int64_t *target,
                                   float *logits, float *stats, void *workspace,
                                   int64_t workspace_bytes, int64_t M, int64_t K, int64_t V,
                                   int64_t ignore_index, int32_t *status, lmh_stream_t stream);

/* Scratch bytes lmhead_fwd_ce needs: 2 * ceil(V / 256) blocks x M tokens x
 * 8 bytes (2 MB for M = 1024, V = 32768).  -1 for sizes out of range. */
LMH_API int64_t lmhead_fwd_ce_workspace_bytes(int64_t M, int64_t V);

/* lmhead_fwd_ce for callers that cannot allocate device memory (no
 * counterpart on the pages).  Some callers cannot give the library a scratch
 * buffer: plug-ins whose host framework owns all device memory and offers
 * them no allocator, and code on paths where calling cudaMalloc (which may
 * synchronise the device) is not allowed.  This call computes exactly what
 * lmhead_fwd_ce computes (same arguments minus the workspace) but keeps the
 * partial statistics in a fixed 8 MiB array inside the library, which every
 * GPU that loads the library holds until the process exits.  It allocates
 * nothing and calls no allocating routine.
 *   Limit: M * 2 * ceil(V / 256) <= 1048576 (e.g. M = 4096 with V up to
 *   32768); larger problems return LMH_ERR_INVALID_ARG before anything is
 *   launched.  (When V % 4 != 0 or logits is not 16-byte aligned the call
 *   runs lmhead_fwd then ce_fwd, which need no scratch, at any size.)
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  The address is kept for the life of the
 *   process: do not use this call on a device after cudaDeviceReset (or
 *   after its primary context has been destroyed), when the library's
 *   device image, and the array with it, may be loaded at another address.
 *   Every call shares the one array per device: calls that may run at the
 *   same time on the GPU (different streams, or different host threads)
 *   race and corrupt each other's results.  Nothing in the array has to start
 *   at zero: each call writes every entry it later reads. */
LMH_API lmh_status_t lmhead_fwd_ce_noalloc(const void *X, const void *W, const int64_t *target,
                                           float *logits, float *stats, int64_t M, int64_t K,
                                           int64_t V, int64_t ignore_index, int32_t *status,
                                           lmh_stream_t stream);

/* Vocabulary-parallel cross-entropy (the vocabulary split across devices, as
 * Megatron's VocabParallelCrossEntropy does, named in [P2] "Description").
 * Device r holds logits[M, V_r] for vocabulary entries [offset_r, offset_r +
 * V_r) of a vocabulary of vocab_total; targets are global ids.  The three
 * calls below are the per-device parts; the exchange between devices (an
 * all-gather of the [M,4] shard records) is the caller's.
 *
 * ce_fwd_shard: per row of this shard, shard_stats[M,4] = {m_r, d_r, x_y or 0,
 *   1 if the target is in this shard else 0}: m_r = the max over the shard's
 *   columns, d_r = sum of exp(x - m_r) over them, leaving out the target's own
 *   term in the shard that holds it; ignored rows (target ==
 *   ignore_index) and bad targets (outside [0, vocab_total)) give zeros, bad
 *   targets also set LMH_DEV_BAD_TARGET.
 *   Requirements: 0 <= vocab_offset, vocab_offset + V <= vocab_total. */
LMH_API lmh_status_t ce_fwd_shard(const float *logits, const int64_t *target, float *shard_stats,
                                  int64_t M, int64_t V, int64_t vocab_offset, int64_t vocab_total,
                                  int64_t ignore_index, int32_t *status, lmh_stream_t stream);

/* ce_merge_shards: stats[M,4] = {m, d, x_y, loss} of the whole vocabulary
 * from the num_shards records of every shard, laid out shard-major
 * (shard_stats[r][M][4]): m = max_r m_r, s = sum_r d_r exp(m_r - m) taken in
 * shard order (deterministic; every column but the target), x_y from the
 * owning shard, d = s + exp(x_y - m), loss = log1p(s exp(m - x_y)).  The
 * result is what ce_fwd gives on the whole rows, up to the order of the sums. */
LMH_API lmh_status_t ce_merge_shards(const float *shard_stats, int64_t num_shards,
                                     const int64_t *target, float *stats, int64_t M,
                                     int64_t vocab_total, int64_t ignore_index, int32_t *status,
                                     lmh_stream_t stream);

/* ce_bwd_shard: ce_bwd on a shard, with the merged stats: dl[i,j] =
 * (exp(x_ij - m_i) / d_i - [vocab_offset + j == target_i]) * g_i, the target's
 * entry as in ce_bwd. */
LMH_API lmh_status_t ce_bwd_shard(const float *logits, const int64_t *target, const float *stats,
                                  const float *grad_loss, int64_t grad_loss_stride, void *dlogits,
                                  int32_t dl_dtype, int64_t M, int64_t V, int64_t vocab_offset,
                                  int64_t vocab_total, int64_t ignore_index, int32_t *status,
                                  lmh_stream_t stream);

/* dX = dlogits . W, the input gradient of logits = X . W^T
 * ([P1] "What does this PR do?", backward under the GEMM contract: the
 * gradient GEMMs take the BF16 dlogits cast from the FP32 backward).
 *   dlogits [M,V] BF16.  W [V,K] BF16.
 *   dX      [M,K] FP32 (LMH_F32) or BF16 (LMH_BF16).
 *   Requirements: V % 8 == 0 and K % 8 == 0 (16-byte rows), inputs 16-byte
 *   aligned.  Deterministic.  With an FP32 dX the output tiles of a last
 *   wave that would leave most SMs idle are computed as two halves of the
 *   reduction that are both added into rows of dX the call first zeroes on
 *   the stream; with two addends the order of the additions does not change
 *   the result. */
LMH_API lmh_status_t lmhead_bwd_dx(const void *dlogits, const void *W, void *dX, int32_t out_dtype,
                           int64_t M, int64_t K, int64_t V, int32_t *status,
                           lmh_stream_t stream);

/* dW = dlogits^T . X, the weight gradient of logits = X . W^T
 * ([P1] "What does this PR do?", backward under the GEMM contract: the
 * gradient GEMMs take the BF16 dlogits cast from the FP32 backward).
 *   dlogits [M,V] BF16.  X [M,K] BF16.
 *   dW      [V,K] FP32 (LMH_F32) or BF16 (LMH_BF16).
 *   Requirements: V % 8 == 0 and K % 8 == 0, inputs 16-byte aligned.
 *   Deterministic. */
LMH_API lmh_status_t lmhead_bwd_dw(const void *dlogits, const void *X, void *dW, int32_t out_dtype,
                           int64_t M, int64_t K, int64_t V, int32_t *status,
                           lmh_stream_t stream);

/* dW += dlogits^T . X: the weight gradient accumulated into an FP32 main
 * gradient (beta = 1), as when gradients of several micro-batches are summed
 * before the optimizer step.
 *   dlogits [M,V] BF16, X [M,K] BF16, dW [V,K] FP32 (read and written).
 *   Each dW element receives exactly one FP32 addition per call (performed
 *   by the TMA reduce-add of the epilogue, or one atomic add where a tensor
 *   map cannot describe dW), so the result does not depend on scheduling:
 *   dW_out = fl(dW_in + fl32-accumulated product).
 *   Requirements as lmhead_bwd_dw. */
LMH_API lmh_status_t lmhead_bwd_dw_acc(const void *dlogits, const void *X, float *dW, int64_t M,
                                       int64_t K, int64_t V, int32_t *status, lmh_stream_t stream);

/* Static, NUL-terminated description of a status value. */
LMH_API const char *lmh_status_string(lmh_status_t s);

/* Library version, major * 10000 + minor * 100 + patch. */
LMH_API int32_t lmh_version(void);

/* Self-test of the pipeline watchdog (failure detection; no counterpart on
 * the pages).  Launches one CTA whose thread waits, with the same bounded
 * wait the GEMM pipelines use, on a shared-memory barrier that nothing
 * arrives at, with a limit of `limit_us` microseconds (1..1000000).  The wait
 * gives up, the CTA unwinds and LMH_DEV_PIPE_TIMEOUT is ORed into *status
 * (device int32, required).  Nothing faults or hangs; the context stays
 * usable.  Asynchronous like every other call. */
LMH_API lmh_status_t lmh_watchdog_selftest(int32_t *status, int64_t limit_us, lmh_stream_t stream);

/* Self-test of the GEMM's own failure path (failure detection; no
 * counterpart on the pages).  Runs lmhead_fwd with FP32 logits, the same
 * kernel selection and arguments, but with every pipeline wait limited to
 * `limit_ns` nanoseconds (1..1000000000) instead of two seconds.  With a limit
 * far below the time one output tile takes (1 ns, say), a wait runs out: the
 * CTA stops, lets every operand copy it issued land and every MMA it issued
 * finish, frees its tensor memory and ORs LMH_DEV_PIPE_TIMEOUT into *status
 * (device int32, required).  The logits are then not valid.  Nothing faults
 * or hangs, and later calls on the stream run normally. */
LMH_API lmh_status_t lmh_gemm_watchdog_selftest(const void *X, const void *W, float *logits,
                                                int64_t M, int64_t K, int64_t V, int64_t limit_ns,
                                                int32_t *status, lmh_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LMHEAD_H_ */
