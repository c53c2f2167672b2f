/*
 * cce.h -- C ABI of libcce.so, Cut Cross-Entropy (CCE) for NVIDIA B200 (sm_100a).
 *
 * What is computed (Cut Cross-Entropy abstract, sentences 4-6 and 9):
 *   for token embeddings E (N x D), classifier C (V x D) and labels y,
 *     lse[i]  = log sum_v exp(E_i . C_v)
 *     loss[i] = lse[i] - E_i . C_{y_i}          (0 where y_i == ignore_index)
 *   without ever writing the N x V logit matrix to global memory; and the
 *   gradients of sum_i dloss[i] * loss[i]:
 *     G[i,v] = dloss[i] * (softmax(E_i C^T)[v] - [v == y_i]),
 *     dE = G C,  dC = G^T E,
 *   where every entry of G whose |softmax - onehot| is below filter_eps is
 *   left out (the abstract's sentence 9: gradient elements too small to
 *   matter at the working precision are skipped).
 *
 * Conventions for every entry point:
 *   - All matrix arguments are DEVICE pointers to row-major, contiguous data.
 *     E, C are bf16 (raw 16-bit storage, passed as void*); y is int64;
 *     loss, lse, dloss, dE, dC are fp32.
 *   - D must be a multiple of 8 and E, C must be 16-byte aligned (the kernels
 *     stream them with TMA).  N, D, V must be positive and fit in int32.
 *   - The caller owns every buffer, including the workspace.  The library
 *     never allocates device memory: the extra global memory of a call is
 *     exactly the workspace, whose size is O(N) (see the *_workspace_size
 *     functions).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and run on the current CUDA device.
 *   - Argument errors are detected on the host: the call returns a non-zero
 *     status and launches nothing.  Conditions found on the device (an
 *     invalid label, a bounded wait that gave up) set bits in the status
 *     block at the head of the workspace, read with cce_read_status.
 *   - Not thread-safe across concurrent calls sharing one workspace.
 */
#ifndef CCE_H_
#define CCE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CCE_API __attribute__((visibility("default")))
#else
#define CCE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CCE_OK = 0,
  CCE_ERR_INVALID_ARG = 1,        /* null pointer, non-positive or too large size, D % 8 != 0 */
  CCE_ERR_MISALIGNED = 2,         /* E, C, or an fp32 vector not suitably aligned */
  CCE_ERR_WORKSPACE_TOO_SMALL = 3,
  CCE_ERR_UNSUPPORTED_DEVICE = 4, /* the current device is not sm_100 */
  CCE_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
  CCE_ERR_TIMEOUT = 6,            /* device: a bounded wait gave up (cce_read_status) */
  CCE_ERR_BAD_LABEL = 7           /* device: a label outside [0, V) (cce_read_status) */
} cce_status_t;

/* Status block decoded by cce_read_status. */
typedef struct {
  uint64_t flags;       /* bit 0: a wait timed out; bit 1: an invalid label was seen */
  uint64_t live_tiles;  /* backward: 32x32 units (tokens x vocabulary rows) holding at
                           least one gradient entry that was added */
  uint64_t dead_tiles;  /* backward: units recomputed and found to hold no entry
                           at or above the filter threshold */
  uint64_t logit_tiles; /* forward: 128x256 logit tiles computed on chip;
                           backward: 128x256 logit tiles recomputed on chip */
  uint64_t pruned_tiles;/* backward: units proven negligible without recomputing
                           them; live + dead + pruned = ceil(N/32) * ceil(V/32)
                           when filter_eps > 0 */
  uint64_t flat_units;  /* backward: the live units that lie in flat token blocks
                           and were formed one correct-token entry at a time,
                           without recomputing a logit tile (included in
                           live_tiles).  Added in version 102. */
} cce_counters_t;

/* Workspace bytes needed by cce_forward for these sizes on the current device
 * (N * splits * 8 bytes of per-split (max, sum) pairs plus a 256-byte status
 * block; splits <= 128, or up to 256 when cce_debug_set_forward_schedule
 * asks for them; 125 on a 256000-entry vocabulary).  Depends on the debug
 * schedule knobs in force.  Returns 0 if the sizes are invalid or no device
 * is usable. */
CCE_API size_t cce_forward_workspace_size(int64_t N, int64_t D, int64_t V);

/* Workspace bytes needed by cce_backward: the status block plus the
 * pre-pass (O(N + V/32): one norm per token, a few words per 128-token
 * block, one bit per vocabulary row).  Returns 0 if the sizes are invalid. */
CCE_API size_t cce_backward_workspace_size(int64_t N, int64_t D, int64_t V);

/* Forward pass (abstract, sentences 4-6): per-token loss and log-sum-exp.
 *   E     [N x D] bf16        token embeddings
 *   C     [V x D] bf16        classifier rows
 *   y     [N]     int64       labels; ignore_index marks tokens without a loss
 *   loss  [N]     fp32 out    lse - correct logit; 0 if ignored; NaN if the
 *                             label is outside [0, V) (status flag bit 1)
 *   lse   [N]     fp32 out    log-sum-exp over the vocabulary (also for ignored rows)
 *   workspace, workspace_bytes: device scratch, >= cce_forward_workspace_size
 * The logits exist only in tensor memory on chip.  If a bounded wait of the
 * logit kernel gave up (status flag bit 0), every loss and lse of the call is
 * NaN. */
CCE_API cce_status_t cce_forward(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D, int64_t V,
                         int64_t ignore_index, float* loss, float* lse, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Backward pass (abstract, sentences 4 and 9): gradients of sum_i dloss[i] * loss[i].
 *   lse   [N] fp32   from cce_forward on the same E, C
 *   dloss [N] fp32   upstream gradient per token (e.g. 1/#kept for a mean)
 *   filter_eps       an entry of (softmax - onehot) below filter_eps in
 *                    magnitude is left out of G; <= 0 keeps every entry
 *                    (exact gradient)
 *   dE    [N x D] fp32 out (overwritten), dC [V x D] fp32 out (overwritten)
 * The logit tiles are recomputed on chip; rows with y == ignore_index
 * contribute nothing.  With filter_eps > 0 a pre-pass bounds every logit by
 * |E_i| max_v |C_v| (Cauchy-Schwarz).  In a 128-token block where that bound
 * puts every softmax probability below filter_eps, only the correct-token
 * entries can survive: they are formed one token at a time (one dot product
 * each) and no logit tile of the block is recomputed.  Other blocks are
 * recomputed tile by tile and tested entry by entry.  The result is the same
 * as testing every entry.  Accumulation order across tiles is not fixed
 * (fp32 atomics), so results may differ in the last bits between runs. */
CCE_API cce_status_t cce_backward(const void* E, const void* C, const int64_t* y, const float* lse, const float* dloss,
                          int64_t N, int64_t D, int64_t V, int64_t ignore_index, float filter_eps, float* dE,
                          float* dC, void* workspace, size_t workspace_bytes, void* stream);

/* Allocation-free forward.  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory when they need the
 * loss -- code handed only its input and output buffers (plugins, hooks), a
 * step running under an allocator that is locked, exhausted or forbids
 * cudaMalloc -- and so cannot supply the workspace cce_forward needs.
 * Inputs, outputs and results are those of cce_forward.  The scratch (status
 * block and per-split partials) lives in a static 8 MiB device array inside
 * the library, which every GPU that loads this part of the library holds
 * until the process exits (with CUDA's lazy module loading the array is
 * created at the first call on the device, not by the call itself; later
 * calls change nothing in the device's free memory).
 *   - Problems whose forward workspace (cce_forward_workspace_size) exceeds
 *     8 MiB are rejected with CCE_ERR_WORKSPACE_TOO_SMALL before anything is
 *     launched (e.g. N = 65536 tokens, V = 262144); invalid sizes or no sm_100
 *     device give CCE_ERR_INVALID_ARG.
 *   - No cudaMalloc, cudaFree or other allocating routine is called.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is cached per device and CUDA
 *     context: after cudaDeviceReset (or on another context) the next call
 *     looks it up again, so that first call after a reset also belongs
 *     before any capture.
 *   - Every call shares the one array and it keeps the last call's contents:
 *     each call clears the status block it needs, and the kernels write
 *     every partial the call reads, but calls whose work overlaps on the GPU
 *     (unordered streams) race on the array and corrupt each other's results.
 *   - The status block is not readable by the caller.  An invalid label shows
 *     as a NaN loss; a bounded wait that gave up (a partial never written)
 *     makes every loss and lse of the call NaN. */
CCE_API cce_status_t cce_forward_noalloc(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D,
                                         int64_t V, int64_t ignore_index, float* loss, float* lse, void* stream);

/* Options of cce_backward_ex (bit flags). */
typedef enum {
  CCE_BWD_DEFAULT = 0,
  /* Bitwise reproducible dE/dC: every per-tile partial product (fp32, from
   * the tensor cores) is rounded once to a 64-bit fixed-point value whose
   * power-of-two scale puts a bound on the largest possible gradient entry
   * (from max|dloss|, max_v|C_v|, max_i|E_i| and N) just under 2^61, and
   * accumulated with integer adds, whose result does not depend on the order
   * in which the tiles finish; a final pass converts to the output type.
   * Needs an extra (N + V) * D * 8 bytes of workspace. */
  CCE_BWD_DETERMINISTIC = 1,
  /* dE and dC are written as bf16 (round to nearest even) instead of fp32.
   * Without CCE_BWD_STRIPES it implies CCE_BWD_DETERMINISTIC (the same
   * fixed-point accumulation, converted once); with CCE_BWD_STRIPES the
   * sums go to fp32 scratch in the workspace ((N + V) * D * 4 bytes) and are
   * rounded to bf16 once at the end. */
  CCE_BWD_BF16_GRADS = 2,
  /* Add this call's gradients to the contents of dE and dC instead of
   * overwriting them (no zeroing pass): gradient accumulation over
   * micro-batches, or zeroing done by the caller where it costs nothing,
   * e.g. on another stream while the compute-bound forward runs.  The
   * caller must have written dE and dC (zeros before a first call).  With
   * CCE_BWD_DETERMINISTIC each output entry gets one add of this call's
   * fixed-point sum, in fp32 (or, with CCE_BWD_BF16_GRADS, the old bf16
   * value plus the sum rounded once to bf16), so the result is still
   * bitwise reproducible.  No extra workspace. */
  CCE_BWD_ACCUMULATE = 4,
  /* cce_backward_prepare has already run on this workspace for the same C,
   * N, D, V (e.g. on a second stream while the forward ran): the backward
   * skips its own pass over C and uses the stored max_v |C_v|.  Same result
   * as without the flag.  No extra workspace. */
  CCE_BWD_PREPARED = 8,
  /* Run the backward through stripes of the softmax gradient: the
   * vocabulary is taken 4096 rows at a time; per stripe the logit tiles are
   * recomputed on chip and G = dloss (softmax - onehot) is stored in bf16
   * into one of three stripe buffers in the workspace, then dC of the
   * stripe's rows = G^T E is formed with every token as the reduction
   * dimension (each entry written once) and dE += G C of the stripe (one bulk
   * reduce-add per 256 x 256 dE tile and stripe).  Only these stripes of G
   * ever exist in global memory: 3 x min(N, 16384) x 4096 x 2 bytes (201 MB
   * at N = 8192), whatever V; tokens beyond 16384 are taken in further
   * launches whose dC contributions are added.  Far less fp32 reduction
   * traffic than adding every logit tile's partial products, so the tensor
   * cores set the pace.  With filter_eps <= 0 this is the dense (exact)
   * backward, the same result as without the flag up to fp32 summation
   * order.  With filter_eps > 0 the pre-pass runs first (flat blocks go to
   * the flat-row kernel, as in the default path); the stripe kernel skips
   * the recompute of 256-token blocks that are entirely flat, zeroes the
   * entries below the threshold (and the flat blocks' rows) in G, and skips
   * the all-zero G tiles in the dC and dE products.  This beats the default
   * filtered path (per-tile contractions of live 32 x 32 units with fp32
   * reduce-adds) when a large share of the units is live, and loses when
   * the gradient is sparse (measured on a Gemma-2-2B-shaped head with peaky
   * logits: 27 ms against 53 ms at 61 % live units; 11.5 ms against 9.7 ms
   * when only the label entries are live; 2 ms against 0.01 ms when every
   * block is flat, the cost of handing out the empty tasks).  With
   * CCE_BWD_DETERMINISTIC the reduce-adds into each dE tile happen in
   * stripe order (and dC is written once per tile), so the fp32 result is
   * bitwise reproducible without the int64 accumulators (with the filter
   * on, every tile is then recomputed: flat blocks are not sent to the
   * flat-row kernel, whose dC additions are unordered).  With
   * CCE_BWD_BF16_GRADS the sums go to fp32 scratch and are rounded to bf16
   * once.  Needs the workspace of cce_backward_workspace_size_ex with this
   * flag. */
  CCE_BWD_STRIPES = 16,
  /* With filter_eps > 0: cce_backward_prepare_rows has stored each token's
   * largest logit max_v E_i . C_v (from cce_forward_ex) in this workspace for
   * the same E, C and N.  The pre-pass then proves token blocks flat with
   * that exact maximum instead of the Cauchy-Schwarz bound |E_i| max_v |C_v|
   * (which can be far looser), and skips both norm passes unless the
   * fixed-point modes need them.  The stored maxima serve one backward call;
   * without a fresh cce_backward_prepare_rows the pre-pass treats every
   * block as not flat (the exact, slower path).  Same result as without the
   * flag.  Ignored with CCE_BWD_STRIPES or filter_eps <= 0.  No extra
   * workspace. */
  CCE_BWD_ROW_MAX = 32
} cce_backward_flags_t;

/* Forward pass that also writes row_max [N] fp32 (device; may be NULL): each
 * token's largest logit max_v E_i . C_v, the maximum the log-sum-exp is
 * taken around (also for ignored rows; NaN where loss is NaN after a wait
 * gave up).  Otherwise the same as cce_forward. */
CCE_API cce_status_t cce_forward_ex(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D, int64_t V,
                                    int64_t ignore_index, float* loss, float* lse, float* row_max, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Stores row_max [N] (device, fp32: each token's largest logit, from
 * cce_forward_ex on the same E and C) in the backward workspace for the next
 * cce_backward_ex with CCE_BWD_ROW_MAX (an asynchronous 4N-byte copy on
 * stream).  Workspace as for cce_backward_workspace_size(N, D, V).  Returns
 * CCE_ERR_INVALID_ARG / CCE_ERR_MISALIGNED / CCE_ERR_WORKSPACE_TOO_SMALL on
 * the host. */
CCE_API cce_status_t cce_backward_prepare_rows(const float* row_max, int64_t N, int64_t D, int64_t V,
                                               void* workspace, size_t workspace_bytes, void* stream);

/* The part of the backward's pre-pass that depends on the classifier alone:
 * max_v |C_v| (one read of all of C, about 0.17 ms for a 256000 x 2304 bf16
 * C on a B200), stored in the backward workspace for a later cce_backward_ex
 * call with CCE_BWD_PREPARED and the same C, N, D, V and workspace.  Since C
 * is known before the forward pass, a caller can run this on another stream
 * concurrently with cce_forward (which is bound by the tensor cores, not by
 * memory) and take it off the backward's critical path.  It reads C only;
 * the two calls may overlap.  The bound feeds the gradient filter's
 * Cauchy-Schwarz pre-pass and the fixed-point scale of the deterministic
 * modes (Cut Cross-Entropy abstract, sentence 9); it changes no result.
 *   C [V x D] bf16 (device), workspace >= cce_backward_workspace_size_ex(N,
 *   D, V, flags) of the backward call that will consume it.
 * Errors as for cce_backward. */
CCE_API cce_status_t cce_backward_prepare(const void* C, int64_t N, int64_t D, int64_t V, void* workspace,
                                          size_t workspace_bytes, void* stream);

/* Workspace bytes for cce_backward_ex with these flags (0 if the sizes or
 * flags are invalid). */
CCE_API size_t cce_backward_workspace_size_ex(int64_t N, int64_t D, int64_t V, unsigned flags);

/* cce_backward with options (see cce_backward_flags_t).  dE and dC are fp32
 * unless CCE_BWD_BF16_GRADS is set, then bf16 (raw 16-bit storage).  With
 * flags == 0 this is exactly cce_backward.  Same filter semantics, parity and
 * error behaviour as cce_backward. */
CCE_API cce_status_t cce_backward_ex(const void* E, const void* C, const int64_t* y, const float* lse,
                                     const float* dloss, int64_t N, int64_t D, int64_t V, int64_t ignore_index,
                                     float filter_eps, unsigned flags, void* dE, void* dC, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* ---- Vocabulary-parallel form (e.g. one classifier shard per GPU) ----
 * The log-sum-exp decomposes over any partition of the vocabulary:
 *   lse = M + log sum_r s_r exp(m_r - M),  M = max_r m_r,
 * where (m_r, s_r) are the max and the sum of exp(z - m_r) over shard r.  So
 * each shard computes 3 floats per token, the shards exchange them (an
 * all-gather of 12 bytes per token per shard, NCCL on multi-GPU), and every
 * shard merges them into the same lse and loss.  Given that lse, each shard's
 * backward yields its own rows of dC exactly and its share of dE; the full dE
 * is the sum of the shares (an all-reduce).  Labels are always global ids.
 * Workspaces: cce_forward_workspace_size / cce_backward_workspace_size with
 * V = V_shard. */

/* Forward on the classifier rows C_shard = C[v_offset : v_offset + V_shard].
 *   stats [3][N] fp32 out: row 0 = max_v z_iv over the shard, row 1 =
 *   sum_v exp(z_iv - max), row 2 = z_{i, y_i} if v_offset <= y_i <
 *   v_offset + V_shard, else 0.  All NaN if a bounded wait gave up. */
CCE_API cce_status_t cce_forward_shard(const void* E, const void* C_shard, const int64_t* y, int64_t N, int64_t D,
                                       int64_t V_shard, int64_t v_offset, int64_t ignore_index, float* stats,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* Merges R shards' stats ([R][3][N] fp32, device) into loss and lse (fp32
 * [N]).  V_total: the full vocabulary size (labels outside [0, V_total) that
 * are not ignore_index give a NaN loss). */
CCE_API cce_status_t cce_merge_shards(const float* stats, int R, int64_t N, const int64_t* y, int64_t V_total,
                                      int64_t ignore_index, float* loss, float* lse, void* stream);

/* Backward for one shard, given the merged (global) lse: dC_shard [V_shard x
 * D] is the exact gradient of the shard's classifier rows; dE_partial [N x D]
 * is this shard's share of dE (sum the shares over shards).  Same filter as
 * cce_backward (the tile grid starts at the shard's first row). */
CCE_API cce_status_t cce_backward_shard(const void* E, const void* C_shard, const int64_t* y, const float* lse,
                                        const float* dloss, int64_t N, int64_t D, int64_t V_shard,
                                        int64_t v_offset, int64_t ignore_index, float filter_eps, float* dE_partial,
                                        float* dC_shard, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then copies the status block of `workspace` (as left
 * by the last call that used it) into *out.  Returns CCE_ERR_TIMEOUT or
 * CCE_ERR_BAD_LABEL if the corresponding flag is set, else CCE_OK. */
CCE_API cce_status_t cce_read_status(const void* workspace, void* stream, cce_counters_t* out);

/* Human-readable name of a status code (static storage). */
CCE_API const char* cce_status_string(cce_status_t status);

/* Library ABI version (major * 100 + minor). */
CCE_API int cce_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CCE_H_ */
