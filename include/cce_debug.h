/*
 * cce_debug.h -- diagnostic entry points of libcce.so (not part of the loss API).
 *
 * These exist so that tests can localise a fault in the fused kernels.  They
 * DO write logits to global memory, which the loss entry points never do.
 */
#ifndef CCE_DEBUG_H_
#define CCE_DEBUG_H_

#include "cce.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Runs the forward kernel's tensor-core mainloop unchanged and additionally
 * stores every raw logit tile it forms:
 *   logits [N x ceil(V/256)*256] fp32 device out, row-major; column v < V
 *   holds E_i . C_v; the padding columns v >= V are unspecified (the kernel
 *   skips 32-column groups that lie wholly past V).
 * loss/lse/workspace are as for cce_forward (which this call also computes). */
CCE_API cce_status_t cce_debug_forward_logits(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D,
                                      int64_t V, int64_t ignore_index, float* loss, float* lse, float* logits,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Upper bound (ns) on any single wait inside the kernels; a wait that runs
 * longer gives up, sets the timeout status flag and the kernel exits.
 * Default 1e9 (one second).  Process-wide. */
CCE_API void cce_debug_set_wait_limit_ns(uint64_t limit_ns);

/* Failure-detection test hook.  While on, the fused kernels' TMA producer
 * warps issue no copies, so the tensor-core and epilogue warps wait on data
 * that never comes.  Each wait gives up after the wait limit (see
 * cce_debug_set_wait_limit_ns), the CTA unwinds, frees its tensor memory and
 * exits, and the call's status block carries the timeout flag
 * (cce_read_status returns CCE_ERR_TIMEOUT).  Outputs are meaningless while
 * it is on.  Process-wide; 0 turns it off. */
CCE_API void cce_debug_withhold_loads(int on);

/* L2 prefetch distances, in 64-wide K slices, of the operand streams of the
 * forward and backward kernels: while loading slice k into shared memory the
 * TMA producer also asks for slice k + distance to be brought into L2
 * (`cp.async.bulk.prefetch.tensor`, a hint with no completion).  0 turns the
 * prefetch off.  Same results; for A/B measurement.  Process-wide.  Returns
 * CCE_ERR_INVALID_ARG outside [0, 64]. */
CCE_API cce_status_t cce_debug_set_prefetch(int fwd_slices, int bwd_slices);

/* Schedule knobs of the forward logit/LSE kernels, for A/B measurement.
 * n_split (0..256; 0 = chosen per shape: the fewest splits that minimise the
 * most-loaded worker's vocabulary tiles) is the number of vocabulary ranges
 * per token block, i.e. of (max, sum) partials per token; group_m (>= 0; 0 =
 * chosen per shape: ~48 MB of E rows in the round-robin order, ~24 MB per
 * L2 half in the two-queue order) is the number of token blocks per raster
 * group; l2_hints (0..3, default 0; CTA-pair kernel only) gives the
 * E slices the evict_last L2 policy (bit 0) and the C slices evict_first
 * (bit 1); stages (0 = the default 7, or 6 or 7; CTA-pair kernel only) is
 * the number of 32 KB operand stages per CTA (7 fill the 227 KB of shared
 * memory; 1 % faster than 6 on the Gemma-2-2B-shaped head).  Same loss and lse up to fp32 rounding order.  The forward
 * workspace size depends on n_split: query cce_forward_workspace_size after
 * changing it.  Process-wide.  Returns CCE_ERR_INVALID_ARG for other
 * values. */
CCE_API cce_status_t cce_debug_set_forward_schedule(int n_split, int group_m, int l2_hints, int stages);

/* Unit order of the CTA-pair forward kernel, for A/B measurement.  0: the
 * (token block, vocabulary split) units are dealt round-robin to the pairs.
 * 1 (the default): two queues, one per L2 half of the GPU.  The L2 is split between the
 * two dies, every line has a home half, and an SM reading a line homed in
 * the other half keeps a copy in its own, so E (re-read for every vocabulary
 * tile) fills both halves when every pair reads every token block.  Order 1
 * gives each half its own token blocks (in proportion to its SMs; which SM
 * is in which half is measured once per device and process by a small probe
 * kernel, from the latency of atomics, which are served at a line's home),
 * and the pairs draw units at run time from their half's queue, taking the
 * other queue's units when theirs runs out or runs ahead.  Drawing units at
 * run time also keeps the pairs that share C rows in step, and the units are
 * short (at most ~8 vocabulary tiles).  DRAM reads of one forward (ncu):
 * 1.9-2.9 -> 1.23 GB on the Gemma-2-2B-shaped head (C read once), 27.6 ->
 * 6.0 GB on the Llama-3-8B-shaped head (16384 x 4096, V = 128256), 141 ->
 * 7.6 GB on the N = 65536 sweep; the last two 10-14 % faster.  Each unit is computed
 * the same way whoever computes it, so loss and lse are bitwise those of
 * order 0; the split count may differ between the orders (the raster group
 * enters its choice), so query cce_forward_workspace_size after changing
 * the order.  Process-wide.  Returns CCE_ERR_INVALID_ARG for other
 * values. */
CCE_API cce_status_t cce_debug_set_forward_order(int order);

/* The L2 half of each SM as the two-queue order's probe found it on the
 * current device: half_of_sm[s] = 1 or 2 for SM id s (1: the half that is
 * home to the probe's first line), 0 if not found (no forward in the
 * two-queue order has run yet, or the SM's lines could not be told apart).
 * Host memory, max_sms entries at most (SM ids 0..255 are kept).  Reads
 * device memory synchronously: synchronize the stream of the forward first.
 * Returns the number of entries written, or -1 (null pointer, max_sms <= 0,
 * CUDA error). */
CCE_API int cce_debug_l2_halves(int* half_of_sm, int max_sms);

/* The forward's launch plan for these sizes on a GPU with `sms` SMs, as
 * cce_forward would choose it under the knobs in force (host arithmetic
 * only: no device needed).  out[6] (host memory) receives: 1 if the
 * CTA-pair kernel runs, the token blocks (of 256 rows for pairs, 128
 * otherwise), the 256-wide vocabulary tiles, the vocabulary splits, the
 * token blocks per raster group, and the grid in CTAs.  The workspace is
 * 256 + N * splits * 8 bytes, rounded up to 256.  Returns 0, or -1 for
 * invalid sizes, sms <= 0 or a null pointer. */
CCE_API int cce_debug_forward_plan(int64_t N, int64_t D, int64_t V, int sms, int* out);

/* Tuning knobs of the dense stripe backward (CCE_BWD_STRIPES), for A/B
 * measurement: tokens_per_launch (a multiple of 256, at most 16384; 0 = the
 * default 16384) bounds the tokens one launch takes (fewer tokens per launch
 * keep the stripe buffers, E and dE of a launch in L2, at the cost of adding
 * dC over more launches); dE_prefetch (0 or 1, default 0) asks for the dE
 * rows of each dE-tile task in L2 when the task starts; vtiles_per_stripe
 * (0..32; 0 = the default 8) sets the stripe width in 256-wide vocabulary
 * tiles (wider stripes: fewer reduce-adds into dE, larger stripe buffers).
 * Same results up to fp32 summation order.  The workspace size depends on
 * the stripe width: query cce_backward_workspace_size_ex after changing it.
 * Process-wide.  Returns CCE_ERR_INVALID_ARG for other values. */
CCE_API cce_status_t cce_debug_set_stripe_params(int tokens_per_launch, int dE_prefetch, int vtiles_per_stripe);

/* L2 prefetch distance, in 64-wide K slices, of the fp32 dE / dC rows that
 * the filtered backward kernel's bulk reduce-adds add into: while loading
 * the operands of contraction slice k, its TMA producer asks for the live
 * 32-row pieces of slice k - distance (the pass runs d descending) to be
 * brought into L2, so the reductions find their lines there.  0 turns it
 * off.  Same results; for A/B measurement.  Process-wide.  Returns
 * CCE_ERR_INVALID_ARG outside [0, 64]. */
CCE_API cce_status_t cce_debug_set_reduce_prefetch(int slices);

/* L2 eviction priorities in the filtered backward kernel: while on, its TMA
 * producer loads the classifier slices with an evict-first cache policy and
 * its epilogue adds into dE with an evict-last policy, so the streamed
 * classifier leaves L2 before the dE rows the reductions keep returning to.
 * Hints only: same results.  For A/B measurement; 0 (the default) is off.
 * Process-wide.  Returns CCE_ERR_INVALID_ARG for values other than 0, 1. */
CCE_API cce_status_t cce_debug_set_l2_hints(int on);

/* Profiling hook for the backward kernel's per-tile timeline.  While set,
 * every backward launch writes, for each CTA b (one per SM) and each of its
 * first tiles_per_cta tiles k, four u64 at trace[(b * tiles_per_cta + k) * 4]:
 * the GPU's globaltimer (ns) when the CTA's epilogue starts on the tile, when
 * the tile's recomputed logits are complete in tensor memory, when its
 * softmax-gradient tile and live mask are published, and the 32-bit live
 * mask; after its last tile the CTA writes the end time into word 0 of the
 * next entry (if < tiles_per_cta).  `trace` is a device buffer owned by the
 * caller with room for (number of SMs) * tiles_per_cta * 32 bytes; the
 * library does not clear it.  The dense stripe backward (CCE_BWD_STRIPES)
 * writes through the same hook, per CTA pair p (leader CTA) and task k, at
 * trace[(p * tiles_per_cta + k) * 4]: the time the task was handed out, the
 * time its accumulator was complete, the time its epilogue finished, and the
 * task kind (0 recompute and store G, 1 dC tile, 2 dE tile) | (ns spent
 * waiting for the task's inputs << 8).  NULL turns the hook off.
 * Process-wide.
 * Returns CCE_ERR_INVALID_ARG for tiles_per_cta outside [1, 2^20]. */
CCE_API cce_status_t cce_debug_set_backward_trace(uint64_t* trace, int64_t tiles_per_cta);

/* Host-only view of the task order of the stripe backward (CCE_BWD_STRIPES)
 * for a launch of n_m2 256-token blocks, n_vtile 256-row vocabulary tiles,
 * n_dc 256-wide d-chunks, vt_per_s tiles per stripe, nbuf stripe buffers
 * and the order of cce_debug_set_stripe_order (order, group_m2, lag):
 * writes min(total + 1, max_tasks) task descriptors, four int32 each (kind:
 * -1 end, 0 recompute-and-store G, 1 dC tile, 2 dE tile; stripe; then
 * (token block, vocabulary tile), (vocabulary tile, d-chunk) or (token
 * block, d-chunk)), into out (host memory; may be NULL) and returns the
 * number of tasks, or -1 for invalid arguments.  Runs no kernel. */
CCE_API int64_t cce_debug_stripe_schedule(int n_m2, int n_vtile, int n_dc, int vt_per_s, int nbuf, int order,
                                          int group_m2, int lag, int32_t* out, int64_t max_tasks);

/* Task order of the stripe backward, for A/B measurement.  order 0 (the
 * default): recompute tasks of stripe s, then the dC and dE tasks of stripe
 * s - 1.  order 1: per stripe, the token blocks in groups of group_m2; each
 * group's recompute tasks are followed by the dE tasks of the group lag
 * groups earlier (their G rows still in L2), then the last groups' dE tasks
 * and the stripe's dC tasks.  Same results up to fp32 summation order (bit
 * for bit in the deterministic mode).  Process-wide.  Returns
 * CCE_ERR_INVALID_ARG unless order is 0 or 1 and group_m2, lag are in
 * [1, 64]. */
CCE_API cce_status_t cce_debug_set_stripe_order(int order, int group_m2, int lag);

/* Selects the forward logit/LSE kernel: 1 = CTA pairs (two SMs per 256 x 256
 * logit tile through tcgen05 cta_group::2, two thirds of the operand traffic
 * per SM; the default), 0 = one SM per 128 x 256 logit tile.  Both give the
 * same loss up to fp32 rounding order; the switch exists for A/B measurement
 * (on the power-capped B200 the pairs are ~3 % faster on the Gemma-2-2B
 * head in long runs).  The forward workspace size depends on the variant:
 * query cce_forward_workspace_size after switching.
 * Process-wide.  Returns CCE_ERR_INVALID_ARG for other values. */
CCE_API cce_status_t cce_debug_set_forward_variant(int variant);

/* Selects the backward kernel's buffering: 0 = three operand pipeline stages
 * and one 4 KB reduction staging buffer per epilogue warp (the default),
 * 1 = two stages and two staging buffers (the staging of a block overlaps the
 * bulk read of the previous one), 2 = two stages and eight epilogue warps
 * (two per TMEM lane group, splitting the gradient columns and the
 * reduction pieces), 3 = as 0 but the fp32 reductions go through vector
 * atomics (red.global.add.v4.f32) instead of the TMA engine.  Same results
 * up to fp32 summation order; for A/B measurement.
 * Process-wide.  Returns CCE_ERR_INVALID_ARG for other values. */
CCE_API cce_status_t cce_debug_set_backward_variant(int variant);

/* Profiling hook.  While set, every launch of the selected kernel records
 * `start_event` on the call's stream immediately before the launch and
 * `stop_event` immediately after it, so the caller can time that kernel alone
 * with cudaEventElapsedTime.  kernel: 0 = forward logit/LSE kernel,
 * 1 = backward kernel.  Events are cudaEvent_t handles created by the caller
 * (passed as void*); NULL clears the hook.  Process-wide, not thread-safe.
 * Returns CCE_ERR_INVALID_ARG for an unknown kernel id. */
CCE_API cce_status_t cce_debug_set_kernel_events(int kernel, void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* CCE_DEBUG_H_ */
