// CCE forward: fused logit GEMM + online log-sum-exp, then a small merge.
//
// Cut Cross-Entropy abstract, sentences 4-6: the loss is computed without
// writing the logit matrix to global memory; only the correct-token logit is
// formed explicitly and the log-sum-exp over the vocabulary is evaluated on
// the fly, with the matrix products and the reduction kept on chip.
//
// fwd_lse_kernel  persistent, warp-specialised tcgen05 kernel.  A work unit is
//                 (token block m of 128 rows, vocabulary split r), dealt in
//                 groups of token blocks whose E rows fit in L2.  For every
//                 256-wide vocabulary tile of the split the logit tile
//                 S = E_m C_tile^T is accumulated in TMEM (double buffered),
//                 and the epilogue warps fold it into a per-row running
//                 (max, sum exp(z - max)).  One (max, sum) pair per row and
//                 split goes to the workspace; logits never leave the SM.
// fwd_lse_pair_kernel  the same on clusters of two CTAs (the default): one
//                 256 x 256 logit tile per pair through tcgen05 cta_group::2,
//                 each CTA loading 128 rows of E and 128 rows of C per slice.
//                 Units are dealt round-robin, or (two-queue order) drawn at
//                 run time from one queue per L2 half of the GPU, so that each
//                 half keeps only its own token blocks' E rows in its L2.
// l2_half_probe   tells the two L2 halves apart once per process: per SM,
//                 the latency of atomics on eight lines 4 KB apart (an atomic
//                 is served where its line is homed, ~2.5x faster in the SM's
//                 own half).
// fwd_finalize    one warp per token: merges the split partials into lse,
//                 forms the correct-token logit E_i . C_{y_i} with coalesced
//                 16-byte loads, and writes loss = lse - z_y (0 if ignored).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace cce {

// Fold one 128 x 256 logit tile held in TMEM (this thread's lane = one token
// row) into the row's running (max, sum exp(z - max)).  Columns >= V are
// masked to -inf; DUMP additionally stores the raw logits (debug entry only).
template <bool DUMP>
__device__ __forceinline__ void lse_fold_tile(uint32_t tbase, int col0, int row, const FwdArgs& a, float& mrun,
                                              float& srun) {
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    const int cbase = col0 + c * 32;
    if (cbase >= a.V) break;  // uniform across the warp
    float x[32];
    tmem_ld32(tbase + (uint32_t)(c * 32), x);
    if constexpr (DUMP) {
      if (row < a.N) {
        float* dst = a.dbg_logits + (size_t)row * ((size_t)a.n_vtile * BN) + cbase;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[j] = x[j];
      }
    }
    const int nvalid = a.V - cbase;
    if (nvalid < 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j >= nvalid) x[j] = -INFINITY;
    }
    float cm0 = x[0], cm1 = x[1];
#pragma unroll
    for (int j = 2; j < 32; j += 2) {
      cm0 = fmaxf(cm0, x[j]);
      cm1 = fmaxf(cm1, x[j + 1]);
    }
    const float mnew = fmaxf(mrun, fmaxf(cm0, cm1));
    const float ms = mnew * LOG2E;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      s0 += ex2_approx(fmaf(x[j], LOG2E, -ms));
      s1 += ex2_approx(fmaf(x[j + 1], LOG2E, -ms));
      s2 += ex2_approx(fmaf(x[j + 2], LOG2E, -ms));
      s3 += ex2_approx(fmaf(x[j + 3], LOG2E, -ms));
    }
    srun = srun * ex2_approx(fmaf(mrun, LOG2E, -ms)) + ((s0 + s1) + (s2 + s3));
    mrun = mnew;
  }
}

template <bool DUMP>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_lse_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC,
                   const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + FWD_STAGES * A_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + FWD_STAGES * B_STAGE_BYTES);
  uint64_t* full = bars;                       // TMA -> MMA, per stage
  uint64_t* empty = bars + FWD_STAGES;         // MMA -> TMA, per stage
  uint64_t* tfull = bars + 2 * FWD_STAGES;     // MMA -> epilogue, per TMEM buffer
  uint64_t* tempty = tfull + 2;                // epilogue -> MMA, per TMEM buffer
  uint64_t* drain = tempty + 2;                // MMA self-drain at exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < FWD_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], BM);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_map(&tmE);
    tma_prefetch_map(&tmC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, a.wait_limit_ns};
  const int nkb = (a.D + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;  // stages armed at least once
      // withhold_loads (test hook): no copy is issued, so the MMA warp's first
      // wait can only end by its time limit; that path must unwind cleanly.
      for (int u = a.withhold_loads ? a.n_units : blockIdx.x; u < a.n_units; u += gridDim.x) {
        int r, m;
        unit_coords(u, a.n_mblk, a.n_split, a.group_m, r, m);
        int v0, v1;
        split_range(r, a.n_vtile, a.n_split, v0, v1);
        for (int vt = v0; vt < v1; ++vt) {
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
            mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
            tma_load_2d(sA + stage * A_STAGE_BYTES, &tmE, &full[stage], kb * BK, m * BM);
            tma_load_2d(sB + stage * B_STAGE_BYTES, &tmC, &full[stage], kb * BK, vt * BN);
            armed |= 1u << stage;
            if (a.pf) {  // L2 prefetch of the C slice a.pf slices ahead in this unit's stream
              const int s2 = (vt - v0) * nkb + kb + a.pf;
              if (s2 < (v1 - v0) * nkb) tma_prefetch_l2_2d(&tmC, (s2 % nkb) * BK, (v0 + s2 / nkb) * BN);
            }
            if (++stage == FWD_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    producer_done:
      // Let every issued copy land before the CTA can exit: the last arming
      // of stage s completed phase parity ((s < stage) ? phase : phase ^ 1).
      {
        WaitCtl exit_wc{abort_flag, a.wait_limit_ns};
        int dummy = 0;
        exit_wc.abort_flag = &dummy;
        for (int s = 0; s < FWD_STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (s < stage) ? phase : (phase ^ 1u), exit_wc);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
        int r, m;
        unit_coords(u, a.n_mblk, a.n_split, a.group_m, r, m);
        int v0, v1;
        split_range(r, a.n_vtile, a.n_split, v0, v1);
        for (int vt = v0; vt < v1; ++vt) {
          if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) goto mma_done;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&full[stage], phase, wc)) goto mma_done;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + stage * A_STAGE_BYTES);
            const uint32_t b_addr = smem_u32(sB + stage * B_STAGE_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              umma_bf16(d_tmem, sdesc_sw128(a_addr + k * 32, 16, 1024), sdesc_sw128(b_addr + k * 32, 16, 1024),
                        IDESC, (kb | k) != 0);
            }
            umma_commit(&empty[stage]);
            if (++stage == FWD_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          umma_commit(&tfull[acc]);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
    mma_done:
      // Wait until every UMMA this thread issued has finished before TMEM is freed.
      umma_commit(drain);
      {
        int dummy = 0;
        WaitCtl exit_wc{&dummy, a.wait_limit_ns};
        mbar_wait(drain, 0, exit_wc);
      }
    }
  } else {
    // ---------------- epilogue: 4 warps, one TMEM lane (token row) per thread ----------------
    const int lane_grp = warp & 3;  // a warp may only touch TMEM lanes 32*(warp%4) .. +31
    const int row_in_blk = lane_grp * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(lane_grp * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
      int r, m;
        unit_coords(u, a.n_mblk, a.n_split, a.group_m, r, m);
      int v0, v1;
      split_range(r, a.n_vtile, a.n_split, v0, v1);
      float mrun = -INFINITY, srun = 0.f;
      bool ok = true;
      for (int vt = v0; vt < v1; ++vt) {
        if (!mbar_wait(&tfull[acc], acc_phase, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        lse_fold_tile<DUMP>(tmem_base + lane_addr + (uint32_t)(acc * BN), vt * BN, m * BM + row_in_blk, a, mrun,
                            srun);
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      const int row = m * BM + row_in_blk;
      if (row < a.N) a.partial[(size_t)r * a.N + row] = make_float2(mrun, srun);
    }
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(a.status + ST_FLAGS, SF_TIMEOUT);
  if (threadIdx.x == 0 && blockIdx.x == 0 && !*abort_flag) {
    atomicAdd(a.status + ST_TILES, (unsigned long long)a.n_mblk * (unsigned long long)a.n_vtile);
  }
}


// ----------------------------------------------------------------------------
// L2 halves.  The L2 of this GPU is split between its two dies: every line has
// a home half, and an SM that reads a line homed in the other half keeps a
// copy in its own half.  Data that all SMs read (E, re-read for every
// vocabulary tile) therefore fills both halves, and at N = 8192 on the 256K
// vocabulary (37.7 MB of E) C is streamed from DRAM 1.7 times instead of once
// (1.15 times at N = 2048).  The two-queue order gives each half its own token
// blocks; this kernel finds which half each SM belongs to.
//
// An atomic is performed at the line's home, so its latency tells near from
// far (about 260 against 690 SM cycles at 1.97 GHz).  Each block times short
// chains of atomics (adding 0) on eight lines 4 KB apart, which the home hash
// spreads over both halves; lines faster than the midpoint of its fastest and
// slowest are near.  The SM's half is then "line 0 is near" (1) or not (2).
// If no two lines differ by 1.5x the SM stays unknown (0).  The tables live
// as long as the process; a table entry is written once (compare-and-swap),
// so the kernel may run again (a replayed graph) without changing anything.
// ----------------------------------------------------------------------------
constexpr int kMaxSmid = 256;
__device__ __align__(4096) unsigned long long g_l2_probe[8 * 512];  // 8 lines, 4 KB apart
__device__ unsigned g_sm_half[kMaxSmid];                            // 0 unknown, 1 or 2
__device__ unsigned g_half_sms[2];                                  // SMs found in half 1, half 2

__device__ __forceinline__ unsigned sm_id() {
  unsigned s;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(s));
  return s;
}

__global__ void __launch_bounds__(32) l2_half_probe_kernel() {
  if (threadIdx.x != 0) return;
  const unsigned smid = sm_id();
  if (smid >= (unsigned)kMaxSmid || *(volatile unsigned*)&g_sm_half[smid] != 0u) return;
  long long lat[8];
  unsigned long long v = 0ull;
  for (int j = 0; j < 8; ++j) {
    const int line = (blockIdx.x + j) & 7;  // blocks start on different lines
    unsigned long long* p = g_l2_probe + line * 512;
    const long long c0 = clock64();
    for (int s = 0; s < 3; ++s) {
      // each address depends on the previous result (v >> 63 is 0: the lines hold 0)
      asm volatile("atom.global.add.u64 %0, [%1], 0;" : "=l"(v) : "l"(p + (v >> 63)) : "memory");
    }
    lat[line] = clock64() - c0 + (long long)(v >> 63);
  }
  long long mn = lat[0], mx = lat[0];
  for (int j = 1; j < 8; ++j) {
    mn = min(mn, lat[j]);
    mx = max(mx, lat[j]);
  }
  if (2 * mx < 3 * mn) return;  // the lines could not be told apart
  const unsigned half = 2 * lat[0] < mn + mx ? 1u : 2u;
  if (atomicCAS(&g_sm_half[smid], 0u, half) == 0u) atomicAdd(&g_half_sms[half - 1], 1u);
}

cudaError_t launch_l2_half_probe(int sms, cudaStream_t stream) {
  // four blocks per SM, so that every SM is all but certain to run one
  l2_half_probe_kernel<<<4 * sms, 32, 0, stream>>>();
  return cudaGetLastError();
}

// Copies the half of SMs 0 .. n-1 (0 unknown, 1, 2) to host memory.
cudaError_t read_l2_halves(unsigned* out, int n) {
  return cudaMemcpyFromSymbol(out, g_sm_half, (size_t)n * sizeof(unsigned));
}

// ----------------------------------------------------------------------------
// CTA-pair variant: a cluster of two CTAs on two SMs computes 256 x 256 logit
// tiles with tcgen05.mma.cta_group::2 (M = 256 split over the pair).  Each CTA
// loads its own 128 token rows of E and 128 vocabulary rows of C per stage
// (32 KB instead of 48 KB per SM for the same MMA work, so 7 stages fit), and
// each CTA's TMEM holds its 128 rows x 256 columns of every tile, which its own
// epilogue folds exactly as in the single-CTA kernel.  Only the even (leader)
// CTA issues UMMAs; its full barriers count both CTAs' copies, its commits
// arrive on both CTAs' barriers, and both epilogues release the accumulator
// on the leader's barrier.  No TMA multicast is used.
// ----------------------------------------------------------------------------
template <bool DUMP, int S>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    fwd_lse_pair_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmCh,
                        const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                    // S x [128 tok][64 d]
  uint8_t* sB = smem + S * A_STAGE_BYTES;      // S x [128 voc][64 d]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * A_STAGE_BYTES);
  uint64_t* full = bars;                      // leader: both CTAs' copies landed
  uint64_t* empty = bars + S;       // each CTA: stage free again
  uint64_t* tfull = bars + 2 * S;   // each CTA: accumulator ready
  uint64_t* tempty = tfull + 2;               // leader: both epilogues done with the accumulator
  uint64_t* drain = tempty + 2;               // leader: UMMA drain at exit
  uint64_t* unit_full = drain + 1;            // each CTA [2]: two-queue order, a unit was published
  uint64_t* unit_empty = unit_full + 2;       // leader [2]: every consumer has read the slot
  int4* unit_slot = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(unit_empty + 2) + 15) & ~uintptr_t(15));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_slot + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  // readers of a published unit: the leader's MMA thread and 4 epilogue
  // warps, the peer's producer and 4 epilogue warps
  constexpr uint32_t UNIT_CONSUMERS = 10;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // one arrival per epilogue warp of both CTAs
      mbar_init(&unit_full[b], 1);
      mbar_init(&unit_empty[b], UNIT_CONSUMERS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_map(&tmE);
    tma_prefetch_map(&tmCh);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, a.wait_limit_ns};
  const int nkb = (a.D + BK - 1) / BK;

  // Round-robin order: unit k of this pair is pair + k * n_pairs.  Two-queue
  // order: the leader's producer draws each unit and publishes its (split,
  // token block) to both CTAs through a two-slot ring; r < 0 ends the stream.
  auto static_unit = [&](int k, int& r, int& m2) -> bool {
    const int u = pair + k * n_pairs;
    if (u >= a.n_units) return false;
    unit_coords(u, a.n_mblk, a.n_split, a.group_m, r, m2);
    return true;
  };
  const uint32_t unit_empty_leader = mapa_shared(smem_u32(&unit_empty[0]), 0);
  // Reads published unit k (bounded wait) and frees the slot on the leader.
  // With whole_warp, lane 0 waits and reads and the warp follows its outcome.
  auto take_unit = [&](int k, int& r, int& m2, bool whole_warp) -> bool {
    const int slot = k & 1;
    int ok = 1, rr = -1, mm = -1;
    if (!whole_warp || lane == 0) {
      ok = mbar_wait_cluster(&unit_full[slot], (uint32_t)(k >> 1) & 1u, wc) ? 1 : 0;
      if (ok) {
        const volatile int* vs = reinterpret_cast<const volatile int*>(&unit_slot[slot]);
        rr = vs[0];
        mm = vs[1];
        mbar_arrive_cluster(unit_empty_leader + (uint32_t)(slot * 8));
      }
    }
    if (whole_warp) {
      ok = __shfl_sync(0xffffffffu, ok, 0);
      rr = __shfl_sync(0xffffffffu, rr, 0);
      mm = __shfl_sync(0xffffffffu, mm, 0);
    }
    r = rr;
    m2 = mm;
    return ok != 0;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0, armed = 0;
      // optional L2 eviction priorities: E (re-read for every vocabulary
      // tile) kept, C (read by every token block in turn) evicted first
      const uint64_t pol_e = l2_policy_evict_last(), pol_c = l2_policy_evict_first();
      const bool hint_e = (a.l2_hints & 1) != 0, hint_c = (a.l2_hints & 2) != 0;
      // Two-queue order (leader): queue q holds the units of token blocks
      // [m_lo[q], m_lo[q] + nq[q]), split-major in raster groups, and the
      // token blocks are divided between the queues in proportion to the
      // SMs of each L2 half.  The pair serves the queue of its own half.
      int own = 0, nq[2] = {0, 0}, m_lo[2] = {0, 0}, gm_q[2] = {1, 1};
      long long units_q[2] = {0, 0};
      unsigned long long* qctr = a.status + ST_FWD_QUEUE;
      if (a.sched && leader) {
        const unsigned c1 = *(volatile unsigned*)&g_half_sms[0], c2 = *(volatile unsigned*)&g_half_sms[1];
        int m_half = a.n_mblk / 2;
        if (c1 != 0u && c2 != 0u)
          m_half = (int)(((long long)a.n_mblk * c1 + (c1 + c2) / 2) / (c1 + c2));
        m_half = max(0, min(a.n_mblk, m_half));
        const unsigned smid = sm_id();
        unsigned h = smid < (unsigned)kMaxSmid ? *(volatile unsigned*)&g_sm_half[smid] : 0u;
        if (h == 0u) h = 1u + (unsigned)(pair & 1);  // half unknown: alternate
        own = (int)h - 1;
        nq[0] = m_half;
        nq[1] = a.n_mblk - m_half;
        m_lo[1] = m_half;
        for (int q = 0; q < 2; ++q) {
          units_q[q] = (long long)nq[q] * a.n_split;
          // raster groups of at most group_m blocks, as even as possible
          const int ng = max(1, (nq[q] + a.group_m - 1) / a.group_m);
          gm_q[q] = max(1, (nq[q] + ng - 1) / ng);
        }
      }
      // Next unit of the two-queue order.  The own queue first, unless it is
      // more than one split ahead of the other (units are split-major inside
      // a raster group, gm_q per split): then the other queue's, so both
      // halves walk the vocabulary together and C rows are read by both while
      // in L2.  When one queue is empty the other's units are taken.
      auto draw = [&](int& r, int& m2) -> bool {
        const int other = 1 - own;
        int first = own;
        if (units_q[own] > 0 && units_q[other] > 0) {
          const long long io = (long long)*(volatile unsigned long long*)(qctr + own);
          const long long ix = (long long)*(volatile unsigned long long*)(qctr + other);
          if (ix < units_q[other] && io * gm_q[other] > (ix + gm_q[other]) * gm_q[own]) first = other;
        }
        for (int t = 0; t < 2; ++t) {
          const int q = t == 0 ? first : 1 - first;
          if (units_q[q] == 0) continue;
          const unsigned long long i = atomicAdd(qctr + q, 1ull);
          if (i < (unsigned long long)units_q[q]) {
            int mloc;
            unit_coords((int)i, nq[q], a.n_split, gm_q[q], r, mloc);
            m2 = m_lo[q] + mloc;
            return true;
          }
        }
        return false;
      };
      // publishes unit k (r < 0: the end) to both CTAs
      auto publish = [&](int k, int r, int m2) -> bool {
        const int slot = k & 1;
        if (!mbar_wait(&unit_empty[slot], ((uint32_t)(k >> 1) & 1u) ^ 1u, wc)) return false;
        const int4 d = make_int4(r, m2, 0, 0);
        unit_slot[slot] = d;
        st_shared_cluster_v4(mapa_shared(smem_u32(&unit_slot[slot]), 1), d);
        mbar_arrive(&unit_full[slot]);
        mbar_arrive_release_cluster(mapa_shared(smem_u32(&unit_full[slot]), 1));
        return true;
      };
      // The leader draws one unit ahead: the next unit is drawn after the
      // first load of the current one, while the stages are full, so the
      // round trips of the draw never stall the operand stream at a unit
      // boundary.
      int next_r = -1, next_m2 = -1;
      bool draw_pending = false;
      if (a.withhold_loads) goto producer_done;  // test hook: nothing is loaded or published
      if (a.sched && leader && !draw(next_r, next_m2)) next_r = next_m2 = -1;
      for (int k = 0;; ++k) {
        int r = -1, m2 = -1;
        if (!a.sched) {
          if (!static_unit(k, r, m2)) break;
        } else if (leader) {
          r = next_r;
          m2 = next_m2;
          if (!publish(k, r, m2)) goto producer_done;
          if (r < 0) break;
          draw_pending = true;
        } else {
          if (!take_unit(k, r, m2, false)) goto producer_done;
          if (r < 0) break;
        }
        int v0, v1;
        split_range(r, a.n_vtile, a.n_split, v0, v1);
        for (int vt = v0; vt < v1; ++vt) {
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * PAIR_STAGE_BYTES);
            void* dA = sA + stage * A_STAGE_BYTES;
            void* dB = sB + stage * A_STAGE_BYTES;
            const int yE = m2 * (2 * BM) + rank * BM, yC = vt * BN + rank * BM;
            if (hint_e)
              tma_load_2d_pair_hint(dA, &tmE, &full[stage], kb * BK, yE, pol_e);
            else
              tma_load_2d_pair(dA, &tmE, &full[stage], kb * BK, yE);
            if (hint_c)
              tma_load_2d_pair_hint(dB, &tmCh, &full[stage], kb * BK, yC, pol_c);
            else
              tma_load_2d_pair(dB, &tmCh, &full[stage], kb * BK, yC);
            armed |= 1u << stage;
            if (draw_pending) {
              if (!draw(next_r, next_m2)) next_r = next_m2 = -1;
              draw_pending = false;
            }
            // L2 prefetch of this CTA's C rows a.pf slices ahead in the unit's
            // stream, by the pair on the first token block of the raster group
            // only (the other pairs on this split read the same rows)
            if (a.pf && m2 % a.group_m == 0) {
              const int s2 = (vt - v0) * nkb + kb + a.pf;
              if (s2 < (v1 - v0) * nkb)
                tma_prefetch_l2_2d(&tmCh, (s2 % nkb) * BK, (v0 + s2 / nkb) * BN + rank * BM);
            }
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (draw_pending) {  // a unit without loads (not reached: every split has a tile, D >= 8)
          if (!draw(next_r, next_m2)) next_r = next_m2 = -1;
          draw_pending = false;
        }
      }
    producer_done:
      // The leader's full barriers count both CTAs' copies: once they have
      // completed, nothing is in flight (the cluster sync below holds the
      // peer until then).
      if (leader) {
        int dummy = 0;
        WaitCtl exit_wc{&dummy, a.wait_limit_ns};
        for (int s = 0; s < S; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (s < stage) ? phase : (phase ^ 1u), exit_wc);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- UMMA issuer (leader only) ----------------
      constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, BN, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int k = 0;; ++k) {
        int r, m2;
        if (!a.sched) {
          if (!static_unit(k, r, m2)) break;
        } else {
          if (!take_unit(k, r, m2, false)) goto mma_done;
          if (r < 0) break;
        }
        int v0, v1;
        split_range(r, a.n_vtile, a.n_split, v0, v1);
        for (int vt = v0; vt < v1; ++vt) {
          if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) goto mma_done;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&full[stage], phase, wc)) goto mma_done;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + stage * A_STAGE_BYTES);
            const uint32_t b_addr = smem_u32(sB + stage * A_STAGE_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16_pair(d_tmem, sdesc_sw128(a_addr + k * 32, 16, 1024), sdesc_sw128(b_addr + k * 32, 16, 1024),
                             IDESC, (kb | k) != 0);
            umma_commit_pair_mc(&empty[stage], 0x3);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
          umma_commit_pair_mc(&tfull[acc], 0x3);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
    mma_done:
      umma_commit_pair_mc(drain, 0x1);
      {
        int dummy = 0;
        WaitCtl exit_wc{&dummy, a.wait_limit_ns};
        mbar_wait(drain, 0, exit_wc);
      }
    }
  } else {
    // ---------------- epilogue: 4 warps per CTA, one TMEM lane (token row) each ----------------
    const int lane_grp = warp & 3;
    const int row_in_blk = lane_grp * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(lane_grp * 32) << 16;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int k = 0;; ++k) {
      int r, m2;
      if (!a.sched) {
        if (!static_unit(k, r, m2)) break;
      } else {
        if (!take_unit(k, r, m2, true)) break;
        if (r < 0) break;
      }
      int v0, v1;
      split_range(r, a.n_vtile, a.n_split, v0, v1);
      const int row = m2 * (2 * BM) + (int)rank * BM + row_in_blk;
      float mrun = -INFINITY, srun = 0.f;
      bool ok = true;
      for (int vt = v0; vt < v1; ++vt) {
        if (!mbar_wait(&tfull[acc], acc_phase, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        lse_fold_tile<DUMP>(tmem_base + lane_addr + (uint32_t)(acc * BN), vt * BN, row, a, mrun, srun);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      if (row < a.N) a.partial[(size_t)r * a.N + row] = make_float2(mrun, srun);
    }
  }

  // ---------------- teardown ----------------
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrival or copy can target an exited CTA
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(a.status + ST_FLAGS, SF_TIMEOUT);
  if (threadIdx.x == 0 && blockIdx.x == 0 && !*abort_flag)
    atomicAdd(a.status + ST_TILES, (unsigned long long)(a.N + BM - 1) / BM * (unsigned long long)a.n_vtile);
}

// One warp per token row.
__global__ void __launch_bounds__(256) fwd_finalize_kernel(const __nv_bfloat16* __restrict__ E,
                                                           const __nv_bfloat16* __restrict__ C,
                                                           const int64_t* __restrict__ y, const FinArgs a,
                                                           float* __restrict__ loss, float* __restrict__ lse) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= a.N) return;

  // A bounded wait of the logit kernel gave up: some partials were never
  // written (the workspace may hold an earlier call's values), so every
  // output of this call is NaN rather than a plausible wrong number.
  if (a.status[ST_FLAGS] & SF_TIMEOUT) {
    if (lane == 0) {
      const float qnan = __int_as_float(0x7fc00000);
      if (a.shard_stats) {
        a.shard_stats[row] = qnan;
        a.shard_stats[(size_t)a.N + row] = qnan;
        a.shard_stats[2 * (size_t)a.N + row] = qnan;
      } else {
        lse[row] = qnan;
        loss[row] = qnan;
        if (a.row_max) a.row_max[row] = qnan;
      }
    }
    return;
  }

  // merge the per-split (max, sum) pairs: lse = M + log(sum_r s_r exp(m_r - M))
  float M = -INFINITY;
  for (int r = lane; r < a.n_split; r += 32) M = fmaxf(M, a.partial[(size_t)r * a.N + row].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float s = 0.f;
  for (int r = lane; r < a.n_split; r += 32) {
    const float2 p = a.partial[(size_t)r * a.N + row];
    if (p.x != -INFINITY) s += p.y * expf(p.x - M);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float L = M + logf(s);
  if (lane == 0 && a.row_max && !a.shard_stats) a.row_max[row] = M;

  if (a.shard_stats) {
    // vocabulary shard: (max, sum exp(z - max)) over the shard and the target
    // logit if the label falls in it (0 otherwise; exactly one shard owns it)
    const long long tg = y[row];
    const long long tl = tg - a.v_offset;
    float z = 0.f;
    if (tg != a.ignore_index && tl >= 0 && tl < a.V) {
      const uint4* er = reinterpret_cast<const uint4*>(E + (size_t)row * a.D);
      const uint4* cr = reinterpret_cast<const uint4*>(C + (size_t)tl * a.D);
      float z0 = 0.f, z1 = 0.f;
      for (int i = lane; i < (a.D >> 3); i += 32) {
        const uint4 ev = __ldg(er + i), cv = __ldg(cr + i);
        const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&ev);
        const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&cv);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 ef = __bfloat1622float2(e2[j]);
          const float2 cf = __bfloat1622float2(c2[j]);
          z0 = fmaf(ef.x, cf.x, z0);
          z1 = fmaf(ef.y, cf.y, z1);
        }
      }
      z = z0 + z1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    }
    if (lane == 0) {
      a.shard_stats[row] = M;
      a.shard_stats[(size_t)a.N + row] = s;
      a.shard_stats[2 * (size_t)a.N + row] = z;
    }
    return;
  }

  const long long t = y[row];
  float out;
  if (t == a.ignore_index) {
    out = 0.f;
  } else if (t >= 0 && t < a.V) {
    // correct-token logit z = E_row . C_t, 8 bf16 per 16-byte load
    const uint4* er = reinterpret_cast<const uint4*>(E + (size_t)row * a.D);
    const uint4* cr = reinterpret_cast<const uint4*>(C + (size_t)t * a.D);
    const int nvec = a.D >> 3;
    float z0 = 0.f, z1 = 0.f;
    for (int i = lane; i < nvec; i += 32) {
      const uint4 ev = __ldg(er + i), cv = __ldg(cr + i);
      const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&ev);
      const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&cv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 ef = __bfloat1622float2(e2[j]);
        const float2 cf = __bfloat1622float2(c2[j]);
        z0 = fmaf(ef.x, cf.x, z0);
        z1 = fmaf(ef.y, cf.y, z1);
      }
    }
    float z = z0 + z1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    out = L - z;
  } else {
    out = __int_as_float(0x7fc00000);  // NaN: the label is invalid
    if (lane == 0) atomicOr(a.status + ST_FLAGS, SF_BAD_LABEL);
  }
  if (lane == 0) {
    lse[row] = L;
    loss[row] = out;
  }
}

// Merge R vocabulary shards' (max, sum exp, target) statistics into the
// per-token loss and lse: lse = M + log sum_r s_r exp(m_r - M), M = max_r m_r;
// the target logit is the sum over shards (only the owner contributes).
__global__ void __launch_bounds__(256) merge_shards_kernel(const float* __restrict__ stats, int R, int N,
                                                           const int64_t* __restrict__ y, long long V_total,
                                                           long long ignore_index, float* __restrict__ loss,
                                                           float* __restrict__ lse, unsigned long long* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const size_t sh = 3 * (size_t)N;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, stats[r * sh + i]);
  float s = 0.f, z = 0.f;
  for (int r = 0; r < R; ++r) {
    const float m = stats[r * sh + i];
    if (m != -INFINITY) s += stats[r * sh + N + i] * expf(m - M);
    z += stats[r * sh + 2 * (size_t)N + i];
  }
  const float L = M + logf(s);
  const long long t = y[i];
  float out;
  if (t == ignore_index) {
    out = 0.f;
  } else if (t >= 0 && t < V_total) {
    out = L - z;
  } else {
    out = __int_as_float(0x7fc00000);
    if (status) atomicOr(status + ST_FLAGS, SF_BAD_LABEL);
  }
  lse[i] = L;
  loss[i] = out;
}

cudaError_t launch_merge_shards(const float* stats, int R, int N, const int64_t* y, long long V_total,
                                long long ignore_index, float* loss, float* lse, cudaStream_t stream) {
  merge_shards_kernel<<<(N + 255) / 256, 256, 0, stream>>>(stats, R, N, y, V_total, ignore_index, loss, lse,
                                                           nullptr);
  return cudaGetLastError();
}

size_t fwd_smem_bytes() { return 1024 + (size_t)FWD_STAGES * STAGE_BYTES + 256; }
size_t fwd_pair_smem_bytes(int stages) { return 1024 + (size_t)stages * PAIR_STAGE_BYTES + 256; }

namespace {
template <bool DUMP, int S>
cudaError_t launch_pair_stages(const CUtensorMap& tmE, const CUtensorMap& tmCh, const FwdArgs& a, int grid,
                               cudaStream_t stream) {
  const size_t smem = fwd_pair_smem_bytes(S);
  cudaError_t e = cudaFuncSetAttribute(fwd_lse_pair_kernel<DUMP, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  fwd_lse_pair_kernel<DUMP, S><<<grid, NUM_THREADS, smem, stream>>>(tmE, tmCh, a);
  return cudaGetLastError();
}
}  // namespace

// grid: an even number of CTAs (pairs); stages: PAIR_STAGES or PAIR_STAGES_MAX
// operand stages per CTA (the latter fills the 227 KB of shared memory)
cudaError_t launch_fwd_lse_pair(const CUtensorMap& tmE, const CUtensorMap& tmCh, const FwdArgs& a, int grid,
                                int stages, cudaStream_t stream) {
  if (stages == PAIR_STAGES_MAX)
    return a.dbg_logits ? launch_pair_stages<true, PAIR_STAGES_MAX>(tmE, tmCh, a, grid, stream)
                        : launch_pair_stages<false, PAIR_STAGES_MAX>(tmE, tmCh, a, grid, stream);
  return a.dbg_logits ? launch_pair_stages<true, PAIR_STAGES>(tmE, tmCh, a, grid, stream)
                      : launch_pair_stages<false, PAIR_STAGES>(tmE, tmCh, a, grid, stream);
}

cudaError_t launch_fwd_lse(const CUtensorMap& tmE, const CUtensorMap& tmC, const FwdArgs& a, int grid,
                           cudaStream_t stream) {
  const size_t smem = fwd_smem_bytes();
  if (a.dbg_logits) {
    cudaError_t e = cudaFuncSetAttribute(fwd_lse_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_lse_kernel<true><<<grid, NUM_THREADS, smem, stream>>>(tmE, tmC, a);
  } else {
    cudaError_t e = cudaFuncSetAttribute(fwd_lse_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_lse_kernel<false><<<grid, NUM_THREADS, smem, stream>>>(tmE, tmC, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_fwd_finalize(const void* E, const void* C, const int64_t* y, const FinArgs& a, float* loss,
                                float* lse, cudaStream_t stream) {
  const int rows_per_block = 8;
  const int grid = (a.N + rows_per_block - 1) / rows_per_block;
  fwd_finalize_kernel<<<grid, rows_per_block * 32, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(E), reinterpret_cast<const __nv_bfloat16*>(C), y, a, loss, lse);
  return cudaGetLastError();
}

}  // namespace cce
