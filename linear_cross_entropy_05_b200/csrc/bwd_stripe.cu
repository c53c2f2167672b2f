// CCE backward through stripes of the softmax gradient: the dense path
// (filter off), and with the entry filter for heads whose softmax is not
// flat (CCE_BWD_STRIPES with filter_eps > 0).
//
// Cut Cross-Entropy abstract, sentences 4 and 9: the logits are recomputed,
// never stored; the backward forms G = dloss * (softmax - onehot) and
// contracts it into dE = G C and dC = G^T E.  When nothing is filtered every
// logit tile contributes to both products, and adding each tile's fp32
// partial products to dE and dC ((256 + 256) x D values per 256 x 256 tile)
// would move far more bytes through L2 than the tensor cores need time for.
// Instead the vocabulary is processed in stripes of Vs = vt_per_s * 256
// columns; for each stripe (task kinds, see StripePlan in common.cuh):
//   A  recompute the logit tiles of the stripe (E C^T on the tensor cores,
//      tcgen05 cta_group::2, as in the forward), form G in registers and
//      store it in bf16 into a stripe buffer in global memory (L2-resident:
//      nbuf x 256-row blocks x Vs columns);
//   B  dC[stripe rows] = G^T E with the whole token range as the reduction
//      dimension: each dC tile is written exactly once;
//   C  dE += G C[stripe rows]: one bulk reduce-add of a 256 x 256 dE tile per
//      stripe instead of one per logit tile.
// So the logits never exist in global memory: only nbuf stripes of G do,
// O(N) bytes for a fixed stripe width (Vs = 4096: 24 KB per token with three
// buffers), against N x V x 4 bytes of fp32 logits.
//
// With the filter on, entries below filter_eps are zeroed in G, and work is
// skipped at two grains: an A task whose two 128-token blocks the pre-pass
// proved flat is not recomputed (the flat-row kernel adds those blocks'
// label entries afterwards; a flat half of a recomputed task gets zero rows),
// and each A task flags its 256 x 256 G tile if it holds a kept entry, so a
// B or C task streams only the K blocks (token blocks, resp. vocabulary
// tiles) whose G tile is flagged; the mask travels with the task.  A task
// left with nothing to do (an A task of two flat blocks, a dC task that adds
// into dC with no flagged block, an unordered dE task with none) never
// reaches the other roles: the producer retires it on the spot, raising its
// completion counters by all of its arrivals.
//
// One persistent kernel runs all three kinds on clusters of two CTAs.  Tasks
// are drawn in a fixed global order from a counter by the leader CTA's
// producer thread, which also waits (bounded) until the task's inputs are
// complete (counters in global memory, released by the epilogues that wrote
// them), then hands the task to both CTAs through a small ring in shared
// memory.  Roles per CTA (320 threads): warp 0 TMA producer, warp 1 UMMA
// issuer (leader CTA only), warps 2-9 epilogue (two per TMEM lane group, one
// per 128-column half).  Each CTA stages 32 KB of
// operands per 64-wide K slice (5 stages) and double-buffers a 128 x 256 fp32
// accumulator in TMEM, so the epilogue of one task overlaps the MMAs of the
// next.  No TMA multicast: every load reads this GPU's memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace cce {

namespace {

constexpr int SP_STAGES = 5;
constexpr int SP_STAGE_BYTES = 32768;          // per CTA: two 16 KB operand regions
constexpr int SP_EPI_WARPS = 8;                // two per TMEM lane group, one per 128-column half
constexpr int SP_THREADS = 64 + 32 * SP_EPI_WARPS;
constexpr int SP_STAGING_PER_WARP = 8192;      // epilogue staging: two 4 KB boxes (bf16 G or fp32 blocks)
constexpr int SP_RING = 4;                     // task hand-off slots
constexpr int SP_CONSUMERS = 2 + 2 * SP_EPI_WARPS;  // leader: MMA + epilogue warps; peer: producer + epilogue warps
constexpr unsigned SP_DONE = 2 * SP_EPI_WARPS; // completion arrivals per task (epilogue warps of both CTAs)

// d-columns of a dC / dE task's chunk: 256, or 128 for a last chunk that
// narrow (D = 896: three chunks of 256 and one of 128), so the tensor cores
// do not multiply columns that lie past D.
__device__ __forceinline__ int chunk_width(int D, int dc) { return D - dc * 256 <= 128 ? 128 : 256; }

struct StripeMaps {
  CUtensorMap eA;    // E   bf16 [N][D]        box {64, 128}: A tasks, K-major token rows
  CUtensorMap cA;    // C   bf16 [V][D]        box {64, 128}: A tasks, K-major vocabulary rows
  CUtensorMap gSt;   // G   bf16 [nbuf*Ns][Vs] box {64, 32}:  A tasks store one warp's rows
  CUtensorMap gK;    // G   bf16               box {64, 128}: C tasks, K-major token rows
  CUtensorMap gM;    // G   bf16               box {64, 64}:  B tasks, vocabulary-contiguous (MN-major)
  CUtensorMap eM;    // E   bf16               box {64, 64}:  B tasks, d-contiguous (MN-major)
  CUtensorMap cM;    // C   bf16               box {64, 64}:  C tasks, d-contiguous (MN-major)
  CUtensorMap dE;    // dE  fp32 [N][D]        box {32, 32}: reduce-add
  CUtensorMap dC;    // dC  fp32 [V][D]        box {32, 32}: store / reduce-add
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// A 32 x 32 fp32 block held one row per lane goes to global memory through
// the TMA engine: written into a 4 KB staging buffer in the 128-byte-swizzled
// layout of a {32, 32} fp32 box, then stored or reduce-added at (x, y).
__device__ __forceinline__ void stage_f32_block(uint8_t* xb, int lane, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(xb + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SP_THREADS, 1)
    bwd_stripe_kernel(const __grid_constant__ StripeMaps mp, const StripeArgs a, __nv_bfloat16* G) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;                                          // SP_STAGES x 32 KB
  uint8_t* staging = smem + SP_STAGES * SP_STAGE_BYTES;            // SP_EPI_WARPS x 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + SP_EPI_WARPS * SP_STAGING_PER_WARP);
  uint64_t* full = bars;                          // leader: both CTAs' copies of a stage landed
  uint64_t* empty = bars + SP_STAGES;             // each CTA: stage free again
  uint64_t* tfull = bars + 2 * SP_STAGES;         // each CTA: accumulator ready [2]
  uint64_t* tempty = tfull + 2;                   // leader: both epilogues done with it [2]
  uint64_t* drain = tempty + 2;                   // leader: UMMA drain at exit
  uint64_t* task_full = drain + 1;                // each CTA [SP_RING]
  uint64_t* task_empty = task_full + SP_RING;     // leader [SP_RING]
  // each CTA [SP_RING][2], 16-byte aligned (written with 16-byte stores):
  // the task, then its 64-bit mask of live K blocks (B / C tasks)
  int4* task_slot = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(task_empty + SP_RING) + 15) & ~uintptr_t(15));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(task_slot + 2 * SP_RING);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const StripePlan& P = a.p;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * SP_EPI_WARPS);
    }
    mbar_init(drain, 1);
    for (int r = 0; r < SP_RING; ++r) {
      mbar_init(&task_full[r], 1);
      mbar_init(&task_empty[r], SP_CONSUMERS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_map(&mp.eA);
    tma_prefetch_map(&mp.cA);
    tma_prefetch_map(&mp.gSt);
    tma_prefetch_map(&mp.gK);
    tma_prefetch_map(&mp.gM);
    tma_prefetch_map(&mp.eM);
    tma_prefetch_map(&mp.cM);
    tma_prefetch_map(&mp.dE);
    tma_prefetch_map(&mp.dC);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, a.wait_limit_ns};
  const uint32_t task_empty_leader0 = mapa_shared(smem_u32(&task_empty[0]), 0);

  // Reads task k from this CTA's ring, then frees the slot on the leader
  // (one arrival per consumer).  With whole_warp, lane 0 waits and reads and
  // the warp follows its outcome, so the lanes never part ways on a wait.
  auto take_task = [&](int k, StripeTaskDesc& t, unsigned long long& mask, bool whole_warp) -> bool {
    const int slot = k & (SP_RING - 1);
    int4 d = make_int4(TASK_END, 0, 0, 0);
    unsigned mlo = 0u, mhi = 0u;
    int ok = 1;
    if (!whole_warp || lane == 0) {
      ok = mbar_wait_cluster(&task_full[slot], (uint32_t)(k / SP_RING) & 1u, wc) ? 1 : 0;
      if (ok) {
        const volatile int* vs = reinterpret_cast<const volatile int*>(&task_slot[2 * slot]);
        d = make_int4(vs[0], vs[1], vs[2], vs[3]);
        mlo = (unsigned)vs[4];
        mhi = (unsigned)vs[5];
        mbar_arrive_cluster(task_empty_leader0 + (uint32_t)(slot * 8));
      }
    }
    if (whole_warp) {
      ok = __shfl_sync(0xffffffffu, ok, 0);
      d.x = __shfl_sync(0xffffffffu, d.x, 0);
      d.y = __shfl_sync(0xffffffffu, d.y, 0);
      d.z = __shfl_sync(0xffffffffu, d.z, 0);
      d.w = __shfl_sync(0xffffffffu, d.w, 0);
      mlo = __shfl_sync(0xffffffffu, mlo, 0);
      mhi = __shfl_sync(0xffffffffu, mhi, 0);
    }
    t = StripeTaskDesc{d.x, d.y, d.z, d.w};
    mask = ((unsigned long long)mhi << 32) | mlo;
    return ok != 0;
  };
  // K blocks (256 wide: a token block for B, a vocabulary tile for C) of a
  // B or C task, and which of them hold a nonzero G tile.  Read after the
  // task's inputs are complete; without the filter every block is live.
  auto k_blocks = [&](const StripeTaskDesc& t) -> int {
    return t.type == TASK_B ? a.Ns_pad / 256 : stripe_tiles(P, t.s);
  };
  auto live_mask = [&](const StripeTaskDesc& t) -> unsigned long long {
    if (t.type == TASK_A) {
      // 1: recompute; 0: both 128-token blocks are flat (or past N), skip
      if (a.blk_flat == nullptr) return 1ull;
      const int row0 = a.tok0 + t.a * 256;
      const bool f0 = __ldcg(a.blk_flat + row0 / BM) != 0;
      const bool f1 = row0 + BM >= a.N || __ldcg(a.blk_flat + row0 / BM + 1) != 0;
      return (f0 && f1) ? 0ull : 1ull;
    }
    const int nb = k_blocks(t);
    const unsigned long long all = nb >= 64 ? ~0ull : ((1ull << nb) - 1ull);
    if (t.type == TASK_END || a.nz == nullptr) return all;
    unsigned long long m = 0ull;
    if (t.type == TASK_B) {
      const unsigned char* f = a.nz + (size_t)t.s * P.n_m2 * P.vt_per_s + (t.a - t.s * P.vt_per_s);
      for (int b = 0; b < nb; ++b)
        if (__ldcg(f + (size_t)b * P.vt_per_s)) m |= 1ull << b;
    } else {
      const unsigned char* f = a.nz + ((size_t)t.s * P.n_m2 + t.a) * P.vt_per_s;
      for (int b = 0; b < nb; ++b)
        if (__ldcg(f + b)) m |= 1ull << b;
    }
    return m;
  };
  // Bounded wait taken by lane 0 for the whole warp (warp-uniform outcome).
  auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    int ok = 0;
    if (lane == 0) ok = mbar_wait(bar, parity, wc) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
  };
  auto k_steps = [&](const StripeTaskDesc& t) -> int {
    if (t.type == TASK_A) return (a.D + BK - 1) / BK;
    if (t.type == TASK_B) return a.Ns_pad / BK;
    return stripe_tiles(P, t.s) * (BN / BK);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer (both CTAs); the leader also deals the tasks ----------------
      int stage = 0;
      uint32_t phase = 0, armed = 0;
      const long long total = stripe_total(P);
      unsigned long long* trace = (a.trace && leader) ? a.trace + (size_t)(blockIdx.x >> 1) * a.trace_cap * 4 : nullptr;
      // The leader draws task k+1 while it issues task k's loads, and reads
      // the counter of its inputs a few stages before the end of task k, so
      // neither round trip stalls the operand stream between tasks.
      unsigned long long drawn_next = leader ? atomicAdd(a.next, 1ull) : 0ull;
      StripeTaskDesc t_next{TASK_END, 0, 0, 0};
      const unsigned* dep_ctr = nullptr;
      unsigned dep_want = 0, dep_seen = 0;
      bool next_known = false;
      auto look_ahead = [&]() {
        t_next = drawn_next < (unsigned long long)total ? stripe_decode(P, (long long)drawn_next)
                                                        : StripeTaskDesc{TASK_END, 0, 0, 0};
        dep_ctr = nullptr;
        dep_want = 0;
        if (t_next.type == TASK_A) {
          if (t_next.s >= P.nbuf) {
            const int s0 = t_next.s - P.nbuf;
            dep_ctr = a.doneBC + s0;
            dep_want = SP_DONE * (unsigned)(stripe_nB(P, s0) + stripe_nC(P));
          }
        } else if (t_next.type == TASK_B) {
          dep_ctr = a.doneA_v + t_next.a;
          dep_want = SP_DONE * (unsigned)P.n_m2;
        } else if (t_next.type == TASK_C) {
          dep_ctr = a.doneA_ms + (size_t)t_next.s * P.n_m2 + t_next.a;
          dep_want = SP_DONE * (unsigned)stripe_tiles(P, t_next.s);
        }
        dep_seen = dep_ctr ? ld_acquire_gpu(dep_ctr) : dep_want;
        next_known = true;
      };
      for (int k = 0;; ++k) {
        StripeTaskDesc t;
        unsigned long long tmask = 0ull;
        if (leader) {
          const int slot = k & (SP_RING - 1);
          if (!mbar_wait(&task_empty[slot], ((uint32_t)(k / SP_RING) & 1u) ^ 1u, wc)) goto producer_done;
          const uint64_t t_dep0 = trace ? global_timer_ns() : 0;
          // Draw until a task with work: a task with nothing to do (a
          // recompute task of two flat blocks, a dC task that would add
          // zeros, an unordered dE task with no live block) is retired here,
          // its completion counters bumped for all its arrivals at once.
          while (true) {
            if (!next_known) look_ahead();
            t = t_next;
            next_known = false;
            // wait until the task's inputs are complete (bounded)
            if (t.type != TASK_END) {
              if (dep_seen < dep_want) {
                const uint64_t t0 = global_timer_ns();
                bool ok = false;
                while (true) {
                  __nanosleep(256);
                  if (ld_acquire_gpu(dep_ctr) >= dep_want) {
                    ok = true;
                    break;
                  }
                  if (*abort_flag) break;
                  if (global_timer_ns() - t0 > a.wait_limit_ns) {
                    *abort_flag = 1;
                    break;
                  }
                }
                if (!ok) goto producer_done;
              }
              fence_proxy_async_global();  // the inputs were written by other CTAs' bulk stores
            }
            tmask = live_mask(t);
            const bool idle = tmask == 0ull && ((t.type == TASK_A) || (t.type == TASK_B && a.dC_add) ||
                                                (t.type == TASK_C && !a.ordered));
            if (!idle) break;
            if (t.type == TASK_A) {
              red_release_gpu_add(a.doneA_v + t.b, SP_DONE);
              red_release_gpu_add(a.doneA_ms + (size_t)t.s * P.n_m2 + t.a, SP_DONE);
            } else {
              red_release_gpu_add(a.doneBC + t.s, SP_DONE);
            }
            drawn_next = atomicAdd(a.next, 1ull);
          }
          const int4 d = make_int4(t.type, t.s, t.a, t.b);
          const int4 dm = make_int4((int)(unsigned)tmask, (int)(unsigned)(tmask >> 32), 0, 0);
          task_slot[2 * slot] = d;
          task_slot[2 * slot + 1] = dm;
          st_shared_cluster_v4(mapa_shared(smem_u32(&task_slot[2 * slot]), 1), d);
          st_shared_cluster_v4(mapa_shared(smem_u32(&task_slot[2 * slot + 1]), 1), dm);
          mbar_arrive(&task_full[slot]);
          mbar_arrive_release_cluster(mapa_shared(smem_u32(&task_full[slot]), 1));
          if (t.type != TASK_END) drawn_next = atomicAdd(a.next, 1ull);
          if (trace && k < a.trace_cap && t.type != TASK_END) {
            const uint64_t now = global_timer_ns();
            trace[k * 4 + 0] = now;
            trace[k * 4 + 3] = (unsigned long long)t.type | ((now - t_dep0) << 8);
          }
        } else {
          if (!take_task(k, t, tmask, false)) goto producer_done;
          fence_proxy_async_global();
        }
        if (t.type == TASK_END) break;
        // live K slices of the task, in order (A tasks: all of K = D)
        const int nk = t.type == TASK_A ? (tmask ? k_steps(t) : 0) : 4 * __popcll(tmask);
        const int r = (int)rank;
        if (t.type == TASK_C && a.dE_prefetch && !a.withhold_loads) {
          // the dE rows this task's epilogue will add into: into L2 while it computes
          const int row0 = a.tok0 + t.a * 256 + r * 128;
#pragma unroll 1
          for (int g = 0; g < 4; ++g)
#pragma unroll 1
            for (int c = 0; c < 8; ++c)
              if (row0 + 32 * g < a.N && t.b * 256 + 32 * c < a.D)
                tma_prefetch_l2_2d(&mp.dE, t.b * 256 + 32 * c, row0 + 32 * g);
        }
        // B / C tasks: this CTA's half of the chunk's d columns, in 64-wide boxes
        const int nd = t.type == TASK_A ? 256 : chunk_width(a.D, t.b);
        const int half_boxes = nd / 128;                 // 2, or 1 for a 128-wide chunk
        const uint32_t cta_bytes = 16384u + (t.type == TASK_A ? 16384u : 8192u * (uint32_t)half_boxes);
        unsigned long long rest = tmask;  // B / C: live K blocks not yet streamed
        int blk = -1;
        for (int j = 0; j < nk; ++j) {
          if (leader && j == (nk > SP_STAGES ? nk - SP_STAGES : 0)) look_ahead();
          if (t.type != TASK_A && (j & 3) == 0) {
            blk = __ffsll((long long)rest) - 1;
            rest &= rest - 1ull;
          }
          const int kb = t.type == TASK_A ? j : 4 * blk + (j & 3);
          if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
          uint8_t* X = stages + stage * SP_STAGE_BYTES;
          uint8_t* Y = X + 16384;
          if (leader) mbar_arrive_expect_tx(&full[stage], 2u * cta_bytes);
          if (!a.withhold_loads) {
            if (t.type == TASK_A) {
              // X = E[token rows of this CTA][64 d], Y = C[vocabulary rows of this CTA][64 d]
              tma_load_2d_pair(X, &mp.eA, &full[stage], kb * BK, a.tok0 + t.a * 256 + r * 128);
              tma_load_2d_pair(Y, &mp.cA, &full[stage], kb * BK, t.b * BN + r * 128);
            } else if (t.type == TASK_B) {
              // X = G[64 tokens][this CTA's 128 vocabulary columns] (two 64-column boxes),
              // Y = E[64 tokens][this CTA's 128 d columns]
              const int gcol = (t.a - t.s * P.vt_per_s) * BN + r * 128;
              const int grow = (t.s % P.nbuf) * a.Ns_pad + kb * BK;
              tma_load_2d_pair(X, &mp.gM, &full[stage], gcol, grow);
              tma_load_2d_pair(X + 8192, &mp.gM, &full[stage], gcol + 64, grow);
              const int d0 = t.b * 256 + r * (nd / 2);
              tma_load_2d_pair(Y, &mp.eM, &full[stage], d0, a.tok0 + kb * BK);
              if (half_boxes == 2) tma_load_2d_pair(Y + 8192, &mp.eM, &full[stage], d0 + 64, a.tok0 + kb * BK);
            } else {
              // X = G[this CTA's 128 token rows][64 stripe columns],
              // Y = C[64 stripe rows][this CTA's 128 d columns]
              tma_load_2d_pair(X, &mp.gK, &full[stage], kb * BK,
                               (t.s % P.nbuf) * a.Ns_pad + t.a * 256 + r * 128);
              const int v0 = t.s * P.vt_per_s * BN + kb * BK;
              const int d0 = t.b * 256 + r * (nd / 2);
              tma_load_2d_pair(Y, &mp.cM, &full[stage], d0, v0);
              if (half_boxes == 2) tma_load_2d_pair(Y + 8192, &mp.cM, &full[stage], d0 + 64, v0);
            }
            armed |= 1u << stage;
          }
          if (++stage == SP_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      if (leader) {
        int dummy = 0;
        WaitCtl exit_wc{&dummy, a.wait_limit_ns};
        for (int s = 0; s < SP_STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&full[s], (s < stage) ? phase : (phase ^ 1u), exit_wc);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- UMMA issuer (leader) ----------------
      constexpr uint32_t IDESC_A = idesc_bf16_f32(2 * BM, BN, false, false);
      constexpr uint32_t IDESC_B = idesc_bf16_f32(2 * BM, BN, true, true);
      constexpr uint32_t IDESC_C = idesc_bf16_f32(2 * BM, BN, false, true);
      constexpr uint32_t IDESC_B128 = idesc_bf16_f32(2 * BM, 128, true, true);
      constexpr uint32_t IDESC_C128 = idesc_bf16_f32(2 * BM, 128, false, true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int k = 0;; ++k) {
        StripeTaskDesc t;
        unsigned long long tmask;
        if (!take_task(k, t, tmask, false)) goto mma_done;
        if (t.type == TASK_END) break;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, wc)) goto mma_done;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        // the live K slices the producer streams, in the same order (a task
        // with none leaves the accumulator untouched; its epilogue knows)
        const int nk = t.type == TASK_A ? (tmask ? k_steps(t) : 0) : 4 * __popcll(tmask);
        const bool narrow = t.type != TASK_A && chunk_width(a.D, t.b) == 128;
        const uint32_t idesc_b = narrow ? IDESC_B128 : IDESC_B;
        const uint32_t idesc_c = narrow ? IDESC_C128 : IDESC_C;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, wc)) goto mma_done;
          tc_fence_after();
          const uint32_t xa = smem_u32(stages + stage * SP_STAGE_BYTES);
          const uint32_t ya = xa + 16384;
#pragma unroll
          for (int k16 = 0; k16 < BK / 16; ++k16) {
            const uint32_t acc_on = (kb | k16) != 0;
            if (t.type == TASK_A) {
              umma_bf16_pair(d_tmem, sdesc_sw128(xa + k16 * 32, 16, 1024), sdesc_sw128(ya + k16 * 32, 16, 1024),
                             IDESC_A, acc_on);
            } else if (t.type == TASK_B) {
              // A = G^T (M = vocabulary, 64-column groups 8 KB apart; K = tokens, 128 B rows)
              // B = E (N = d, 64-column groups 8 KB apart; K = tokens)
              umma_bf16_pair(d_tmem, sdesc_sw128(xa + k16 * 2048, 8192, 1024),
                             sdesc_sw128(ya + k16 * 2048, 8192, 1024), idesc_b, acc_on);
            } else {
              // A = G (K-major token rows), B = C (N = d groups 8 KB apart; K = vocabulary rows)
              umma_bf16_pair(d_tmem, sdesc_sw128(xa + k16 * 32, 16, 1024),
                             sdesc_sw128(ya + k16 * 2048, 8192, 1024), idesc_c, acc_on);
            }
          }
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == SP_STAGES) {
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
    mma_done:
      umma_commit_pair_mc(drain, 0x1);
      {
        int dummy = 0;
        WaitCtl exit_wc{&dummy, a.wait_limit_ns};
        mbar_wait(drain, 0, exit_wc);
      }
    }
  } else {
    // ---------------- epilogue: 8 warps per CTA, one TMEM lane (row) per thread ----------------
    // Warp w may only read TMEM lanes 32 (w % 4) .. +31; warps 2-5 take the
    // first 128 accumulator columns and warps 6-9 the last 128, so each lane
    // group has one warp per half.
    const int lg = warp & 3;                 // TMEM lane group of this warp
    const int hsel = (warp - 2) >> 2;        // 128-column half of this warp
    const uint32_t lane_addr = (uint32_t)(lg * 32) << 16;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    uint8_t* stg = staging + (warp - 2) * SP_STAGING_PER_WARP;
    const int r = (int)rank;
    int acc = 0;
    uint32_t acc_phase = 0;
    unsigned long long n_tiles = 0, n_units = 0, n_live = 0, n_inrange = 0;
    unsigned long long* trace = (a.trace && leader && warp == 2 && lane == 0)
                                    ? a.trace + (size_t)(blockIdx.x >> 1) * a.trace_cap * 4
                                    : nullptr;
    for (int k = 0;; ++k) {
      StripeTaskDesc t;
      unsigned long long tmask;
      if (!take_task(k, t, tmask, true)) break;
      if (t.type == TASK_END) break;
      if (!warp_wait(&tfull[acc], acc_phase)) break;
      tc_fence_after();
      if (trace && k < a.trace_cap) trace[k * 4 + 1] = global_timer_ns();
      const uint32_t tacc = tmem_base + lane_addr + (uint32_t)(acc * BN);
      if (t.type == TASK_A) {
        // (an A task of two flat blocks never gets here: the producer retired
        // it, and its G tile keeps flag 0, so no B or C task reads it)
        // row = token; columns = this warp's 128 of the 256 vocabulary entries of tile t.b
        const int row = a.tok0 + t.a * 256 + r * 128 + lg * 32 + lane;
        // a flat block's rows of G are zero: its label entries go to the flat-row kernel
        const int blk_row0 = a.tok0 + t.a * 256 + r * 128;
        const bool blk_is_flat = a.blk_flat != nullptr && blk_row0 < a.N && a.blk_flat[blk_row0 / BM] != 0;
        bool valid = row < a.N && !blk_is_flat;
        long long yl = valid ? a.y[row] : a.ignore_index;
        if (yl == a.ignore_index) valid = false;
        if (a.shard_mode) {
          yl -= a.v_offset;
        } else if (valid && (yl < 0 || yl >= a.V)) {
          valid = false;
          atomicOr(a.status + ST_FLAGS, SF_BAD_LABEL);
        }
        const float lse2 = valid ? a.lse[row] * LOG2E : 0.f;
        const float dl = valid ? a.dloss[row] : 0.f;
        const long long yrel = yl - (long long)t.b * BN;
        const int ycol = (valid && yrel >= 0 && yrel < BN) ? (int)yrel : -1;
        const int ncols = min(BN, a.V - t.b * BN);
        const int sw = lane & 7;
        const int gcol = (t.b - t.s * P.vt_per_s) * BN + hsel * 128;
        const int grow = (t.s % P.nbuf) * a.Ns_pad + t.a * 256 + r * 128 + lg * 32;
        unsigned live_units = 0;  // of this warp's four 32 x 32 units (filter on)
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          const int c = hsel * 4 + cc;  // 32-column chunk of the accumulator
          float x[32];
          tmem_ld32(tacc + (uint32_t)(c * 32), x);
          uint32_t pk[16];
          bool kept = false;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float g2[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int col = c * 32 + j + q;
              const float p = ex2_approx(fmaf(x[j + q], LOG2E, -lse2));
              float d = (col == ycol) ? p - 1.f : p;
              d = (valid && col < ncols) ? d : 0.f;
              // the entry filter (eps <= 0 keeps every entry)
              const bool keep = fabsf(d) >= a.filter_eps && d != 0.f;
              kept |= keep;
              g2[q] = keep ? dl * d : 0.f;
            }
            pk[j >> 1] = pack_bf16x2(g2[0], g2[1]);
          }
          live_units += __any_sync(0xffffffffu, kept) ? 1u : 0u;
          // staging box cc / 2 (64 columns), this lane's 128-byte row, 128B swizzle
          uint8_t* rowp = stg + (cc >> 1) * 4096 + lane * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = ((cc & 1) * 4 + q) ^ sw;
            *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        // every column this warp needs is read from TMEM
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&mp.gSt, stg, gcol, grow);
          tma_store_2d(&mp.gSt, stg + 4096, gcol + 64, grow);
          bulk_commit_group();
          // this G tile holds a kept entry: B and C tasks must read it
          if (a.nz && live_units)
            a.nz[((size_t)t.s * P.n_m2 + t.a) * P.vt_per_s + (t.b - t.s * P.vt_per_s)] = 1;
          n_live += live_units;
          // in-range units of this warp: its 32-row group (if any row is a
          // token of this launch's range) x its 32-column chunks inside V
          if (a.tok0 + t.a * 256 + r * 128 + lg * 32 < a.N && !blk_is_flat)
            n_inrange += (unsigned long long)max(0, min(4, (ncols - hsel * 128 + 31) / 32));
          bulk_wait_group0();
          fence_proxy_async_global();
          red_release_gpu_add(a.doneA_v + t.b, 1u);
          red_release_gpu_add(a.doneA_ms + (size_t)t.s * P.n_m2 + t.a, 1u);
          if (lg == 0 && hsel == 0) {
            const int rows_here = a.N - (a.tok0 + t.a * 256 + r * 128);
            if (rows_here > 0) {
              n_tiles += 1;
              n_units += (unsigned long long)min(4, (rows_here + 31) / 32) * (unsigned long long)((ncols + 31) / 32);
            }
          }
        }
        __syncwarp();
      } else {
        // B: rows = vocabulary (dC), C: rows = tokens (dE); this warp's half
        // of the chunk's d columns
        const bool isB = t.type == TASK_B;
        const int row0 = isB ? t.a * BN + r * 128 + lg * 32 : a.tok0 + t.a * 256 + r * 128 + lg * 32;
        const int rows_lim = isB ? a.V : a.N;
        const CUtensorMap* map = isB ? &mp.dC : &mp.dE;
        const bool add = isB ? (a.dC_add != 0) : true;
        const int nd = chunk_width(a.D, t.b);
        unsigned* tile_ctr = isB ? nullptr : a.doneC + (size_t)t.a * P.n_dc + t.b;
        if (!isB && a.ordered && t.s > 0) {
          // Ordered mode: this dE tile's reduce-adds follow those of the
          // previous stripe, so every entry is summed in stripe order and the
          // result does not depend on timing (bitwise reproducible).
          int ok = 1;
          if (lane == 0) {
            const unsigned want = SP_DONE * (unsigned)t.s;
            if (ld_acquire_gpu(tile_ctr) < want) {
              const uint64_t t0 = global_timer_ns();
              ok = 0;
              while (true) {
                __nanosleep(128);
                if (ld_acquire_gpu(tile_ctr) >= want) {
                  ok = 1;
                  break;
                }
                if (*abort_flag) break;
                if (global_timer_ns() - t0 > a.wait_limit_ns) {
                  *abort_flag = 1;
                  break;
                }
              }
            }
            fence_proxy_async_global();
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          __syncwarp();
          if (!ok) break;
        }
        // no live K block: the accumulator was not written; the tile is zero
        // (stored as zeros by a dC task that writes, skipped by one that adds)
        const bool empty_task = tmask == 0ull;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          const int c = hsel * 4 + cc;
          if (c * 32 >= nd) break;  // a 128-wide chunk fills only the first half
          if (empty_task && add) break;
          float v[32];
          if (empty_task) {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = 0.f;
          } else {
            tmem_ld32(tacc + (uint32_t)(c * 32), v);
          }
          const int x0 = t.b * 256 + c * 32;
          if (row0 < rows_lim && x0 < a.D) {
            // Two staging buffers in turn: the block staged here two pieces ago
            // has been read once at most one group is still reading.  (Pieces
            // are skipped only from some c on, so the turn never breaks.)
            uint8_t* xb = stg + (cc & 1) * 4096;
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
            stage_f32_block(xb, lane, v);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (add)
                tma_reduce_add_2d(map, xb, x0, row0);
              else
                tma_store_2d(map, xb, x0, row0);
              bulk_commit_group();
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        if (lane == 0) {
          bulk_wait_group0();
          fence_proxy_async_global();
          red_release_gpu_add(a.doneBC + t.s, 1u);
          if (tile_ctr) red_release_gpu_add(tile_ctr, 1u);
        }
        __syncwarp();
      }
      if (trace && k < a.trace_cap) trace[k * 4 + 2] = global_timer_ns();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_group0();
    if (lg == 0 && hsel == 0 && lane == 0) {
      atomicAdd(a.status + ST_TILES, n_tiles);
      // without the filter every recomputed unit counts as live; with it, the
      // units holding a kept entry are live and the others dead
      if (!a.nz) atomicAdd(a.status + ST_LIVE_TILES, n_units);
    }
    if (a.nz && lane == 0) {
      // (counted by every epilogue warp: in-range units of its rows and columns)
      atomicAdd(a.status + ST_LIVE_TILES, n_live);
      atomicAdd(a.status + ST_DEAD_TILES, n_inrange - n_live);
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
}

size_t bwd_stripe_smem_bytes() {
  return 1024 + (size_t)SP_STAGES * SP_STAGE_BYTES + (size_t)SP_EPI_WARPS * SP_STAGING_PER_WARP + 512;
}

// maps: the nine tensor maps in the order of StripeMaps; grid: an even number of CTAs.
cudaError_t launch_bwd_stripe(const CUtensorMap* maps, const StripeArgs& a, void* G, int grid, cudaStream_t stream) {
  StripeMaps mp;
  mp.eA = maps[0];
  mp.cA = maps[1];
  mp.gSt = maps[2];
  mp.gK = maps[3];
  mp.gM = maps[4];
  mp.eM = maps[5];
  mp.cM = maps[6];
  mp.dE = maps[7];
  mp.dC = maps[8];
  const size_t smem = bwd_stripe_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(bwd_stripe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  bwd_stripe_kernel<<<grid, SP_THREADS, smem, stream>>>(mp, a, reinterpret_cast<__nv_bfloat16*>(G));
  return cudaGetLastError();
}

}  // namespace cce
