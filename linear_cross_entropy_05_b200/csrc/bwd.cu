// CCE backward: recompute logit tiles on chip, form the softmax gradient,
// skip negligible tiles, contract the rest into dE and dC.
//
// Cut Cross-Entropy abstract, sentences 4 and 9: the logits are never stored,
// so the backward pass recomputes each 128 x 256 logit tile S = E_m C_v^T in
// TMEM and forms P = exp(S - lse) and D = P - onehot(y) in registers.  The
// filter drops every entry with |D| below filter_eps (gradient elements too
// small to matter at the working precision) by writing it to the shared
// memory tile of G = dloss * D as zero.  The skipping of work is coarser:
// 32 x 32 units (one epilogue warp's 32 rows x one 32-column chunk, 32 per
// logit tile) left with no entry are "dead", and
// the tensor cores contract only whole blocks that hold a live unit:
//     dE[m-block, d-chunk] += sum over live 64-column quarters q of G_q . C_q[d-chunk]   (M=128, N=64, K=64 each)
//     dC[v-half h, d-chunk] += G_h^T . E[m-block, d-chunk]  for halves with a live unit  (M=128, N=64, K=128)
// and only the 32-row pieces of dE and dC that a live unit touches are added
// to global memory (the others are exactly zero).
// The C and E slices are the same TMA tiles the recompute streams (128-byte
// swizzled rows of 64 d values); read K-major for S and MN-major for the
// contractions.  Partial products are added to fp32 dE/dC by the TMA engine
// (bulk tensor reduce-add from a swizzled shared staging tile).
//
// Roles (192 threads): warp 0 TMA producer, warp 1 UMMA issuer, warps 2-5
// epilogue (one TMEM lane = one token row / one vocabulary row per thread).
// TMEM columns: [0,256) logit tile; [256,512) two contraction buffers of a
// dE chunk and one half's dC chunk each.  Because the two never overlap, the
// next tile's logits are recomputed while this tile's products drain: once a
// tile's gradient tile is published, the operand stream interleaves its
// contraction slices with the next tile's recompute slices.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace cce {

namespace {
constexpr uint32_t TM_S = 0;
// Contraction accumulators, double-buffered beside the logit tile: buffer b =
// TMEM columns [256 + 128 b, 384 + 128 b): a dE chunk (64 columns) then one
// half's dC chunk (64 columns).
__device__ __forceinline__ uint32_t tm_de(int b) { return 256u + 128u * (uint32_t)b; }
__device__ __forceinline__ uint32_t tm_dc(int b) { return 320u + 128u * (uint32_t)b; }

// Live mask of a logit tile: bit 8 * g + c is the 32 x 32 filter unit of
// token rows [32g, 32g + 32) and columns [32c, 32c + 32).
__device__ __forceinline__ bool quarter_live(uint32_t u, int q) { return (u & (0x03030303u << (2 * q))) != 0; }
__device__ __forceinline__ bool half_live(uint32_t u, int h) { return (u & (0x0F0F0F0Fu << (4 * h))) != 0; }
__device__ __forceinline__ bool chunk_live(uint32_t u, int c) { return (u & (0x01010101u << c)) != 0; }
__device__ __forceinline__ bool rows_live(uint32_t u, int g) { return ((u >> (8 * g)) & 0xFFu) != 0; }

__device__ __forceinline__ void tile_coords(int t, int n_mblk, int n_vtile, int group_m, int& m, int& vt) {
  // Raster: groups of group_m token blocks; inside a group the token block
  // varies fastest so concurrent CTAs share the same C tile in L2 while the
  // group's E rows stay resident.
  const int gsize = group_m * n_vtile;
  const int g = t / gsize;
  const int rem = t - g * gsize;
  const int gm = min(group_m, n_mblk - g * group_m);
  vt = rem / gm;
  m = g * group_m + (rem - vt * gm);
}

// Adds a 32 x 32 fp32 block held one row per lane (32 consecutive columns
// each) to global memory through the TMA engine: the block is written to one
// of the warp's NXB 4 KB staging buffers (used in rotation) in the
// 128-byte-swizzled layout of a {32, 32} fp32 box and reduced into the tensor
// at (x = column, y = row) by one bulk tensor reduce-add.  Rows/columns past
// the tensor's extent are clipped.
template <int NXB>
__device__ __forceinline__ void tma_red_block32(uint8_t* xb, int lane, const float (&v)[32], const CUtensorMap* map,
                                                int x, int y, uint64_t policy = 0) {
  // the block issued NXB pieces ago (which used this buffer) has left it
  if (lane == 0) bulk_wait_group_read<NXB - 1>();
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(xb + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if (policy)
      tma_reduce_add_2d_hint(map, xb, x, y, policy);
    else
      tma_reduce_add_2d(map, xb, x, y);
    bulk_commit_group();
  }
}

// The same 32 x 32 fp32 block added with vector atomics on the load/store
// path instead of the TMA engine: staged in the same swizzled layout, then
// each warp instruction `red.global.add.v4.f32` covers four rows x 128
// contiguous bytes.  nrows / ncols clip the block at the tensor's edge
// (ncols is a multiple of 8).
__device__ __forceinline__ void lsu_red_block32(uint8_t* xb, int lane, const float (&v)[32], float* base, size_t ld,
                                                int nrows, int ncols) {
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(xb + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const int c4 = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = i * 4 + (lane >> 3);
    const float4 x = *reinterpret_cast<const float4*>(xb + r * 128 + ((c4 ^ (r & 7)) << 4));
    if (r < nrows && c4 * 4 < ncols) red_add_v4(base + (size_t)r * ld + c4 * 4, x.x, x.y, x.z, x.w);
  }
  __syncwarp();
}

// Work item t -> (token block m, vocabulary tile vt).  Dense mode rasters the
// whole grid; list mode visits every tile of each token block that is not
// flat, vocabulary-major (the flat blocks are handled by the flat-row kernel).
struct TileMap {
  int T, nnf;
  __device__ __forceinline__ void init(const BwdArgs& a) {
    if (a.list_mode) {
      T = (int)a.hdr[HDR_T];
      nnf = (int)a.hdr[HDR_NNF];
    } else {
      T = a.n_tiles;
      nnf = 0;
    }
  }
  __device__ __forceinline__ void get(const BwdArgs& a, int t, int& m, int& vt) const {
    if (!a.list_mode) {
      tile_coords(t, a.n_mblk, a.n_vtile, a.group_m, m, vt);
    } else {
      vt = t / nnf;
      m = a.nonflat[t - vt * nnf];
    }
  }
};

// Deterministic-mode counterpart of tma_red_block32: the 32 x 32 block is
// staged the same way, read back one row at a time (lane = column), each value
// rounded to fixed point round(x * scale) and added to the int64 accumulator
// with a 64-bit integer atomic (a warp covers 256 contiguous bytes per row).
// Integer addition is associative, so the totals do not depend on the order
// in which CTAs deliver their tiles.
__device__ __forceinline__ void fixed_red_block32(uint8_t* xb, int lane, const float (&v)[32],
                                                  unsigned long long* base, size_t ld, uint32_t row_ok, int ncols,
                                                  float scale) {
  if (lane == 0) bulk_wait_group_read0();  // a bulk copy may still be reading the buffer
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(xb + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const bool col_ok = lane < ncols;
#pragma unroll 4
  for (int r = 0; r < 32; ++r) {
    const float x = *reinterpret_cast<const float*>(xb + r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + (lane & 3) * 4);
    if (((row_ok >> r) & 1u) && col_ok)
      atomicAdd(base + (size_t)r * ld + lane, (unsigned long long)__float2ll_rn(x * scale));
  }
  __syncwarp();
}

// Deterministic mode through the TMA engine: the 32 x 32 block, each value
// rounded once to 64-bit fixed point round(x * scale), is added to the int64
// accumulator by two bulk tensor reduce-adds (the map's element type is u64
// and its box {16, 32}: 128-byte rows, 128-byte swizzle), the halves staged
// in turn in the warp's 4 KB buffer.  Integer addition is associative, so
// the totals do not depend on the order in which the operations land.
// Columns from ncols on lie past the tensor and are not sent.
__device__ __forceinline__ void tma_fixed_block32(uint8_t* xb, int lane, const float (&v)[32], const CUtensorMap* map,
                                                  int x, int y, int ncols, float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (16 * h >= ncols) break;
    if (lane == 0) bulk_wait_group_read0();  // the buffer's previous contents have been read
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const long long a0 = __float2ll_rn(v[16 * h + 2 * q] * scale);
      const long long a1 = __float2ll_rn(v[16 * h + 2 * q + 1] * scale);
      *reinterpret_cast<longlong2*>(xb + lane * 128 + ((q ^ (lane & 7)) << 4)) = make_longlong2(a0, a1);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_reduce_add_2d(map, xb, x + 16 * h, y);
      bulk_commit_group();
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
}  // namespace

// NST: operand pipeline stages; NXB: reduction staging buffers per epilogue
// warp; RED: 0 = fp32 reductions by the TMA engine (bulk tensor reduce-add),
// 1 = by vector atomics on the load/store path; EPG: epilogue warps per TMEM lane group (1 or 2; with 2, the two
// warps of a lane group split the softmax-gradient columns by 128-column half
// and deal the reduction pieces of each chunk between them).
template <int NST, int NXB, int EPG, int RED>
__global__ void __launch_bounds__(64 + 128 * EPG, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC,
               const __grid_constant__ CUtensorMap tmCq,
               const __grid_constant__ CUtensorMap tmdE, const __grid_constant__ CUtensorMap tmdC, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                   // NST x [128][64] bf16 (E slices)
  uint8_t* sB = smem + NST * A_STAGE_BYTES;      // NST x [256][64] bf16 (C slices)
  uint8_t* sG = sB + NST * B_STAGE_BYTES;        // 4 x [128][64] bf16, swizzled (G tile)
  uint8_t* sX = sG + G_BYTES;                           // 4*EPG x NXB x 4 KB reduction staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + 4 * EPG * NXB * 4096);
  constexpr int NEPI = 128 * EPG;                       // epilogue threads
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* s_full = bars + 2 * NST;
  uint64_t* s_empty = s_full + 1;
  uint64_t* g_full = s_full + 2;
  uint64_t* g_empty = s_full + 3;
  uint64_t* c_full = s_full + 4;   // [2] per accumulator buffer
  uint64_t* c_empty = s_full + 6;  // [2]
  uint64_t* drain = s_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  // Per-tile live votes, a ring of 8 slots indexed by the CTA's tile counter.
  // Slot kt%8 is written by the epilogue before g_full(kt) completes and read by
  // every role after it; the epilogue clears slot (kt+4)%8 at tile kt, long
  // after its last reader (tile kt-4) and before its next writer (tile kt+4).
  volatile int* live_ring = reinterpret_cast<volatile int*>(tmem_slot + 2);
  // Work items are handed out at run time (a global counter), so CTAs that
  // draw cheap tiles take more of them.  The producer draws the CTA's kt-th
  // item, writes it to tile_ring[kt%8] (-1: no more work) and arrives on
  // tile_full[kt%2]; the MMA and epilogue roles wait on that barrier (phase
  // kt/2) before reading the slot.  The producer cannot run two tiles ahead
  // of either role (it needs tile kt's live mask before tile kt+1), so
  // neither barrier can complete twice between a role's waits.
  volatile int* tile_ring = live_ring + 8;
  uint64_t* tile_full = reinterpret_cast<uint64_t*>(tmem_slot + 20);  // [2], 8-byte aligned

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, NEPI);
    mbar_init(g_full, NEPI);
    mbar_init(g_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c_full[b], 1);
      mbar_init(&c_empty[b], NEPI);
    }
    mbar_init(drain, 1);
    mbar_init(&tile_full[0], 1);
    mbar_init(&tile_full[1], 1);
    *abort_flag = 0;
    for (int i = 0; i < 8; ++i) live_ring[i] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_map(&tmE);
    tma_prefetch_map(&tmC);
    tma_prefetch_map(&tmCq);
    tma_prefetch_map(&tmdE);
    tma_prefetch_map(&tmdC);
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
      uint32_t phase = 0, gph = 0, armed = 0;
      TileMap tm;
      tm.init(a);
      // withhold_loads (test hook): tiles are handed out but no copy is
      // issued, so the other roles wait on data that never comes.
      //
      // Stage order (the MMA warp consumes the ring in the same order): the
      // first tile's recompute slices (d ascending); then, per tile kt, once
      // its live mask is known, its contraction slices (d descending, so the
      // slices fetched last, most likely still in L2, come first: the E
      // slice and only the live 64-row quarters of the C slice, the only C
      // rows its dE products read) interleaved one to one with the next
      // tile's recompute slices, so that the next logits are computed while
      // this tile's partial products drain.
      auto draw = [&](int k) -> int {
        const unsigned long long drawn = atomicAdd(a.status + ST_NEXT_TILE, 1ull);
        const int t = drawn < (unsigned long long)tm.T ? (int)drawn : -1;
        tile_ring[k & 7] = t;
        mbar_arrive(&tile_full[k & 1]);
        return t;
      };
      auto advance = [&]() {
        if (++stage == NST) {
          stage = 0;
          phase ^= 1u;
        }
      };
      // With a.l2_hints the C slices (streamed, shared only by the CTAs on the
      // same vocabulary tile at about the same time) leave L2 first, so the
      // dE rows the reductions keep returning to stay there.
      const uint64_t pol_c = a.l2_hints ? l2_policy_evict_first() : 0ull;
      auto load_c = [&](void* dst, const CUtensorMap* map, int x, int y) {
        if (pol_c)
          tma_load_2d_hint(dst, map, &full[stage], x, y, pol_c);
        else
          tma_load_2d(dst, map, &full[stage], x, y);
      };
      auto load_s = [&](int m, int vt, int kb) {  // one recompute slice (stage already free)
        if (a.withhold_loads) return;
        mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
        tma_load_2d(sA + stage * A_STAGE_BYTES, &tmE, &full[stage], kb * BK, m * BM);
        load_c(sB + stage * B_STAGE_BYTES, &tmC, kb * BK, vt * BN);
        armed |= 1u << stage;
        if (a.pf && kb + a.pf < nkb) {  // L2 prefetch of the slices a.pf ahead
          tma_prefetch_l2_2d(&tmE, (kb + a.pf) * BK, m * BM);
          tma_prefetch_l2_2d(&tmC, (kb + a.pf) * BK, vt * BN);
        }
      };
      int t = draw(0);
      int m = 0, vt = 0;
      if (t >= 0) {
        tm.get(a, t, m, vt);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
          load_s(m, vt, kb);
          advance();
        }
      }
      for (int kt = 0; t >= 0; ++kt) {
        if (!mbar_wait(g_full, gph, wc)) goto producer_done;
        gph ^= 1u;
        const uint32_t umask = (uint32_t)live_ring[kt & 7];
        const int tn = draw(kt + 1);
        int mn = 0, vtn = 0;
        if (tn >= 0) tm.get(a, tn, mn, vtn);
        uint32_t qmask = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) qmask |= (quarter_live(umask, q) ? 1u : 0u) << q;
        const uint32_t c_bytes = A_STAGE_BYTES + (uint32_t)__popc(qmask) * QUARTER_BYTES;  // one d slice
        // A tile with a single live quarter needs 24 KB per d slice: two
        // slices share one stage (E of the second slice at B + 8 KB, the
        // quarters at B + 0 and B + 24 KB), halving its contraction stages.
        const int cpack = __popc(qmask) == 1 ? 2 : 1;
        const int q1 = __ffs(qmask) - 1;
        const int n_cst = umask ? (nkb + cpack - 1) / cpack : 0;
        const int n_sst = tn >= 0 ? nkb : 0;
        // L2 prefetch of the fp32 dE / dC rows this tile's reductions add
        // into (the live 32-row pieces of d slice kb), a.red_pf slices ahead
        // of the slice being loaded, so the reduce-adds find their lines in
        // L2 instead of filling them from DRAM one by one.
        auto pf_red = [&](int kb) {
          if (kb < 0 || kb >= nkb) return;
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            const int x = kb * BK + q * 32;
            if (x >= a.D) break;
#pragma unroll 1
            for (int g = 0; g < 4; ++g)
              if (rows_live(umask, g) && m * BM + 32 * g < a.N) tma_prefetch_l2_2d(&tmdE, x, m * BM + 32 * g);
#pragma unroll 1
            for (int c = 0; c < 8; ++c)
              if (chunk_live(umask, c) && vt * BN + 32 * c < a.V) tma_prefetch_l2_2d(&tmdC, x, vt * BN + 32 * c);
          }
        };
        const bool red_pf = a.red_pf > 0 && umask != 0u && a.accE == nullptr && RED == 0;
        if (red_pf)
          for (int i = 0; i < a.red_pf; ++i) pf_red(nkb - 1 - i);
        for (int j = 0; j < max(n_cst, n_sst); ++j) {
          if (j < n_cst) {
            const int kb0 = nkb - 1 - cpack * j;
            const int ns = (cpack == 2 && kb0 >= 1) ? 2 : 1;  // d slices in this stage
            if (red_pf)
              for (int sl = 0; sl < ns; ++sl) pf_red(kb0 - sl - a.red_pf);
            if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
            mbar_arrive_expect_tx(&full[stage], (uint32_t)ns * c_bytes);
            uint8_t* b_st = sB + stage * B_STAGE_BYTES;
            tma_load_2d(sA + stage * A_STAGE_BYTES, &tmE, &full[stage], kb0 * BK, m * BM);
            if (cpack == 2) {
              load_c(b_st, &tmCq, kb0 * BK, vt * BN + q1 * 64);
              if (ns == 2) {
                tma_load_2d(b_st + QUARTER_BYTES, &tmE, &full[stage], (kb0 - 1) * BK, m * BM);
                load_c(b_st + QUARTER_BYTES + A_STAGE_BYTES, &tmCq, (kb0 - 1) * BK, vt * BN + q1 * 64);
              }
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if ((qmask >> q) & 1) load_c(b_st + q * QUARTER_BYTES, &tmCq, kb0 * BK, vt * BN + q * 64);
            }
            armed |= 1u << stage;
            for (int sl = 0; a.pf && sl < ns; ++sl) {  // L2 prefetch of the contraction slices a.pf further on
              const int kp = kb0 - sl - a.pf * cpack;         // (d descending)
              if (kp < 0) break;
              tma_prefetch_l2_2d(&tmE, kp * BK, m * BM);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if ((qmask >> q) & 1) tma_prefetch_l2_2d(&tmCq, kp * BK, vt * BN + q * 64);
            }
            advance();
          }
          if (j < n_sst) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, wc)) goto producer_done;
            load_s(mn, vtn, j);
            advance();
          }
        }
        t = tn;
        m = mn;
        vt = vtn;
      }
    producer_done : {
      int dummy = 0;
      WaitCtl exit_wc{&dummy, a.wait_limit_ns};
      for (int s = 0; s < NST; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (s < stage) ? phase : (phase ^ 1u), exit_wc);
    }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer ----------------
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_DE = idesc_bf16_f32(BM, 64, false, true);
      constexpr uint32_t IDESC_DC = idesc_bf16_f32(BM, 64, true, true);
      const uint32_t g_addr = smem_u32(sG);
      int stage = 0;
      uint32_t phase = 0, sph = 0, gph = 0;
      uint32_t cfill0 = 0u, cfill1 = 0u;  // fills of contraction buffers 0 / 1 so far
      int fb = 0;                         // contraction buffer of the next fill
      auto advance = [&]() {
        if (++stage == NST) {
          stage = 0;
          phase ^= 1u;
        }
      };
      // one k-block of the logit tile S = E_m C_vt^T into TMEM columns [0, 256)
      auto s_block = [&](int kb) {
        const uint32_t a_addr = smem_u32(sA + stage * A_STAGE_BYTES);
        const uint32_t b_addr = smem_u32(sB + stage * B_STAGE_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          umma_bf16(tmem_base + TM_S, sdesc_sw128(a_addr + k * 32, 16, 1024),
                    sdesc_sw128(b_addr + k * 32, 16, 1024), IDESC_S, (kb | k) != 0);
        umma_commit(&empty[stage]);
      };
      int t = -1;
      if (!mbar_wait(&tile_full[0], 0u, wc)) goto mma_done;
      t = tile_ring[0];
      if (t >= 0) {
        if (!mbar_wait(s_empty, sph ^ 1u, wc)) goto mma_done;
        sph ^= 1u;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, wc)) goto mma_done;
          tc_fence_after();
          s_block(kb);
          advance();
        }
        umma_commit(s_full);
      }
      for (int kt = 0; t >= 0; ++kt) {
        if (!mbar_wait(g_full, gph, wc)) goto mma_done;
        gph ^= 1u;
        tc_fence_after();
        const uint32_t umask = (uint32_t)live_ring[kt & 7];  // live 32 x 32 units of the tile
        if (!mbar_wait(&tile_full[(kt + 1) & 1], (uint32_t)((kt + 1) >> 1) & 1u, wc)) goto mma_done;
        const int tn = tile_ring[(kt + 1) & 7];
        if (tn >= 0) {
          // the epilogue has read this tile's logits: the next tile may overwrite them
          if (!mbar_wait(s_empty, sph ^ 1u, wc)) goto mma_done;
          sph ^= 1u;
          tc_fence_after();
        }
        // Contraction fills per 64-wide d slice: the first holds the dE chunk
        // (every live quarter) and the dC chunk of the first live half, the
        // second (only when both halves are live) the dC chunk of half 1.
        const int h_first = half_live(umask, 0) ? 0 : 1;
        const bool both = half_live(umask, 0) && half_live(umask, 1);
        uint32_t qmask = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) qmask |= (quarter_live(umask, q) ? 1u : 0u) << q;
        // stage packing as in the producer: one live quarter -> two d slices per stage
        const int cpack = __popc(qmask) == 1 ? 2 : 1;
        const int n_cst = umask ? (nkb + cpack - 1) / cpack : 0;
        const int n_sst = tn >= 0 ? nkb : 0;
        for (int j = 0; j < max(n_cst, n_sst); ++j) {
          if (j < n_cst) {
            const int kb0 = nkb - 1 - cpack * j;
            const int ns = (cpack == 2 && kb0 >= 1) ? 2 : 1;
            if (!mbar_wait(&full[stage], phase, wc)) goto mma_done;
            const uint32_t a_st = smem_u32(sA + stage * A_STAGE_BYTES);
            const uint32_t b_st = smem_u32(sB + stage * B_STAGE_BYTES);
            for (int sl = 0; sl < ns; ++sl) {
              // E[m-block, d slice]: 128 tok x 64 d; C rows of the live quarters
              const uint32_t e_addr = sl == 0 ? a_st : b_st + QUARTER_BYTES;
              const uint32_t c_base = sl == 0 ? b_st : b_st + QUARTER_BYTES + A_STAGE_BYTES;
              for (int f = 0; f < (both ? 2 : 1); ++f) {
                const int b = fb;
                fb ^= 1;
                if (!mbar_wait(&c_empty[b], ((b ? cfill1 : cfill0) & 1u) ^ 1u, wc)) goto mma_done;
                if (b) ++cfill1; else ++cfill0;
                tc_fence_after();
                if (f == 0) {
                  uint32_t acc_de = 0;
#pragma unroll
                  for (int q = 0; q < 4; ++q) {
                    if (!quarter_live(umask, q)) continue;
                    // C rows of quarter q: packed stages hold the single live quarter at c_base
                    const uint32_t cq = cpack == 2 ? c_base : c_base + q * QUARTER_BYTES;
                    // dE chunk += G_q (128 tok x 64 voc, K-major) . C_q chunk (K = voc rows, MN = d)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                      umma_bf16(tmem_base + tm_de(b),
                                sdesc_sw128(g_addr + q * (BM * 128) + k * 32, 16, 1024),
                                sdesc_sw128(cq + k * 2048, 16384, 1024), IDESC_DE, acc_de);
                      acc_de = 1;
                    }
                  }
                }
                const int h = f == 0 ? h_first : 1;
                // dC chunk of half h = G_h^T (MN = voc, K = tok) . Echunk (K = tok rows, MN = d)
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)
                  umma_bf16(tmem_base + tm_dc(b),
                            sdesc_sw128(g_addr + (2 * h) * (BM * 128) + k * 2048, BM * 128, 1024),
                            sdesc_sw128(e_addr + k * 2048, 16384, 1024), IDESC_DC, k != 0);
                umma_commit(&c_full[b]);
              }
            }
            umma_commit(&empty[stage]);
            advance();
          }
          if (j < n_sst) {
            if (!mbar_wait(&full[stage], phase, wc)) goto mma_done;
            tc_fence_after();
            s_block(j);
            advance();
          }
        }
        umma_commit(g_empty);  // this tile's gradient tile may be overwritten once these products are done
        if (tn >= 0) umma_commit(s_full);
        t = tn;
      }
    mma_done:
      umma_commit(drain);
      {
        int dummy = 0;
        WaitCtl exit_wc{&dummy, a.wait_limit_ns};
        mbar_wait(drain, 0, exit_wc);
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int lane_grp = warp & 3;
    const int ew = warp - 2;               // epilogue warp 0 .. 4*EPG-1
    const int hsel = ew >> 2;              // with EPG = 2: the 128-column half this warp forms G for
    const int rib = lane_grp * 32 + lane;  // row inside the tile (token, or vocab for dC)
    const uint32_t lane_addr = (uint32_t)(lane_grp * 32) << 16;
    const float eps = a.filter_eps;
    const bool filter_on = eps > 0.f;
    uint32_t sph = 0, gph = 0;
    uint32_t cfe0 = 0u, cfe1 = 0u;  // drains of contraction buffers 0 / 1 so far
    int fb = 0;                     // contraction buffer of the next fill
    unsigned long long n_live = 0, n_dead = 0, n_tiles = 0;
    uint8_t* g_row = sG + rib * 128;
    uint8_t* const xb0 = sX + ew * NXB * 4096;
    int xbi = 0;  // next staging buffer of this warp (rotation over NXB)
    auto next_xb = [&]() -> uint8_t* {
      uint8_t* p = xb0 + xbi * 4096;
      xbi = (xbi + 1 == NXB) ? 0 : xbi + 1;
      return p;
    };
    const bool fixed = a.accE != nullptr;
    const uint64_t pol_de = a.l2_hints ? l2_policy_evict_last() : 0ull;
    float fx_scale = 0.f;
    if (fixed)
      fx_scale = ldexpf(1.f, fixed_point_exponent(__uint_as_float(a.hdr[HDR_CMAX]), __uint_as_float(a.hdr[HDR_EMAX]),
                                                  __uint_as_float(a.hdr[HDR_DLMAX]), a.N));
    const int sw = rib & 7;
    int kt = 0;
    TileMap tm;
    tm.init(a);
    const bool tracer = a.trace != nullptr && ew == 0 && lane == 0;
    unsigned long long* trace_cta = a.trace ? a.trace + (size_t)blockIdx.x * a.trace_cap * 4 : nullptr;
    for (;; ++kt) {
      if (tracer && kt < a.trace_cap) trace_cta[kt * 4 + 0] = global_timer_ns();
      if (!mbar_wait(&tile_full[kt & 1], (uint32_t)(kt >> 1) & 1u, wc)) break;
      const int t = tile_ring[kt & 7];
      if (t < 0) break;
      int m, vt;
      tm.get(a, t, m, vt);
      const int row = m * BM + rib;
      bool valid = row < a.N;
      long long yl = valid ? a.y[row] : a.ignore_index;
      if (yl == a.ignore_index) valid = false;
      if (a.shard_mode) {
        // vocabulary shard: labels are global ids; a label outside the shard
        // contributes no one-hot entry here but the token's softmax row does
        yl -= a.v_offset;
      } else if (valid && (yl < 0 || yl >= a.V)) {
        valid = false;
        atomicOr(a.status + ST_FLAGS, SF_BAD_LABEL);
      }
      const float lse2 = valid ? a.lse[row] * LOG2E : 0.f;
      const float dl = valid ? a.dloss[row] : 0.f;
      const long long yrel = yl - (long long)vt * BN;
      const int ycol = (valid && yrel >= 0 && yrel < BN) ? (int)yrel : -1;
      const int ncols = min(BN, a.V - vt * BN);

      if (!mbar_wait(s_full, sph, wc)) break;
      sph ^= 1u;
      if (tracer && kt < a.trace_cap) trace_cta[kt * 4 + 1] = global_timer_ns();
      if (!mbar_wait(g_empty, gph ^ 1u, wc)) break;
      tc_fence_after();
      // This warp's units: its 32 rows (if any of them is a token) x each
      // 32-column chunk inside V.  A unit is live if some |D| >= eps in it
      // (every existing unit when the filter is off).
      const int n_groups = min(4, (a.N - m * BM + 31) >> 5);  // token row groups of this block
      const int n_chunks = (ncols + 31) >> 5;
      const uint32_t my_chunks = lane_grp < n_groups ? (1u << n_chunks) - 1u : 0u;
      uint32_t live = 0;
      constexpr int NC = (BN / 32) / EPG;  // 32-column chunks of S handled by this warp
#pragma unroll 1
      for (int c = hsel * NC; c < hsel * NC + NC; ++c) {
        float x[32];
        tmem_ld32(tmem_base + lane_addr + TM_S + c * 32, x);
        uint32_t pk[16];
        bool big = false;  // some |D| >= eps in this lane's 32 entries
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float g2[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int col = c * 32 + j + q;
            float p = ex2_approx(fmaf(x[j + q], LOG2E, -lse2));
            float d = (col == ycol) ? p - 1.f : p;
            d = (valid && col < ncols) ? d : 0.f;
            // entries below the threshold are dropped one by one (with the
            // filter off eps <= 0 keeps every entry)
            const bool keep = fabsf(d) >= eps;
            big |= keep;
            g2[q] = keep ? dl * d : 0.f;
          }
          pk[j >> 1] = pack_bf16x2(g2[0], g2[1]);
        }
        const bool unit_live = filter_on ? __any_sync(0xffffffffu, big) : ((my_chunks >> c) & 1u) != 0;
        if (!unit_live) {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;  // a dropped unit contributes nothing
        }
        live |= (unit_live ? 1u : 0u) << (8 * lane_grp + c);
        // 32 columns = 64 bytes = four 16-byte chunks of the 128-byte row of
        // K block (c / 2); 128B swizzle: chunk index ^= row % 8.
        uint8_t* blk = g_row + (c >> 1) * (BM * 128);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c & 1) * 4 + q) ^ sw;
          *reinterpret_cast<uint4*>(blk + chunk * 16) = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(s_empty);
      fence_proxy_async_smem();
      if (live && lane == 0) atomicOr(const_cast<int*>(&live_ring[kt & 7]), (int)live);
      __syncwarp();
      if (rib == 0) live_ring[(kt + 4) & 7] = 0;
      mbar_arrive(g_full);
      if (!mbar_wait(g_full, gph, wc)) break;
      gph ^= 1u;
      const uint32_t umask = (uint32_t)live_ring[kt & 7];
      if (tracer && kt < a.trace_cap) {
        trace_cta[kt * 4 + 2] = global_timer_ns();
        trace_cta[kt * 4 + 3] = umask;
      }
      n_live += __popc(umask);
      n_dead += (unsigned)(n_groups * n_chunks) - __popc(umask);
      ++n_tiles;
      if (!umask) continue;
      const bool de_rows_live = rows_live(umask, lane_grp);  // this warp's 32 token rows
      bool ok = true;
      const int row0 = m * BM + lane_grp * 32;           // first dE row of this warp
      const uint32_t rows_valid = __ballot_sync(0xffffffffu, valid);  // kept tokens among those rows
      // the fills of each d slice, in the MMA warp's order (see there)
      const int h_first = half_live(umask, 0) ? 0 : 1;
      const bool both = half_live(umask, 0) && half_live(umask, 1);
      for (int j = 0; j < nkb && ok; ++j) {
        const int d0 = (nkb - 1 - j) * BK;  // the contraction pass runs d descending
        // Reduction pieces of this slice (32 rows of this lane group x 32
        // columns each): dE q0, dE q1 and dC q0, q1 of the first live half,
        // then dC q0, q1 of half 1 if both are live.  With EPG = 2 the
        // pieces alternate between the two warps of the lane group.
        int piece = 0;
        for (int f = 0; f < (both ? 2 : 1); ++f) {
          const int b = fb;
          fb ^= 1;
          if (!mbar_wait(&c_full[b], (b ? cfe1 : cfe0) & 1u, wc)) {
            ok = false;
            break;
          }
          if (b) ++cfe1; else ++cfe0;
          tc_fence_after();
          if (f == 0) {
#pragma unroll 1
            for (int q = 0; q < 2; ++q, ++piece) {
              const bool mine = (piece % EPG) == hsel && de_rows_live;
              float v[32];
              if (mine) tmem_ld32(tmem_base + lane_addr + tm_de(b) + q * 32, v);
              if (mine && d0 + q * 32 < a.D && row0 < a.N) {
                if (fixed && RED == 0)
                  tma_fixed_block32(next_xb(), lane, v, &tmdE, d0 + q * 32, row0, min(32, a.D - (d0 + q * 32)),
                                    fx_scale);
                else if (fixed)
                  fixed_red_block32(next_xb(), lane, v, a.accE + (size_t)row0 * a.D + d0 + q * 32, (size_t)a.D,
                                    rows_valid, min(32, a.D - (d0 + q * 32)), fx_scale);
                else if (RED == 1)
                  lsu_red_block32(next_xb(), lane, v, a.dE + (size_t)row0 * a.D + d0 + q * 32, (size_t)a.D,
                                  min(32, a.N - row0), min(32, a.D - (d0 + q * 32)));
                else
                  tma_red_block32<NXB>(next_xb(), lane, v, &tmdE, d0 + q * 32, row0, pol_de);
              }
            }
          }
          const int h = f == 0 ? h_first : 1;
          const int vr0 = vt * BN + h * BM + lane_grp * 32;
          // this warp's 32 vocabulary rows are column chunk 4h + lane_grp
          const bool dc_rows_live = chunk_live(umask, 4 * h + lane_grp);
#pragma unroll 1
          for (int q = 0; q < 2; ++q, ++piece) {
            const bool mine = (piece % EPG) == hsel && dc_rows_live;
            float v[32];
            if (mine) tmem_ld32(tmem_base + lane_addr + tm_dc(b) + q * 32, v);
            if (mine && d0 + q * 32 < a.D && vr0 < a.V) {
              if (fixed && RED == 0)
                tma_fixed_block32(next_xb(), lane, v, &tmdC, d0 + q * 32, vr0, min(32, a.D - (d0 + q * 32)),
                                  fx_scale);
              else if (fixed)
                fixed_red_block32(next_xb(), lane, v, a.accC + (size_t)vr0 * a.D + d0 + q * 32, (size_t)a.D,
                                  __ballot_sync(0xffffffffu, vr0 + lane < a.V), min(32, a.D - (d0 + q * 32)),
                                  fx_scale);
              else if (RED == 1)
                lsu_red_block32(next_xb(), lane, v, a.dC + (size_t)vr0 * a.D + d0 + q * 32, (size_t)a.D,
                                min(32, a.V - vr0), min(32, a.D - (d0 + q * 32)));
              else
                tma_red_block32<NXB>(next_xb(), lane, v, &tmdC, d0 + q * 32, vr0);
            }
          }
          tc_fence_before();
          mbar_arrive(&c_empty[b]);
        }
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_group0();  // every reduction issued by this warp has landed
    if (tracer && kt < a.trace_cap) trace_cta[kt * 4 + 0] = global_timer_ns();  // end of the last tile
    if (rib == 0 && hsel == 0) {
      atomicAdd(a.status + ST_LIVE_TILES, n_live);
      atomicAdd(a.status + ST_DEAD_TILES, n_dead);
      atomicAdd(a.status + ST_TILES, n_tiles);
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
}

template <int NST, int NXB, int EPG, int RED>
size_t bwd_smem_bytes() {
  return 1024 + (size_t)NST * STAGE_BYTES + G_BYTES + (size_t)4 * EPG * NXB * 4096 + 256;
}

template <int NST, int NXB, int EPG, int RED>
cudaError_t launch_bwd_t(const CUtensorMap& tmE, const CUtensorMap& tmC, const CUtensorMap& tmCq, const CUtensorMap& tmdE,
                         const CUtensorMap& tmdC, const BwdArgs& a, int grid, cudaStream_t stream) {
  const size_t smem = bwd_smem_bytes<NST, NXB, EPG, RED>();
  cudaError_t e =
      cudaFuncSetAttribute(bwd_kernel<NST, NXB, EPG, RED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  bwd_kernel<NST, NXB, EPG, RED><<<grid, 64 + 128 * EPG, smem, stream>>>(tmE, tmC, tmCq, tmdE, tmdC, a);
  return cudaGetLastError();
}

// variant 0: 3 operand stages, one staging buffer, 4 epilogue warps (default);
// variant 1: 2 stages, two staging buffers per warp (staging overlaps the bulk
//            read of the previous block);
// variant 2: 2 stages, 8 epilogue warps (two per TMEM lane group);
// variant 3: as 0 with the fp32 reductions on the load/store path.
cudaError_t launch_bwd(const CUtensorMap& tmE, const CUtensorMap& tmC, const CUtensorMap& tmCq, const CUtensorMap& tmdE,
                       const CUtensorMap& tmdC, const BwdArgs& a, int grid, int variant, cudaStream_t stream) {
  if (variant == 1) return launch_bwd_t<2, 2, 1, 0>(tmE, tmC, tmCq, tmdE, tmdC, a, grid, stream);
  if (variant == 2) return launch_bwd_t<2, 1, 2, 0>(tmE, tmC, tmCq, tmdE, tmdC, a, grid, stream);
  if (variant == 3) return launch_bwd_t<BWD_STAGES, 1, 1, 1>(tmE, tmC, tmCq, tmdE, tmdC, a, grid, stream);
  return launch_bwd_t<BWD_STAGES, 1, 1, 0>(tmE, tmC, tmCq, tmdE, tmdC, a, grid, stream);
}

}  // namespace cce
