// Definitions shared by the CCE kernels and the C-ABI front end.
#pragma once

#include <cstdint>

namespace cce {

// Tile geometry of the fused logit kernels.
//   BM token rows (one TMEM lane each) x BN vocabulary columns per tile,
//   BK = 64 bf16 along D per pipeline stage (one 128-byte swizzle row).
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int A_STAGE_BYTES = BM * BK * 2;  // E slice  [128 rows][64 d]
constexpr int B_STAGE_BYTES = BN * BK * 2;  // C slice  [256 rows][64 d]
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int QUARTER_BYTES = 64 * BK * 2;   // C slice [64 rows][64 d]: one K block of the dE product
constexpr int NUM_THREADS = 192;            // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int FWD_STAGES = 4;
constexpr int PAIR_STAGES = 6;                          // CTA-pair forward: E half + C half per stage (A/B)
constexpr int PAIR_STAGES_MAX = 7;                      // the default: the most that fit in 227 KB of shared memory
constexpr int PAIR_STAGE_BYTES = 2 * A_STAGE_BYTES;     // [128][64] bf16 of E and of C
constexpr int BWD_STAGES = 3;
constexpr int G_BYTES = BM * BN * 2;        // bf16 softmax-gradient tile (4 swizzled K blocks)

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// Status block at the head of every workspace (32 x u64, zeroed per call;
// cce_read_status reads words 0-7).
enum StatusWord : int {
  ST_FLAGS = 0,        // bit mask of StatusFlag
  ST_LIVE_TILES = 1,   // backward: 32x32 filter units whose contraction ran
  ST_DEAD_TILES = 2,   // backward: filter units recomputed and found negligible
  ST_TILES = 3,        // forward: 128x256 logit tiles computed; backward: logit tiles recomputed
  ST_PRUNED = 4,       // backward: filter units proven negligible without recomputing them
  ST_NEXT_TILE = 5,    // backward: next work item to hand out (CTAs take tiles as they free up)
  ST_FLAT = 6,         // backward: live units of flat blocks, formed without recomputing a tile
  ST_FWD_QUEUE = 8,    // forward, two-queue order: next unit of queue 0 (word 8) and queue 1 (word 9)
};
// Header words of the backward pre-pass (u32, after the status block).
enum PrepHeader : int {
  HDR_CMAX = 0,  // max_v |C_v| as float bits
  HDR_NNF = 1,   // token blocks that are not flat (visited densely)
  HDR_ROWMAX = 2,// nonzero: the workspace holds each token's maximum logit (cce_backward_prepare_rows)
  HDR_T = 3,     // tiles to visit: NNF * n_vtile
  HDR_EMAX = 4,  // max_i |E_i| as float bits (fixed-point accumulation)
  HDR_DLMAX = 5, // max_i |dloss_i| as float bits (fixed-point accumulation)
};
constexpr int HDR_BYTES = 256;
enum StatusFlag : unsigned long long {
  SF_TIMEOUT = 1ull,    // a bounded wait gave up; outputs are incomplete
  SF_BAD_LABEL = 2ull,  // a label outside [0, V) that is not ignore_index
};
constexpr int STATUS_BYTES = 256;

struct FwdArgs {
  int N, D, V;
  int n_mblk;      // token blocks: ceil(N / BM), or ceil(N / 2BM) for the CTA-pair kernel
  int n_vtile;     // ceil(V / BN)
  int n_split;     // vocabulary splits per token block
  int n_units;     // n_mblk * n_split
  int group_m;     // token blocks per raster group (their E rows stay in L2)
  float2* partial; // [n_split][N]: (running max, sum of exp(z - max)) per split
  float* dbg_logits;           // optional [N][n_vtile * BN] raw logits (debug build entry only)
  unsigned long long* status;
  unsigned long long wait_limit_ns;
  int withhold_loads;          // test hook: the TMA producer issues nothing
  int pf;                      // L2 prefetch distance of the C stream in K slices (0: off)
  int l2_hints;                // CTA-pair kernel: bit 0 E slices evict_last, bit 1 C slices evict_first
  // CTA-pair kernel, unit order.  0: units dealt round-robin to the pairs.
  // 1: two queues, one per L2 half: the token blocks are split between the
  // halves of the GPU (in proportion to their SMs), each pair draws units of
  // its own half's blocks at run time, and takes the other queue's units when
  // its own runs out or runs more than one vocabulary split ahead.
  int sched;
};

struct FinArgs {
  int N, D, V, n_split;
  long long ignore_index;
  const float2* partial;
  unsigned long long* status;
  // vocabulary shard (C holds rows v_offset .. v_offset + V - 1 of the full
  // classifier): write per-token (max, sum exp(z - max), target logit or 0)
  // to shard_stats [3][N] instead of loss / lse
  float* shard_stats;
  long long v_offset;
  float* row_max;        // optional [N]: max_v z_iv, the largest logit of each token
};

struct PrepArgs {
  int N, D, V, n_mblk, n_vtile;
  long long ignore_index;
  int shard_mode;         // labels are global ids; C is the shard [v_offset, v_offset + V)
  long long v_offset;
  float log_eps;          // ln(filter_eps)
  unsigned* hdr;          // PrepHeader words
  unsigned* rowbits;      // [ceil(V / 32)] bit v: row v of dC is a label of a flat block's kept token
  int* blk_flat;          // [n_mblk]
  int* nonflat;           // [n_mblk] ids of blocks that are not flat
  float* enorm;           // [N] |E_i|
  const float* row_max;   // [N] max_v E_i . C_v from the forward, or null (then |E_i| max_v |C_v| bounds it)
  unsigned long long* status;
};

// Flat token blocks (the pre-pass proved every non-label entry of their
// softmax rows below filter_eps): the only entry left per kept token is its
// label entry, handled without recomputing any logit tile.
struct FlatArgs {
  int N, D, V;
  long long ignore_index;
  int shard_mode;
  long long v_offset;
  float filter_eps;
  int accumulate;              // dE rows are added to instead of written
  const int* blk_flat;         // [n_mblk] from the pre-pass
  const unsigned* hdr;         // pre-pass header (fixed-point scale)
  float* dE;                   // fp32 [N][D] (unless accE)
  float* dC;                   // fp32 [V][D] (unless accC)
  unsigned long long* accE;    // fixed-point accumulators (deterministic mode) or null
  unsigned long long* accC;
  unsigned long long* status;
};

struct BwdArgs {
  int N, D, V;
  int n_mblk, n_vtile;
  int n_tiles;          // tiles to visit (dense mode)
  int group_m;          // token blocks per raster group (dense mode)
  int list_mode;        // 1: visit the tiles of the blocks that are not flat (hdr, nonflat)
  int shard_mode;       // 1: C is a vocabulary shard starting at global id v_offset
  long long v_offset;
  const unsigned* hdr;
  const int* nonflat;
  float filter_eps;     // <= 0: every tile is live
  long long ignore_index;
  const int64_t* y;
  const float* lse;
  const float* dloss;
  float* dE;            // [N][D] fp32, accumulated
  float* dC;            // [V][D] fp32, accumulated
  // fixed-point accumulation (deterministic mode): when accE is non-null the
  // contributions go to these int64 buffers instead of dE/dC
  unsigned long long* accE;  // [N][D]
  unsigned long long* accC;  // [V][D]
  unsigned long long* status;
  unsigned long long wait_limit_ns;
  int withhold_loads;   // test hook: the TMA producer issues nothing
  int pf;               // L2 prefetch distance of the operand streams in K slices (0: off)
  int red_pf;           // L2 prefetch distance, in K slices, of the dE/dC rows the reductions add into (0: off)
  int l2_hints;         // 1: C slices loaded evict-first, dE reduce-adds evict-last (keeps dE in L2)
  // profiling hook: per CTA and tile, globaltimer stamps (ns) at the start of
  // the tile, when its logits are in TMEM and when its gradient tile and
  // live mask are published; [grid][trace_cap][4] u64, null when off
  unsigned long long* trace;
  int trace_cap;
};

// ----------------------------------------------------------------------------
// Dense backward through softmax-gradient stripes (filter off).
//
// The vocabulary is cut into stripes of vt_per_s 256-wide tiles.  For each
// stripe s three kinds of 256 x 256 CTA-pair tasks run:
//   A(s): (token block m2 of 256, vocabulary tile vt of the stripe): recompute
//         the logit tile, form G = dloss (softmax - onehot) and store it in
//         bf16 into stripe buffer s % nbuf;
//   B(s): (vt of the stripe, d-chunk dc of 256): dC[vt, dc] = G[:, vt]^T E[:, dc]
//         over every token of the launch (written once);
//   C(s): (m2, dc): dE[m2, dc] += G[m2, stripe] C[stripe, dc].
// Global task order: A(0); then for s = 1 .. n_s - 1: A(s), B(s-1), C(s-1);
// then B(n_s - 1), C(n_s - 1).  Every task depends only on tasks earlier in
// this order (B(s), C(s) on A(s); A(s) on B(s - nbuf), C(s - nbuf), which
// free its buffer), so CTA pairs that take tasks in this order always make
// progress.
// ----------------------------------------------------------------------------
struct StripePlan {
  int n_m2;      // 256-token blocks of this launch
  int n_vtile;   // 256-wide vocabulary tiles (all of V)
  int n_dc;      // 256-wide d-chunks
  int vt_per_s;  // vocabulary tiles per stripe
  int n_s;       // stripes
  int nbuf;      // stripe buffers (<= n_s)
  int order;     // 0: stripe-major (above); 1: interleaved (below)
  int gm;        // order 1: token blocks per group
  int lag;       // order 1: groups between a group's A tasks and its C tasks (>= 1)
};
enum StripeTask : int { TASK_END = -1, TASK_A = 0, TASK_B = 1, TASK_C = 2 };
struct StripeTaskDesc {
  int type, s, a, b;  // A: a = m2, b = vt; B: a = vt, b = dc; C: a = m2, b = dc
};

__host__ __device__ inline int stripe_tiles(const StripePlan& p, int s) {
  const int t = p.n_vtile - s * p.vt_per_s;
  return t < p.vt_per_s ? t : p.vt_per_s;
}
__host__ __device__ inline long long stripe_nA(const StripePlan& p, int s) {
  return (long long)p.n_m2 * stripe_tiles(p, s);
}
__host__ __device__ inline long long stripe_nB(const StripePlan& p, int s) {
  return (long long)stripe_tiles(p, s) * p.n_dc;
}
__host__ __device__ inline long long stripe_nC(const StripePlan& p) { return (long long)p.n_m2 * p.n_dc; }
__host__ __device__ inline long long stripe_total(const StripePlan& p) {
  long long t = 0;
  for (int s = 0; s < p.n_s; ++s) t += stripe_nA(p, s) + stripe_nB(p, s) + stripe_nC(p);
  return t;
}

// Inside A(s): the token block varies fastest, so the pairs running at the
// same time share a vocabulary tile of C; inside B(s) and C(s) the d-chunk
// varies fastest (pairs share the stripe columns, resp. the token rows, of G).
__host__ __device__ inline StripeTaskDesc stripe_A(const StripePlan& p, int s, long long k) {
  return StripeTaskDesc{TASK_A, s, (int)(k % p.n_m2), s * p.vt_per_s + (int)(k / p.n_m2)};
}
__host__ __device__ inline StripeTaskDesc stripe_BC(const StripePlan& p, int s, long long k) {
  const long long nB = stripe_nB(p, s);
  if (k < nB) return StripeTaskDesc{TASK_B, s, s * p.vt_per_s + (int)(k / p.n_dc), (int)(k % p.n_dc)};
  k -= nB;
  return StripeTaskDesc{TASK_C, s, (int)(k / p.n_dc), (int)(k % p.n_dc)};
}

// Interleaved order (order 1): each stripe is one run of tasks.  Its token
// blocks are taken gm at a time; a group's A tasks (vocabulary tile outer,
// token block inner, so the pairs running together share a C tile) are
// followed by the C tasks of the group `lag` groups earlier, whose G rows
// were written recently and are still in L2; the C tasks of the last `lag`
// groups and then the stripe's B tasks close the run.  Every task still
// comes after the tasks it reads: C(s, m2) after all A(s, m2, .), B(s, vt)
// after all A(s, ., vt), A(s) after the B and C tasks of earlier stripes.
__host__ __device__ inline int stripe_group_size(const StripePlan& p, int grp) {
  const int r = p.n_m2 - grp * p.gm;
  return r < p.gm ? r : p.gm;
}
__host__ __device__ inline StripeTaskDesc stripe_local_interleaved(const StripePlan& p, int s, long long k) {
  const int T = stripe_tiles(p, s), nd = p.n_dc;
  const int ng = (p.n_m2 + p.gm - 1) / p.gm;
  const int L = p.lag < ng ? p.lag : ng;
  const int vt0 = s * p.vt_per_s;
  long long off = 0;
  for (int grp = 0; grp < ng; ++grp) {
    const int mc = stripe_group_size(p, grp);
    const long long nA = (long long)T * mc;
    if (k < off + nA) {
      const long long i = k - off;
      return StripeTaskDesc{TASK_A, s, grp * p.gm + (int)(i % mc), vt0 + (int)(i / mc)};
    }
    off += nA;
    if (grp >= L) {
      const int cg = grp - L;
      const long long nC = (long long)stripe_group_size(p, cg) * nd;
      if (k < off + nC) {
        const long long i = k - off;
        return StripeTaskDesc{TASK_C, s, cg * p.gm + (int)(i / nd), (int)(i % nd)};
      }
      off += nC;
    }
  }
  for (int cg = ng - L; cg < ng; ++cg) {
    const long long nC = (long long)stripe_group_size(p, cg) * nd;
    if (k < off + nC) {
      const long long i = k - off;
      return StripeTaskDesc{TASK_C, s, cg * p.gm + (int)(i / nd), (int)(i % nd)};
    }
    off += nC;
  }
  const long long i = k - off;
  return StripeTaskDesc{TASK_B, s, vt0 + (int)(i / nd), (int)(i % nd)};
}

// Task t of the global order.  Every stripe but the last has the same task
// counts, so the position is found without walking the stripes.
__host__ __device__ inline StripeTaskDesc stripe_decode(const StripePlan& p, long long t) {
  if (t < 0) return StripeTaskDesc{TASK_END, 0, 0, 0};
  if (p.order == 1) {
    const long long per = stripe_nA(p, 0) + stripe_nC(p) + stripe_nB(p, 0);
    const long long full = (long long)(p.n_s - 1) * per;
    if (t < full) return stripe_local_interleaved(p, (int)(t / per), t % per);
    t -= full;
    const int L = p.n_s - 1;
    if (t < stripe_nA(p, L) + stripe_nC(p) + stripe_nB(p, L)) return stripe_local_interleaved(p, L, t);
    return StripeTaskDesc{TASK_END, 0, 0, 0};
  }
  const long long nA = stripe_nA(p, 0);
  if (p.n_s == 1) {
    if (t < nA) return stripe_A(p, 0, t);
    t -= nA;
    if (t < stripe_nB(p, 0) + stripe_nC(p)) return stripe_BC(p, 0, t);
    return StripeTaskDesc{TASK_END, 0, 0, 0};
  }
  if (t < nA) return stripe_A(p, 0, t);
  t -= nA;
  // groups g = 1 .. n_s - 2: A(g) (full), then B/C(g - 1) (full)
  const long long nBCf = stripe_nB(p, 0) + stripe_nC(p);
  const long long gsz = nA + nBCf;
  const long long full_groups = p.n_s - 2;
  if (t < full_groups * gsz) {
    const int g = 1 + (int)(t / gsz);
    const long long k = t % gsz;
    return k < nA ? stripe_A(p, g, k) : stripe_BC(p, g - 1, k - nA);
  }
  t -= full_groups * gsz;
  const int L = p.n_s - 1;  // the last stripe (possibly narrower)
  const long long nAL = stripe_nA(p, L);
  if (t < nAL) return stripe_A(p, L, t);
  t -= nAL;
  const long long nBCp = stripe_nB(p, L - 1) + stripe_nC(p);
  if (t < nBCp) return stripe_BC(p, L - 1, t);
  t -= nBCp;
  if (t < stripe_nB(p, L) + stripe_nC(p)) return stripe_BC(p, L, t);
  return StripeTaskDesc{TASK_END, 0, 0, 0};
}

// Counters of the stripe backward (u32, zeroed per launch): one arrival per
// epilogue warp (4 per CTA, 8 per pair) for each finished task.
//   doneA_v[n_vtile]        A tasks of vocabulary tile vt
//   doneA_ms[n_s][n_m2]     A tasks of token block m2 in stripe s
//   doneBC[n_s]             B and C tasks of stripe s
//   doneC[n_m2][n_dc]       C tasks of each dE tile (ordered mode)
//   next                    the next task to hand out
struct StripeArgs {
  StripePlan p;
  int N, D, V;
  int tok0;              // first token of this launch (token super-block)
  int Ns_pad;            // rows of one stripe buffer: n_m2 * 256
  int Vs;                // columns of one stripe buffer: vt_per_s * 256
  int dC_add;            // 1: B tasks add into dC (later super-blocks, or accumulation)
  long long ignore_index;
  int shard_mode;        // labels are global ids; C is the shard [v_offset, v_offset + V)
  long long v_offset;
  const int64_t* y;
  const float* lse;
  const float* dloss;
  unsigned* doneA_v;
  unsigned* doneA_ms;
  unsigned* doneBC;
  unsigned* doneC;       // [n_m2][n_dc] C tasks of each dE tile (ordered mode)
  unsigned long long* next;
  int ordered;           // 1: the stripes' reduce-adds into a dE tile happen in stripe order
  int dE_prefetch;       // 1: dE-tile tasks ask for their dE rows in L2 when they start
  // profiling hook: per CTA pair and task, globaltimer stamps (ns) when the
  // task was handed out, when its accumulator was complete and when its
  // epilogue finished, then the task kind | (ns spent waiting for its inputs
  // << 8); [pairs][trace_cap][4] u64, null when off
  unsigned long long* trace;
  int trace_cap;
  unsigned long long* status;
  unsigned long long wait_limit_ns;
  int withhold_loads;    // test hook: the TMA producers issue nothing
  float filter_eps;      // > 0: entries of G with |P - onehot| below it are zeroed
  // filter on: [n_s][n_m2][vt_per_s] bytes, 1 where the 256 x 256 G tile of
  // an A task holds a kept entry (zeroed per launch); B and C tasks skip the
  // K blocks whose G tile is all zero
  unsigned char* nz;
  // filter on: [ceil(N / 128)] from the pre-pass, nonzero for a flat 128-token
  // block (its label entries go to the flat-row kernel; its rows of G are
  // zero, and a recompute task whose two blocks are both flat is skipped)
  const int* blk_flat;
};

// Fixed-point exponent s: contributions are stored as round(x * 2^s) in int64.
// Every gradient entry is bounded by
//   |dE_id| <= max_i|dloss_i| * 2 * max_v|C_v|   and
//   |dC_vd| <= sum_i |dloss_i| * max_i|E_i| <= N * max|dloss| * max|E_i|,
// so with B = 2 * max of both (and a factor 2 of headroom) the final sums stay
// inside +-2^62 when s = 61 - ceil(log2 B).  Integer wrap-around in between
// cancels, so only the final value needs the bound.
__host__ __device__ inline int fixed_point_exponent(float cmax, float emax, float dlmax, int N) {
  const float b1 = 2.f * dlmax * cmax;
  const float b2 = (float)N * dlmax * emax;
  float B = 2.f * fmaxf(b1, b2);
  if (!(B > 0.f)) return 60;                  // nothing to accumulate
  int e = 0;
  frexpf(B, &e);                              // B < 2^e
  int s = 61 - e;
  return s < -60 ? -60 : (s > 100 ? 100 : s);
}

// Work unit u -> (vocabulary split r, token block m).  Units are grouped by
// group_m token blocks; inside a group the token block varies fastest, so the
// CTAs running at the same time share a few splits (C tiles) and a bounded
// set of E rows, both L2-resident.
__host__ __device__ inline void unit_coords(int u, int n_mblk, int n_split, int group_m, int& r, int& m) {
  const int gsz = group_m * n_split;
  const int g = u / gsz;
  const int rem = u - g * gsz;
  const int gm = min(group_m, n_mblk - g * group_m);
  r = rem / gm;
  m = g * group_m + (rem - r * gm);
}

__host__ __device__ inline void split_range(int r, int n_vtile, int n_split, int& v0, int& v1) {
  v0 = (int)(((long long)r * n_vtile) / n_split);
  v1 = (int)(((long long)(r + 1) * n_vtile) / n_split);
}

}  // namespace cce
