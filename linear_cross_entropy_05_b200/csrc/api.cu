// C-ABI front end of libcce.so: argument validation, workspace carving,
// TMA descriptor construction and kernel launches.  See include/cce.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "../../include/cce.h"
#include "../../include/cce_debug.h"
#include "common.cuh"

namespace cce {
cudaError_t launch_fwd_lse(const CUtensorMap& tmE, const CUtensorMap& tmC, const FwdArgs& a, int grid,
                           cudaStream_t stream);
cudaError_t launch_l2_half_probe(int sms, cudaStream_t stream);
cudaError_t read_l2_halves(unsigned* out, int n);
cudaError_t launch_fwd_lse_pair(const CUtensorMap& tmE, const CUtensorMap& tmCh, const FwdArgs& a, int grid,
                                int stages, cudaStream_t stream);
cudaError_t launch_fwd_finalize(const void* E, const void* C, const int64_t* y, const FinArgs& a, float* loss,
                                float* lse, cudaStream_t stream);
cudaError_t launch_merge_shards(const float* stats, int R, int N, const int64_t* y, long long V_total,
                                long long ignore_index, float* loss, float* lse, cudaStream_t stream);
cudaError_t launch_bwd(const CUtensorMap& tmE, const CUtensorMap& tmC, const CUtensorMap& tmCq, const CUtensorMap& tmdE,
                       const CUtensorMap& tmdC, const BwdArgs& a, int grid, int variant, cudaStream_t stream);
cudaError_t launch_prep(const void* E, const void* C, const int64_t* y, const float* lse, const PrepArgs& p,
                        int sms, cudaStream_t stream);
cudaError_t launch_cnorm(const void* C, const PrepArgs& p, int sms, cudaStream_t stream);
cudaError_t launch_enorm(const void* E, const PrepArgs& p, int sms, cudaStream_t stream);
cudaError_t launch_fixed_prep(const float* dloss, const PrepArgs& p, int sms, cudaStream_t stream);
cudaError_t launch_bwd_stripe(const CUtensorMap* maps, const StripeArgs& a, void* G, int grid, cudaStream_t stream);
cudaError_t launch_fixed_to_out(const unsigned long long* acc, void* out, int rows, int D, const unsigned* hdr,
                                int N, bool bf16, bool accumulate, const unsigned* rowbits, int sms,
                                cudaStream_t stream);
cudaError_t launch_clear_visited_rows(unsigned long long* acc, int V, int D, const unsigned* rowbits,
                                      const unsigned* hdr, int sms, cudaStream_t stream);
cudaError_t launch_flat_rows(const void* E, const void* C, const int64_t* y, const float* lse, const float* dloss,
                             const FlatArgs& f, cudaStream_t stream);
cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, bool accumulate, int sms, cudaStream_t stream);
}  // namespace cce

using namespace cce;

namespace {

std::atomic<unsigned long long> g_wait_limit_ns{1000000000ull};

// Forward kernel variant: 1 = CTA pairs (cta_group::2, the default), 0 = single CTAs.
std::atomic<int> g_fwd_variant{1};
// Backward kernel variant: 0 = 3 stages / 1 staging buffer (default), 1 = 2 stages / 2 buffers,
// 2 = 2 stages / 8 epilogue warps, 3 = as 0 with load/store-path reductions.
std::atomic<int> g_bwd_variant{0};

// Test hook: when set, the next launches' TMA producers issue no copies.
std::atomic<int> g_withhold_loads{0};
std::atomic<int> g_fwd_pf{0};  // L2 prefetch distances (K slices) of the forward / backward operand streams
std::atomic<int> g_fwd_split{0};     // forward vocabulary splits per token block (0: chosen per shape)
std::atomic<int> g_fwd_group_m{0};   // forward token blocks per raster group (0: chosen per shape)
std::atomic<int> g_fwd_l2_hints{0};  // forward CTA-pair kernel: L2 eviction priorities (A/B)
std::atomic<int> g_fwd_stages{PAIR_STAGES_MAX};  // forward CTA-pair kernel: operand stages per CTA
std::atomic<int> g_fwd_order{1};     // forward CTA-pair kernel: 0 round-robin units, 1 one queue per L2 half
constexpr int kMaxDevices = 64;
std::atomic<bool> g_l2_probed[kMaxDevices];  // the L2-half probe was launched on this device
std::atomic<int> g_bwd_pf{0};
std::atomic<int> g_bwd_red_pf{0};  // L2 prefetch distance (K slices) of the backward's reduction targets
std::atomic<int> g_bwd_l2_hints{0};  // L2 eviction priorities in the filtered backward (A/B)
std::atomic<unsigned long long*> g_bwd_trace{nullptr};
std::atomic<int> g_bwd_trace_cap{0};

// Optional per-kernel timing events (debug hook): [kernel][0 = start, 1 = stop].
std::atomic<void*> g_events[2][2] = {{{nullptr}, {nullptr}}, {{nullptr}, {nullptr}}};

cudaError_t record_event(int kernel, int which, cudaStream_t s) {
  void* ev = g_events[kernel][which].load();
  return ev ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), s) : cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  bool ok = false;
  int sms = 0;
};

// Per-device facts, cached (at most 64 devices).
DeviceInfo device_info() {
  static DeviceInfo cache[64];
  static std::once_flag flags[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{};
  std::call_once(flags[dev], [dev] {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return;
    cache[dev].ok = (major == 10 && minor == 0);
    cache[dev].sms = sms;
  });
  return cache[dev];
}

bool sizes_ok(int64_t N, int64_t D, int64_t V) {
  return N > 0 && D > 0 && V > 0 && N <= INT_MAX && V <= INT_MAX && D <= INT_MAX && (D % 8) == 0 &&
         N * D <= (int64_t)1 << 40 && V * D <= (int64_t)1 << 40;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Vocabulary splits per 128-row token block.  Work units (block, split) are
// dealt to the persistent CTAs round-robin; pick the split count that
// minimises (units per CTA) x (tiles per unit).
// Largest number of vocabulary tiles any worker gets when the n_mblk * s
// work units are dealt round-robin (unit u to worker u % workers, as the
// forward kernels take them) and unit_coords maps a unit to its split.
long long max_worker_tiles(int n_mblk, int n_vtile, int s, int workers, int group_m) {
  std::vector<long long> load((size_t)workers, 0);
  const int units = n_mblk * s;
  for (int u = 0; u < units; ++u) {
    int r, m;
    unit_coords(u, n_mblk, s, group_m, r, m);
    int v0, v1;
    split_range(r, n_vtile, s, v0, v1);
    load[(size_t)(u % workers)] += v1 - v0;
  }
  return *std::max_element(load.begin(), load.end());
}

// Splits per token block: the fewest that minimise the most-loaded worker's
// vocabulary tiles (the kernel's duration).  The load is counted exactly
// while a candidate has at most 2^16 units (every workload here), else
// estimated as ceil(units / workers) * ceil(n_vtile / s).  Memoised per shape.
int choose_splits(int n_mblk, int n_vtile, int workers, int group_m) {
  static std::mutex mu;
  static std::map<std::array<int, 4>, int> memo;
  const std::array<int, 4> key{n_mblk, n_vtile, workers, group_m};
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = memo.find(key);
    if (it != memo.end()) return it->second;
  }
  long long best = LLONG_MAX;
  int best_s = 1;
  const int smax = std::min(64, n_vtile);
  for (int s = 1; s <= smax; ++s) {
    const long long units = (long long)n_mblk * s;
    const long long cost = units <= (1ll << 16) ? max_worker_tiles(n_mblk, n_vtile, s, workers, group_m)
                                                : ((units + workers - 1) / workers) * ((n_vtile + s - 1) / s);
    if (cost < best) {
      best = cost;
      best_s = s;
    }
  }
  std::lock_guard<std::mutex> lk(mu);
  if (memo.size() > 256) memo.clear();
  memo[key] = best_s;
  return best_s;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t D, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 gradient tensor [rows][D] as 32 x 32 boxes with 128-byte swizzle: the
// target of the backward kernel's bulk reduce-adds.
bool make_map_f32(CUtensorMap* map, const void* base, int64_t rows, int64_t D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// int64 fixed-point accumulator [rows][D] as {16, 32} boxes of u64 with
// 128-byte swizzle (16 values = one 128-byte row): the target of the
// deterministic backward's bulk reduce-adds.
bool make_map_u64(CUtensorMap* map, const void* base, int64_t rows, int64_t D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 8};
  cuuint32_t box[2] = {16, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct FwdPlan {
  bool pair;       // CTA-pair kernel: token blocks of 2 x BM rows, grid in pairs
  int n_mblk, n_vtile, n_split, grid, group_m;
  size_t ws_bytes;
};

// The forward's launch plan for a GPU with `sms` SMs (host arithmetic only).
bool plan_forward_for(int64_t N, int64_t D, int64_t V, int sms, FwdPlan* p) {
  if (!sizes_ok(N, D, V) || sms <= 0) return false;
  p->pair = g_fwd_variant.load() == 1 && sms >= 2;
  const int rows = p->pair ? 2 * BM : BM;       // token rows per work unit
  const int workers = p->pair ? sms / 2 : sms;  // CTA pairs or CTAs
  p->n_mblk = (int)((N + rows - 1) / rows);
  p->n_vtile = (int)((V + BN - 1) / BN);
  // Token blocks per raster group.  Round-robin order: ~48 MB of E rows in
  // flight.  Two-queue order (CTA pairs): ~24 MB per group of each L2 half;
  // the halves' groups are in flight together, and every line read by the
  // other half also has a copy in its home half, so each half holds about
  // 1.5 x that of E next to the C tiles being streamed.
  const bool two_queues = p->pair && g_fwd_order.load() == 1;
  p->group_m = (int)std::max<int64_t>(
      1, std::min<int64_t>(p->n_mblk, ((two_queues ? 24ll : 48ll) << 20) / ((int64_t)rows * D * 2)));
  if (g_fwd_group_m.load() > 0) p->group_m = std::min(p->n_mblk, g_fwd_group_m.load());
  p->n_split = g_fwd_split.load() > 0 ? std::min(p->n_vtile, g_fwd_split.load())
                                      : choose_splits(p->n_mblk, p->n_vtile, workers, p->group_m);
  if (two_queues && g_fwd_split.load() == 0) {
    // Units of at most ~8 vocabulary tiles (up to 128 splits): the pairs
    // that share a split's C rows then read them within a few tile steps,
    // before they leave L2.  Gemma-2-2B-shaped head: 2.2 GB of DRAM reads
    // at 37 splits, 1.3 GB at 74-128; Llama-3-8B-shaped: 8.6 -> 7.4 GB;
    // the N = 65536 sweep: 17 -> 7.6 GB and 4 % faster.  The split count
    // chosen for balance stays the floor (small problems need the units).
    p->n_split = std::min(p->n_vtile, std::min(128, std::max(p->n_split, (p->n_vtile + 7) / 8)));
  }
  const long long units = (long long)p->n_mblk * p->n_split;
  p->grid = (int)std::min<long long>(units, workers) * (p->pair ? 2 : 1);
  p->ws_bytes = STATUS_BYTES + align_up((size_t)p->n_split * (size_t)N * sizeof(float2), 256);
  return true;
}

bool plan_forward(int64_t N, int64_t D, int64_t V, FwdPlan* p) {
  if (!sizes_ok(N, D, V)) return false;
  const DeviceInfo di = device_info();
  if (!di.ok || di.sms <= 0) return false;
  return plan_forward_for(N, D, V, di.sms, p);
}

// Backward workspace: status | pre-pass header | dC row bits [ceil(V/32)] |
// blk_flat, nonflat [n_mblk] | |E_i| [N] | the tokens' maximum logits [N]
// (cce_backward_prepare_rows).  O(N + V/32).
// Stripe backward (CCE_BWD_STRIPES, filter off): 256-token blocks per launch
// (token super-block; dC gathers the super-blocks by reduce-adds) and
// vocabulary tiles per stripe.
constexpr int kStripeMaxM2 = 64;     // 16384 tokens per launch (upper bound; workspace sized for it)
constexpr int kStripeVtiles = 16;    // 4096 vocabulary columns per stripe (measured: 8 -> 16 tiles +6 %)
constexpr int kStripeBuffers = 3;
std::atomic<int> g_stripe_m2{kStripeMaxM2};  // token blocks per launch actually used (A/B knob)
std::atomic<int> g_stripe_dE_pf{0};          // L2 prefetch of the dE rows of dE-tile tasks (measured: no gain)
std::atomic<int> g_stripe_vt{kStripeVtiles};  // vocabulary tiles per stripe (A/B knob)
std::atomic<int> g_stripe_order{0};  // task order: 0 stripe-major, 1 interleaved (A/B knob)
std::atomic<int> g_stripe_gm{4};     // interleaved order: token blocks per group
std::atomic<int> g_stripe_lag{2};    // interleaved order: groups between A and C tasks

struct StripeLayout {
  StripePlan p;          // of a full super-block
  int n_sb;              // super-blocks (launches)
  int Ns_pad, Vs;
  size_t off_ctr, ctr_bytes, off_G, G_bytes, bytes;
  size_t n_doneA_v, n_doneA_ms, n_doneBC, n_doneC, n_nz;
};

StripeLayout plan_stripes(int64_t N, int64_t D, int64_t V, size_t base) {
  StripeLayout L{};
  const int n_m2_total = (int)((N + 255) / 256);
  L.p.n_m2 = std::min(n_m2_total, kStripeMaxM2);
  L.p.n_vtile = (int)((V + BN - 1) / BN);
  L.p.n_dc = (int)((D + 255) / 256);
  L.p.vt_per_s = std::min(L.p.n_vtile, g_stripe_vt.load());
  L.p.n_s = (L.p.n_vtile + L.p.vt_per_s - 1) / L.p.vt_per_s;
  L.p.nbuf = std::min(L.p.n_s, kStripeBuffers);
  L.p.order = g_stripe_order.load();
  L.p.gm = g_stripe_gm.load();
  L.p.lag = g_stripe_lag.load();
  L.n_sb = (n_m2_total + L.p.n_m2 - 1) / L.p.n_m2;
  L.Ns_pad = L.p.n_m2 * 256;
  L.Vs = L.p.vt_per_s * BN;
  L.n_doneA_v = (size_t)L.p.n_vtile;
  L.n_doneA_ms = (size_t)L.p.n_s * L.p.n_m2;
  L.n_doneBC = (size_t)L.p.n_s;
  L.n_doneC = (size_t)L.p.n_m2 * L.p.n_dc;
  L.off_ctr = base;
  L.n_nz = (size_t)L.p.n_s * L.p.n_m2 * L.p.vt_per_s;
  L.ctr_bytes = align_up(8 + 4 * (L.n_doneA_v + L.n_doneA_ms + L.n_doneBC + L.n_doneC) + L.n_nz, 256);
  L.off_G = L.off_ctr + L.ctr_bytes;
  L.G_bytes = align_up((size_t)L.p.nbuf * L.Ns_pad * L.Vs * 2, 256);
  L.bytes = L.off_G + L.G_bytes;
  return L;
}

struct BwdPlan {
  int n_mblk, n_vtile;
  size_t off_hdr, off_rowbits, off_flat, off_nonflat, off_enorm, off_rowmax, zero_bytes, ws_bytes;
  size_t off_accE, off_accC;  // fixed-point accumulators (deterministic mode only)
  StripeLayout stripes;       // CCE_BWD_STRIPES only
};

constexpr unsigned kBwdFlagsAll = CCE_BWD_DETERMINISTIC | CCE_BWD_BF16_GRADS | CCE_BWD_ACCUMULATE |
                                  CCE_BWD_PREPARED | CCE_BWD_STRIPES | CCE_BWD_ROW_MAX;
// Whether these flags take the int64 fixed-point accumulation.  With
// CCE_BWD_STRIPES the deterministic mode is served by the stripe kernel's
// fixed reduction order instead (filter off only, fp32 outputs).
bool uses_fixed_point(unsigned flags) {
  if (flags & CCE_BWD_STRIPES) return false;  // bf16 outputs: fp32 scratch, converted once
  if (flags & CCE_BWD_BF16_GRADS) return true;
  return (flags & CCE_BWD_DETERMINISTIC) && !(flags & CCE_BWD_STRIPES);
}

bool plan_backward(int64_t N, int64_t D, int64_t V, BwdPlan* p, unsigned flags = 0) {
  if (flags & ~kBwdFlagsAll) return false;
  if (!sizes_ok(N, D, V)) return false;
  p->n_mblk = (int)((N + BM - 1) / BM);
  p->n_vtile = (int)((V + BN - 1) / BN);
  if ((int64_t)p->n_mblk * p->n_vtile >= ((int64_t)1 << 31)) return false;
  const size_t mb4 = align_up((size_t)p->n_mblk * 4, 256);
  p->off_hdr = STATUS_BYTES;
  p->off_rowbits = p->off_hdr + HDR_BYTES;
  p->zero_bytes = p->off_rowbits + align_up((size_t)((V + 31) / 32) * 4, 256);  // status, header, row bits
  p->off_flat = p->zero_bytes;
  p->off_nonflat = p->off_flat + mb4;
  p->off_enorm = p->off_nonflat + mb4;
  p->off_rowmax = p->off_enorm + align_up((size_t)N * sizeof(float), 256);
  p->ws_bytes = p->off_rowmax + align_up((size_t)N * sizeof(float), 256);
  p->off_accE = p->off_accC = 0;
  if ((flags & CCE_BWD_STRIPES) && (flags & CCE_BWD_BF16_GRADS)) {
    // the stripe path with bf16 outputs sums into fp32 dE / dC scratch
    p->off_accE = p->ws_bytes;
    p->off_accC = p->off_accE + align_up((size_t)N * D * 4, 256);
    p->ws_bytes = p->off_accC + align_up((size_t)V * D * 4, 256);
  } else if (uses_fixed_point(flags)) {
    p->off_accE = p->ws_bytes;
    p->off_accC = p->off_accE + align_up((size_t)N * D * 8, 256);
    p->ws_bytes = p->off_accC + align_up((size_t)V * D * 8, 256);
  }
  p->stripes = StripeLayout{};
  if (flags & CCE_BWD_STRIPES) {
    p->stripes = plan_stripes(N, D, V, p->ws_bytes);
    p->ws_bytes = p->stripes.bytes;
  }
  return true;
}

// shard_stats != nullptr: C is the vocabulary shard starting at global id
// v_offset; per-token (max, sum exp, target) go to shard_stats [3][N] and
// loss / lse are not written.
cce_status_t forward_impl(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D, int64_t V,
                          int64_t ignore_index, float* loss, float* lse, float* dbg_logits, void* ws,
                          size_t ws_bytes, void* stream_, float* shard_stats = nullptr, int64_t v_offset = 0,
                          float* row_max = nullptr) {
  if (!E || !C || !y || !ws) return CCE_ERR_INVALID_ARG;
  if (!shard_stats && (!loss || !lse)) return CCE_ERR_INVALID_ARG;
  if (!sizes_ok(N, D, V) || v_offset < 0) return CCE_ERR_INVALID_ARG;
  if (!aligned(E, 16) || !aligned(C, 16) || !aligned(y, 8) || !aligned(loss, 4) || !aligned(lse, 4) ||
      !aligned(shard_stats, 4) || !aligned(row_max, 4) || !aligned(ws, 256))
    return CCE_ERR_MISALIGNED;
  if (!device_info().ok) return CCE_ERR_UNSUPPORTED_DEVICE;
  FwdPlan p;
  if (!plan_forward(N, D, V, &p)) return CCE_ERR_INVALID_ARG;
  if (ws_bytes < p.ws_bytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

  CUtensorMap tmE, tmC;
  if (!make_map(&tmE, E, N, D, BM) || !make_map(&tmC, C, V, D, p.pair ? BM : BN)) return CCE_ERR_CUDA;

  unsigned long long* status = reinterpret_cast<unsigned long long*>(ws);
  float2* partial = reinterpret_cast<float2*>(reinterpret_cast<char*>(ws) + STATUS_BYTES);
  if (cudaMemsetAsync(status, 0, STATUS_BYTES, stream) != cudaSuccess) return CCE_ERR_CUDA;

  FwdArgs a;
  a.N = (int)N;
  a.D = (int)D;
  a.V = (int)V;
  a.n_mblk = p.n_mblk;
  a.n_vtile = p.n_vtile;
  a.n_split = p.n_split;
  a.n_units = p.n_mblk * p.n_split;
  a.group_m = p.group_m;
  a.partial = partial;
  a.dbg_logits = dbg_logits;
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.withhold_loads = g_withhold_loads.load();
  a.pf = g_fwd_pf.load();
  a.l2_hints = g_fwd_l2_hints.load();
  a.sched = p.pair ? g_fwd_order.load() : 0;
  if (a.sched) {
    // which L2 half each SM is in: found once per device and process (the
    // first launch on a stream being captured goes into the graph, where it
    // changes nothing when replayed); until it has run, pairs alternate
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return CCE_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices && !g_l2_probed[dev].exchange(true) &&
        launch_l2_half_probe(device_info().sms, stream) != cudaSuccess)
      return CCE_ERR_CUDA;
  }
  if (record_event(0, 0, stream) != cudaSuccess) return CCE_ERR_CUDA;
  const cudaError_t le =
      p.pair ? launch_fwd_lse_pair(tmE, tmC, a, p.grid, g_fwd_stages.load(), stream)
             : launch_fwd_lse(tmE, tmC, a, p.grid, stream);
  if (le != cudaSuccess) return CCE_ERR_CUDA;
  if (record_event(0, 1, stream) != cudaSuccess) return CCE_ERR_CUDA;

  FinArgs f;
  f.N = (int)N;
  f.D = (int)D;
  f.V = (int)V;
  f.n_split = p.n_split;
  f.ignore_index = ignore_index;
  f.partial = partial;
  f.status = status;
  f.shard_stats = shard_stats;
  f.v_offset = v_offset;
  f.row_max = row_max;
  if (launch_fwd_finalize(E, C, y, f, loss, lse, stream) != cudaSuccess) return CCE_ERR_CUDA;
  return CCE_OK;
}

}  // namespace

extern "C" {

size_t cce_forward_workspace_size(int64_t N, int64_t D, int64_t V) {
  FwdPlan p;
  if (!plan_forward(N, D, V, &p)) return 0;
  return p.ws_bytes;
}

size_t cce_backward_workspace_size(int64_t N, int64_t D, int64_t V) {
  BwdPlan p;
  if (!plan_backward(N, D, V, &p)) return 0;
  return p.ws_bytes;
}

cce_status_t cce_forward(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D, int64_t V,
                         int64_t ignore_index, float* loss, float* lse, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return forward_impl(E, C, y, N, D, V, ignore_index, loss, lse, nullptr, workspace, workspace_bytes, stream);
}

cce_status_t cce_forward_ex(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D, int64_t V,
                            int64_t ignore_index, float* loss, float* lse, float* row_max, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return forward_impl(E, C, y, N, D, V, ignore_index, loss, lse, nullptr, workspace, workspace_bytes, stream,
                      nullptr, 0, row_max);
}

cce_status_t cce_debug_forward_logits(const void* E, const void* C, const int64_t* y, int64_t N, int64_t D,
                                      int64_t V, int64_t ignore_index, float* loss, float* lse, float* logits,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!logits) return CCE_ERR_INVALID_ARG;
  return forward_impl(E, C, y, N, D, V, ignore_index, loss, lse, logits, workspace, workspace_bytes, stream);
}

void cce_debug_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns ? limit_ns : 1000000000ull);
}

void cce_debug_withhold_loads(int on) { g_withhold_loads.store(on ? 1 : 0); }

cce_status_t cce_debug_set_prefetch(int fwd_slices, int bwd_slices) {
  if (fwd_slices < 0 || fwd_slices > 64 || bwd_slices < 0 || bwd_slices > 64) return CCE_ERR_INVALID_ARG;
  g_fwd_pf.store(fwd_slices);
  g_bwd_pf.store(bwd_slices);
  return CCE_OK;
}

cce_status_t cce_debug_set_forward_schedule(int n_split, int group_m, int l2_hints, int stages) {
  if (n_split < 0 || n_split > 256 || group_m < 0 || l2_hints < 0 || l2_hints > 3) return CCE_ERR_INVALID_ARG;
  if (stages != 0 && stages != PAIR_STAGES && stages != PAIR_STAGES_MAX) return CCE_ERR_INVALID_ARG;
  g_fwd_split.store(n_split);
  g_fwd_group_m.store(group_m);
  g_fwd_l2_hints.store(l2_hints);
  g_fwd_stages.store(stages ? stages : PAIR_STAGES_MAX);
  return CCE_OK;
}

int cce_debug_forward_plan(int64_t N, int64_t D, int64_t V, int sms, int* out) {
  if (!out) return -1;
  FwdPlan p;
  if (!plan_forward_for(N, D, V, sms, &p)) return -1;
  out[0] = p.pair ? 1 : 0;
  out[1] = p.n_mblk;
  out[2] = p.n_vtile;
  out[3] = p.n_split;
  out[4] = p.group_m;
  out[5] = p.grid;
  return 0;
}

int cce_debug_l2_halves(int* half_of_sm, int max_sms) {
  if (!half_of_sm || max_sms <= 0) return -1;
  const int n = std::min(max_sms, 256);
  std::vector<unsigned> h((size_t)n, 0u);
  if (read_l2_halves(h.data(), n) != cudaSuccess) return -1;
  for (int i = 0; i < n; ++i) half_of_sm[i] = (int)h[(size_t)i];
  return n;
}

cce_status_t cce_debug_set_forward_order(int order) {
  if (order < 0 || order > 1) return CCE_ERR_INVALID_ARG;
  g_fwd_order.store(order);
  return CCE_OK;
}

cce_status_t cce_debug_set_stripe_params(int tokens_per_launch, int dE_prefetch, int vtiles_per_stripe) {
  if (tokens_per_launch < 0 || tokens_per_launch > kStripeMaxM2 * 256 || tokens_per_launch % 256 != 0 ||
      dE_prefetch < 0 || dE_prefetch > 1 || vtiles_per_stripe < 0 || vtiles_per_stripe > 32)
    return CCE_ERR_INVALID_ARG;
  g_stripe_m2.store(tokens_per_launch ? tokens_per_launch / 256 : kStripeMaxM2);
  g_stripe_dE_pf.store(dE_prefetch);
  g_stripe_vt.store(vtiles_per_stripe ? vtiles_per_stripe : kStripeVtiles);
  return CCE_OK;
}

cce_status_t cce_debug_set_stripe_order(int order, int group_m2, int lag) {
  if (order < 0 || order > 1 || group_m2 <= 0 || group_m2 > 64 || lag <= 0 || lag > 64) return CCE_ERR_INVALID_ARG;
  g_stripe_order.store(order);
  g_stripe_gm.store(group_m2);
  g_stripe_lag.store(lag);
  return CCE_OK;
}

cce_status_t cce_debug_set_reduce_prefetch(int slices) {
  if (slices < 0 || slices > 64) return CCE_ERR_INVALID_ARG;
  g_bwd_red_pf.store(slices);
  return CCE_OK;
}

cce_status_t cce_debug_set_l2_hints(int on) {
  if (on < 0 || on > 1) return CCE_ERR_INVALID_ARG;
  g_bwd_l2_hints.store(on);
  return CCE_OK;
}

cce_status_t cce_debug_set_backward_trace(uint64_t* trace, int64_t tiles_per_cta) {
  if (trace && (tiles_per_cta <= 0 || tiles_per_cta > (1 << 20))) return CCE_ERR_INVALID_ARG;
  g_bwd_trace_cap.store(trace ? (int)tiles_per_cta : 0);
  g_bwd_trace.store(reinterpret_cast<unsigned long long*>(trace));
  return CCE_OK;
}

int64_t cce_debug_stripe_schedule(int n_m2, int n_vtile, int n_dc, int vt_per_s, int nbuf, int order, int group_m2,
                                  int lag, int32_t* out, int64_t max_tasks) {
  if (n_m2 <= 0 || n_vtile <= 0 || n_dc <= 0 || vt_per_s <= 0 || nbuf <= 0) return -1;
  if (order < 0 || order > 1 || group_m2 <= 0 || lag <= 0) return -1;
  StripePlan p{};
  p.n_m2 = n_m2;
  p.n_vtile = n_vtile;
  p.n_dc = n_dc;
  p.vt_per_s = vt_per_s;
  p.n_s = (n_vtile + vt_per_s - 1) / vt_per_s;
  p.nbuf = std::min(nbuf, p.n_s);
  p.order = order;
  p.gm = group_m2;
  p.lag = lag;
  const long long total = stripe_total(p);
  if (out) {
    for (long long t = 0; t < total + 1 && t < max_tasks; ++t) {
      const StripeTaskDesc d = stripe_decode(p, t);
      out[4 * t + 0] = d.type;
      out[4 * t + 1] = d.s;
      out[4 * t + 2] = d.a;
      out[4 * t + 3] = d.b;
    }
  }
  return total;
}

cce_status_t cce_debug_set_forward_variant(int variant) {
  if (variant < 0 || variant > 1) return CCE_ERR_INVALID_ARG;
  g_fwd_variant.store(variant);
  return CCE_OK;
}

cce_status_t cce_debug_set_backward_variant(int variant) {
  if (variant < 0 || variant > 3) return CCE_ERR_INVALID_ARG;
  g_bwd_variant.store(variant);
  return CCE_OK;
}

cce_status_t cce_debug_set_kernel_events(int kernel, void* start_event, void* stop_event) {
  if (kernel < 0 || kernel > 1) return CCE_ERR_INVALID_ARG;
  g_events[kernel][0].store(start_event);
  g_events[kernel][1].store(stop_event);
  return CCE_OK;
}

}  // extern "C"

namespace {

// Dense backward through softmax-gradient stripes (bwd_stripe.cu): one
// launch per token super-block; a: the common backward arguments.
cce_status_t backward_stripes(const void* E, const void* C, void* dE, void* dC, const BwdPlan& bp, const BwdArgs& a,
                              bool accumulate, bool ordered, int sms, char* ws, cudaStream_t stream,
                              const int* blk_flat = nullptr) {
  const StripeLayout& L = bp.stripes;
  void* G = ws + L.off_G;
  CUtensorMap maps[9];
  const int64_t Grows = (int64_t)L.p.nbuf * L.Ns_pad;
  if (!make_map(&maps[0], E, a.N, a.D, 128) || !make_map(&maps[1], C, a.V, a.D, 128) ||
      !make_map(&maps[2], G, Grows, L.Vs, 32) || !make_map(&maps[3], G, Grows, L.Vs, 128) ||
      !make_map(&maps[4], G, Grows, L.Vs, 64) || !make_map(&maps[5], E, a.N, a.D, 64) ||
      !make_map(&maps[6], C, a.V, a.D, 64) || !make_map_f32(&maps[7], dE, a.N, a.D) ||
      !make_map_f32(&maps[8], dC, a.V, a.D))
    return CCE_ERR_CUDA;
  unsigned char* ctr = reinterpret_cast<unsigned char*>(ws + L.off_ctr);
  StripeArgs sa{};
  sa.N = a.N;
  sa.D = a.D;
  sa.V = a.V;
  sa.Vs = L.Vs;
  sa.ignore_index = a.ignore_index;
  sa.shard_mode = a.shard_mode;
  sa.v_offset = a.v_offset;
  sa.y = a.y;
  sa.lse = a.lse;
  sa.dloss = a.dloss;
  sa.next = reinterpret_cast<unsigned long long*>(ctr);
  sa.doneA_v = reinterpret_cast<unsigned*>(ctr + 8);
  sa.doneA_ms = sa.doneA_v + L.n_doneA_v;
  sa.doneBC = sa.doneA_ms + L.n_doneA_ms;
  sa.doneC = sa.doneBC + L.n_doneBC;
  sa.nz = a.filter_eps > 0.f ? reinterpret_cast<unsigned char*>(sa.doneC + L.n_doneC) : nullptr;
  sa.blk_flat = blk_flat;
  sa.ordered = ordered ? 1 : 0;
  sa.status = a.status;
  sa.wait_limit_ns = a.wait_limit_ns;
  sa.withhold_loads = a.withhold_loads;
  sa.trace = a.trace;
  sa.trace_cap = a.trace_cap;
  sa.dE_prefetch = g_stripe_dE_pf.load();
  sa.filter_eps = a.filter_eps;
  const int grid = sms & ~1;
  const int n_m2_total = (a.N + 255) / 256;
  const int m2_per_launch = std::max(1, std::min(L.p.n_m2, g_stripe_m2.load()));
  const int n_sb = (n_m2_total + m2_per_launch - 1) / m2_per_launch;
  if (record_event(1, 0, stream) != cudaSuccess) return CCE_ERR_CUDA;
  for (int sb = 0; sb < n_sb; ++sb) {
    sa.p = L.p;
    sa.p.n_m2 = std::min(m2_per_launch, n_m2_total - sb * m2_per_launch);
    sa.tok0 = sb * m2_per_launch * 256;
    sa.Ns_pad = sa.p.n_m2 * 256;   // buffer row stride of this launch
    sa.dC_add = (accumulate || sb > 0) ? 1 : 0;
    if (cudaMemsetAsync(ctr, 0, L.ctr_bytes, stream) != cudaSuccess) return CCE_ERR_CUDA;
    if (launch_bwd_stripe(maps, sa, G, grid, stream) != cudaSuccess) return CCE_ERR_CUDA;
  }
  if (record_event(1, 1, stream) != cudaSuccess) return CCE_ERR_CUDA;
  return CCE_OK;
}

// shard: C is the vocabulary shard starting at global label id v_offset;
// dC is that shard's gradient and dE this shard's share of the full dE.
cce_status_t backward_impl(const void* E, const void* C, const int64_t* y, const float* lse, const float* dloss,
                           int64_t N, int64_t D, int64_t V, int64_t ignore_index, float filter_eps, unsigned flags,
                           void* dE, void* dC, void* workspace, size_t workspace_bytes, void* stream_,
                           bool shard = false, int64_t v_offset = 0) {
  if (!E || !C || !y || !lse || !dloss || !dE || !dC || !workspace) return CCE_ERR_INVALID_ARG;
  if (v_offset < 0) return CCE_ERR_INVALID_ARG;
  if (flags & ~kBwdFlagsAll) return CCE_ERR_INVALID_ARG;
  const bool fixed = uses_fixed_point(flags);
  const bool bf16_out = (flags & CCE_BWD_BF16_GRADS) != 0;
  const bool accumulate = (flags & CCE_BWD_ACCUMULATE) != 0;
  if (!sizes_ok(N, D, V)) return CCE_ERR_INVALID_ARG;
  if (!(filter_eps == filter_eps)) return CCE_ERR_INVALID_ARG;  // NaN
  if (!aligned(E, 16) || !aligned(C, 16) || !aligned(y, 8) || !aligned(lse, 4) || !aligned(dloss, 4) ||
      !aligned(dE, 16) || !aligned(dC, 16) || !aligned(workspace, 256))
    return CCE_ERR_MISALIGNED;
  BwdPlan bp;
  if (!plan_backward(N, D, V, &bp, flags)) return CCE_ERR_INVALID_ARG;
  DeviceInfo di = device_info();
  if (!di.ok) return CCE_ERR_UNSUPPORTED_DEVICE;
  if (workspace_bytes < bp.ws_bytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

  CUtensorMap tmE, tmC, tmCq, tmdE, tmdC;
  char* ws = reinterpret_cast<char*>(workspace);
  unsigned long long* status = reinterpret_cast<unsigned long long*>(ws);
  unsigned long long* accE = fixed ? reinterpret_cast<unsigned long long*>(ws + bp.off_accE) : nullptr;
  unsigned long long* accC = fixed ? reinterpret_cast<unsigned long long*>(ws + bp.off_accC) : nullptr;
  // the reduction targets: fp32 dE / dC, or in fixed-point mode the int64
  // accumulators (dE / dC may then hold bf16)
  const bool red_maps_ok = fixed ? (make_map_u64(&tmdE, accE, N, D) && make_map_u64(&tmdC, accC, V, D))
                                 : (make_map_f32(&tmdE, dE, N, D) && make_map_f32(&tmdC, dC, V, D));
  if (!make_map(&tmE, E, N, D, BM) || !make_map(&tmC, C, V, D, BN) || !make_map(&tmCq, C, V, D, 64) ||
      !red_maps_ok)
    return CCE_ERR_CUDA;
  const bool filter_on = filter_eps > 0.f;
  const bool prepared = (flags & CCE_BWD_PREPARED) != 0;
  // the tokens' maximum logits from cce_backward_prepare_rows bound the
  // logits exactly; the filter then needs neither |E_i| nor max_v |C_v|
  const bool row_max = (flags & CCE_BWD_ROW_MAX) != 0 && filter_on;
  const bool stripes = (flags & CCE_BWD_STRIPES) != 0 && !fixed;
  // bf16 outputs through the stripe path: every sum goes to fp32 scratch in
  // the workspace (fresh each call), rounded to bf16 once at the end
  const bool stripes_bf16 = stripes && bf16_out;
  float* dE32 = stripes_bf16 ? reinterpret_cast<float*>(ws + bp.off_accE) : reinterpret_cast<float*>(dE);
  float* dC32 = stripes_bf16 ? reinterpret_cast<float*>(ws + bp.off_accC) : reinterpret_cast<float*>(dC);
  const bool acc32 = accumulate && !stripes_bf16;
  if ((prepared || row_max) && (filter_on || fixed)) {
    // keep header words HDR_CMAX (cce_backward_prepare) and HDR_ROWMAX
    // (cce_backward_prepare_rows); clear the rest
    char* hdr0 = ws + bp.off_hdr;
    if (cudaMemsetAsync(ws, 0, bp.off_hdr, stream) != cudaSuccess ||
        (!prepared && cudaMemsetAsync(hdr0 + HDR_CMAX * 4, 0, 4, stream) != cudaSuccess) ||
        cudaMemsetAsync(hdr0 + HDR_NNF * 4, 0, 4, stream) != cudaSuccess ||
        (!row_max && cudaMemsetAsync(hdr0 + HDR_ROWMAX * 4, 0, 4, stream) != cudaSuccess) ||
        cudaMemsetAsync(hdr0 + HDR_T * 4, 0, bp.zero_bytes - bp.off_hdr - HDR_T * 4, stream) != cudaSuccess)
      return CCE_ERR_CUDA;
  } else if (cudaMemsetAsync(ws, 0, (filter_on || fixed) ? bp.zero_bytes : STATUS_BYTES, stream) != cudaSuccess) {
    return CCE_ERR_CUDA;
  }
  if (fixed) {
    if (cudaMemsetAsync(accE, 0, (size_t)N * D * 8, stream) != cudaSuccess) return CCE_ERR_CUDA;
    // with the filter on only visited vocabulary tiles are cleared, after the pre-pass
    if (!filter_on && cudaMemsetAsync(accC, 0, (size_t)V * D * 8, stream) != cudaSuccess) return CCE_ERR_CUDA;
  } else if (!acc32) {
    if (cudaMemsetAsync(dE32, 0, (size_t)N * D * sizeof(float), stream) != cudaSuccess) return CCE_ERR_CUDA;
    // (the stripe path writes every entry of dC)
    if (!stripes && cudaMemsetAsync(dC, 0, (size_t)V * D * sizeof(float), stream) != cudaSuccess)
      return CCE_ERR_CUDA;
  }

  BwdArgs a;
  a.N = (int)N;
  a.D = (int)D;
  a.V = (int)V;
  a.n_mblk = bp.n_mblk;
  a.n_vtile = bp.n_vtile;
  a.n_tiles = bp.n_mblk * bp.n_vtile;
  a.group_m = std::min(a.n_mblk, 64);
  a.list_mode = filter_on ? 1 : 0;
  a.shard_mode = shard ? 1 : 0;
  a.v_offset = v_offset;
  a.hdr = reinterpret_cast<const unsigned*>(ws + bp.off_hdr);
  a.nonflat = reinterpret_cast<const int*>(ws + bp.off_nonflat);
  a.filter_eps = filter_eps;
  a.ignore_index = ignore_index;
  a.y = y;
  a.lse = lse;
  a.dloss = dloss;
  a.dE = reinterpret_cast<float*>(dE);
  a.dC = reinterpret_cast<float*>(dC);
  a.accE = accE;
  a.accC = accC;
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.withhold_loads = g_withhold_loads.load();
  a.pf = g_bwd_pf.load();
  a.red_pf = g_bwd_red_pf.load();
  a.l2_hints = g_bwd_l2_hints.load();
  a.trace = g_bwd_trace.load();
  a.trace_cap = g_bwd_trace_cap.load();

  const bool ordered = (flags & CCE_BWD_DETERMINISTIC) != 0;
  // bf16 outputs of the stripe path: the fp32 scratch sums rounded once
  auto finish_stripes = [&]() -> cce_status_t {
    if (!stripes_bf16) return CCE_OK;
    if (launch_f32_to_bf16(dE32, dE, (size_t)N * D, accumulate, di.sms, stream) != cudaSuccess ||
        launch_f32_to_bf16(dC32, dC, (size_t)V * D, accumulate, di.sms, stream) != cudaSuccess)
      return CCE_ERR_CUDA;
    return CCE_OK;
  };
  // the dense backward, and the stripe-ordered (bitwise reproducible) one
  // with the filter: the stripe kernel alone, no pre-pass (the flat-row
  // kernel's fp32 additions into shared dC rows would not be reproducible)
  if (stripes && (!filter_on || ordered)) {
    const cce_status_t st = backward_stripes(E, C, dE32, dC32, bp, a, acc32, ordered, di.sms, ws, stream);
    return st != CCE_OK ? st : finish_stripes();
  }
  FlatArgs fa{};
  if (filter_on || fixed) {
    PrepArgs pp;
    pp.N = (int)N;
    pp.D = (int)D;
    pp.V = (int)V;
    pp.n_mblk = bp.n_mblk;
    pp.n_vtile = bp.n_vtile;
    pp.ignore_index = ignore_index;
    pp.shard_mode = shard ? 1 : 0;
    pp.v_offset = v_offset;
    pp.log_eps = logf(filter_eps);
    pp.hdr = reinterpret_cast<unsigned*>(ws + bp.off_hdr);
    pp.rowbits = reinterpret_cast<unsigned*>(ws + bp.off_rowbits);
    pp.blk_flat = reinterpret_cast<int*>(ws + bp.off_flat);
    pp.nonflat = reinterpret_cast<int*>(ws + bp.off_nonflat);
    pp.enorm = reinterpret_cast<float*>(ws + bp.off_enorm);
    pp.row_max = row_max ? reinterpret_cast<const float*>(ws + bp.off_rowmax) : nullptr;
    pp.status = status;
    // the norms bound the logits (unless the row maxima do) and scale the
    // fixed-point accumulation
    if (!prepared && (fixed || !row_max) && launch_cnorm(C, pp, di.sms, stream) != cudaSuccess)
      return CCE_ERR_CUDA;
    if ((fixed || !row_max) && launch_enorm(E, pp, di.sms, stream) != cudaSuccess) return CCE_ERR_CUDA;
    if (filter_on && launch_prep(E, C, y, lse, pp, di.sms, stream) != cudaSuccess) return CCE_ERR_CUDA;
    if (fixed && launch_fixed_prep(dloss, pp, di.sms, stream) != cudaSuccess) return CCE_ERR_CUDA;
    if (fixed && filter_on &&
        launch_clear_visited_rows(accC, (int)V, (int)D, pp.rowbits, pp.hdr, di.sms, stream) != cudaSuccess)
      return CCE_ERR_CUDA;
    if (filter_on) {
      // the label entries of the flat blocks (their other entries are all below eps)
      fa.N = (int)N;
      fa.D = (int)D;
      fa.V = (int)V;
      fa.ignore_index = ignore_index;
      fa.shard_mode = shard ? 1 : 0;
      fa.v_offset = v_offset;
      fa.filter_eps = filter_eps;
      fa.accumulate = acc32 ? 1 : 0;
      fa.blk_flat = pp.blk_flat;
      fa.hdr = pp.hdr;
      fa.dE = dE32;
      fa.dC = dC32;
      fa.accE = accE;
      fa.accC = accC;
      fa.status = status;
      if (!stripes && launch_flat_rows(E, C, y, lse, dloss, fa, stream) != cudaSuccess) return CCE_ERR_CUDA;
    }
  }
  if (stripes) {
    // the blocks that are not flat through the stripe kernel (which stores
    // every dC tile), then the flat blocks' label entries added on top
    const cce_status_t st = backward_stripes(E, C, dE32, dC32, bp, a, acc32, ordered, di.sms, ws, stream,
                                             reinterpret_cast<const int*>(ws + bp.off_flat));
    if (st != CCE_OK) return st;
    if (launch_flat_rows(E, C, y, lse, dloss, fa, stream) != cudaSuccess) return CCE_ERR_CUDA;
    return finish_stripes();
  }
  const int grid = filter_on ? di.sms : std::min(a.n_tiles, di.sms);
  if (record_event(1, 0, stream) != cudaSuccess) return CCE_ERR_CUDA;
  if (launch_bwd(tmE, tmC, tmCq, tmdE, tmdC, a, grid, g_bwd_variant.load(), stream) != cudaSuccess) return CCE_ERR_CUDA;
  if (record_event(1, 1, stream) != cudaSuccess) return CCE_ERR_CUDA;
  if (fixed) {
    const unsigned* hdr = reinterpret_cast<const unsigned*>(ws + bp.off_hdr);
    const unsigned* rowbits = filter_on ? reinterpret_cast<const unsigned*>(ws + bp.off_rowbits) : nullptr;
    if (launch_fixed_to_out(accE, dE, (int)N, (int)D, hdr, (int)N, bf16_out, accumulate, nullptr, di.sms,
                            stream) != cudaSuccess ||
        launch_fixed_to_out(accC, dC, (int)V, (int)D, hdr, (int)N, bf16_out, accumulate, rowbits, di.sms,
                            stream) != cudaSuccess)
      return CCE_ERR_CUDA;
  }
  return CCE_OK;
}

}  // namespace

extern "C" {

size_t cce_backward_workspace_size_ex(int64_t N, int64_t D, int64_t V, unsigned flags) {
  BwdPlan p;
  if (!plan_backward(N, D, V, &p, flags)) return 0;
  return p.ws_bytes;
}

cce_status_t cce_backward_ex(const void* E, const void* C, const int64_t* y, const float* lse, const float* dloss,
                             int64_t N, int64_t D, int64_t V, int64_t ignore_index, float filter_eps, unsigned flags,
                             void* dE, void* dC, void* workspace, size_t workspace_bytes, void* stream) {
  return backward_impl(E, C, y, lse, dloss, N, D, V, ignore_index, filter_eps, flags, dE, dC, workspace,
                       workspace_bytes, stream);
}

cce_status_t cce_backward(const void* E, const void* C, const int64_t* y, const float* lse, const float* dloss,
                          int64_t N, int64_t D, int64_t V, int64_t ignore_index, float filter_eps, float* dE,
                          float* dC, void* workspace, size_t workspace_bytes, void* stream) {
  return backward_impl(E, C, y, lse, dloss, N, D, V, ignore_index, filter_eps, 0u, dE, dC, workspace,
                       workspace_bytes, stream);
}

cce_status_t cce_backward_prepare(const void* C, int64_t N, int64_t D, int64_t V, void* workspace,
                                  size_t workspace_bytes, void* stream_) {
  if (!C || !workspace) return CCE_ERR_INVALID_ARG;
  if (!sizes_ok(N, D, V)) return CCE_ERR_INVALID_ARG;
  if (!aligned(C, 16) || !aligned(workspace, 256)) return CCE_ERR_MISALIGNED;
  BwdPlan bp;
  if (!plan_backward(N, D, V, &bp)) return CCE_ERR_INVALID_ARG;
  DeviceInfo di = device_info();
  if (!di.ok) return CCE_ERR_UNSUPPORTED_DEVICE;
  if (workspace_bytes < bp.ws_bytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  char* ws = reinterpret_cast<char*>(workspace);
  unsigned* hdr = reinterpret_cast<unsigned*>(ws + bp.off_hdr);
  if (cudaMemsetAsync(hdr + HDR_CMAX, 0, sizeof(unsigned), stream) != cudaSuccess) return CCE_ERR_CUDA;
  PrepArgs pp{};
  pp.N = (int)N;
  pp.D = (int)D;
  pp.V = (int)V;
  pp.hdr = hdr;
  if (launch_cnorm(C, pp, di.sms, stream) != cudaSuccess) return CCE_ERR_CUDA;
  return CCE_OK;
}

cce_status_t cce_backward_prepare_rows(const float* row_max, int64_t N, int64_t D, int64_t V, void* workspace,
                                       size_t workspace_bytes, void* stream_) {
  if (!row_max || !workspace) return CCE_ERR_INVALID_ARG;
  if (!sizes_ok(N, D, V)) return CCE_ERR_INVALID_ARG;
  if (!aligned(row_max, 4) || !aligned(workspace, 256)) return CCE_ERR_MISALIGNED;
  BwdPlan bp;
  if (!plan_backward(N, D, V, &bp)) return CCE_ERR_INVALID_ARG;
  if (workspace_bytes < bp.ws_bytes) return CCE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  char* ws = reinterpret_cast<char*>(workspace);
  if (cudaMemcpyAsync(ws + bp.off_rowmax, row_max, (size_t)N * sizeof(float), cudaMemcpyDeviceToDevice, stream) !=
          cudaSuccess ||
      cudaMemsetAsync(ws + bp.off_hdr + HDR_ROWMAX * 4, 0x01, 4, stream) != cudaSuccess)
    return CCE_ERR_CUDA;
  return CCE_OK;
}

cce_status_t cce_forward_shard(const void* E, const void* C_shard, const int64_t* y, int64_t N, int64_t D,
                               int64_t V_shard, int64_t v_offset, int64_t ignore_index, float* stats,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!stats) return CCE_ERR_INVALID_ARG;
  return forward_impl(E, C_shard, y, N, D, V_shard, ignore_index, nullptr, nullptr, nullptr, workspace,
                      workspace_bytes, stream, stats, v_offset);
}

cce_status_t cce_merge_shards(const float* stats, int R, int64_t N, const int64_t* y, int64_t V_total,
                              int64_t ignore_index, float* loss, float* lse, void* stream) {
  if (!stats || !y || !loss || !lse || R <= 0 || N <= 0 || N > INT_MAX || V_total <= 0) return CCE_ERR_INVALID_ARG;
  if (!aligned(stats, 4) || !aligned(y, 8) || !aligned(loss, 4) || !aligned(lse, 4)) return CCE_ERR_MISALIGNED;
  if (!device_info().ok) return CCE_ERR_UNSUPPORTED_DEVICE;
  if (launch_merge_shards(stats, R, (int)N, y, V_total, ignore_index, loss, lse,
                          reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return CCE_ERR_CUDA;
  return CCE_OK;
}

cce_status_t cce_backward_shard(const void* E, const void* C_shard, const int64_t* y, const float* lse,
                                const float* dloss, int64_t N, int64_t D, int64_t V_shard, int64_t v_offset,
                                int64_t ignore_index, float filter_eps, float* dE_partial, float* dC_shard,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return backward_impl(E, C_shard, y, lse, dloss, N, D, V_shard, ignore_index, filter_eps, 0u, dE_partial,
                       dC_shard, workspace, workspace_bytes, stream, true, v_offset);
}

cce_status_t cce_read_status(const void* workspace, void* stream, cce_counters_t* out) {
  if (!workspace || !out) return CCE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return CCE_ERR_CUDA;
  unsigned long long h[8];
  if (cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return CCE_ERR_CUDA;
  out->flags = h[ST_FLAGS];
  out->live_tiles = h[ST_LIVE_TILES];
  out->dead_tiles = h[ST_DEAD_TILES];
  out->logit_tiles = h[ST_TILES];
  out->pruned_tiles = h[ST_PRUNED];
  out->flat_units = h[ST_FLAT];
  if (h[ST_FLAGS] & SF_TIMEOUT) return CCE_ERR_TIMEOUT;
  if (h[ST_FLAGS] & SF_BAD_LABEL) return CCE_ERR_BAD_LABEL;
  return CCE_OK;
}

const char* cce_status_string(cce_status_t s) {
  switch (s) {
    case CCE_OK: return "CCE_OK";
    case CCE_ERR_INVALID_ARG: return "CCE_ERR_INVALID_ARG";
    case CCE_ERR_MISALIGNED: return "CCE_ERR_MISALIGNED";
    case CCE_ERR_WORKSPACE_TOO_SMALL: return "CCE_ERR_WORKSPACE_TOO_SMALL";
    case CCE_ERR_UNSUPPORTED_DEVICE: return "CCE_ERR_UNSUPPORTED_DEVICE";
    case CCE_ERR_CUDA: return "CCE_ERR_CUDA";
    case CCE_ERR_TIMEOUT: return "CCE_ERR_TIMEOUT";
    case CCE_ERR_BAD_LABEL: return "CCE_ERR_BAD_LABEL";
  }
  return "CCE_ERR_UNKNOWN";
}

int cce_version(void) { return 103; }

}  // extern "C"
