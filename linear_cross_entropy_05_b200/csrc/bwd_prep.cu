// Backward pre-pass: the list of logit tiles the backward must recompute.
//
// The gradient filter (Cut Cross-Entropy abstract, sentence 9) drops every
// entry of the softmax gradient with |P - onehot| < eps.  For a token i and a
// column v that is not its label, P_iv = exp(E_i.C_v - lse_i) and, by
// Cauchy-Schwarz, E_i.C_v <= |E_i| |C_v| (or, when the forward's maximum
// logit of each token is at hand, E_i.C_v <= max_v E_i.C_v exactly).  So if
// |E_i| * max_v |C_v| (or that maximum) < lse_i + ln(eps) for every kept
// token of a 128-token block, every entry of
// that block's rows except the label entries is dropped, and no logit of the
// block needs to be recomputed: the label entry P_iy - 1 needs only the
// correct-token logit E_i . C_y and lse_i.  Such a block is "flat"; its
// tokens go to the flat-row kernel.  Blocks that are not flat are visited
// densely by the tile kernel, which tests every entry.  The result equals
// that of the dense recompute with the same filter.
//
// Kernels (stream order):
//   prep_cnorm    max_v |C_v| (fp32, atomicMax on the float's bits)
//   prep_enorm    |E_i| per token (and the maximum)
//   prep_blocks   per token block: flatness; marks the dC rows (labels)
//                 that flat blocks can touch
//   prep_totals   totals: the tiles to visit (every tile of each block that
//                 is not flat)
//   flat_rows     the label entries of the flat blocks' tokens, formed
//                 directly (no logit tile is recomputed for a flat block)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace cce {

namespace {

__device__ __forceinline__ float sumsq_bf16x8(const uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(h[j]);
    s = fmaf(f.x, f.x, s);
    s = fmaf(f.y, f.y, s);
  }
  return s;
}

__device__ __forceinline__ float warp_row_norm(const __nv_bfloat16* row, int D, int lane) {
  const uint4* r = reinterpret_cast<const uint4*>(row);
  const int nvec = D >> 3;
  float s = 0.f;
  for (int i = lane; i < nvec; i += 32) s += sumsq_bf16x8(__ldg(r + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return sqrtf(s);
}

__device__ __forceinline__ bool label_ok(long long t, long long ignore_index, int V) {
  return t != ignore_index && t >= 0 && t < V;
}

// Filter units (32 tokens x 32 vocabulary entries) inside token block m and
// inside vocabulary tile v, and the pruned-unit counter's update: it starts
// at the number of all units and loses those of every recomputed tile.
__device__ __forceinline__ unsigned long long unit_rows(const PrepArgs& p, int m) {
  return (unsigned long long)min(BM / 32, (p.N - m * BM + 31) / 32);
}
__device__ __forceinline__ void pruned_sub(const PrepArgs& p, unsigned long long units) {
  atomicAdd(p.status + ST_PRUNED, 0ull - units);  // modulo 2^64: order of the updates is free
}

// Row v of dC can receive a gradient only if some token block is not flat
// (its tiles are all visited) or v is the label of a kept token of a flat
// block (rowbits).  The other rows of dC are exactly zero.
__device__ __forceinline__ bool row_visited(const unsigned* rowbits, const unsigned* hdr, int v) {
  return hdr[HDR_NNF] != 0u || ((rowbits[v >> 5] >> (v & 31)) & 1u) != 0u;
}

}  // namespace

__global__ void __launch_bounds__(256) prep_cnorm_kernel(const __nv_bfloat16* __restrict__ C, PrepArgs p) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  float mx = 0.f;
  for (int v = gw; v < p.V; v += nw) mx = fmaxf(mx, warp_row_norm(C + (size_t)v * p.D, p.D, lane));
  if (lane == 0) atomicMax(p.hdr + HDR_CMAX, __float_as_uint(mx));  // non-negative: bit order = value order
}

// |E_i| for every token (one warp per row, all SMs), and their maximum.
__global__ void __launch_bounds__(256) prep_enorm_kernel(const __nv_bfloat16* __restrict__ E, PrepArgs p) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  float mx = 0.f;
  for (int i = gw; i < p.N; i += nw) {
    const float n = warp_row_norm(E + (size_t)i * p.D, p.D, lane);
    if (lane == 0) p.enorm[i] = n;
    mx = fmaxf(mx, n);
  }
  if (lane == 0) atomicMax(p.hdr + HDR_EMAX, __float_as_uint(mx));
}

// One CTA (128 threads) per token block.
__global__ void __launch_bounds__(128) prep_blocks_kernel(const int64_t* __restrict__ y,
                                                          const float* __restrict__ lse, PrepArgs p) {
  const int m = blockIdx.x;
  const int t = threadIdx.x;
  const int row = m * BM + t;
  long long yl = row < p.N ? y[row] : p.ignore_index;
  // kept token (its softmax row matters for flatness) and, separately, whether
  // its label has a column in this C (always, unless C is a vocabulary shard)
  const bool valid = row < p.N && (p.shard_mode ? yl != p.ignore_index : label_ok(yl, p.ignore_index, p.V));
  if (!p.shard_mode && row < p.N && yl != p.ignore_index && !valid) atomicOr(p.status + ST_FLAGS, SF_BAD_LABEL);
  const long long ylocal = yl - (p.shard_mode ? p.v_offset : 0);
  const bool has_col = valid && ylocal >= 0 && ylocal < p.V;
  // Margins cover the fp32 rounding of the norms (or of the forward's
  // maximum against the backward's recomputed logits) and of the exp2 in
  // the exact test.
  const float margin = 1.0f / 1024.0f;
  bool flat = true;
  if (p.row_max && p.hdr[HDR_ROWMAX] == 0u) {
    flat = false;  // row maxima asked for but not stored for this call: visit every tile (exact, slower)
  } else if (valid) {
    // an upper bound of max_v E_i . C_v: the forward's exact maximum when
    // given, else Cauchy-Schwarz
    const float zmax = p.row_max ? p.row_max[row] + margin * (1.0f + fabsf(p.row_max[row]))
                                 : p.enorm[row] * __uint_as_float(p.hdr[HDR_CMAX]) * (1.0f + margin) + margin;
    flat = zmax < lse[row] + p.log_eps - margin;
  }
  const int all_flat = __syncthreads_and(flat);
  if (t == 0) p.blk_flat[m] = all_flat;
  if (!all_flat) {
    if (t == 0) {
      p.nonflat[atomicAdd(p.hdr + HDR_NNF, 1u)] = m;
      pruned_sub(p, unit_rows(p, m) * (((unsigned long long)p.V + 31ull) / 32ull));  // visited densely
    }
    return;
  }
  // flat block: the flat-row kernel touches row ylocal of dC
  if (has_col) atomicOr(p.rowbits + (ylocal >> 5), 1u << (ylocal & 31));
}

// Totals into the header once every block is classified: the tiles to visit
// are every tile of each block that is not flat (vocabulary-major), and the
// pruned-unit counter starts from all units (prep_blocks took off the dense
// blocks' units, flat_rows takes off the flat blocks' live label units).
__global__ void prep_totals_kernel(PrepArgs p) {
  if (threadIdx.x != 0) return;
  const unsigned nnf = p.hdr[HDR_NNF];
  p.hdr[HDR_T] = (unsigned)((unsigned long long)nnf * (unsigned long long)p.n_vtile);
  p.hdr[HDR_ROWMAX] = 0u;  // the row maxima serve one backward: the next needs cce_backward_prepare_rows again
  atomicAdd(p.status + ST_PRUNED,
            (((unsigned long long)p.N + 31ull) / 32ull) * (((unsigned long long)p.V + 31ull) / 32ull));
}

// Flat token blocks: one CTA (32 warps) per 32-token row group, one warp per
// token.  A kept token whose label column lies in this C has
//   z = E_i . C_y,  p = exp(z - lse_i),  d = p - 1,
// its only entry with |d| >= filter_eps (the pre-pass proved all others
// below it); if |d| >= eps, G = dloss_i d adds G C_y to dE_i (the warp owns
// the row: plain stores) and G E_i to dC_y.  Tokens share labels, so the dC
// row is added with bulk reduce-adds: the warp writes 1 KB pieces of G E_i
// (fp32, or int64 fixed point in the deterministic mode) into one of two
// shared-memory buffers and one lane hands each piece to the TMA engine,
// which adds it at L2 -- 9 operations per 2304-wide row instead of 576
// vector (or 2304 64-bit) atomics.  The live 32 x 32 units of the row group
// are its distinct live label chunks; they move from the pruned to the live
// count.
constexpr int FLAT_PIECE = 1024;                           // bytes per bulk reduce-add
constexpr int FLAT_SMEM = 32 * 2 * FLAT_PIECE;             // two pieces per warp

__global__ void __launch_bounds__(1024) flat_rows_kernel(const __nv_bfloat16* __restrict__ E,
                                                         const __nv_bfloat16* __restrict__ C,
                                                         const int64_t* __restrict__ y,
                                                         const float* __restrict__ lse,
                                                         const float* __restrict__ dloss, FlatArgs f) {
  extern __shared__ __align__(128) uint8_t flat_smem[];
  __shared__ int chunk_of[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g0 = blockIdx.x * 32;              // first token of the row group
  if (!f.blk_flat[g0 / BM]) return;            // whole CTA: a row group lies in one token block
  const int row = g0 + warp;
  int live_chunk = -1;
  if (row < f.N) {
    const long long yg = y[row];
    const long long yl = yg - (f.shard_mode ? f.v_offset : 0);
    if (yg != f.ignore_index && yl >= 0 && yl < f.V) {
      const uint4* er = reinterpret_cast<const uint4*>(E + (size_t)row * f.D);
      const uint4* cr = reinterpret_cast<const uint4*>(C + (size_t)yl * f.D);
      const int nvec = f.D >> 3;
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
      const float d = expf(z - lse[row]) - 1.f;
      if (fabsf(d) >= f.filter_eps) {
        live_chunk = (int)(yl >> 5);
        const float g = dloss[row] * d;
        const bool fixed = f.accE != nullptr;
        const float scale =
            fixed ? ldexpf(1.f, fixed_point_exponent(__uint_as_float(f.hdr[HDR_CMAX]), __uint_as_float(f.hdr[HDR_EMAX]),
                                                     __uint_as_float(f.hdr[HDR_DLMAX]), f.N))
                  : 0.f;
        // elements per piece: 256 fp32 or 128 int64; a lane takes 8 or 4 of them
        const int per_piece = fixed ? FLAT_PIECE / 8 : FLAT_PIECE / 4;
        const int per_lane = per_piece / 32;
        uint8_t* wbuf = flat_smem + warp * 2 * FLAT_PIECE;
        const int npieces = (f.D + per_piece - 1) / per_piece;
        for (int c = 0; c < npieces; ++c) {
          uint8_t* buf = wbuf + (c & 1) * FLAT_PIECE;
          if (c >= 2) {
            if (lane == 0) bulk_wait_group_read<1>();  // the reduce-add of piece c - 2 has read this buffer
            __syncwarp();
          }
          const int e0 = c * per_piece + lane * per_lane;  // this lane's first element
          const int n_el = min(per_piece, f.D - c * per_piece);
          if (e0 < f.D) {
            const size_t oe = (size_t)row * f.D + e0;
            if (fixed) {
              const uint2 ev = *reinterpret_cast<const uint2*>(E + (size_t)row * f.D + e0);
              const uint2 cv = *reinterpret_cast<const uint2*>(C + (size_t)yl * f.D + e0);
              const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&ev);
              const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&cv);
              unsigned long long qe[4], qc[4];
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const float2 ef = __bfloat1622float2(e2[j]);
                const float2 cf = __bfloat1622float2(c2[j]);
                qc[2 * j] = (unsigned long long)__float2ll_rn(g * ef.x * scale);
                qc[2 * j + 1] = (unsigned long long)__float2ll_rn(g * ef.y * scale);
                qe[2 * j] = (unsigned long long)__float2ll_rn(g * cf.x * scale);
                qe[2 * j + 1] = (unsigned long long)__float2ll_rn(g * cf.y * scale);
              }
              // this warp owns dE_i (the accumulator starts at zero)
              ulonglong2* ae = reinterpret_cast<ulonglong2*>(f.accE + oe);
              ae[0] = make_ulonglong2(qe[0], qe[1]);
              ae[1] = make_ulonglong2(qe[2], qe[3]);
              ulonglong2* sb = reinterpret_cast<ulonglong2*>(buf + lane * per_lane * 8);
              sb[0] = make_ulonglong2(qc[0], qc[1]);
              sb[1] = make_ulonglong2(qc[2], qc[3]);
            } else {
              const uint4 ev = *reinterpret_cast<const uint4*>(E + (size_t)row * f.D + e0);
              const uint4 cv = *reinterpret_cast<const uint4*>(C + (size_t)yl * f.D + e0);
              const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&ev);
              const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&cv);
              float ce[8], ee[8];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 cf = __bfloat1622float2(c2[j]);
                const float2 ef = __bfloat1622float2(e2[j]);
                ce[2 * j] = g * cf.x;
                ce[2 * j + 1] = g * cf.y;
                ee[2 * j] = g * ef.x;
                ee[2 * j + 1] = g * ef.y;
              }
              float4* de = reinterpret_cast<float4*>(f.dE + oe);
              float4 a0 = make_float4(ce[0], ce[1], ce[2], ce[3]), a1 = make_float4(ce[4], ce[5], ce[6], ce[7]);
              if (f.accumulate) {
                const float4 o0 = de[0], o1 = de[1];
                a0 = make_float4(o0.x + a0.x, o0.y + a0.y, o0.z + a0.z, o0.w + a0.w);
                a1 = make_float4(o1.x + a1.x, o1.y + a1.y, o1.z + a1.z, o1.w + a1.w);
              }
              de[0] = a0;
              de[1] = a1;
              float4* sb = reinterpret_cast<float4*>(buf + lane * per_lane * 4);
              sb[0] = make_float4(ee[0], ee[1], ee[2], ee[3]);
              sb[1] = make_float4(ee[4], ee[5], ee[6], ee[7]);
            }
          }
          fence_proxy_async_smem();  // the generic-proxy writes above, seen by the TMA engine
          __syncwarp();
          if (lane == 0) {
            const size_t oc = (size_t)yl * f.D + (size_t)c * per_piece;
            if (fixed)
              bulk_reduce_add_u64(f.accC + oc, buf, (uint32_t)n_el * 8u);
            else
              bulk_reduce_add_f32(f.dC + oc, buf, (uint32_t)n_el * 4u);
            bulk_commit_group();
          }
        }
        if (lane == 0) bulk_wait_group0();  // sources read and adds done before the CTA exits
        __syncwarp();
      }
    }
  }
  if (lane == 0) chunk_of[warp] = live_chunk;
  __syncthreads();
  if (warp == 0) {
    const int c = chunk_of[lane];
    const unsigned same = __match_any_sync(0xffffffffu, c);
    const bool first = (__ffs(same) - 1) == lane;  // one lane per distinct chunk
    const unsigned n = __popc(__ballot_sync(0xffffffffu, first && c >= 0));
    if (lane == 0 && n) {
      atomicAdd(f.status + ST_LIVE_TILES, (unsigned long long)n);
      atomicAdd(f.status + ST_FLAT, (unsigned long long)n);
      atomicAdd(f.status + ST_PRUNED, 0ull - (unsigned long long)n);
    }
  }
}

cudaError_t launch_flat_rows(const void* E, const void* C, const int64_t* y, const float* lse, const float* dloss,
                             const FlatArgs& f, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(flat_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FLAT_SMEM);
  if (e != cudaSuccess) return e;
  flat_rows_kernel<<<(f.N + 31) / 32, 1024, FLAT_SMEM, stream>>>(reinterpret_cast<const __nv_bfloat16*>(E),
                                                                 reinterpret_cast<const __nv_bfloat16*>(C), y, lse,
                                                                 dloss, f);
  return cudaGetLastError();
}

// Deterministic mode: max_i |dloss_i| for the fixed-point scale (max_i |E_i|
// comes from prep_enorm; maxima do not depend on the order of the atomics).
__global__ void __launch_bounds__(256) prep_fixed_kernel(const float* __restrict__ dloss, PrepArgs p) {
  const int lane = threadIdx.x & 31;
  float dmax = 0.f;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.N; i += gridDim.x * blockDim.x)
    dmax = fmaxf(dmax, fabsf(dloss[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
  if (lane == 0) atomicMax(p.hdr + HDR_DLMAX, __float_as_uint(dmax));
}

// Deterministic mode: int64 fixed-point accumulators -> fp32 or bf16 output
// (written, or with accumulate added to what the output holds: one add per
// entry, so the result stays reproducible).  The n values are `rows` rows of
// D.  When rowbits is non-null the accumulator is dC and only its visited
// rows (row_visited) were cleared and accumulated: the others are exactly
// zero and are not read (written as zeros, or left alone when accumulating).
// One warp per row.
__global__ void __launch_bounds__(256) fixed_to_out_kernel(const unsigned long long* __restrict__ acc, void* out,
                                                           int rows, int D, const unsigned* __restrict__ hdr, int N,
                                                           int bf16, int accumulate,
                                                           const unsigned* __restrict__ rowbits) {
  const int s = fixed_point_exponent(__uint_as_float(hdr[HDR_CMAX]), __uint_as_float(hdr[HDR_EMAX]),
                                     __uint_as_float(hdr[HDR_DLMAX]), N);
  const double inv = ldexp(1.0, -s);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int h = D >> 1;  // value pairs per row (D is even)
  for (int row = gw; row < rows; row += nw) {
    const bool live_row = rowbits == nullptr || row_visited(rowbits, hdr, row);
    if (!live_row && accumulate) continue;  // adds nothing: the output keeps its contents
    const ulonglong2* a2 = reinterpret_cast<const ulonglong2*>(acc + (size_t)row * D);
    for (int j = lane; j < h; j += 32) {
      const ulonglong2 q = live_row ? a2[j] : make_ulonglong2(0ull, 0ull);
      double x0 = (double)(long long)q.x * inv, x1 = (double)(long long)q.y * inv;
      const size_t i = (size_t)row * h + j;
      if (bf16) {
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out) + i;
        if (accumulate) {
          const float2 old = __bfloat1622float2(*o);
          x0 += (double)old.x;
          x1 += (double)old.y;
        }
        *o = __halves2bfloat162(__double2bfloat16(x0), __double2bfloat16(x1));
      } else {
        float2* o = reinterpret_cast<float2*>(out) + i;
        float2 r = make_float2((float)x0, (float)x1);
        if (accumulate) {
          const float2 old = *o;
          r.x = old.x + r.x;  // fp32 add of this call's sum, rounded once to fp32
          r.y = old.y + r.y;
        }
        *o = r;
      }
    }
  }
}

// Fixed-point dC accumulator: clear the visited rows only (one warp per row).
__global__ void __launch_bounds__(256) clear_visited_rows_kernel(unsigned long long* __restrict__ acc, int V, int D,
                                                                 const unsigned* __restrict__ rowbits,
                                                                 const unsigned* __restrict__ hdr) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int h = D >> 1;
  for (int row = gw; row < V; row += nw) {
    if (!row_visited(rowbits, hdr, row)) continue;
    ulonglong2* a2 = reinterpret_cast<ulonglong2*>(acc + (size_t)row * D);
    for (int j = lane; j < h; j += 32) a2[j] = make_ulonglong2(0ull, 0ull);
  }
}

cudaError_t launch_clear_visited_rows(unsigned long long* acc, int V, int D, const unsigned* rowbits,
                                      const unsigned* hdr, int sms, cudaStream_t stream) {
  clear_visited_rows_kernel<<<sms * 8, 256, 0, stream>>>(acc, V, D, rowbits, hdr);
  return cudaGetLastError();
}

cudaError_t launch_fixed_prep(const float* dloss, const PrepArgs& p, int sms, cudaStream_t stream) {
  prep_fixed_kernel<<<sms, 256, 0, stream>>>(dloss, p);
  return cudaGetLastError();
}

cudaError_t launch_fixed_to_out(const unsigned long long* acc, void* out, int rows, int D, const unsigned* hdr,
                                int N, bool bf16, bool accumulate, const unsigned* rowbits, int sms,
                                cudaStream_t stream) {
  fixed_to_out_kernel<<<sms * 8, 256, 0, stream>>>(acc, out, rows, D, hdr, N, bf16 ? 1 : 0, accumulate ? 1 : 0,
                                                   rowbits);
  return cudaGetLastError();
}

// bf16 gradient outputs of the stripe path: the fp32 sums, rounded once to
// bf16 (with accumulate, added to what the output holds first).  n % 4 == 0.
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ src, uint2* dst, size_t n4,
                                                          int accumulate) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 v = src[i];
    if (accumulate) {
      const uint2 o = dst[i];
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o.y));
      v = make_float4(v.x + a.x, v.y + a.y, v.z + b.x, v.w + b.y);
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    dst[i] = make_uint2(*reinterpret_cast<const unsigned*>(&lo), *reinterpret_cast<const unsigned*>(&hi));
  }
}

cudaError_t launch_f32_to_bf16(const float* src, void* dst, size_t n, bool accumulate, int sms, cudaStream_t stream) {
  f32_to_bf16_kernel<<<sms * 8, 256, 0, stream>>>(reinterpret_cast<const float4*>(src), reinterpret_cast<uint2*>(dst),
                                                  n / 4, accumulate ? 1 : 0);
  return cudaGetLastError();
}

// Norm pre-pass shared by the filter and the fixed-point scale: max_v |C_v|
// (launch_cnorm; HDR_CMAX must start at zero), |E_i| per token and
// max_i |E_i| (launch_enorm).
cudaError_t launch_cnorm(const void* C, const PrepArgs& p, int sms, cudaStream_t stream) {
  prep_cnorm_kernel<<<sms * 8, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(C), p);
  return cudaGetLastError();
}

cudaError_t launch_enorm(const void* E, const PrepArgs& p, int sms, cudaStream_t stream) {
  prep_enorm_kernel<<<sms * 4, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(E), p);
  return cudaGetLastError();
}

cudaError_t launch_prep(const void* E, const void* C, const int64_t* y, const float* lse, const PrepArgs& p,
                        int sms, cudaStream_t stream) {
  // expects launch_cnorm and launch_enorm to have run
  prep_blocks_kernel<<<p.n_mblk, 128, 0, stream>>>(y, lse, p);
  prep_totals_kernel<<<1, 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace cce
