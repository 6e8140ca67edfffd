// Routing of the (t, k) pairs to experts, activation gather and the k-ordered combine.
//
// The experts interface is (hidden_states, top_k_index, top_k_weights) (unsloth-zoo
// issue #850).  Grouping: counts[e] = #pairs routed to e, offsets = exclusive prefix
// sum, perm = the flat pair index p = t*K + k listed by expert and in increasing p
// within an expert (stable).  A pair whose index is outside [0, E) is dropped.
//
// Work is cut into chunks of kRouteChunk consecutive pairs, one warp per chunk, so
// that the stable order comes from walking each chunk in order (32 pairs at a time,
// ranks inside a step from __match_any_sync) and from chunk bases taken in chunk order.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace moeq {

constexpr int kWarpsPerBlock = 8;
constexpr int kSteps = kRouteChunk / 32;

template <typename IdxT>
__device__ __forceinline__ int load_expert(const IdxT *idx, int p, int S, int E, int32_t *status) {
  if (p >= S) return -1;
  const long long e = static_cast<long long>(idx[p]);
  if (e < 0 || e >= E) {
    report(status, MOEQ_ERR_INDEX);
    return -1;
  }
  return static_cast<int>(e);
}

// Per-chunk histograms counts_chunk[chunk][e].
template <typename IdxT>
__global__ void __launch_bounds__(256) k_route_count(const IdxT *__restrict__ idx, int S, int E,
                                                     int nchunks, int32_t *__restrict__ counts_chunk,
                                                     int32_t *status) {
  extern __shared__ int32_t hist[];  // [kWarpsPerBlock][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kWarpsPerBlock + warp;
  if (chunk >= nchunks) return;  // whole warp; no block-wide barrier below
  int32_t *h = hist + warp * E;
  for (int e = lane; e < E; e += 32) h[e] = 0;
  // all of the warp's index loads first, then the histogram updates
  int ev[kSteps];
#pragma unroll
  for (int st = 0; st < kSteps; ++st) ev[st] = load_expert(idx, chunk * kRouteChunk + st * 32 + lane, S, E, status);
  __syncwarp();
#pragma unroll
  for (int st = 0; st < kSteps; ++st)
    if (ev[st] >= 0) atomicAdd(&h[ev[st]], 1);
  __syncwarp();
  int32_t *dst = counts_chunk + static_cast<size_t>(chunk) * E;
  for (int e = lane; e < E; e += 32) dst[e] = h[e];
}

// Exclusive scan of one value per thread over the block (blockDim.x == 1024).
__device__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
    int z = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, z, d);
      if (lane >= d) z += y;
    }
    warp_tot[lane] = z - w;  // exclusive prefix of warp totals
    if (lane == 31) *total = z;
  }
  __syncthreads();
  const int r = warp_tot[warp] + x - v;
  __syncthreads();
  return r;
}

// Totals per expert, offsets, tile prefix and per-(chunk, expert) bases.
__global__ void __launch_bounds__(1024) k_route_scan(const int32_t *__restrict__ counts_chunk,
                                                     int nchunks, int E,
                                                     int32_t *__restrict__ chunk_base,
                                                     int32_t *__restrict__ counts,
                                                     int32_t *__restrict__ offsets,
                                                     int32_t *__restrict__ ntile_prefix) {
  __shared__ int warp_tot[32];
  __shared__ int total_cnt, total_tiles;
  const int e = threadIdx.x;
  int tot = 0;
  if (e < E) {
    // eight chunks' counts in flight at a time
    for (int c0 = 0; c0 < nchunks; c0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (c0 + j < nchunks) ? counts_chunk[static_cast<size_t>(c0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (c0 + j < nchunks) chunk_base[static_cast<size_t>(c0 + j) * E + e] = tot;
        tot += v[j];
      }
    }
  }
  const int off = block_exclusive_scan(tot, warp_tot, &total_cnt);
  const int nt = (tot + kTileN - 1) / kTileN;
  const int ntp = block_exclusive_scan(nt, warp_tot, &total_tiles);
  if (e < E) {
    offsets[e] = off;
    ntile_prefix[e] = ntp;
    if (counts) counts[e] = tot;
    for (int c = 0; c < nchunks; ++c) chunk_base[static_cast<size_t>(c) * E + e] += off;
  }
  if (e == 0) {
    offsets[E] = total_cnt;
    ntile_prefix[E] = total_tiles;
  }
}

// Stable scatter of pair indices into perm.
template <typename IdxT>
__global__ void __launch_bounds__(256) k_route_scatter(const IdxT *__restrict__ idx, int S, int E,
                                                       int nchunks,
                                                       const int32_t *__restrict__ chunk_base,
                                                       int32_t *__restrict__ perm) {
  extern __shared__ int32_t running_all[];  // [kWarpsPerBlock][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kWarpsPerBlock + warp;
  if (chunk >= nchunks) return;
  int32_t *running = running_all + warp * E;
  const int32_t *base = chunk_base + static_cast<size_t>(chunk) * E;
  for (int e = lane; e < E; e += 32) running[e] = base[e];
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  int ev[kSteps];
#pragma unroll
  for (int st = 0; st < kSteps; ++st) ev[st] = load_expert(idx, chunk * kRouteChunk + st * 32 + lane, S, E, nullptr);
#pragma unroll
  for (int st = 0; st < kSteps; ++st) {
    const int p = chunk * kRouteChunk + st * 32 + lane;
    const int e = ev[st];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int rank = __popc(peers & lt);
      perm[running[e] + rank] = p;
    }
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) running[e] += __popc(peers);
    __syncwarp();
  }
}

// The same three steps in one CTA of 1024 threads, for the small problems where launch
// latency dominates (a few thousand pairs): the per-chunk table (at most kFusedChunks chunks, each walked in
// order by one warp) lives in shared memory, so the whole routing is one launch.
constexpr int kFusedChunks = 128;
constexpr int kFusedMaxE = 256;
constexpr int kFusedMaxS = 4096;  // beyond, one SM walking the pairs is slower than three launches

template <typename IdxT>
__global__ void __launch_bounds__(1024) k_route_fused(const IdxT *__restrict__ idx, int S, int E,
                                                     int nchunks, int chunk, int32_t *__restrict__ counts,
                                                     int32_t *__restrict__ offsets,
                                                     int32_t *__restrict__ ntile_prefix,
                                                     int32_t *__restrict__ perm, int32_t *status) {
  extern __shared__ int32_t cc[];  // [nchunks][E]: histograms, then running bases
  __shared__ int warp_tot[32];
  __shared__ int total_cnt, total_tiles;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < nchunks * E; i += blockDim.x) cc[i] = 0;
  __syncthreads();
  // 1: per-chunk histograms
  for (int c = warp; c < nchunks; c += 32) {
    int32_t *h = cc + c * E;
    const int end = min(S, (c + 1) * chunk);
    for (int p0 = c * chunk; p0 < end; p0 += 32) {
      const int p = p0 + lane;
      const int e = p < end ? load_expert(idx, p, S, E, status) : -1;
      if (e >= 0) atomicAdd(&h[e], 1);
    }
  }
  __syncthreads();
  // 2: per expert, the chunks' bases in chunk order; offsets and the token-tile prefix
  const int e = threadIdx.x;
  int tot = 0;
  if (e < E) {
    for (int c = 0; c < nchunks; ++c) {
      const int v = cc[c * E + e];
      cc[c * E + e] = tot;
      tot += v;
    }
  }
  const int off = block_exclusive_scan(tot, warp_tot, &total_cnt);
  const int nt = (tot + kTileN - 1) / kTileN;
  const int ntp = block_exclusive_scan(nt, warp_tot, &total_tiles);
  if (e < E) {
    offsets[e] = off;
    ntile_prefix[e] = ntp;
    if (counts) counts[e] = tot;
    for (int c = 0; c < nchunks; ++c) cc[c * E + e] += off;
  }
  if (e == 0) {
    offsets[E] = total_cnt;
    ntile_prefix[E] = total_tiles;
  }
  __syncthreads();
  // 3: stable scatter, each chunk walked in order by the warp that counted it
  const unsigned lt = (1u << lane) - 1u;
  for (int c = warp; c < nchunks; c += 32) {
    int32_t *running = cc + c * E;
    const int end = min(S, (c + 1) * chunk);
    for (int p0 = c * chunk; p0 < end; p0 += 32) {
      const int p = p0 + lane;
      const int ex = p < end ? load_expert(idx, p, S, E, nullptr) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, ex);
      if (ex >= 0) perm[running[ex] + __popc(peers & lt)] = p;
      __syncwarp();
      if (ex >= 0 && (peers & lt) == 0) running[ex] += __popc(peers);
      __syncwarp();
    }
  }
}

cudaError_t launch_route(const void *idx, bool idx64, int S, int E, int nchunks,
                         int32_t *counts_chunk, int32_t *chunk_base, int32_t *counts,
                         int32_t *offsets, int32_t *ntile_prefix, int32_t *perm, int32_t *status,
                         cudaStream_t s, int *launches) {
  if (S <= kFusedMaxS && E <= kFusedMaxE) {
    // chunks of a multiple of 32 pairs, at most kFusedChunks of them
    const int per = (S + kFusedChunks - 1) / kFusedChunks;
    const int chunk = ((per + 31) / 32) * 32 > 32 ? ((per + 31) / 32) * 32 : 32;
    const int nfc = (S + chunk - 1) / chunk;
    const size_t shm = static_cast<size_t>(nfc) * E * sizeof(int32_t);
    static bool attr = false;
    if (!attr) {
      const int mx = kFusedChunks * kFusedMaxE * static_cast<int>(sizeof(int32_t));
      if (cudaFuncSetAttribute(k_route_fused<long long>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess ||
          cudaFuncSetAttribute(k_route_fused<int32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess)
        return cudaGetLastError();
      attr = true;
    }
    if (idx64) k_route_fused<long long><<<1, 1024, shm, s>>>(static_cast<const long long *>(idx), S, E, nfc, chunk, counts, offsets, ntile_prefix, perm, status);
    else k_route_fused<int32_t><<<1, 1024, shm, s>>>(static_cast<const int32_t *>(idx), S, E, nfc, chunk, counts, offsets, ntile_prefix, perm, status);
    *launches += 1;
    return cudaGetLastError();
  }
  const int blocks = (nchunks + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const size_t shm = static_cast<size_t>(kWarpsPerBlock) * E * sizeof(int32_t);
  if (idx64) k_route_count<long long><<<blocks, 256, shm, s>>>(static_cast<const long long *>(idx), S, E, nchunks, counts_chunk, status);
  else k_route_count<int32_t><<<blocks, 256, shm, s>>>(static_cast<const int32_t *>(idx), S, E, nchunks, counts_chunk, status);
  k_route_scan<<<1, 1024, 0, s>>>(counts_chunk, nchunks, E, chunk_base, counts, offsets, ntile_prefix);
  if (idx64) k_route_scatter<long long><<<blocks, 256, shm, s>>>(static_cast<const long long *>(idx), S, E, nchunks, chunk_base, perm);
  else k_route_scatter<int32_t><<<blocks, 256, shm, s>>>(static_cast<const int32_t *>(idx), S, E, nchunks, chunk_base, perm);
  *launches += 3;
  return cudaGetLastError();
}

// xg[s] = fp16(x[perm[s] / K]) for s < offsets[E]: one warp per row, 16-byte vectors.
// bf16 -> fp16 is exact for 6.1e-5 <= |x| <= 65504; larger magnitudes saturate to
// +-65504 and raise MOEQ_ERR_RANGE.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_sat(uint32_t w, bool &over) {
  float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
  over |= (fabsf(lo) > 65504.0f) || (fabsf(hi) > 65504.0f);
  lo = fminf(fmaxf(lo, -65504.0f), 65504.0f);
  hi = fminf(fmaxf(hi, -65504.0f), 65504.0f);
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(256) k_gather_rows(const uint4 *__restrict__ x,
                                                     const int32_t *__restrict__ perm,
                                                     const int32_t *__restrict__ offsets, int E,
                                                     int S, int K, int vec_per_row,
                                                     uint4 *__restrict__ xg, int32_t *status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= S || row >= offsets[E]) return;
  const int t = perm[row] / K;
  const uint4 *src = x + static_cast<size_t>(t) * vec_per_row;
  uint4 *dst = xg + static_cast<size_t>(row) * vec_per_row;
  bool over = false;
  for (int v = lane; v < vec_per_row; v += 32) {
    const uint4 a = src[v];
    uint4 b;
    b.x = bf16x2_to_f16x2_sat(a.x, over);
    b.y = bf16x2_to_f16x2_sat(a.y, over);
    b.z = bf16x2_to_f16x2_sat(a.z, over);
    b.w = bf16x2_to_f16x2_sat(a.w, over);
    dst[v] = b;
  }
  if (over) report(status, MOEQ_ERR_RANGE);
}

cudaError_t launch_gather_rows(const void *x, const int32_t *perm, const int32_t *offsets, int E,
                               int S, int K, int H, void *xg, int32_t *status, cudaStream_t s,
                               int *launches) {
  const int blocks = (S + 7) / 8;
  k_gather_rows<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(x), perm, offsets, E, S, K, H / 8,
                                       static_cast<uint4 *>(xg), status);
  ++*launches;
  return cudaGetLastError();
}

// out[t, i] = sum over k = 0..K-1, in order, of slots[t*K + k, i] (fp32), skipping
// dropped pairs; stored as fp32 or rounded once to bf16.  One thread per 8 features.
template <typename IdxT, bool F32OUT>
__global__ void __launch_bounds__(256) k_combine(const float4 *__restrict__ slots,
                                                 const IdxT *__restrict__ idx, int T, int K, int E,
                                                 int H8, void *__restrict__ out) {
  const size_t g = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= static_cast<size_t>(T) * H8) return;
  const size_t t = g / H8, j = g - t * H8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int k = 0; k < K; ++k) {
    const long long e = static_cast<long long>(idx[t * K + k]);
    if (e < 0 || e >= E) continue;
    const float4 *src = slots + ((t * K + k) * H8 + j) * 2;
    const float4 a = src[0], b = src[1];
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
  if (F32OUT) {
    float4 *o = reinterpret_cast<float4 *>(out) + g * 2;
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  } else {
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      p[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    reinterpret_cast<uint4 *>(out)[g] = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

cudaError_t launch_combine(const float *slots, const void *idx, bool idx64, int T, int K, int E,
                           int H, void *out, bool f32_out, cudaStream_t s, int *launches) {
  const int H8 = H / 8;
  const size_t n = static_cast<size_t>(T) * H8;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
  const float4 *sp = reinterpret_cast<const float4 *>(slots);
  const long long *i64 = static_cast<const long long *>(idx);
  const int32_t *i32 = static_cast<const int32_t *>(idx);
  if (idx64 && f32_out) k_combine<long long, true><<<blocks, 256, 0, s>>>(sp, i64, T, K, E, H8, out);
  else if (idx64) k_combine<long long, false><<<blocks, 256, 0, s>>>(sp, i64, T, K, E, H8, out);
  else if (f32_out) k_combine<int32_t, true><<<blocks, 256, 0, s>>>(sp, i32, T, K, E, H8, out);
  else k_combine<int32_t, false><<<blocks, 256, 0, s>>>(sp, i32, T, K, E, H8, out);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace moeq
