// Quantizers and dequantizers for fused 3-D expert tensors (HBM-bound kernels).
//
// Definitions ("MoE Expert Quantization", Implementation details; bitsandbytes issue
// #1849, maintainer comments on blocksize 64 and per-expert absmax):
//   NF4:  per 64-element block along C, absmax = max|x|, n = fl(x / absmax), code =
//         nearest NormalFloat-4 level (ties to the lower index), 2 codes per byte with
//         the first element in the high nibble.
//   DQ:   absmax as int8 blocks of 256 with an fp32 scale and a per-expert mean offset.
//   int8: per row absmax, q = rint(fl(127 x) / absmax).
// Every result is bit-exact: fp32 operations are written as explicit round-to-nearest
// intrinsics and this file is built with -fmad=false, so nothing contracts to an FMA
// except the FMAs written on purpose in the division below.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moeq {

// The 16 NormalFloat-4 levels (4-bit normal-quantile table, exact 0 at index 7),
// as fp32 constants.
__constant__ float kNF4[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
    0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};

// ---------------------------------------------------------------------------
// Nearest-level lookup without 15 compares per element.
//
// code(n) = #{j : n > t_j} with t_j = the fp32 value just at or below the midpoint
// (c_j + c_{j+1}) / 2 (for an fp32 n, "n > t_j" is then the same as "n above the exact
// midpoint", so an exact midpoint goes to the lower level).  The interval [-1, 1] is
// cut into 31 cells by cell(n) = RN(15 n + 12582927) - 12582912, a monotone map.
// No two thresholds share a cell (the cells are 1/15 wide, the thresholds at least
// 0.08 apart), so with base[m] = #{j : cell(t_j) < m} and thr[m] the threshold in
// cell m (+inf if none), monotonicity gives exactly
//   code(n) = base[cell(n)] + (n > thr[cell(n)]).
// The two tables live in shared memory as one 32-entry array of (thr, base) pairs: one
// 8-byte load per element.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int nf4_cell(float n) {
  return __float_as_int(__fmaf_rn(n, 15.0f, 12582927.0f)) & 31;
}

__device__ void build_nf4_cells(uint2 *cells) {
  const int m = threadIdx.x;
  if (m < 32) {
    int b = 0;
    float th = __int_as_float(0x7f800000);  // +inf
    for (int j = 0; j < 15; ++j) {
      const double mid = (static_cast<double>(kNF4[j]) + static_cast<double>(kNF4[j + 1])) * 0.5;
      const float t = __double2float_rd(mid);
      const int cj = nf4_cell(t);
      if (cj < m) ++b;
      else if (cj == m) th = t;
    }
    cells[m] = make_uint2(__float_as_uint(th), static_cast<uint32_t>(b));
  }
}

// (acc << 4) + code(n), n in cell c: appends the 4-bit code of n below the codes in acc
__device__ __forceinline__ uint32_t nf4_push(uint32_t acc, float n, int c, const uint2 *cells) {
  const uint2 tb = cells[c];
  return (acc << 4) + tb.y + (n > __uint_as_float(tb.x) ? 1u : 0u);
}

// fl(x / a) for |x| <= a, a a normal fp32 number >= 2^-120, r = RN(1/a):
// q0 = RN(x r); e = x - a q0 (exact, one FMA); q = RN(q0 + e r).  This is Markstein's
// correction step (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990); it returns the
// correctly rounded quotient for these operands, which the exhaustive bf16 parity
// tests confirm against the oracle's IEEE divide.
__device__ __forceinline__ float div_by(float x, float a, float r) {
  const float q0 = __fmul_rn(x, r);
  const float e = __fmaf_rn(-a, q0, x);
  return __fmaf_rn(e, r, q0);
}

// Packed fp32x2 arithmetic: each lane of the pair is one IEEE round-to-nearest
// operation, exactly as the scalar form.
__device__ __forceinline__ uint64_t f2u(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float lo_f(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 32 bytes in one 256-bit load (the address must be 32-byte aligned)
__device__ __forceinline__ void ld_stream_v8(const void *p, uint4 &a, uint4 &b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}

// the 32 bytes of quarter q: one 256-bit load when the source is 32-byte aligned, else two
// 16-byte loads
template <bool V8>
__device__ __forceinline__ void load_quarter(const uint4 *w, size_t q, uint4 &a, uint4 &b) {
  if (V8) {
    ld_stream_v8(w + 2 * q, a, b);
  } else {
    a = ld_stream_u4(w + 2 * q);
    b = ld_stream_u4(w + 2 * q + 1);
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __int_as_float(w[i] << 16);
    f[2 * i + 1] = __int_as_float(w[i] & 0xffff0000u);
  }
}

// ---------------------------------------------------------------------------
// a1: NF4 quantize.  One thread per 16 consecutive elements (a quarter of a block),
// 4 lanes per block, absmax by two xor-shuffles inside the 4-lane group.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void nf4_quarter(const uint4 v0, const uint4 v1, size_t q, uint32_t lane,
                                            const uint2 *cells, uint2 *codes, float *absmax) {
  float x[16];
  {
    float a8[8], b8[8];
    unpack_bf16x8(v0, a8);
    unpack_bf16x8(v1, b8);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[i] = a8[i];
      x[8 + i] = b8[i];
    }
  }
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(x[i]));
  const uint32_t gmask = 0xFu << (lane & 28u);
  m = fmaxf(m, __shfl_xor_sync(gmask, m, 1, 4));
  m = fmaxf(m, __shfl_xor_sync(gmask, m, 2, 4));
  const float a = m;
  // word h of the output holds elements 8h..8h+7; byte k of it is (code(2k) << 4) | code(2k+1),
  // so the codes are pushed in the order 6 7 4 5 2 3 0 1
  uint32_t out[2] = {0u, 0u};
  if (a == 0.0f || a >= 0x1p-120f) {
    // the division and the cell map two elements at a time (fp32x2)
    const float r = (a == 0.0f) ? 0.0f : __frcp_rn(a);
    const uint64_t r2 = f2u(r, r), na2 = f2u(-a, -a);
    const uint64_t k15 = f2u(15.0f, 15.0f), kc = f2u(12582927.0f, 12582927.0f);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int p = 3; p >= 0; --p) {
        const int i = 8 * h + 2 * p;
        const uint64_t x2 = f2u(x[i], x[i + 1]);
        const uint64_t q0 = mul2(x2, r2);
        const uint64_t e = fma2(na2, q0, x2);
        const uint64_t n2 = fma2(e, r2, q0);
        const uint64_t f2 = fma2(n2, k15, kc);
        out[h] = nf4_push(out[h], lo_f(n2), static_cast<int>(static_cast<uint32_t>(f2) & 31u), cells);
        out[h] = nf4_push(out[h], hi_f(n2), static_cast<int>(static_cast<uint32_t>(f2 >> 32) & 31u), cells);
      }
    }
  } else {  // tiny (subnormal-range) absmax: plain IEEE divide
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int p = 3; p >= 0; --p) {
        const int i = 8 * h + 2 * p;
        const float n0 = __fdiv_rn(x[i], a), n1 = __fdiv_rn(x[i + 1], a);
        out[h] = nf4_push(out[h], n0, nf4_cell(n0), cells);
        out[h] = nf4_push(out[h], n1, nf4_cell(n1), cells);
      }
    }
  }
  codes[q] = make_uint2(out[0], out[1]);
  if ((lane & 3u) == 0) absmax[q >> 2] = a;
}

template <bool V8>
__global__ void __launch_bounds__(256) k_quant_nf4(const uint4 *__restrict__ w,
                                                   uint2 *__restrict__ codes,
                                                   float *__restrict__ absmax, size_t nquarters) {
  __shared__ uint2 cells[32];
  build_nf4_cells(cells);
  __syncthreads();
  const uint32_t lane = threadIdx.x & 31u;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t q = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  // two quarters in flight per thread
  for (; q + stride < nquarters; q += 2 * stride) {
    uint4 a0, a1, b0, b1;
    load_quarter<V8>(w, q, a0, a1);
    load_quarter<V8>(w, q + stride, b0, b1);
    nf4_quarter(a0, a1, q, lane, cells, codes, absmax);
    nf4_quarter(b0, b1, q + stride, lane, cells, codes, absmax);
  }
  if (q < nquarters) {
    uint4 a0, a1;
    load_quarter<V8>(w, q, a0, a1);
    nf4_quarter(a0, a1, q, lane, cells, codes, absmax);
  }
}

// ---------------------------------------------------------------------------
// a2: double quantization of absmax [E, nb] (fixed-order fp64 mean, int8 blocks of 256)
// ---------------------------------------------------------------------------
// Chunk sums: kDqSumChunks chunks of 256 per block, staged in shared memory (coalesced
// loads, row pitch 257 so that the summing threads hit distinct banks), each summed
// sequentially by one thread (the order is part of the definition).
constexpr int kDqSumChunks = 64;
__global__ void __launch_bounds__(256) k_dq_chunk_sum(const float *__restrict__ absmax, int nb,
                                                      int nblk, int nchunks_total,
                                                      double *__restrict__ S) {
  extern __shared__ float buf[];  // [kDqSumChunks][257]
  const int c0 = blockIdx.x * kDqSumChunks;
  // thread t stages element t of every chunk (256 threads = one chunk row), 16 chunks' loads
  // in flight before their shared-memory stores
  const int i = threadIdx.x;
  for (int j0 = 0; j0 < kDqSumChunks; j0 += 16) {
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int g = c0 + j0 + u;
      v[u] = 0.0f;
      if (g < nchunks_total) {
        const int e = g / nblk, c = g - e * nblk;
        const int at = c * 256 + i;
        if (at < nb) v[u] = absmax[static_cast<size_t>(e) * nb + at];
      }
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) buf[(j0 + u) * 257 + i] = v[u];
  }
  __syncthreads();
  if (threadIdx.x < kDqSumChunks) {
    const int g = c0 + threadIdx.x;
    if (g < nchunks_total) {
      double s = 0.0;
      for (int i = 0; i < 256; ++i) s = __dadd_rn(s, static_cast<double>(buf[threadIdx.x * 257 + i]));
      S[g] = s;
    }
  }
}

// One warp per expert: the lanes stage the expert's chunk sums in shared memory (coalesced,
// all loads in flight together), then lane 0 adds them in chunk order (the sequential sum).
constexpr int kDqOffWarps = 8;
constexpr int kDqOffMaxChunks = 512;   // chunk sums staged per pass (8 warps x 4 KB)
__global__ void __launch_bounds__(kDqOffWarps * 32) k_dq_offset(const double *__restrict__ S, int E, int nb,
                                                                int nblk, float *__restrict__ off) {
  __shared__ double buf[kDqOffWarps][kDqOffMaxChunks];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kDqOffWarps + warp;
  if (e >= E) return;  // whole warp; no block-wide barrier below
  const double *src = S + static_cast<size_t>(e) * nblk;
  double t = 0.0;
  for (int c0 = 0; c0 < nblk; c0 += kDqOffMaxChunks) {
    const int n = min(kDqOffMaxChunks, nblk - c0);
    for (int c = lane; c < n; c += 32) buf[warp][c] = src[c0 + c];
    __syncwarp();
    if (lane == 0)
      for (int c = 0; c < n; ++c) t = __dadd_rn(t, buf[warp][c]);
    __syncwarp();
  }
  if (lane == 0) off[e] = __double2float_rn(__ddiv_rn(t, static_cast<double>(nb)));
}

// One warp per 256-block: v = fl(a - off), s = max|v|, q = rint(fl(fl(127 v) / s)).
__global__ void __launch_bounds__(256) k_dq_quant(const float *__restrict__ absmax,
                                                  const float *__restrict__ off, int E, int nb,
                                                  int nblk, int8_t *__restrict__ q_out,
                                                  float *__restrict__ scale) {
  const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (g >= E * nblk) return;  // whole warp leaves together
  const int e = g / nblk, c = g - e * nblk;
  const float o = off[e];
  const float *src = absmax + static_cast<size_t>(e) * nb;
  float v[8];
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = c * 256 + lane * 8 + j;
    v[j] = (i < nb) ? __fsub_rn(src[i], o) : 0.0f;
    m = fmaxf(m, fabsf(v[j]));
  }
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
  int8_t *dst = q_out + static_cast<size_t>(e) * nb;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = c * 256 + lane * 8 + j;
    if (i < nb) {
      int q = 0;
      if (m != 0.0f) q = __float2int_rn(__fdiv_rn(__fmul_rn(127.0f, v[j]), m));
      dst[i] = static_cast<int8_t>(q);
    }
  }
  if (lane == 0) scale[g] = m;
}

// ---------------------------------------------------------------------------
// a3: int8 row-wise.  One CTA per row; the row stays in registers (NV 16-byte
// vectors per thread) between the absmax reduction and the quantization.
// ---------------------------------------------------------------------------
template <int NV>
__global__ void k_quant_int8_row(const uint4 *__restrict__ w, uint2 *__restrict__ codes,
                                 float *__restrict__ absmax, int C) {
  __shared__ float red[32];
  const size_t row = blockIdx.x;
  const int nvec = C >> 3;
  const uint4 *src = w + row * nvec;
  uint2 *dst = codes + row * nvec;
  uint4 v[NV];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int idx = threadIdx.x + i * blockDim.x;
    if (idx < nvec) {
      v[i] = ld_stream_u4(src + idx);
      float f[8];
      unpack_bf16x8(v[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(f[j]));
    }
  }
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = (static_cast<int>(threadIdx.x) < nw) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, d));
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float a = red[0];
  const bool fast = (a == 0.0f || a >= 0x1p-120f);
  const float r = (a == 0.0f) ? 0.0f : __frcp_rn(a);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int idx = threadIdx.x + i * blockDim.x;
    if (idx < nvec) {
      float f[8];
      unpack_bf16x8(v[i], f);
      uint32_t b[8];
      if (fast) {
        const uint64_t r2 = f2u(r, r), na2 = f2u(-a, -a), k127 = f2u(127.0f, 127.0f);
        const uint64_t kr = f2u(12582912.0f, 12582912.0f);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          const uint64_t p2 = mul2(k127, f2u(f[j], f[j + 1]));  // 127 x, exact for bf16 x
          const uint64_t q0 = mul2(p2, r2);
          const uint64_t e = fma2(na2, q0, p2);
          const uint64_t n2 = fma2(e, r2, q0);                  // fl(127 x / absmax)
          // rint (half to even) by adding 1.5*2^23; |n| <= 127 keeps this exact
          uint64_t one = f2u(1.0f, 1.0f);
          const uint64_t rr = fma2(n2, one, kr);
          b[j] = static_cast<uint32_t>(rr) & 0xffu;
          b[j + 1] = static_cast<uint32_t>(rr >> 32) & 0xffu;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float p = __fmul_rn(127.0f, f[j]);
          const float n = __fdiv_rn(p, a);
          b[j] = static_cast<uint32_t>(__float_as_int(__fadd_rn(n, 12582912.0f))) & 0xffu;
        }
      }
      uint2 o;
      o.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
      o.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
      dst[idx] = o;
    }
  }
  if (threadIdx.x == 0) absmax[row] = a;
}

// ---------------------------------------------------------------------------
// a4: dequantize.  One thread per 16 elements.
// ---------------------------------------------------------------------------
template <bool DQ, bool F32OUT>
__global__ void __launch_bounds__(256) k_dequant_nf4(const uint2 *__restrict__ codes,
                                                     const float *__restrict__ absmax,
                                                     const int8_t *__restrict__ aq,
                                                     const float *__restrict__ ascale,
                                                     const float *__restrict__ aoff, size_t nb_per_expert,
                                                     size_t nblk, size_t nquarters,
                                                     void *__restrict__ out) {
  __shared__ float cb[16];
  if (threadIdx.x < 16) cb[threadIdx.x] = kNF4[threadIdx.x];
  __syncthreads();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t q = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < nquarters;
       q += stride) {
    const size_t b = q >> 2;  // global 64-block index
    float a;
    if (DQ) {
      const size_t e = b / nb_per_expert, bb = b - e * nb_per_expert;
      const float step = __fdiv_rn(ascale[e * nblk + (bb >> 8)], 127.0f);
      a = __fadd_rn(__fmul_rn(static_cast<float>(aq[b]), step), aoff[e]);
    } else {
      a = absmax[b];
    }
    const uint2 cw = codes[q];
    float wv[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t b0 = (cw.x >> (8 * k)) & 0xffu, b1 = (cw.y >> (8 * k)) & 0xffu;
      wv[2 * k] = __fmul_rn(cb[b0 >> 4], a);
      wv[2 * k + 1] = __fmul_rn(cb[b0 & 15u], a);
      wv[8 + 2 * k] = __fmul_rn(cb[b1 >> 4], a);
      wv[8 + 2 * k + 1] = __fmul_rn(cb[b1 & 15u], a);
    }
    if (F32OUT) {
      float4 *o = reinterpret_cast<float4 *>(out) + q * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = make_float4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
    } else {
      uint4 *o = reinterpret_cast<uint4 *>(out) + q * 2;
      uint32_t p[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(wv[2 * i], wv[2 * i + 1]);
        p[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
      o[0] = make_uint4(p[0], p[1], p[2], p[3]);
      o[1] = make_uint4(p[4], p[5], p[6], p[7]);
    }
  }
}

template <bool F32OUT>
__global__ void __launch_bounds__(256) k_dequant_int8(const uint4 *__restrict__ codes,
                                                      const float *__restrict__ absmax, int C,
                                                      size_t nvec16, void *__restrict__ out) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t per_row = static_cast<size_t>(C) >> 4;
  for (size_t v = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec16; v += stride) {
    const size_t row = v / per_row;
    const float step = __fdiv_rn(absmax[row], 127.0f);
    const uint4 cw = codes[v];
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
    float wv[16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int8_t qv = static_cast<int8_t>((w4[i] >> (8 * k)) & 0xffu);
        wv[4 * i + k] = __fmul_rn(static_cast<float>(qv), step);
      }
    if (F32OUT) {
      float4 *o = reinterpret_cast<float4 *>(out) + v * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = make_float4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
    } else {
      uint4 *o = reinterpret_cast<uint4 *>(out) + v * 2;
      uint32_t p[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(wv[2 * i], wv[2 * i + 1]);
        p[i] = *reinterpret_cast<const uint32_t *>(&h);
      }
      o[0] = make_uint4(p[0], p[1], p[2], p[3]);
      o[1] = make_uint4(p[4], p[5], p[6], p[7]);
    }
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
static int grid_for(size_t work_threads, int threads, int sm_count, int per_sm) {
  const size_t need = (work_threads + threads - 1) / threads;
  const size_t cap = static_cast<size_t>(sm_count) * per_sm;
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

cudaError_t launch_quant_nf4(const void *w, size_t n_elems, uint8_t *codes, float *absmax,
                             int sm_count, cudaStream_t s, int *launches) {
  const size_t nq = n_elems / 16;
  const int grid = grid_for((nq + 1) / 2, 256, sm_count, 8);
  if ((reinterpret_cast<uintptr_t>(w) & 31u) == 0)
    k_quant_nf4<true><<<grid, 256, 0, s>>>(reinterpret_cast<const uint4 *>(w), reinterpret_cast<uint2 *>(codes),
                                           absmax, nq);
  else
    k_quant_nf4<false><<<grid, 256, 0, s>>>(reinterpret_cast<const uint4 *>(w), reinterpret_cast<uint2 *>(codes),
                                            absmax, nq);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_double_quant(const float *absmax_f32, int E, int nb, double *chunk_sums,
                                int8_t *q_out, float *scale, float *off, cudaStream_t s,
                                int *launches) {
  const int nblk = (nb + 255) / 256;
  const int total = E * nblk;
  const size_t sum_smem = static_cast<size_t>(kDqSumChunks) * 257 * sizeof(float);
  static bool sum_attr = false;
  if (!sum_attr) {
    const cudaError_t e = cudaFuncSetAttribute(k_dq_chunk_sum, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(sum_smem));
    if (e != cudaSuccess) return e;
    sum_attr = true;
  }
  k_dq_chunk_sum<<<(total + kDqSumChunks - 1) / kDqSumChunks, 256, sum_smem, s>>>(absmax_f32, nb, nblk, total,
                                                                                  chunk_sums);
  k_dq_offset<<<(E + kDqOffWarps - 1) / kDqOffWarps, kDqOffWarps * 32, 0, s>>>(chunk_sums, E, nb, nblk, off);
  k_dq_quant<<<(total + 7) / 8, 256, 0, s>>>(absmax_f32, off, E, nb, nblk, q_out, scale);
  *launches += 3;
  return cudaGetLastError();
}

cudaError_t launch_quant_int8_row(const void *w, size_t rows, int C, int8_t *codes, float *absmax,
                                  cudaStream_t s, int *launches) {
  const int nvec = C / 8;
  int threads = 128;
  while (threads < 1024 && (nvec + threads - 1) / threads > 16) threads *= 2;
  const int per = (nvec + threads - 1) / threads;
  const uint4 *wp = reinterpret_cast<const uint4 *>(w);
  uint2 *cp = reinterpret_cast<uint2 *>(codes);
  const unsigned grid = static_cast<unsigned>(rows);
  if (per <= 1) k_quant_int8_row<1><<<grid, threads, 0, s>>>(wp, cp, absmax, C);
  else if (per <= 2) k_quant_int8_row<2><<<grid, threads, 0, s>>>(wp, cp, absmax, C);
  else if (per <= 4) k_quant_int8_row<4><<<grid, threads, 0, s>>>(wp, cp, absmax, C);
  else if (per <= 8) k_quant_int8_row<8><<<grid, threads, 0, s>>>(wp, cp, absmax, C);
  else if (per <= 16) k_quant_int8_row<16><<<grid, threads, 0, s>>>(wp, cp, absmax, C);
  else return cudaErrorInvalidValue;
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_dequant(const moeq_packed *p, void *out, bool f32, int sm_count, cudaStream_t s,
                           int *launches) {
  const size_t n = static_cast<size_t>(p->E) * p->R * p->C;
  if (p->mode == MOEQ_INT8_ROW) {
    const size_t nv = n / 16;
    const int grid = grid_for(nv, 256, sm_count, 8);
    const uint4 *c = reinterpret_cast<const uint4 *>(p->codes);
    if (f32) k_dequant_int8<true><<<grid, 256, 0, s>>>(c, p->absmax, p->C, nv, out);
    else k_dequant_int8<false><<<grid, 256, 0, s>>>(c, p->absmax, p->C, nv, out);
  } else {
    const size_t nq = n / 16;
    const size_t nbpe = static_cast<size_t>(p->R) * p->C / 64;
    const size_t nblk = (nbpe + 255) / 256;
    const int grid = grid_for(nq, 256, sm_count, 8);
    const uint2 *c = reinterpret_cast<const uint2 *>(p->codes);
    if (p->mode == MOEQ_NF4_DQ) {
      if (f32) k_dequant_nf4<true, true><<<grid, 256, 0, s>>>(c, nullptr, p->absmax_q, p->absmax_scale, p->absmax_offset, nbpe, nblk, nq, out);
      else k_dequant_nf4<true, false><<<grid, 256, 0, s>>>(c, nullptr, p->absmax_q, p->absmax_scale, p->absmax_offset, nbpe, nblk, nq, out);
    } else {
      if (f32) k_dequant_nf4<false, true><<<grid, 256, 0, s>>>(c, p->absmax, nullptr, nullptr, nullptr, nbpe, nblk, nq, out);
      else k_dequant_nf4<false, false><<<grid, 256, 0, s>>>(c, p->absmax, nullptr, nullptr, nullptr, nbpe, nblk, nq, out);
    }
  }
  ++*launches;
  return cudaGetLastError();
}

}  // namespace moeq
