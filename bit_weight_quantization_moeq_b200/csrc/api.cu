// C ABI entry points (include/moeq.h): argument checks on the host, then kernel launches
// on the caller's stream.  Nothing here allocates device memory.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/moeq.h"
#include "kernels.h"

using namespace moeq;

namespace {

std::atomic<unsigned long long> g_launches{0};

thread_local void *const *t_trace_events = nullptr;
thread_local int t_trace_n = 0;

// Records the k-th trace event on `s` when tracing is on for this thread.
void trace_mark(int k, cudaStream_t s) {
  if (t_trace_events && k < t_trace_n)
    cudaEventRecord(reinterpret_cast<cudaEvent_t>(t_trace_events[k]), s);
}

struct DevInfo {
  int sm_count = 0;
  bool ok = false;
};

moeq_status device_info(DevInfo *out) {
  static thread_local int cached_dev = -1;
  static thread_local DevInfo cached;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOEQ_ERR_CUDA;
  if (dev != cached_dev) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOEQ_ERR_CUDA;
    cached.sm_count = sms;
    cached.ok = (major == 10 && minor == 0);
    cached_dev = dev;
  }
  *out = cached;
  return cached.ok ? MOEQ_OK : MOEQ_ERR_DEVICE;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

moeq_status finish(cudaError_t e, int launches) {
  g_launches.fetch_add(static_cast<unsigned long long>(launches));
  return e == cudaSuccess ? MOEQ_OK : MOEQ_ERR_CUDA;
}

// Checks a packed descriptor: mode, shape, pointers present and aligned.
moeq_status check_packed(const moeq_packed *p) {
  if (!p) return MOEQ_ERR_NULL;
  if (p->mode < MOEQ_NF4 || p->mode > MOEQ_INT8_ROW) return MOEQ_ERR_DTYPE;
  if (p->E < 0 || p->R < 0 || p->C < 0) return MOEQ_ERR_SHAPE;
  if (p->C % 64) return MOEQ_ERR_BLOCKSIZE;
  const size_t n = static_cast<size_t>(p->E) * p->R * p->C;
  if (n == 0) return MOEQ_OK;
  if (!p->codes) return MOEQ_ERR_NULL;
  if (!aligned16(p->codes)) return MOEQ_ERR_ALIGN;
  if (p->mode == MOEQ_NF4_DQ) {
    if (!p->absmax_q || !p->absmax_scale || !p->absmax_offset) return MOEQ_ERR_NULL;
    if (!aligned16(p->absmax_q) || !aligned16(p->absmax_scale) || !aligned16(p->absmax_offset))
      return MOEQ_ERR_ALIGN;
  } else {
    if (!p->absmax) return MOEQ_ERR_NULL;
    if (!aligned16(p->absmax)) return MOEQ_ERR_ALIGN;
  }
  return MOEQ_OK;
}

struct QuantWs {
  size_t absmax, sums, total;
};
QuantWs quant_ws_layout(int E, int R, int C) {
  QuantWs l{};
  const size_t nb = static_cast<size_t>(R) * C / 64;
  const size_t nblk = (nb + 255) / 256;
  l.absmax = 0;
  l.sums = align256(static_cast<size_t>(E) * nb * sizeof(float));
  l.total = l.sums + align256(static_cast<size_t>(E) * nblk * sizeof(double));
  return l;
}

struct FwdWs {
  size_t counts_chunk, chunk_base, counts, offsets, ntp, perm, status, route_end, xg, h, slots, total;
};
FwdWs fwd_ws_layout(long long T, int K, int E, int H, int I) {
  FwdWs l{};
  const long long S = T * K;
  const long long nchunks = (S + kRouteChunk - 1) / kRouteChunk;
  size_t o = 0;
  l.counts_chunk = o; o += align256(static_cast<size_t>(nchunks) * E * 4);
  l.chunk_base = o;   o += align256(static_cast<size_t>(nchunks) * E * 4);
  l.counts = o;       o += align256(static_cast<size_t>(E) * 4);
  l.offsets = o;      o += align256(static_cast<size_t>(E + 1) * 4);
  l.ntp = o;          o += align256(static_cast<size_t>(E + 1) * 4);
  l.perm = o;         o += align256(static_cast<size_t>(S) * 4);
  l.status = o;       o += 256;
  l.route_end = o;
  l.xg = o;           o += align256(static_cast<size_t>(S) * H * 2);
  l.h = o;            o += align256(static_cast<size_t>(S) * I * 2);
  l.slots = o;        o += align256(static_cast<size_t>(S) * H * 4);
  l.total = o;
  return l;
}

template <typename T>
T *at(void *base, size_t off) {
  return reinterpret_cast<T *>(static_cast<uint8_t *>(base) + off);
}

}  // namespace

extern "C" {

size_t moeq_packed_bytes(int mode, int E, int R, int C, size_t out_sizes[5]) {
  size_t sz[5] = {0, 0, 0, 0, 0};
  if (E < 0 || R < 0 || C < 0 || C % 64) return 0;
  const size_t n = static_cast<size_t>(E) * R * C;
  const size_t nb = static_cast<size_t>(R) * C / 64;
  switch (mode) {
    case MOEQ_NF4:
      sz[0] = n / 2;
      sz[1] = static_cast<size_t>(E) * nb * 4;
      break;
    case MOEQ_NF4_DQ:
      sz[0] = n / 2;
      sz[2] = static_cast<size_t>(E) * nb;
      sz[3] = static_cast<size_t>(E) * ((nb + 255) / 256) * 4;
      sz[4] = static_cast<size_t>(E) * 4;
      break;
    case MOEQ_INT8_ROW:
      sz[0] = n;
      sz[1] = static_cast<size_t>(E) * R * 4;
      break;
    default:
      return 0;
  }
  if (out_sizes) std::memcpy(out_sizes, sz, sizeof(sz));
  return sz[0] + sz[1] + sz[2] + sz[3] + sz[4];
}

size_t moeq_quantize_workspace(int mode, int E, int R, int C) {
  if (mode != MOEQ_NF4_DQ || E <= 0 || R <= 0 || C <= 0 || C % 64) return 0;
  return quant_ws_layout(E, R, C).total;
}

size_t moeq_route_workspace(int T, int K, int E) {
  if (T < 0 || K <= 0 || E <= 0) return 0;
  return fwd_ws_layout(T, K, E, 0, 0).route_end;
}

size_t moeq_forward_workspace(int T, int K, int E, int H, int I) {
  if (T < 0 || K <= 0 || E <= 0 || H <= 0 || I <= 0) return 0;
  return fwd_ws_layout(T, K, E, H, I).total;
}

unsigned long long moeq_kernel_launches(void) { return g_launches.load(); }

void moeq_set_trace_events(void *const *events, int n) {
  t_trace_events = (events && n > 0) ? events : nullptr;
  t_trace_n = t_trace_events ? n : 0;
}

moeq_status moeq_quantize_nf4(const void *w_bf16, int E, int R, int C, int double_quant,
                              const moeq_packed *out, void *ws, size_t ws_bytes,
                              moeq_stream_t stream) {
  if (!out) return MOEQ_ERR_NULL;
  if (E < 0 || R < 0 || C < 0) return MOEQ_ERR_SHAPE;
  if (C % 64) return MOEQ_ERR_BLOCKSIZE;
  const int want_mode = double_quant ? MOEQ_NF4_DQ : MOEQ_NF4;
  if (out->mode != want_mode) return MOEQ_ERR_DTYPE;
  if (out->E != E || out->R != R || out->C != C) return MOEQ_ERR_SHAPE;
  const size_t n = static_cast<size_t>(E) * R * C;
  if (n == 0) return MOEQ_OK;
  if (!w_bf16) return MOEQ_ERR_NULL;
  if (!aligned16(w_bf16)) return MOEQ_ERR_ALIGN;
  moeq_status st = check_packed(out);
  if (st != MOEQ_OK) return st;
  if (double_quant) {
    if (!ws || ws_bytes < moeq_quantize_workspace(MOEQ_NF4_DQ, E, R, C)) return MOEQ_ERR_WORKSPACE;
    if (!aligned16(ws)) return MOEQ_ERR_ALIGN;
  }
  DevInfo di;
  if ((st = device_info(&di)) != MOEQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int launches = 0;
  float *absmax = out->absmax;
  QuantWs l{};
  if (double_quant) {
    l = quant_ws_layout(E, R, C);
    absmax = at<float>(ws, l.absmax);
  }
  cudaError_t e = launch_quant_nf4(w_bf16, n, static_cast<uint8_t *>(out->codes), absmax, di.sm_count, s,
                                   &launches);
  if (e == cudaSuccess && double_quant) {
    const int nb = static_cast<int>(static_cast<size_t>(R) * C / 64);
    e = launch_double_quant(absmax, E, nb, at<double>(ws, l.sums), out->absmax_q, out->absmax_scale,
                            out->absmax_offset, s, &launches);
  }
  return finish(e, launches);
}

moeq_status moeq_quantize_int8_rowwise(const void *w_bf16, int E, int R, int C,
                                       const moeq_packed *out, moeq_stream_t stream) {
  if (!out) return MOEQ_ERR_NULL;
  if (E < 0 || R < 0 || C < 0) return MOEQ_ERR_SHAPE;
  if (C % 64) return MOEQ_ERR_BLOCKSIZE;
  if (C > 131072) return MOEQ_ERR_SHAPE;
  if (out->mode != MOEQ_INT8_ROW) return MOEQ_ERR_DTYPE;
  if (out->E != E || out->R != R || out->C != C) return MOEQ_ERR_SHAPE;
  const size_t rows = static_cast<size_t>(E) * R;
  if (rows == 0 || C == 0) return MOEQ_OK;
  if (!w_bf16) return MOEQ_ERR_NULL;
  if (!aligned16(w_bf16)) return MOEQ_ERR_ALIGN;
  moeq_status st = check_packed(out);
  if (st != MOEQ_OK) return st;
  DevInfo di;
  if ((st = device_info(&di)) != MOEQ_OK) return st;
  int launches = 0;
  const cudaError_t e = launch_quant_int8_row(w_bf16, rows, C, static_cast<int8_t *>(out->codes), out->absmax,
                                              reinterpret_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

moeq_status moeq_dequantize(const moeq_packed *p, void *out, int out_dtype, moeq_stream_t stream) {
  moeq_status st = check_packed(p);
  if (st != MOEQ_OK) return st;
  if (out_dtype != MOEQ_BF16 && out_dtype != MOEQ_F32) return MOEQ_ERR_DTYPE;
  const size_t n = static_cast<size_t>(p->E) * p->R * p->C;
  if (n == 0) return MOEQ_OK;
  if (!out) return MOEQ_ERR_NULL;
  if (!aligned16(out)) return MOEQ_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di)) != MOEQ_OK) return st;
  int launches = 0;
  const cudaError_t e =
      launch_dequant(p, out, out_dtype == MOEQ_F32, di.sm_count, reinterpret_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

moeq_status moeq_route(const void *top_k_index, int index_dtype, int T, int K, int E, int32_t *counts,
                       int32_t *offsets, int32_t *perm, void *ws, size_t ws_bytes, int32_t *d_status,
                       moeq_stream_t stream) {
  if (T < 0 || K <= 0 || E <= 0 || E > 1024) return MOEQ_ERR_SHAPE;
  if (index_dtype != MOEQ_I32 && index_dtype != MOEQ_I64) return MOEQ_ERR_DTYPE;
  if (static_cast<long long>(T) * K > 0x7fffffffLL) return MOEQ_ERR_SHAPE;
  if (T == 0) return MOEQ_OK;
  if (!top_k_index || !counts || !offsets || !perm) return MOEQ_ERR_NULL;
  if (!aligned16(top_k_index) || !aligned16(counts) || !aligned16(offsets) || !aligned16(perm))
    return MOEQ_ERR_ALIGN;
  const FwdWs l = fwd_ws_layout(T, K, E, 0, 0);
  if (!ws || ws_bytes < l.route_end) return MOEQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOEQ_ERR_ALIGN;
  DevInfo di;
  moeq_status st = device_info(&di);
  if (st != MOEQ_OK) return st;
  const int S = T * K;
  const int nchunks = (S + kRouteChunk - 1) / kRouteChunk;
  int launches = 0;
  const cudaError_t e = launch_route(top_k_index, index_dtype == MOEQ_I64, S, E, nchunks, at<int32_t>(ws, l.counts_chunk),
                                     at<int32_t>(ws, l.chunk_base), counts, offsets, at<int32_t>(ws, l.ntp), perm,
                                     d_status, reinterpret_cast<cudaStream_t>(stream), &launches);
  return finish(e, launches);
}

moeq_status moeq_experts_forward(const void *hidden, const void *top_k_index, int index_dtype,
                                 const void *top_k_weights, int weight_dtype, int T, int K,
                                 const moeq_packed *gate_up, const moeq_packed *down, void *out,
                                 int out_dtype, void *ws, size_t ws_bytes, int32_t *d_status,
                                 moeq_stream_t stream) {
  if (T < 0 || K <= 0) return MOEQ_ERR_SHAPE;
  if (out_dtype != MOEQ_BF16 && out_dtype != MOEQ_F32) return MOEQ_ERR_DTYPE;
  if (index_dtype != MOEQ_I32 && index_dtype != MOEQ_I64) return MOEQ_ERR_DTYPE;
  if (weight_dtype != MOEQ_F32 && weight_dtype != MOEQ_BF16) return MOEQ_ERR_DTYPE;
  moeq_status st;
  if ((st = check_packed(gate_up)) != MOEQ_OK) return st;
  if ((st = check_packed(down)) != MOEQ_OK) return st;
  if (gate_up->mode != down->mode) return MOEQ_ERR_DTYPE;
  const int E = gate_up->E, H = gate_up->C, I = down->C;
  if (E <= 0 || E > 1024 || down->E != E) return MOEQ_ERR_SHAPE;
  if (gate_up->R != 2 * I || down->R != H) return MOEQ_ERR_SHAPE;
  if (H <= 0 || I <= 0 || H % 128 || I % 64) return MOEQ_ERR_SHAPE;
  if (static_cast<long long>(T) * K > 0x7fffffffLL) return MOEQ_ERR_SHAPE;
  if (T == 0) return MOEQ_OK;
  if (!hidden || !top_k_index || !top_k_weights || !out) return MOEQ_ERR_NULL;
  if (!aligned16(hidden) || !aligned16(top_k_index) || !aligned16(top_k_weights) || !aligned16(out))
    return MOEQ_ERR_ALIGN;
  const FwdWs l = fwd_ws_layout(T, K, E, H, I);
  if (!ws || ws_bytes < l.total) return MOEQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOEQ_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di)) != MOEQ_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int S = T * K;
  const int nchunks = (S + kRouteChunk - 1) / kRouteChunk;
  int32_t *status = d_status ? d_status : at<int32_t>(ws, l.status);
  int32_t *offsets = at<int32_t>(ws, l.offsets), *ntp = at<int32_t>(ws, l.ntp), *perm = at<int32_t>(ws, l.perm);
  int launches = 0;
  trace_mark(0, s);
  cudaError_t e = launch_route(top_k_index, index_dtype == MOEQ_I64, S, E, nchunks, at<int32_t>(ws, l.counts_chunk),
                               at<int32_t>(ws, l.chunk_base), at<int32_t>(ws, l.counts), offsets, ntp, perm, status,
                               s, &launches);
  trace_mark(1, s);
  void *xg = at<void>(ws, l.xg);
  void *h = at<void>(ws, l.h);
  float *slots = at<float>(ws, l.slots);
  if (e == cudaSuccess) e = launch_gather_rows(hidden, perm, offsets, E, S, K, H, xg, status, s, &launches);
  trace_mark(2, s);
  if (e == cudaSuccess) {
    GemmLaunch g{};
    g.mode = gate_up->mode;
    g.kind = 0;
    g.w = gate_up;
    g.I = I;
    g.S = S;
    g.act = xg;
    g.offsets = offsets;
    g.ntile_prefix = ntp;
    g.perm = perm;
    g.h_out = h;
    g.status = status;
    e = launch_moe_gemm(g, di.sm_count, s, &launches);
  }
  trace_mark(3, s);
  if (e == cudaSuccess) {
    GemmLaunch g{};
    g.mode = down->mode;
    g.kind = 1;
    g.w = down;
    g.I = I;
    g.S = S;
    g.act = h;
    g.offsets = offsets;
    g.ntile_prefix = ntp;
    g.perm = perm;
    g.slot_out = slots;
    g.topk_w = top_k_weights;
    g.w_bf16 = weight_dtype == MOEQ_BF16;
    g.status = status;
    e = launch_moe_gemm(g, di.sm_count, s, &launches);
  }
  trace_mark(4, s);
  if (e == cudaSuccess) e = launch_combine(slots, top_k_index, index_dtype == MOEQ_I64, T, K, E, H, out, out_dtype == MOEQ_F32, s,
                                          &launches);
  trace_mark(5, s);
  return finish(e, launches);
}

const char *moeq_status_string(moeq_status s) {
  switch (s) {
    case MOEQ_OK: return "ok";
    case MOEQ_ERR_NULL: return "null pointer";
    case MOEQ_ERR_SHAPE: return "bad shape";
    case MOEQ_ERR_DTYPE: return "bad dtype or mode";
    case MOEQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MOEQ_ERR_BLOCKSIZE: return "reduction dim not a multiple of 64";
    case MOEQ_ERR_WORKSPACE: return "workspace missing or too small";
    case MOEQ_ERR_CUDA: return "CUDA error";
    case MOEQ_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MOEQ_ERR_INDEX: return "top_k_index out of range (pair dropped)";
    case MOEQ_ERR_DEVICE: return "device is not sm_100 (B200)";
    case MOEQ_ERR_RANGE: return "activation beyond fp16 range was saturated";
  }
  return "unknown status";
}

}  // extern "C"
