// moeq_route_noalloc: the routing step of the experts forward (moeq_route) for callers
// that cannot give the library a workspace.
//
// Some callers cannot call cudaMalloc: a host runtime that has reserved the device's
// memory for its own pool and forbids allocations outside it, or a latency-critical
// loop where cudaMalloc / cudaFree would synchronise the device and stall its other
// streams.  This entry point needs no workspace: its scratch (the per-chunk expert
// counts, the per-chunk bases and the token-tile prefix) lives in a file-scope
// __device__ array of kRouteScratchBytes, which every GPU that loads the library holds
// until the process exits.  The caller still passes the inputs and the outputs.
//
// The host cannot use the array's name as a device address: in host code it is only a
// stand-in, and a kernel given it would fault (or, where the GPU can reach host memory,
// silently use the wrong memory).  So the first call on each device, with that device
// current, asks the runtime for the array's device address (cudaGetSymbolAddress) and
// keeps it; later calls on that device reuse it.  That first call should come before
// any stream capture on the device.
//
// Every call shares the one array.  Nothing in it needs to start at zero: every word
// the routing kernels read is written earlier in the same call.  It keeps the last
// call's contents, and two calls whose work overlaps on the GPU (different streams,
// no ordering between them) race on it.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/moeq.h"
#include "kernels.h"

namespace {

constexpr size_t kRouteScratchBytes = size_t(2) << 20;  // 2 MiB per device
__device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device (set up on first use).
moeq_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOEQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOEQ_ERR_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MOEQ_ERR_CUDA;
  if (major != 10 || minor != 0) return MOEQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return MOEQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOEQ_OK;
}

}  // namespace

extern "C" moeq_status moeq_route_noalloc(const void *top_k_index, int index_dtype, int T, int K, int E,
                                          int32_t *counts, int32_t *offsets, int32_t *perm,
                                          int32_t *d_status, moeq_stream_t stream) {
  if (T < 0 || K <= 0 || E <= 0 || E > 1024) return MOEQ_ERR_SHAPE;
  if (index_dtype != MOEQ_I32 && index_dtype != MOEQ_I64) return MOEQ_ERR_DTYPE;
  if (static_cast<long long>(T) * K > 0x7fffffffLL) return MOEQ_ERR_SHAPE;
  if (T == 0) return MOEQ_OK;
  if (!top_k_index || !counts || !offsets || !perm) return MOEQ_ERR_NULL;
  if (!aligned16(top_k_index) || !aligned16(counts) || !aligned16(offsets) || !aligned16(perm))
    return MOEQ_ERR_ALIGN;
  const int S = T * K;
  const int nchunks = (S + moeq::kRouteChunk - 1) / moeq::kRouteChunk;
  const size_t table = align256(static_cast<size_t>(nchunks) * E * sizeof(int32_t));
  const size_t need = 2 * table + align256(static_cast<size_t>(E + 1) * sizeof(int32_t));
  if (need > kRouteScratchBytes) return MOEQ_ERR_WORKSPACE;  // beyond the fixed scratch
  void *scratch = nullptr;
  const moeq_status st = scratch_address(&scratch);
  if (st != MOEQ_OK) return st;
  uint8_t *base = static_cast<uint8_t *>(scratch);
  int launches = 0;
  const cudaError_t e = moeq::launch_route(
      top_k_index, index_dtype == MOEQ_I64, S, E, nchunks, reinterpret_cast<int32_t *>(base),
      reinterpret_cast<int32_t *>(base + table), counts, offsets, reinterpret_cast<int32_t *>(base + 2 * table),
      perm, d_status, reinterpret_cast<cudaStream_t>(stream), &launches);
  return e == cudaSuccess ? MOEQ_OK : MOEQ_ERR_CUDA;
}
