// Internal launcher declarations shared by the translation units of libmoeq.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moeq.h"

namespace moeq {

// quant.cu
cudaError_t launch_quant_nf4(const void *w, size_t n_elems, uint8_t *codes, float *absmax,
                             int sm_count, cudaStream_t s, int *launches);
cudaError_t launch_double_quant(const float *absmax_f32, int E, int nb, double *chunk_sums,
                                int8_t *q_out, float *scale, float *off, cudaStream_t s,
                                int *launches);
cudaError_t launch_quant_int8_row(const void *w, size_t rows, int C, int8_t *codes, float *absmax,
                                  cudaStream_t s, int *launches);
cudaError_t launch_dequant(const moeq_packed *p, void *out, bool f32, int sm_count, cudaStream_t s,
                           int *launches);

// route.cu
constexpr int kRouteChunk = 512;  // (t,k) pairs per routing chunk (one warp, 16 x 32)
constexpr int kTileN = 192;       // tokens per GEMM tile (UMMA N upper bound)
cudaError_t launch_route(const void *idx, bool idx64, int S, int E, int nchunks,
                         int32_t *counts_chunk, int32_t *chunk_base, int32_t *counts,
                         int32_t *offsets, int32_t *ntile_prefix, int32_t *perm, int32_t *status,
                         cudaStream_t s, int *launches);
cudaError_t launch_gather_rows(const void *x, const int32_t *perm, const int32_t *offsets, int E,
                               int S, int K, int H, void *xg, int32_t *status, cudaStream_t s,
                               int *launches);
cudaError_t launch_combine(const float *slots, const void *idx, bool idx64, int T, int K, int E,
                           int H, void *out, bool f32_out, cudaStream_t s, int *launches);

// gemm.cu
struct GemmLaunch {
  int mode;       // moeq_mode
  int kind;       // 0 = gate_up (+ SiLU*up epilogue), 1 = down (+ weighted slot epilogue)
  const moeq_packed *w;
  int I;          // intermediate size (gate_up: R = 2I; down: C = I)
  int S;          // rows of the activation operand (T*K)
  const void *act;  // fp16 [S, C] activation rows in expert-sorted order
  const int32_t *offsets, *ntile_prefix, *perm;
  void *h_out;      // gate_up: fp16 [S, I]
  float *slot_out;  // down: f32 [T*K, H]
  const void *topk_w;
  int w_bf16;
  int32_t *status;
};
cudaError_t launch_moe_gemm(const GemmLaunch &g, int sm_count, cudaStream_t s, int *launches);

}  // namespace moeq
