/*
 * moeq.h - C ABI of the quantized fused-MoE experts library (one NVIDIA B200, sm_100a).
 *
 * What the library computes, and where each operation is defined:
 *
 *   The fused expert layout is that of "Failed to quant MoE models with fused expert
 *   weights in transformers v5" (bitsandbytes issue #1849), section "Description":
 *   gate_up_proj [E, 2I, H] and down_proj [E, H, I], bf16, one tensor per layer.
 *   A 3-D weight is written W[E, R, C] row-major with C the reduction dim
 *   (in_features): gate_up has R = 2I, C = H; down has R = H, C = I.
 *
 *   Quantize-on-load ("MoE Expert Quantization", section "Implementation details":
 *   each expert tensor is quantized as it loads and the bf16 original freed at once):
 *     - NF4: blocks of 64 consecutive elements along C; absmax = max|x| (fp32);
 *       n = x / absmax (IEEE fp32 divide); code = nearest of the 16 NormalFloat-4
 *       levels, ties to the lower index; two codes per byte, the first element in
 *       the high nibble.  absmax == 0 gives code 7 (the 0.0 level) everywhere.
 *       Blocksize 64 and C % 64 == 0 follow the maintainer comments in #1849.
 *     - NF4 with double quantization (#1849: compress_statistics): each expert's
 *       absmax vector (nb = R*C/64 values) is stored as int8 blocks of 256 with an
 *       fp32 scale per block and an fp32 mean offset per expert:
 *         off = fp32(fp64 sum, fixed order: 256-chunks sequentially, then chunks
 *               sequentially) / nb;  v = fl(a - off); s = max|v| per block;
 *         q = rint(fl(fl(127 v) / s)), q = 0 where s == 0;
 *         decoded absmax = fl(fl(q * fl(s / 127)) + off).
 *     - int8 row-wise ("MoE Expert Quantization": a row-wise int8 parametrization
 *       with bitsandbytes dequantization): per row absmax; q = rint(fl(127 x) / absmax)
 *       half to even; dequantized w = fl(q * fl(absmax / 127)).
 *
 *   Forward (unsloth-zoo issue #850: the experts interface
 *   (hidden_states, top_k_index, top_k_weights); gate is the first I rows of dim 1
 *   of gate_up, never inferred from the shape):
 *     out[t] = sum_k w[t,k] * down_e( silu(gate_e x_t) * up_e x_t ),  e = idx[t,k],
 *   with silu(z) = z / (1 + exp(-z)), fp32 accumulation, the k terms added in k
 *   order, the result rounded once to bf16 (or returned in fp32, out_dtype MOEQ_F32).
 *   top_k_weights are used as given.  The tensor-core operands are fp16 (the compute
 *   dtype of the pages' bitsandbytes reproduction, bnb_4bit_compute_dtype=float16):
 *   the hidden rows (converted from bf16, exact for 6.1e-5 <= |x| <= 65504), the
 *   intermediate h, and the weights decoded in the GEMM: fp16(fp16(level) *
 *   fp16(absmax)) for NF4, the exact code q for int8 (its row scale is applied to the
 *   fp32 accumulator).  Larger magnitudes saturate and report MOEQ_ERR_RANGE.
 *   moeq_dequantize is unaffected: it returns the exact dequantized values above.
 *
 * Conventions (every entry point):
 *   - Memory: every pointer argument is a DEVICE pointer, 16-byte aligned, unless the
 *     comment says host.  The library never allocates or frees device memory; the
 *     caller owns every buffer (inputs, outputs, workspace) and frees the bf16
 *     source after quantizing it.
 *   - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns before it runs.  Calls keep no state between them
 *     and may be made from several host threads on different streams.
 *   - Errors found on the host (null pointers, shapes, alignment, C % 64, workspace
 *     size, unsupported device) return a status before anything is enqueued.  A
 *     failed launch returns MOEQ_ERR_CUDA.  Errors in the data (a top_k_index outside
 *     [0, E)) never trap: the pair is dropped (adds nothing) and MOEQ_ERR_INDEX is
 *     written to *d_status when d_status is not NULL.
 *   - Empty inputs: T == 0 (forward) or E*R*C == 0 (quantize/dequantize) return
 *     MOEQ_OK and enqueue nothing.
 */
#ifndef MOEQ_H_
#define MOEQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *moeq_stream_t; /* same object as cudaStream_t */

typedef enum {
  MOEQ_OK = 0,
  MOEQ_ERR_NULL = 1,       /* a required pointer is NULL */
  MOEQ_ERR_SHAPE = 2,      /* a size is negative, zero where it may not be, or mismatched */
  MOEQ_ERR_DTYPE = 3,      /* unknown dtype or mode code */
  MOEQ_ERR_ALIGN = 4,      /* a pointer is not 16-byte aligned */
  MOEQ_ERR_BLOCKSIZE = 5,  /* C % 64 != 0 (NF4 blocks may not straddle rows) */
  MOEQ_ERR_WORKSPACE = 6,  /* workspace NULL or smaller than the *_workspace() size */
  MOEQ_ERR_CUDA = 7,       /* a CUDA call or kernel launch failed */
  MOEQ_ERR_TIMEOUT = 8,    /* device: a pipeline wait ran past its limit (a bug) */
  MOEQ_ERR_INDEX = 9,      /* device: a top_k_index value outside [0, E) was dropped */
  MOEQ_ERR_DEVICE = 10,    /* the current device is not compute capability 10.0 */
  MOEQ_ERR_RANGE = 11      /* device: an activation (hidden or h) or an NF4 block absmax
                              beyond the fp16 range of the tensor-core operands
                              (|v| > 65504) was saturated */
} moeq_status;

typedef enum { MOEQ_NF4 = 0, MOEQ_NF4_DQ = 1, MOEQ_INT8_ROW = 2 } moeq_mode;
typedef enum { MOEQ_BF16 = 0, MOEQ_F32 = 1, MOEQ_I32 = 2, MOEQ_I64 = 3 } moeq_dtype;

/* Describes one packed 3-D weight W[E, R, C].  The caller fills the pointers with
 * buffers of the sizes moeq_packed_bytes() reports; the library only reads or writes
 * through them.  This is the storage the bitsandbytes #1849 thread settles on: the
 * packed weight as one plain tensor plus module-owned quantization metadata, absmax
 * kept per expert ([num_experts, blocks_per_expert]) so experts stay sliceable. */
typedef struct {
  int32_t mode;          /* moeq_mode */
  int32_t E, R, C;       /* C = reduction dim; C % 64 == 0 */
  void *codes;           /* NF4*: u8 [E, R, C/2], element 2j -> high nibble of byte j,
                            element 2j+1 -> low nibble.  INT8_ROW: i8 [E, R, C] */
  float *absmax;         /* NF4: f32 [E, R, C/64].  INT8_ROW: f32 [E, R].  NF4_DQ: unused */
  int8_t *absmax_q;      /* NF4_DQ: i8 [E, R*C/64] */
  float *absmax_scale;   /* NF4_DQ: f32 [E, ceil(R*C/64/256)] */
  float *absmax_offset;  /* NF4_DQ: f32 [E] */
} moeq_packed;

/* Bytes of each buffer of a packed [E, R, C] weight in `mode`.  out_sizes (host,
 * may be NULL) receives {codes, absmax, absmax_q, absmax_scale, absmax_offset}; an
 * unused buffer has size 0.  Returns the total, or 0 for an invalid mode or shape.
 * Host only; no device work. */
size_t moeq_packed_bytes(int mode, int E, int R, int C, size_t out_sizes[5]);

/* Device workspace bytes moeq_quantize_nf4 needs (0 unless mode == MOEQ_NF4_DQ,
 * which needs the fp32 absmax and the fixed-order fp64 chunk sums).  Host only. */
size_t moeq_quantize_workspace(int mode, int E, int R, int C);

/* NF4 quantization of w_bf16 [E, R, C] (bf16, device) into the buffers of *out
 * (host struct; out->mode must be MOEQ_NF4 when double_quant == 0, MOEQ_NF4_DQ
 * otherwise, and out->E/R/C must match).  ws: device workspace of at least
 * moeq_quantize_workspace(out->mode, E, R, C) bytes (may be NULL when that is 0).
 * Codes, absmax and the double-quant fields are bit-exact to the definition above. */
moeq_status moeq_quantize_nf4(const void *w_bf16, int E, int R, int C, int double_quant,
                              const moeq_packed *out, void *ws, size_t ws_bytes,
                              moeq_stream_t stream);

/* Row-wise int8 quantization of w_bf16 [E, R, C] into *out (out->mode ==
 * MOEQ_INT8_ROW).  No workspace.  Bit-exact to the definition above. */
moeq_status moeq_quantize_int8_rowwise(const void *w_bf16, int E, int R, int C,
                                       const moeq_packed *out, moeq_stream_t stream);

/* Dequantize *p into out [E, R, C] as bf16 (out_dtype MOEQ_BF16: round to nearest
 * even of the fp32 value) or fp32 (MOEQ_F32).  NF4: w = fl(c[code] * absmax');
 * INT8_ROW: w = fl(q * fl(absmax / 127)).  Bit-exact. */
moeq_status moeq_dequantize(const moeq_packed *p, void *out, int out_dtype,
                            moeq_stream_t stream);

/* Device workspace bytes moeq_experts_forward needs for T tokens, top-K, E experts,
 * hidden H and intermediate I (routing tables, the expert-sorted activations, the
 * intermediate h and the per-(token, k) partial outputs).  Host only. */
size_t moeq_forward_workspace(int T, int K, int E, int H, int I);

/* Routed experts forward from packed weights.
 *   hidden        bf16 [T, H]
 *   top_k_index   [T, K], int32 (index_dtype MOEQ_I32) or int64 (MOEQ_I64)
 *   top_k_weights [T, K], fp32 (weight_dtype MOEQ_F32) or bf16 (MOEQ_BF16)
 *   gate_up       packed [E, 2I, H];  down: packed [E, H, I]; same mode and E
 *                 (modes NF4, NF4_DQ or INT8_ROW; H % 128 == 0, I % 64 == 0)
 *   out           [T, H], fully overwritten: bf16 (out_dtype MOEQ_BF16, the fp32 sum
 *                 rounded once, to nearest even) or fp32 (MOEQ_F32, the sum itself)
 *   ws            device workspace of at least moeq_forward_workspace(T, K, E, H, I)
 *   d_status      optional device int32, zeroed by the caller: when the device finds
 *                 bad data it writes a moeq_status code there if the word is still 0
 *                 (first error wins); left untouched otherwise.
 * The result is deterministic: identical inputs give identical output bits. */
moeq_status moeq_experts_forward(const void *hidden, const void *top_k_index, int index_dtype,
                                 const void *top_k_weights, int weight_dtype, int T, int K,
                                 const moeq_packed *gate_up, const moeq_packed *down,
                                 void *out, int out_dtype, void *ws, size_t ws_bytes,
                                 int32_t *d_status, moeq_stream_t stream);

/* Routing step of the forward on its own (the grouping of the (t, k) pairs by
 * expert): counts [E] (int32), offsets [E+1] (int32, exclusive prefix sum of counts)
 * and perm [T*K] (int32: the flat pair index t*K+k listed by expert, in increasing
 * pair order within an expert; only the first offsets[E] entries are written).
 * Indices outside [0, E) are dropped and reported through d_status (as in the
 * forward).  ws: device workspace of at least moeq_route_workspace(T, K, E) bytes. */
moeq_status moeq_route(const void *top_k_index, int index_dtype, int T, int K, int E,
                       int32_t *counts, int32_t *offsets, int32_t *perm, void *ws,
                       size_t ws_bytes, int32_t *d_status, moeq_stream_t stream);

/* The routing step of moeq_route without a workspace, for callers that cannot allocate
 * device memory: a host runtime that keeps the whole device for its own memory pool and
 * forbids allocations outside it, or a latency-critical loop in which cudaMalloc/cudaFree
 * would synchronise the device.  (The pages have no counterpart: this is a library
 * convenience, not part of the method.)  Same arguments and results as moeq_route, minus
 * ws/ws_bytes.  Its scratch is a fixed 2 MiB __device__ array inside the library, held by
 * every GPU that loads the library until the process exits; it covers
 * 2*ceil(T*K/512)*E*4 + (E+1)*4 bytes (each part rounded up to 256) and larger problems
 * return MOEQ_ERR_WORKSPACE.  The first call on a device looks up the array's device
 * address with that device current: make that first call before any stream capture.
 * All calls share the array; calls that overlap on the GPU (e.g. on two unordered
 * streams) race on it.  Allocates nothing, frees nothing. */
moeq_status moeq_route_noalloc(const void *top_k_index, int index_dtype, int T, int K, int E,
                               int32_t *counts, int32_t *offsets, int32_t *perm,
                               int32_t *d_status, moeq_stream_t stream);

/* Device workspace bytes moeq_route needs.  Host only. */
size_t moeq_route_workspace(int T, int K, int E);

/* Number of kernels this library has enqueued since it was loaded, all devices and
 * threads together (a host-side counter, for launch accounting).  Host only. */
unsigned long long moeq_kernel_launches(void);

/* Launch tracing (instrumentation, for timing each kernel with CUDA events on the
 * stream it runs on).  `events` (host array of n cudaEvent_t handles, created by the
 * caller) is kept for the calling host thread; every later moeq_experts_forward on
 * that thread records events[0] before its first kernel and events[1..5] after its
 * routing kernels, the row gather, the gate_up GEMM, the down GEMM and the combine
 * (fewer if n < 6).  Pass NULL / 0 to stop.  Host only. */
void moeq_set_trace_events(void *const *events, int n);

/* Human-readable name of a status code (static string). */
const char *moeq_status_string(moeq_status s);

#ifdef __cplusplus
}
#endif
#endif /* MOEQ_H_ */
