// Grouped expert GEMMs straight from packed NF4 / int8 weights (sm_100a, tcgen05 + TMEM).
//
// What is computed (bitsandbytes issue #1849, "Description": gate_up_proj [E, 2I, H],
// down_proj [E, H, I], act = SiLU; the fused grouped NF4 GEMM described later in that
// thread decodes NF4 inside the mainloop with fp32 accumulation and never materialises
// a dequantized weight tensor):
//   gate_up:  h[s, j] = silu(x_s . G_e[j]) * (x_s . U_e[j]),  G = rows [0, I), U = rows
//             [I, 2I) of gate_up[e]  (gate is never inferred from the shape: unsloth-zoo
//             issue #850 on the square OLMoE gate_up)
//   down:     slot[p, i] = w_p * (h_s . D_e[i])   with p = perm[s] the (t, k) pair of s
// over the expert-sorted rows s of each expert e.
//
// Tile = 128 weight rows (UMMA M, operand A) x up to 192 tokens (UMMA N, operand B) x
// K in steps of 64 (one NF4 block).  Both operands are fp16 (weights dequantized to fp16,
// activations and h stored as fp16), accumulation fp32.  The dequantized weights never
// touch shared memory: the dequant warps store them straight into tensor memory
// (tcgen05.st) and the MMA reads operand A from there; only the token tiles (TMA, 128B
// swizzle) and the packed codes go through shared memory.
//   warps 0-7   epilogue: TMEM -> registers (tcgen05.ld), SiLU*up or weighted slot stores;
//               warp w reads TMEM lanes 32*(w%4).. and half the tile's columns
//   warps 8-23  dequant: packed codes (TMA'd into SMEM) -> fp16 A stage in TMEM, one
//               weight row per thread; four groups of 4 warps take K stages in turn
//   warp 24     TMA of the packed-code tiles
//   warp 25     TMA of the token tiles, a pair of K stages at a time
//   warp 26     TMEM allocation and the single-thread tcgen05.mma issue (8 MMAs per pair)
//   warp 27     relay: a pair's token tiles have landed -> the pair's full barrier
// TMEM (512 columns): two 192-column fp32 accumulators (the epilogue of one tile overlaps
// the mainloop of the next) and 4 32-column fp16 A stages (2 pairs).  The CTA is
// persistent over a tile list derived on the device from the routing (per-expert token
// counts).  Every mbarrier wait is bounded (2 s); a timeout raises MOEQ_ERR_TIMEOUT and
// the CTA drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace moeq {

constexpr int BM = 128;
constexpr int BN = kTileN;  // 192
constexpr int BK = 64;
// The operand rings advance in pairs of K stages: one pair = 2 x 64 of K = 8 MMAs of
// K = 16, and one full/empty barrier pair covers both the A and B halves of a pair.  The
// single MMA-issuing thread then waits and commits once per 8 MMAs: at N = 192 an MMA
// runs ~96 cycles and the tensor core queues few instructions, so a wait and a commit
// per 4 MMAs leave the tensor pipe idle between stages.
constexpr int kPairSlots = 2;        // pairs of A stages in TMEM
constexpr int kAStages = 2 * kPairSlots;  // dequantized weight stages in TMEM
constexpr int kBPairs = 3;           // pairs of token tiles in shared memory (a 48 KB pair
                                     // takes ~1000 cycles to land: two pairs of lead)
constexpr int kBStages = 2 * kBPairs;
constexpr int kDonePairs = 6;        // pair-completion barriers (a multiple of 2 and 3)
constexpr uint32_t kAccCols = BN;    // fp32 columns per accumulator
constexpr uint32_t kACol0 = 2 * kAccCols;  // first TMEM column of the A ring
constexpr uint32_t kAStageCols = 32;       // 64 fp16 per row = 32 columns
static_assert(kACol0 + kAStages * kAStageCols <= 512, "accumulators and A ring fit in TMEM");
constexpr int kEpiWarps = 8;
constexpr int kDequantGroups = 4;    // groups take K stages in turn
constexpr int kGroupWarps = 4;       // per group: 128 rows, one per thread
constexpr int kDequantWarps = kDequantGroups * kGroupWarps;
static_assert((kDequantGroups & (kDequantGroups - 1)) == 0, "groups are picked with a mask");
constexpr int kDequantThread0 = kEpiWarps * 32;
constexpr int kCodeProducerWarp = kEpiWarps + kDequantWarps;
constexpr int kBProducerWarp = kCodeProducerWarp + 1;
constexpr int kMmaWarp = kBProducerWarp + 1;
constexpr int kRelayWarp = kMmaWarp + 1;
constexpr int kThreads = (kRelayWarp + 1) * 32;
constexpr int kGroupM = 16;  // m-tiles walked per token tile before moving on (L2 reuse)
constexpr uint32_t kBBytes = BN * BK * 2;
constexpr int kMaxExperts = 1024;  // the largest expert count the entry points accept
// NF4 pair table: for every code byte (two 4-bit codes) the two levels as an fp16 pair,
// one copy per lane: entry (byte, lane) at byte*128 + lane*4, so a warp's 32 lookups hit
// 32 different banks, and the address is a byte permute and a shift.
constexpr uint32_t kLutBytes = 256 * 128;

// Ring depths.  The packed codes stream from HBM once per token tile, so their ring is
// the deep one: each dequant group finds several of its stages already landed (a group
// copies its codes to registers and frees the slot at once).
template <int MODE>
struct Cfg {
  static constexpr uint32_t kCodeRow = (MODE == MOEQ_INT8_ROW) ? 64 : 32;  // bytes/row/stage
  static constexpr uint32_t kCodeBytes = BM * kCodeRow;
  static constexpr int kCStages = (MODE == MOEQ_INT8_ROW) ? 8 : 10;  // packed-code tiles
  static constexpr uint32_t kBOff = 0;
  static constexpr uint32_t kCOff = kBOff + kBStages * kBBytes;
  static constexpr uint32_t kLutOff = kCOff + kCStages * kCodeBytes;
  static constexpr uint32_t kLut = (MODE == MOEQ_INT8_ROW) ? 0 : kLutBytes;
  static constexpr uint32_t kCtrlOff = kLutOff + kLut;
  static constexpr int kNumBars = kPairSlots + kDonePairs + kBPairs + 2 * kCStages + 5;
  // per-expert token-tile prefix and row offsets, copied once so that every role decodes
  // its next tile from shared memory instead of a chain of dependent global loads
  static constexpr uint32_t kTabOff = kCtrlOff + kNumBars * 8 + 16;
  static constexpr uint32_t kSmem = kTabOff + 2 * (kMaxExperts + 1) * 4 + 1024;
  static_assert(kSmem <= 232448, "shared memory per block");
};

// The 16 NormalFloat-4 levels (fp32), the table the packed codes index.
__constant__ float kNF4Levels[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
    0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};

__device__ __forceinline__ uint32_t box_rows(int nbox) { return nbox < 4 ? (16u << nbox) : 192u; }

struct TmapSet {
  CUtensorMap b[5];  // activation rows, boxes of 16, 32, 64, 128, 192 rows x 64 elements
  CUtensorMap codes; // packed codes, [E*R rows, bytes per row], box 64 rows x kCodeRow
};

struct GemmArgs {
  const float *absmax;      // NF4: [E*R, C/64]; INT8: [E*R]
  const int8_t *aq;         // NF4_DQ
  const float *ascale;      // NF4_DQ
  const float *aoff;        // NF4_DQ
  int E, R, C, I, MT, nk, nb, nblk;
  const int32_t *offsets;
  const int32_t *ntp;
  const int32_t *perm;
  __half *h_out;
  float *slot_out;
  const void *topk_w;
  int w_bf16;
  int32_t *status;
};

struct Tile {
  int e, m, row0, count, nbox;
};

// ntp / offs: the expert tables in shared memory (E + 1 entries each)
__device__ __forceinline__ Tile decode_tile(int tile, const GemmArgs &a, const int *ntp, const int *offs) {
  int lo = 0, hi = a.E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ntp[mid] * a.MT <= tile) lo = mid;
    else hi = mid;
  }
  Tile t;
  t.e = lo;
  const int NT = ntp[lo + 1] - ntp[lo];
  const int local = tile - ntp[lo] * a.MT;
  const int gfull = NT * kGroupM;
  const int g = local / gfull;
  const int rem = local - g * gfull;
  const int Gg = min(kGroupM, a.MT - g * kGroupM);
  const int nt = rem / Gg;
  t.m = g * kGroupM + (rem - nt * Gg);
  const int off = offs[lo];
  const int n_e = offs[lo + 1] - off;
  const int n0 = nt * BN;
  t.count = min(BN, n_e - n0);
  t.row0 = off + n0;
  t.nbox = t.count <= 16 ? 0 : t.count <= 32 ? 1 : t.count <= 64 ? 2 : t.count <= 128 ? 3 : 4;
  return t;
}

// Shared-memory accesses as plain loads/stores through the dynamic shared buffer, so the
// compiler is free to interleave the many independent table lookups of a dequant thread.
__device__ __forceinline__ uint32_t lds_u32(const uint8_t *smem, uint32_t off) {
  return *reinterpret_cast<const uint32_t *>(smem + off);
}
__device__ __forceinline__ uint4 lds_u4(const uint8_t *smem, uint32_t off) {
  return *reinterpret_cast<const uint4 *>(smem + off);
}

// packed fp16 a - b (round to nearest; exact for the small integers it is used on)
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Decode step s/127 of the double-quantized absmax, kept for the 256-block group it
// belongs to (a thread walks one weight row, so the group rarely changes).
struct DqStep {
  int group = -1;
  float step = 0.0f;
};

// fp32 absmax of weight row `wr` (expert e), NF4 block kb
template <int MODE>
__device__ __forceinline__ float load_absmax(const GemmArgs &a, int e, int wr, int kb, DqStep &dq) {
  if (MODE == MOEQ_NF4) {
    return __ldg(a.absmax + (static_cast<size_t>(e) * a.R + wr) * (a.C / 64) + kb);
  } else if (MODE == MOEQ_NF4_DQ) {
    const int b = wr * (a.C / 64) + kb;  // block index inside expert e
    const float q = static_cast<float>(__ldg(a.aq + static_cast<size_t>(e) * a.nb + b));
    const int g = e * a.nblk + (b >> 8);
    if (g != dq.group) {
      dq.group = g;
      dq.step = __fdiv_rn(__ldg(a.ascale + g), 127.0f);
    }
    return __fadd_rn(__fmul_rn(q, dq.step), __ldg(a.aoff + e));
  }
  return 0.0f;
}

template <int MODE, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    k_moe_gemm(const __grid_constant__ TmapSet maps, const GemmArgs args) {
  using CF = Cfg<MODE>;
  constexpr int kCS = CF::kCStages;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, kept as shared-array arithmetic so accesses stay shared loads
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint8_t *ctrl = smem + CF::kCtrlOff;
  const uint32_t bar0 = smem_u32(ctrl);
  // barriers: FULL (a pair's A stages are in TMEM and its token tiles have landed: what
  // the MMA waits on), DONE (the MMAs of pair j have completed, on DONE(j % 6)), BFULL
  // (a pair's token-tile copies), code ring full/empty, accumulator full/empty (x2), drain
  auto FULL = [&](uint32_t i) -> uint32_t { return bar0 + 8u * i; };
  auto DONE = [&](uint32_t i) -> uint32_t { return bar0 + 8u * (kPairSlots + i); };
  auto BFULL = [&](uint32_t i) -> uint32_t { return bar0 + 8u * (kPairSlots + kDonePairs + i); };
  constexpr int kC0 = kPairSlots + kDonePairs + kBPairs;
  auto C_FULL = [&](uint32_t i) -> uint32_t { return bar0 + 8u * (kC0 + i); };
  auto C_EMPTY = [&](uint32_t i) -> uint32_t { return bar0 + 8u * (kC0 + kCS + i); };
  constexpr int kAcc0 = kC0 + 2 * kCS;
  auto ACC_FULL = [&](int b) -> uint32_t { return bar0 + 8u * (kAcc0 + b); };
  auto ACC_EMPTY = [&](int b) -> uint32_t { return bar0 + 8u * (kAcc0 + 2 + b); };
  const uint32_t DRAIN = bar0 + 8u * (kAcc0 + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctrl + CF::kNumBars * 8);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + CF::kNumBars * 8 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPairSlots; ++i) {
      // the relay (token tiles landed) and, per K stage of the pair, one arrival per warp
      // of the dequant group that wrote it (a lone last stage arrives twice)
      mbar_init(FULL(i), 2 * kGroupWarps + 1);
    }
    for (int i = 0; i < kDonePairs; ++i) mbar_init(DONE(i), 1);  // MMA commit
    for (int i = 0; i < kBPairs; ++i) mbar_init(BFULL(i), 1);    // producer arrive + tx bytes
    for (int i = 0; i < kCS; ++i) {
      mbar_init(C_FULL(i), 1);            // producer arrive + tx bytes
      mbar_init(C_EMPTY(i), kGroupWarps); // the group has read the codes
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(ACC_FULL(b), 1);          // MMA commit
      mbar_init(ACC_EMPTY(b), kEpiWarps); // one arrival per epilogue warp
    }
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (MODE != MOEQ_INT8_ROW) {
    // NF4 pair table (see kLutBytes): entry (byte, lane) = (c[byte >> 4], c[byte & 15])
    for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
      const int byte = i >> 5, l = i & 31;
      *reinterpret_cast<__half2 *>(smem + CF::kLutOff + byte * 128 + l * 4) =
          __floats2half2_rn(kNF4Levels[byte >> 4], kNF4Levels[byte & 15]);
    }
  }
  int *s_ntp = reinterpret_cast<int *>(smem + CF::kTabOff);
  int *s_off = s_ntp + (kMaxExperts + 1);
  for (int i = threadIdx.x; i <= args.E; i += kThreads) {
    s_ntp[i] = __ldg(args.ntp + i);
    s_off[i] = __ldg(args.offsets + i);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kBProducerWarp && lane == 0) {
    for (int i = 0; i < 5; ++i) tma_prefetch_desc(&maps.b[i]);
  }
  if (warp == kCodeProducerWarp && lane == 0) tma_prefetch_desc(&maps.codes);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total_tiles = s_ntp[args.E] * args.MT;
  const int nk = args.nk;

  if (warp == kCodeProducerWarp) {
    // ---------------- packed-code producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const Tile t = decode_tile(tile, args, s_ntp, s_off);
        int y0, y1;
        if (KIND == 0) {
          y0 = t.e * args.R + t.m * 64;
          y1 = y0 + args.I;
        } else {
          y0 = t.e * args.R + t.m * 128;
          y1 = y0 + 64;
        }
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kCS, ph = (it / kCS) & 1u;
          if (!mbar_wait(C_EMPTY(s), ph ^ 1u, abort_flag, args.status)) { ok = false; break; }
          const uint32_t dst = sbase + CF::kCOff + s * CF::kCodeBytes;
          mbar_arrive_expect_tx(C_FULL(s), CF::kCodeBytes);
          tma_load_2d(dst, &maps.codes, kb * CF::kCodeRow, y0, C_FULL(s));
          tma_load_2d(dst + 64 * CF::kCodeRow, &maps.codes, kb * CF::kCodeRow, y1, C_FULL(s));
        }
      }
      // drain: every copy issued lands before the CTA may exit
      const uint32_t n = it < static_cast<uint32_t>(kCS) ? it : static_cast<uint32_t>(kCS);
      for (uint32_t d = 0; d < n; ++d) {
        const uint32_t j = it - 1 - d;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(C_FULL(j % kCS), (j / kCS) & 1u)) {
          if (globaltimer() - t0 > kWaitLimitNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == kBProducerWarp) {
    // ---------------- token-tile producer (one pair of K stages at a time) ----------------
    if (lane == 0) {
      uint32_t pr = 0;  // pairs issued by this CTA
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const Tile t = decode_tile(tile, args, s_ntp, s_off);
        const uint32_t box = box_rows(t.nbox) * 128u;
        for (int kb = 0; kb < nk; kb += 2, ++pr) {
          // the slot pair pr % 3 was last read by the MMAs of pair pr - 3
          if (pr >= static_cast<uint32_t>(kBPairs)) {
            const uint32_t j = pr - kBPairs;
            if (!mbar_wait(DONE(j % kDonePairs), (j / kDonePairs) & 1u, abort_flag, args.status)) { ok = false; break; }
          }
          const uint32_t bs = pr % kBPairs;
          const int nst = min(2, nk - kb);
          mbar_arrive_expect_tx(BFULL(bs), box * nst);
          for (int h = 0; h < nst; ++h)
            tma_load_2d(sbase + CF::kBOff + (2 * bs + h) * kBBytes, &maps.b[t.nbox], (kb + h) * BK, t.row0,
                        BFULL(bs));
        }
      }
      // drain: the copies of the last pairs land before the CTA may exit
      const uint32_t n = pr < static_cast<uint32_t>(kBPairs) ? pr : static_cast<uint32_t>(kBPairs);
      for (uint32_t d = 0; d < n; ++d) {
        const uint32_t j = pr - 1 - d;
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(BFULL(j % kBPairs), (j / kBPairs) & 1u)) {
          if (globaltimer() - t0 > kWaitLimitNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == kRelayWarp) {
    // ---------------- relay: a pair's token tiles have landed -> its FULL barrier ----------------
    // (the MMA thread then waits on a single barrier per pair; the token ring is deeper
    // than the A ring, so its copies are tracked on barriers of their own)
    if (lane == 0) {
      uint32_t pr = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < nk; kb += 2, ++pr) {
          if (!mbar_wait(BFULL(pr % kBPairs), (pr / kBPairs) & 1u, abort_flag, args.status)) { ok = false; break; }
          // this arrival must count toward pair pr: FULL(pr % 2) has to be done with pair pr - 2
          if (pr >= 2 && !mbar_wait(FULL(pr & 1u), ((pr - 2) >> 1) & 1u, abort_flag, args.status)) { ok = false; break; }
          mbar_arrive(FULL(pr & 1u));
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // The issue loop is kept minimal: the tensor core queues few MMAs, so every cycle
      // this thread spends between two MMAs can leave the tensor pipe idle.  Operand
      // addresses advance by adding to precomputed bases (the descriptor's start field is
      // the shared-memory address >> 4; no carry leaves its 14 bits below 256 KB).
      const uint32_t a_base = tmem_base + kACol0;
      const uint64_t b_base = umma_desc_sw128(sbase + CF::kBOff);
      constexpr uint32_t kBStep = kBBytes >> 4;  // one token tile in descriptor units
      uint32_t pr = 0, acc_it = 0, bs = 0, ds = 0;  // pair, its token slot pair (pr % 3) and DONE (pr % 6)
      bool ok = true;
      bool ready = false;  // the next pair's barrier was already seen complete
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++acc_it) {
        const Tile t = decode_tile(tile, args, s_ntp, s_off);
        const uint32_t b = acc_it & 1u, aph = (acc_it >> 1) & 1u;
        if (!mbar_wait(ACC_EMPTY(b), aph ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kAccCols;
        const uint32_t idesc = umma_idesc_f16_m128(static_cast<uint32_t>((t.count + 15) & ~15));
        for (int kb = 0; kb < nk; kb += 2, ++pr) {
          const uint32_t ps = pr & 1u;
          if (!ready && !mbar_wait(FULL(ps), (pr >> 1) & 1u, abort_flag, args.status)) { ok = false; break; }
          tc_fence_after();
          // look at the next pair's barrier now, while this pair's MMAs queue up
          ready = mbar_try_wait(FULL(ps ^ 1u), ((pr + 1) >> 1) & 1u);
          const uint32_t a = a_base + ps * (2 * kAStageCols);
          const uint64_t bd = b_base + bs * (2 * kBStep);
          // K = 16 per MMA: +8 TMEM columns of A, +32 bytes (+2 in the start field) of B
          umma_f16_ts(d_tmem, a, bd, idesc, kb != 0 ? 1u : 0u);
          umma_f16_ts(d_tmem, a + 8u, bd + 2u, idesc, 1u);
          umma_f16_ts(d_tmem, a + 16u, bd + 4u, idesc, 1u);
          umma_f16_ts(d_tmem, a + 24u, bd + 6u, idesc, 1u);
          if (kb + 1 < nk) {
            umma_f16_ts(d_tmem, a + kAStageCols, bd + kBStep, idesc, 1u);
            umma_f16_ts(d_tmem, a + kAStageCols + 8u, bd + kBStep + 2u, idesc, 1u);
            umma_f16_ts(d_tmem, a + kAStageCols + 16u, bd + kBStep + 4u, idesc, 1u);
            umma_f16_ts(d_tmem, a + kAStageCols + 24u, bd + kBStep + 6u, idesc, 1u);
          }
          umma_commit(DONE(ds));
          if (++bs == static_cast<uint32_t>(kBPairs)) bs = 0;
          if (++ds == static_cast<uint32_t>(kDonePairs)) ds = 0;
        }
        if (!ok) break;
        umma_commit(ACC_FULL(b));
      }
      // drain: all issued MMAs complete before TMEM is freed
      umma_commit(DRAIN);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(DRAIN, 0)) {
        if (globaltimer() - t0 > kWaitLimitNs) break;
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarps) {
    // ---------------- dequant (four groups, K stages in turn) ----------------
    // A group decodes its stage into registers first and only then waits for the TMEM
    // slot, so that the slot (freed when the MMAs of the pair two back complete) is
    // refilled with a few tcgen05.st.
    const int dt = threadIdx.x - kDequantThread0;
    const int group = dt / (kGroupWarps * 32);
    const int r = dt - group * (kGroupWarps * 32);  // tile row = TMEM lane (warp%4 quadrant)
    const uint32_t lane8 = static_cast<uint32_t>(lane) * 8u;
    const uint32_t trow = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kACol0;
    uint32_t it = 0, cs = 0, cph = 0, pr0 = 0;  // K stages, code slot/phase, pairs before this tile
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, pr0 += (nk + 1) >> 1) {
      const Tile t = decode_tile(tile, args, s_ntp, s_off);
      int wr, cr;  // weight row inside the expert, row inside the staged code tile
      if (KIND == 0) {
        const int sgate = r & 1, i = r >> 1;
        wr = sgate * args.I + t.m * 64 + i;
        cr = sgate * 64 + i;
      } else {
        wr = t.m * 128 + r;
        cr = r;
      }
      float a_pref = 0.f;
      bool have_pref = false;
      DqStep dq;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const uint32_t my_cs = cs, my_cph = cph;
        if (++cs == static_cast<uint32_t>(kCS)) { cs = 0; cph ^= 1u; }
        if (static_cast<int>(it & (kDequantGroups - 1)) != group) continue;
        float a = 0.f;
        if (MODE != MOEQ_INT8_ROW) {
          a = have_pref ? a_pref : load_absmax<MODE>(args, t.e, wr, kb, dq);
          have_pref = kb + kDequantGroups < nk;
          if (have_pref) a_pref = load_absmax<MODE>(args, t.e, wr, kb + kDequantGroups, dq);
        }
        if (!mbar_wait(C_FULL(my_cs), my_cph, abort_flag, args.status)) { ok = false; break; }
        // this thread's codes: its row of the stage, 32 bytes (NF4) or 64 bytes (int8)
        const uint32_t crow = CF::kCOff + my_cs * CF::kCodeBytes + cr * CF::kCodeRow;
        uint4 cw[CF::kCodeRow / 16];
#pragma unroll
        for (int i = 0; i < static_cast<int>(CF::kCodeRow / 16); ++i) cw[i] = lds_u4(smem, crow + 16 * i);
        // the codes are in registers: hand the slot back to the producer (the proxy fence
        // orders these generic-proxy reads before its next TMA write into the slot)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(C_EMPTY(my_cs));
        uint32_t o[32];  // the row's 64 fp16 weights, two per word, in K order
        if (MODE == MOEQ_INT8_ROW) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t wv[4] = {cw[q].x, cw[q].y, cw[q].z, cw[q].w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
              // fp16 0x64XX is 1024 + XX (ulp 1 on [1024, 2048)), so with byte = q + 128
              // the pair (0x64 byte0, 0x64 byte1) minus 1152 is (q0, q1), exactly
              const uint32_t bw = wv[wi] ^ 0x80808080u;
              o[8 * q + 2 * wi] = hsub2_u32(__byte_perm(bw, 0x64646464u, 0x4140u), 0x64806480u);
              o[8 * q + 2 * wi + 1] = hsub2_u32(__byte_perm(bw, 0x64646464u, 0x4342u), 0x64806480u);
            }
          }
        } else {
          // w = fp16(level) * fp16(absmax), rounded to fp16 (an absmax beyond the fp16 range
          // is reported and clamped)
          if (!(a <= 65504.0f)) {
            report(args.status, MOEQ_ERR_RANGE);
            a = 65504.0f;
          }
          const __half2 a2 = __float2half2_rn(a);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint32_t wv[4] = {cw[q].x, cw[q].y, cw[q].z, cw[q].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                // byte k of the word holds elements 2k (high nibble) and 2k+1; its entry is at
                // byte*128 + lane*4 = ((byte << 8) | lane*8) >> 1
                const uint32_t addr = __byte_perm(wv[j], lane8, 0x5504u | (static_cast<uint32_t>(k) << 4)) >> 1;
                const __half2 c = *reinterpret_cast<const __half2 *>(smem + CF::kLutOff + addr);
                const __half2 w = __hmul2(c, a2);
                o[16 * q + 4 * j + k] = *reinterpret_cast<const uint32_t *>(&w);
              }
            }
          }
        }
        // this stage's A slot: half (kb & 1) of slot pr % 2, last read by the MMAs of pair pr - 2
        const uint32_t pr = pr0 + (kb >> 1), ps = pr & 1u;
        if (pr >= 2) {
          const uint32_t j = pr - 2;
          if (!mbar_wait(DONE(j % kDonePairs), (j / kDonePairs) & 1u, abort_flag, args.status)) { ok = false; break; }
        }
        tc_fence_after();
        const uint32_t tcol = trow + (2 * ps + (kb & 1)) * kAStageCols;
        tmem_st_32x32b_x16(tcol, *reinterpret_cast<const uint32_t(*)[16]>(o));
        tmem_st_32x32b_x16(tcol + 16u, *reinterpret_cast<const uint32_t(*)[16]>(o + 16));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          // a lone last stage (odd K / 64) stands for both halves of its pair
          if ((nk & 1) && kb == nk - 1) mbar_arrive_cnt(FULL(ps), 2);
          else mbar_arrive(FULL(ps));
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 0-7) ----------------
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int col0 = (warp >> 2) * (BN / 2);   // this warp's half of the tile's columns
    const int r = quad * 32 + lane;
    uint32_t acc_it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++acc_it) {
      const Tile t = decode_tile(tile, args, s_ntp, s_off);
      const uint32_t b = acc_it & 1u, aph = (acc_it >> 1) & 1u;
      if (!mbar_wait(ACC_FULL(b), aph, abort_flag, args.status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * kAccCols;
      const int ncols = min(BN / 2, t.count - col0);   // may be <= 0: nothing to do
      const int nch = ncols > 0 ? (ncols + 31) >> 5 : 0;
      if (KIND == 0) {
        const int sgate = lane & 1;
        const int j = t.m * 64 + (r >> 1);
        float step = 1.0f;
        if (MODE == MOEQ_INT8_ROW)
          step = __fdiv_rn(__ldg(args.absmax + static_cast<size_t>(t.e) * args.R + sgate * args.I + j), 127.0f);
        for (int c = 0; c < nch; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + col0 + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            float own = __uint_as_float(sgate ? v[16 + q] : v[q]);
            float snd = __uint_as_float(sgate ? v[q] : v[16 + q]);
            if (MODE == MOEQ_INT8_ROW) {
              own *= step;
              snd *= step;
            }
            const float rcv = __shfl_xor_sync(0xffffffffu, snd, 1);
            const float g = sgate ? rcv : own;
            const float u = sgate ? own : rcv;
            const int col = col0 + c * 32 + (sgate ? 16 : 0) + q;
            float hval = __fdividef(g, 1.0f + __expf(-g)) * u;
            if (col < t.count) {
              if (fabsf(hval) > 65504.0f) {
                report(args.status, MOEQ_ERR_RANGE);
                hval = fminf(fmaxf(hval, -65504.0f), 65504.0f);
              }
              args.h_out[static_cast<size_t>(t.row0 + col) * args.I + j] = __float2half_rn(hval);
            }
          }
        }
      } else {
        const int i = t.m * 128 + r;
        float step = 1.0f;
        if (MODE == MOEQ_INT8_ROW)
          step = __fdiv_rn(__ldg(args.absmax + static_cast<size_t>(t.e) * args.R + i), 127.0f);
        for (int c = 0; c < nch; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + col0 + c * 32, v);
          tmem_ld_wait();
          const int colL = col0 + c * 32 + lane;
          int p = 0;
          float wv = 0.0f;
          if (colL < t.count) {
            p = __ldg(args.perm + t.row0 + colL);
            if (args.w_bf16)
              wv = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(args.topk_w)[p]);
            else
              wv = __ldg(reinterpret_cast<const float *>(args.topk_w) + p);
          }
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int pq = __shfl_sync(0xffffffffu, p, q);
            const float wq = __shfl_sync(0xffffffffu, wv, q);
            if (col0 + c * 32 + q < t.count)
              args.slot_out[static_cast<size_t>(pq) * args.R + i] =
                  MODE == MOEQ_INT8_ROW ? wq * (__uint_as_float(v[q]) * step) : wq * __uint_as_float(v[q]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ACC_EMPTY(b));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

static bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner,
                      uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int KIND>
static cudaError_t launch_t(const TmapSet &maps, const GemmArgs &a, int grid, cudaStream_t s) {
  using CF = Cfg<MODE>;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(k_moe_gemm<MODE, KIND>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, CF::kSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  k_moe_gemm<MODE, KIND><<<grid, kThreads, CF::kSmem, s>>>(maps, a);
  return cudaGetLastError();
}

cudaError_t launch_moe_gemm(const GemmLaunch &g, int sm_count, cudaStream_t s, int *launches) {
  const moeq_packed *w = g.w;
  TmapSet maps;
  const int C = w->C;
  const uint32_t code_row = (g.mode == MOEQ_INT8_ROW) ? 64u : 32u;
  for (int i = 0; i < 5; ++i) {
    if (!encode_2d(&maps.b[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.act, C, g.S, static_cast<uint64_t>(C) * 2,
                   64, i < 4 ? (16u << i) : 192u, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  const uint64_t row_bytes = (g.mode == MOEQ_INT8_ROW) ? C : C / 2;
  if (!encode_2d(&maps.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, row_bytes,
                 static_cast<uint64_t>(w->E) * w->R, row_bytes, code_row, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;

  GemmArgs a;
  a.absmax = w->absmax;
  a.aq = w->absmax_q;
  a.ascale = w->absmax_scale;
  a.aoff = w->absmax_offset;
  a.E = w->E;
  a.R = w->R;
  a.C = C;
  a.I = g.I;
  a.MT = (g.kind == 0) ? g.I / 64 : w->R / 128;
  a.nk = C / 64;
  a.nb = static_cast<int>(static_cast<long long>(w->R) * C / 64);
  a.nblk = (a.nb + 255) / 256;
  a.offsets = g.offsets;
  a.ntp = g.ntile_prefix;
  a.perm = g.perm;
  a.h_out = static_cast<__half *>(g.h_out);
  a.slot_out = g.slot_out;
  a.topk_w = g.topk_w;
  a.w_bf16 = g.w_bf16;
  a.status = g.status;

  const long long max_tiles = (static_cast<long long>(w->E) + (g.S + BN - 1) / BN) * a.MT;
  const int grid = static_cast<int>(max_tiles < sm_count ? max_tiles : sm_count);
  cudaError_t e;
  if (g.mode == MOEQ_NF4) e = g.kind == 0 ? launch_t<MOEQ_NF4, 0>(maps, a, grid, s) : launch_t<MOEQ_NF4, 1>(maps, a, grid, s);
  else if (g.mode == MOEQ_NF4_DQ) e = g.kind == 0 ? launch_t<MOEQ_NF4_DQ, 0>(maps, a, grid, s) : launch_t<MOEQ_NF4_DQ, 1>(maps, a, grid, s);
  else e = g.kind == 0 ? launch_t<MOEQ_INT8_ROW, 0>(maps, a, grid, s) : launch_t<MOEQ_INT8_ROW, 1>(maps, a, grid, s);
  ++*launches;
  return e;
}

}  // namespace moeq
