"""Plain, slow CPU oracle for quantizing fused MoE expert tensors and running the
routed experts forward. TEST INFRASTRUCTURE ONLY: the product path never calls it.

Everything here is written from the statement of the problem on the source pages:

* "MoE Expert Quantization" (axolotl docs), section "Implementation details":
  expert tensors (3-D, "expert" in the name) are quantized on load, 4-bit through
  the bitsandbytes NF4 parametrization, 8-bit through a row-wise int8
  parametrization with bitsandbytes-style dequantization.
* "Failed to quant MoE models with fused expert weights in transformers v5"
  (bitsandbytes issue #1849): section "Description" gives the fused layout
  ``gate_up_proj [E, 2I, H]`` and ``down_proj [E, H, I]`` with an activation
  ``ACT2FN[hidden_act]`` (SiLU for Qwen3-MoE); the maintainer comments fix the
  blocksize (default 64, in_features divisible by it, blocks never straddle
  experts), the per-expert absmax buffer ``[num_experts, blocks_per_expert]`` and
  name double quantization (``compress_statistics``/``bnb_4bit_use_double_quant``).
* unsloth-zoo issue #850 ("quantize-coverage vs route-coverage"): the experts
  interface ``(hidden_states, top_k_index, top_k_weights)`` and the warning that the
  square OLMoE gate_up (2*1024 == 2048) makes its orientation impossible to infer
  from the shape: gate is the first I rows of dim 1, always.

Where the pages are silent the plainest reading is taken; each one is marked
"READING" below.

Conventions.
* bf16 tensors are numpy ``uint16`` arrays holding the raw bf16 bit patterns.
* ``fl(.)`` is one IEEE fp32 operation, round to nearest even. numpy float32
  ``+ - * /`` on float32 arrays are exactly that, one rounding per operation.
* No function here reorders, blocks or fuses arithmetic beyond what the
  definition it follows states.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
(closed forms, exhaustive checks, brute force on tiny inputs, library routines).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "NF4_CODEBOOK", "NF4_BLOCK", "DQ_BLOCK",
    "bf16_to_f32", "f32_to_bf16",
    "nf4_code", "quantize_nf4", "double_quantize_absmax", "quantize_int8_rowwise",
    "nf4_absmax_decoded", "dequantize", "route", "experts_forward",
    "packed_nbytes",
]

# ----------------------------------------------------------------------------
# NF4 codebook.  READING: the pages name "NF4" ("MoE Expert Quantization",
# Implementation details: "bitsandbytes NF4 parametrization") but do not print
# the levels.  The 16 levels are the 4-bit NormalFloat table (normal quantiles,
# asymmetric: 8 positive, 7 negative, one exact zero, normalised to [-1, 1]).
# They are frozen here as fp32 constants; the pins rebuild them from the normal
# quantile construction to within a few ulp.
# ----------------------------------------------------------------------------
NF4_CODEBOOK = np.array([
    -1.0, -0.6961928009986877, -0.5250730514526367, -0.39491748809814453,
    -0.28444138169288635, -0.18477343022823334, -0.09105003625154495, 0.0,
    0.07958029955625534, 0.16093020141124725, 0.24611230194568634, 0.33791524171829224,
    0.44070982933044434, 0.5626170039176941, 0.7229568362236023, 1.0,
], dtype=np.float32)

NF4_BLOCK = 64   # bitsandbytes #1849 maintainer comment: default blocksize 64
DQ_BLOCK = 256   # READING: int8 double-quant blocks of 256 absmax values


# ----------------------------------------------------------------------------
# bf16 <-> fp32
# ----------------------------------------------------------------------------
def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening: a bf16 bit pattern is the top half of an fp32 one."""
    u16 = np.asarray(u16, dtype=np.uint16)
    return (u16.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 with round-to-nearest-even (NaN stays NaN, quiet)."""
    f = np.ascontiguousarray(f, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        r = r.copy()
        r[nan] = ((u[nan] >> np.uint64(16)) | np.uint64(0x0040)).astype(np.uint16)
    return r


# ----------------------------------------------------------------------------
# a1: NF4 blockwise quantization
# ----------------------------------------------------------------------------
def nf4_code(n: np.ndarray) -> np.ndarray:
    """Index of the nearest NF4 level to each fp32 ``n`` in [-1, 1]; ties go to
    the lower index.

    Written as a count: code = #{ j in [0, 15) : 2n > c_j + c_{j+1} }.  Both sides
    are exact in fp64 (n and c_j are fp32; a sum of two fp32 is exact in fp64), so
    "2n is above the midpoint sum" is decided exactly and an exact midpoint stays
    with the lower level.
    """
    n64 = np.asarray(n, dtype=np.float32).astype(np.float64)
    c = NF4_CODEBOOK.astype(np.float64)
    mid2 = c[:-1] + c[1:]                                   # 15 exact sums
    return (2.0 * n64[..., None] > mid2).sum(axis=-1).astype(np.uint8)


def quantize_nf4(w_bf16: np.ndarray, double_quant: bool = False) -> dict:
    """NF4 quantization of one fused 3-D expert tensor ``W[E, R, C]`` (C is the
    reduction dim, in_features; the pages require C % 64 == 0 so that no block
    straddles a row or an expert).

    Per block of 64 consecutive elements along C:
      absmax = max |x|                          (fp32, exact)
      n      = fl(x / absmax)                   (IEEE fp32 divide; READING: a
                                                 divide, not a reciprocal multiply)
      code   = nearest NF4 level, ties -> lower index
    absmax == 0 (READING, pages silent): every code is 7 (the 0.0 level), absmax
    stored as 0.  Packing (READING, pages silent): byte k of a row holds
    (code[2k] << 4) | code[2k+1], first element in the high nibble.

    Returns codes u8 [E, R, C/2] and absmax f32 [E, R, C/64]; with double_quant the
    absmax is replaced by its int8 encoding (see ``double_quantize_absmax``).
    """
    w = np.asarray(w_bf16, dtype=np.uint16)
    E, R, C = w.shape
    if C % NF4_BLOCK:
        raise ValueError("C must be a multiple of 64")
    x = bf16_to_f32(w).reshape(-1, NF4_BLOCK)
    absmax = np.abs(x).max(axis=1)
    codes = np.empty(x.shape, dtype=np.uint8)
    chunk = 1 << 16
    for b0 in range(0, x.shape[0], chunk):
        xb, ab = x[b0:b0 + chunk], absmax[b0:b0 + chunk]
        zero = ab == 0
        denom = np.where(zero, np.float32(1), ab).astype(np.float32)
        n = (xb / denom[:, None]).astype(np.float32)
        n[zero] = 0.0
        codes[b0:b0 + chunk] = nf4_code(n)
    packed = ((codes[:, 0::2] << 4) | codes[:, 1::2]).astype(np.uint8)
    out = {
        "mode": "nf4_dq" if double_quant else "nf4",
        "E": E, "R": R, "C": C,
        "codes": packed.reshape(E, R, C // 2),
    }
    absmax = absmax.astype(np.float32).reshape(E, R, C // NF4_BLOCK)
    if double_quant:
        out.update(double_quantize_absmax(absmax.reshape(E, -1)))
    else:
        out["absmax"] = absmax
    return out


# ----------------------------------------------------------------------------
# a2: double quantization of the absmax values
# ----------------------------------------------------------------------------
def double_quantize_absmax(absmax: np.ndarray) -> dict:
    """Int8 encoding of each expert's absmax vector (``[E, nb]``, nb = R*C/64).

    The pages only name the option (bitsandbytes #1849: ``compress_statistics`` /
    ``bnb_4bit_use_double_quant``, "absmax / double-quant layout ... per-expert").
    READING (int8 blocks of 256, fp32 scale, mean offset, per expert so that experts
    stay independently sliceable):
      1. offset: chunk sums S_c over consecutive 256-value chunks, each summed
         sequentially in fp64; the chunk sums added sequentially in fp64;
         off_e = fp32(fp64(total / nb)).
      2. per block of 256 (the last may be partial): v = fl(a - off_e),
         s = max |v|; q = rint(fl(fl(127 * v) / s)) (half to even), q = 0 if s == 0.
      3. decode: a' = fl(fl(q * fl(s / 127)) + off_e)   (``nf4_absmax_decoded``)
    Returns absmax_q i8 [E, nb], absmax_scale f32 [E, ceil(nb/256)],
    absmax_offset f32 [E].
    """
    a = np.asarray(absmax, dtype=np.float32)
    E, nb = a.shape
    nblk = -(-nb // DQ_BLOCK)
    pad = np.zeros((E, nblk * DQ_BLOCK), dtype=np.float64)
    pad[:, :nb] = a
    chunks = pad.reshape(E, nblk, DQ_BLOCK)
    # 1. fixed-order fp64 sums (each chunk sequential in its element index; padding
    #    zeros add exactly nothing)
    S = np.zeros((E, nblk), dtype=np.float64)
    for i in range(DQ_BLOCK):
        S = S + chunks[:, :, i]
    total = np.zeros(E, dtype=np.float64)
    for cidx in range(nblk):
        total = total + S[:, cidx]
    off = (total / np.float64(nb)).astype(np.float32)
    # 2. int8 blocks
    v = (a - off[:, None]).astype(np.float32)
    vpad = np.zeros((E, nblk * DQ_BLOCK), dtype=np.float32)
    vpad[:, :nb] = v
    vb = vpad.reshape(E, nblk, DQ_BLOCK)
    s = np.abs(vb).max(axis=2).astype(np.float32)
    p = (np.float32(127.0) * vb).astype(np.float32)
    sden = np.where(s == 0, np.float32(1), s).astype(np.float32)
    qf = (p / sden[:, :, None]).astype(np.float32)
    q = np.rint(qf)
    q[s == 0] = 0
    q = q.reshape(E, -1)[:, :nb].astype(np.int8)
    return {"absmax_q": q, "absmax_scale": s, "absmax_offset": off}


def nf4_absmax_decoded(packed: dict) -> np.ndarray:
    """fp32 absmax used by NF4 dequantization, ``[E, R, C/64]``."""
    E, R, C = packed["E"], packed["R"], packed["C"]
    if packed["mode"] == "nf4":
        return np.asarray(packed["absmax"], dtype=np.float32)
    q = packed["absmax_q"].astype(np.float32)
    s = packed["absmax_scale"].astype(np.float32)
    off = packed["absmax_offset"].astype(np.float32)
    nb = q.shape[1]
    step = (s / np.float32(127.0)).astype(np.float32)          # fl(s / 127)
    blk = np.arange(nb) // DQ_BLOCK
    prod = (q * step[:, blk]).astype(np.float32)                # fl(q * step)
    dec = (prod + off[:, None]).astype(np.float32)              # fl(. + off)
    return dec.reshape(E, R, C // NF4_BLOCK)


# ----------------------------------------------------------------------------
# a3: row-wise int8
# ----------------------------------------------------------------------------
def quantize_int8_rowwise(w_bf16: np.ndarray) -> dict:
    """Row-wise int8 ("MoE Expert Quantization", Implementation details: "a custom
    row-wise int8 parametrization with bitsandbytes dequantization").

    Per row of length C: absmax = max |x| (fp32); q = rint(fl(127 * x) / absmax)
    with an IEEE fp32 divide and half-to-even rounding (READING: round() on a
    tensor is half-to-even); q = 0 where absmax == 0.  127 * x is exact for a bf16 x.
    Returns codes i8 [E, R, C] and absmax f32 [E, R].
    """
    w = np.asarray(w_bf16, dtype=np.uint16)
    E, R, C = w.shape
    x = bf16_to_f32(w).reshape(E * R, C)
    absmax = np.abs(x).max(axis=1).astype(np.float32)
    p = (np.float32(127.0) * x).astype(np.float32)
    den = np.where(absmax == 0, np.float32(1), absmax).astype(np.float32)
    q = np.rint((p / den[:, None]).astype(np.float32))
    q[absmax == 0] = 0
    return {"mode": "int8", "E": E, "R": R, "C": C,
            "codes": q.astype(np.int8).reshape(E, R, C),
            "absmax": absmax.reshape(E, R)}


# ----------------------------------------------------------------------------
# a4: dequantization
# ----------------------------------------------------------------------------
def dequantize(packed: dict, experts=None) -> np.ndarray:
    """fp32 weights ``[E', R, C]`` (all experts, or the listed ones).

    NF4:    w = fl(c[code] * absmax')            (absmax' decoded if double-quant)
    int8:   w = fl(q * fl(absmax / 127))         (bitsandbytes-style row dequant)
    A bf16 output is the round-to-nearest-even of this fp32 value.
    """
    E, R, C = packed["E"], packed["R"], packed["C"]
    ex = np.arange(E) if experts is None else np.asarray(experts)
    if packed["mode"] == "int8":
        q = packed["codes"][ex].astype(np.float32)
        step = (packed["absmax"][ex].astype(np.float32) / np.float32(127.0)).astype(np.float32)
        return (q * step[:, :, None]).astype(np.float32)
    codes = packed["codes"][ex]
    hi = (codes >> 4) & 0xF
    lo = codes & 0xF
    idx = np.empty(codes.shape[:-1] + (C,), dtype=np.uint8)
    idx[..., 0::2] = hi
    idx[..., 1::2] = lo
    a = nf4_absmax_decoded(packed)[ex]
    cval = NF4_CODEBOOK[idx].reshape(len(ex), R, C // NF4_BLOCK, NF4_BLOCK)
    return (cval * a[..., None]).astype(np.float32).reshape(len(ex), R, C)


# ----------------------------------------------------------------------------
# a5: routing (token -> expert grouping)
# ----------------------------------------------------------------------------
def route(top_k_index: np.ndarray, E: int):
    """Group the (t, k) pairs by expert.

    counts[e] = #pairs routed to e; offsets = exclusive prefix sum (length E+1);
    perm lists the flat pair index p = t*K + k sorted by expert, and by p within an
    expert (stable).  Pairs whose index is outside [0, E) are dropped.
    """
    idx = np.asarray(top_k_index).reshape(-1).astype(np.int64)
    valid = (idx >= 0) & (idx < E)
    counts = np.zeros(E, dtype=np.int64)
    for e in idx[valid]:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    perm = np.empty(int(offsets[E]), dtype=np.int64)
    fill = offsets[:-1].copy()
    for p in range(idx.size):          # walking p in order keeps each group stable
        e = idx[p]
        if 0 <= e < E:
            perm[fill[e]] = p
            fill[e] += 1
    return counts, offsets, perm


# ----------------------------------------------------------------------------
# a6 + a7: routed experts forward
# ----------------------------------------------------------------------------
def _silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def experts_forward(hidden_bf16: np.ndarray, top_k_index: np.ndarray,
                    top_k_weights: np.ndarray, w_gate_up: np.ndarray,
                    w_down: np.ndarray, tokens=None) -> np.ndarray:
    """out[t] = sum_k w[t,k] * down_e(silu(gate_e x) * up_e x), e = top_k_index[t,k].

    ``w_gate_up`` is ``[E, 2I, H]`` and ``w_down`` ``[E, H, I]`` (fp32 dequantized
    weights; the layout of bitsandbytes #1849 "Description").  Gate is rows [0, I)
    of dim 1 and up is rows [I, 2I): never inferred from the shape (unsloth-zoo
    #850, the square OLMoE gate_up).  silu(z) = z / (1 + exp(-z)).  The weights are
    used as given (no renormalisation).  Arithmetic in fp64 on the fp32 weights;
    the k terms are added in k order.  Pairs with an index outside [0, E) add
    nothing.  ``tokens`` selects a subset of rows of ``hidden`` (default: all).
    Returns fp64 ``[len(tokens), H]``.
    """
    x_all = bf16_to_f32(np.asarray(hidden_bf16, dtype=np.uint16))
    idx_all = np.asarray(top_k_index).astype(np.int64)
    wk_all = np.asarray(top_k_weights, dtype=np.float64)
    t_sel = np.arange(x_all.shape[0]) if tokens is None else np.asarray(tokens)
    x = x_all[t_sel].astype(np.float64)
    idx, wk = idx_all[t_sel], wk_all[t_sel]
    E, twoI, H = w_gate_up.shape
    I = twoI // 2
    T, K = idx.shape
    out = np.zeros((T, H), dtype=np.float64)
    for k in range(K):                      # k order
        yk = np.zeros((T, H), dtype=np.float64)
        for e in np.unique(idx[:, k]):
            if not (0 <= e < E):
                continue
            rows = np.nonzero(idx[:, k] == e)[0]
            wgu = w_gate_up[e].astype(np.float64)
            g = x[rows] @ wgu[:I].T
            u = x[rows] @ wgu[I:].T
            h = _silu(g) * u
            yk[rows] = h @ w_down[e].astype(np.float64).T
        valid = (idx[:, k] >= 0) & (idx[:, k] < E)
        out += np.where(valid[:, None], wk[:, k:k + 1] * yk, 0.0)
    return out


# ----------------------------------------------------------------------------
# storage size (closed form)
# ----------------------------------------------------------------------------
def packed_nbytes(mode: str, E: int, R: int, C: int) -> int:
    """Bytes of the packed representation of one ``[E, R, C]`` tensor."""
    if mode == "nf4":
        return E * R * C // 2 + 4 * E * R * C // NF4_BLOCK
    if mode == "nf4_dq":
        nb = R * C // NF4_BLOCK
        return E * R * C // 2 + E * nb + 4 * E * math.ceil(nb / DQ_BLOCK) + 4 * E
    if mode == "int8":
        return E * R * C + 4 * E * R
    raise ValueError(mode)
