"""Pins of the CPU oracle against facts fixed outside it: the normal-quantile
construction of the NF4 table, exhaustive and brute-force code selection, closed
forms, exact rational arithmetic (fractions.Fraction), textbook/library routines
(torch's bf16 cast and SwiGLU via torch.nn.functional, Python's stable sort,
math.fsum) and the figures printed on the source pages.  CPU only."""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
C64 = O.NF4_CODEBOOK.astype(np.float64)


# ---------------------------------------------------------------------------
# exact fp32 rounding of a rational (ties to even), independent of numpy
# ---------------------------------------------------------------------------
def fl32(q: Fraction) -> float:
    if q == 0:
        return 0.0
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    m = a / ulp
    lo = math.floor(m)
    r = m - lo
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * float(lo * ulp)


def fr(x) -> Fraction:
    return Fraction(float(x))


def rand_bf16(shape, seed, scale=0.02):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).view(torch.uint16).numpy()


def to_bf16_bits(vals) -> np.ndarray:
    return torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


# ---------------------------------------------------------------------------
# codebook
# ---------------------------------------------------------------------------
def test_codebook_table_properties():
    c = O.NF4_CODEBOOK
    assert c.dtype == np.float32 and c.shape == (16,)
    assert np.all(np.diff(c.astype(np.float64)) > 0)
    assert c[0] == -1.0 and c[15] == 1.0
    assert np.count_nonzero(c == 0.0) == 1 and c[7] == 0.0
    assert np.count_nonzero(c > 0) == 8 and np.count_nonzero(c < 0) == 7


def test_codebook_rebuilt_from_normal_quantiles():
    from scipy.stats import norm
    offset = 0.9677083  # (1 - 1/(2*15) + 1 - 1/(2*16)) / 2
    pos = norm.ppf(np.linspace(offset, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(offset, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v = (v / np.abs(v).max()).astype(np.float32)
    ulps = np.abs(v.view(np.int32).astype(np.int64) - O.NF4_CODEBOOK.view(np.int32).astype(np.int64))
    assert ulps.max() <= 8, ulps


# ---------------------------------------------------------------------------
# bf16 conversions against torch's cast
# ---------------------------------------------------------------------------
def test_bf16_conversions_match_torch():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(100000, generator=g) * s for s in (1e-38, 1e-3, 1.0, 1e30)])
    special = torch.tensor([0.0, -0.0, float("inf"), -float("inf"), 1.0 + 2**-8, 1.0 + 3 * 2**-8,
                            3.3895e38, 1e-45, -1e-45, 1.00390625, 1.01171875])
    x = torch.cat([x, special]).to(torch.float32)
    ours = O.f32_to_bf16(x.numpy())
    ref = x.to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(ours, ref)
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.uint16)
    back = O.bf16_to_f32(bits.numpy())
    refb = bits.view(torch.bfloat16).to(torch.float32).numpy()
    fin = np.isfinite(refb)
    assert np.array_equal(back[fin], refb[fin]) and np.array_equal(np.isnan(back), np.isnan(refb))
    assert np.isnan(O.bf16_to_f32(O.f32_to_bf16(np.array([np.nan], np.float32))))[0]


# ---------------------------------------------------------------------------
# code selection
# ---------------------------------------------------------------------------
def _argmin_ref(n: np.ndarray) -> np.ndarray:
    d = np.abs(n.astype(np.float64)[:, None] - C64[None, :])
    return np.argmin(d, axis=1)  # first minimum: ties go to the lower index


def test_nf4_code_near_every_midpoint_exhaustive():
    for j in range(15):
        m = (C64[j] + C64[j + 1]) / 2
        b0 = np.array([m], dtype=np.float32).view(np.int32)[0]
        bits = np.arange(b0 - 65536, b0 + 65537, dtype=np.int64)
        n = bits.astype(np.int32).view(np.float32)
        n = n[np.isfinite(n) & (np.abs(n) <= 1)]
        assert np.array_equal(O.nf4_code(n), _argmin_ref(n)), j
        # an exactly representable midpoint goes to the lower level
        if float(np.float32(m)) == m:
            assert O.nf4_code(np.array([m], np.float32))[0] == j


def test_nf4_code_strided_sample_of_all_fp32_in_unit_interval():
    pos = np.arange(0, 0x3F800001, 4099, dtype=np.int64).astype(np.int32).view(np.float32)
    n = np.concatenate([pos, -pos, np.array([1.0, -1.0, 0.0], np.float32)])
    assert np.array_equal(O.nf4_code(n), _argmin_ref(n))
    assert np.array_equal(O.nf4_code(O.NF4_CODEBOOK), np.arange(16))


@pytest.mark.slow
def test_nf4_code_exhaustive_all_fp32_in_unit_interval():
    step = 1 << 24
    for sgn in (1, -1):
        for b in range(0, 0x3F800001, step):
            bits = np.arange(b, min(b + step, 0x3F800001), dtype=np.int64).astype(np.int32)
            n = bits.view(np.float32) * np.float32(sgn)
            assert np.array_equal(O.nf4_code(n), _argmin_ref(n))


# ---------------------------------------------------------------------------
# NF4 quantize / dequantize through the bf16 interface
# ---------------------------------------------------------------------------
def test_nf4_levels_round_trip_through_bf16_blocks():
    for k in (-20, -7, 0, 3):
        A = 2.0 ** k
        vals = np.concatenate([O.NF4_CODEBOOK * np.float32(A)] * 4).astype(np.float32)
        w = to_bf16_bits(vals).reshape(1, 1, 64)
        p = O.quantize_nf4(w)
        assert p["absmax"][0, 0, 0] == np.float32(A)
        codes = np.empty(64, np.uint8)
        codes[0::2] = p["codes"][0, 0] >> 4
        codes[1::2] = p["codes"][0, 0] & 15
        assert np.array_equal(codes, np.tile(np.arange(16), 4))
        dq = O.dequantize(p)[0, 0]
        assert np.array_equal(dq, np.tile(O.NF4_CODEBOOK * np.float32(A), 4))


def test_nf4_packing_bytes():
    w = to_bf16_bits(np.tile(O.NF4_CODEBOOK, 4)).reshape(1, 1, 64)
    p = O.quantize_nf4(w)
    expect = np.tile(np.array([0x01, 0x23, 0x45, 0x67, 0x89, 0xAB, 0xCD, 0xEF], np.uint8), 4)
    assert np.array_equal(p["codes"][0, 0], expect)


def test_nf4_block_extremes_and_zero():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 0.02, size=(4, 64)).astype(np.float32)
    x[0, 5] = 0.5      # positive absmax element
    x[1, 9] = -0.5     # negative absmax element
    x[2, :] = 0.0      # all-zero block
    x[3, 17] = 0.0
    w = to_bf16_bits(x).reshape(1, 4, 64)
    p = O.quantize_nf4(w)
    codes = np.empty((4, 64), np.uint8)
    codes[:, 0::2] = p["codes"][0] >> 4
    codes[:, 1::2] = p["codes"][0] & 15
    assert codes[0, 5] == 15 and codes[1, 9] == 0
    assert np.all(codes[2] == 7) and p["absmax"][0, 2, 0] == 0.0
    assert codes[3, 17] == 7
    assert np.all(O.dequantize(p)[0, 2] == 0.0)


def test_nf4_error_bound_and_nearest_level():
    w = rand_bf16((3, 32, 256), seed=11)
    w[0, 0, :7] = to_bf16_bits([1.0, -3.0, 1e-30, -1e-30, 0.4, 200.0, -0.001])
    p = O.quantize_nf4(w)
    x = O.bf16_to_f32(w).astype(np.float64).reshape(-1, 64)
    dq = O.dequantize(p).astype(np.float64).reshape(-1, 64)
    a = p["absmax"].astype(np.float64).reshape(-1, 1)
    half_gap = np.max(np.diff(C64)) / 2
    # half the widest level gap, plus the fp32 roundings of x/absmax and of c*absmax
    assert np.all(np.abs(x - dq) <= (half_gap + 2.0 ** -22) * a)
    # the chosen level is a nearest level of the exact ratio, brute force
    n = x / np.where(a == 0, 1, a)
    codes = np.empty(x.shape, np.int64)
    cb = p["codes"].reshape(-1, 32)
    codes[:, 0::2] = cb >> 4
    codes[:, 1::2] = cb & 15
    d_chosen = np.abs(n - C64[codes])
    d_best = np.min(np.abs(n[..., None] - C64), axis=-1)
    assert np.all(d_chosen <= d_best + 1e-6)


def test_nf4_quotient_and_product_rounding_exact_rationals():
    w = rand_bf16((2, 4, 128), seed=5)
    p = O.quantize_nf4(w)
    x = O.bf16_to_f32(w).reshape(-1, 64)
    a = p["absmax"].reshape(-1)
    dq = O.dequantize(p).reshape(-1, 64)
    rng = np.random.default_rng(0)
    cb = p["codes"].reshape(-1, 32)
    for _ in range(300):
        b, i = rng.integers(0, x.shape[0]), rng.integers(0, 64)
        A = Fraction(float(a[b]))
        n = fl32(fr(x[b, i]) / A)                      # fl(x / absmax)
        # nearest level by exact distance, ties to the lower index
        dists = [abs(Fraction(n) - fr(c)) for c in O.NF4_CODEBOOK]
        code = min(range(16), key=lambda j: (dists[j], j))
        byte = int(cb[b, i // 2])
        got = (byte >> 4) if i % 2 == 0 else (byte & 15)
        assert got == code
        assert float(dq[b, i]) == fl32(fr(O.NF4_CODEBOOK[code]) * A)   # fl(c * absmax)


# ---------------------------------------------------------------------------
# double quantization
# ---------------------------------------------------------------------------
def test_double_quant_offset_scale_and_error():
    rng = np.random.default_rng(1)
    E, nb = 3, 300  # one full block and one partial block per expert
    a = np.abs(rng.normal(0.05, 0.02, size=(E, nb))).astype(np.float32)
    a[1, :] = np.float32(0.03)          # constant absmax: v == 0 everywhere, s == 0
    d = O.double_quantize_absmax(a)
    for e in range(E):
        exact = math.fsum(float(v) for v in a[e]) / nb
        off = float(d["absmax_offset"][e])
        assert abs(off - exact) <= float(np.spacing(np.float32(exact)))
    assert np.all(d["absmax_q"][1] == 0) and np.all(d["absmax_scale"][1] == 0)
    packed = {"mode": "nf4_dq", "E": E, "R": 1, "C": nb * 64, **d}
    dec = O.nf4_absmax_decoded(packed).reshape(E, nb).astype(np.float64)
    s = np.repeat(d["absmax_scale"].astype(np.float64), 256, axis=1)[:, :nb]
    tol = s / 254 * (1 + 2.0 ** -18) + 4 * np.spacing(np.maximum(np.abs(a), np.abs(dec)).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(dec - a) <= tol)
    assert np.array_equal(dec[1], np.full(nb, 0.03, np.float32).astype(np.float64))
    # int8 range and the block's extreme maps to +-127
    q = d["absmax_q"].astype(np.int64)
    assert q.min() >= -127 and q.max() <= 127
    assert np.abs(q[0, :256]).max() == 127 and np.abs(q[0, 256:]).max() == 127


def test_double_quant_sum_order_is_sequential():
    # values whose fp64 sum depends on the order: a huge value first, then many tiny ones
    a = np.full((1, 512), np.float32(2.0 ** -30), dtype=np.float32)
    a[0, 0] = np.float32(2.0 ** 30)
    a[0, 256] = np.float32(2.0 ** 30)
    d = O.double_quantize_absmax(a)
    s0 = 0.0
    for v in a[0, :256]:
        s0 += float(v)
    s1 = 0.0
    for v in a[0, 256:]:
        s1 += float(v)
    expect = np.float32((0.0 + s0 + s1) / 512)
    assert d["absmax_offset"][0] == expect


# ---------------------------------------------------------------------------
# int8 row-wise
# ---------------------------------------------------------------------------
def test_int8_half_even_and_extremes():
    row = np.zeros(64, np.float32)
    row[:8] = [127.0, 2.5, 3.5, -2.5, 0.5, 1.5, -127.0, 0.0]
    w = to_bf16_bits(np.stack([row, np.zeros(64, np.float32)])).reshape(1, 2, 64)
    p = O.quantize_int8_rowwise(w)
    assert list(p["codes"][0, 0, :8]) == [127, 2, 4, -2, 0, 2, -127, 0]
    assert p["absmax"][0, 0] == 127.0
    assert np.all(p["codes"][0, 1] == 0) and p["absmax"][0, 1] == 0.0
    assert np.all(O.dequantize(p)[0, 1] == 0.0)


def test_int8_error_bound_with_outliers_and_exact_rationals():
    g = torch.Generator().manual_seed(9)
    x = torch.randn((2, 16, 256), generator=g) * 0.02
    m = torch.rand((2, 16, 256), generator=g) < 0.01
    x = torch.where(m, x * 20, x)
    w = x.to(torch.bfloat16).view(torch.uint16).numpy()
    p = O.quantize_int8_rowwise(w)
    xf = O.bf16_to_f32(w).astype(np.float64)
    a = p["absmax"].astype(np.float64)[..., None]
    dq = O.dequantize(p).astype(np.float64)
    # a/254 from rounding q, plus fl(a/127) times |q| <= 127 and the final product
    # rounding: 2 * 2^-24 * a at most
    assert np.all(np.abs(xf - dq) <= a / 254 + a * 2.0 ** -23)
    am = np.argmax(np.abs(xf), axis=-1)
    q = p["codes"].astype(np.int64)
    assert np.all(np.abs(np.take_along_axis(q, am[..., None], -1)) == 127)
    rng = np.random.default_rng(2)
    for _ in range(300):
        e, r, c = rng.integers(0, 2), rng.integers(0, 16), rng.integers(0, 256)
        A = fr(p["absmax"][e, r])
        n = Fraction(fl32(Fraction(127) * fr(xf[e, r, c])) ) / A
        nq = Fraction(fl32(n))
        fl_ = math.floor(nq)
        rq = fl_ + 1 if (nq - fl_ > Fraction(1, 2) or (nq - fl_ == Fraction(1, 2) and fl_ % 2)) else fl_
        assert int(p["codes"][e, r, c]) == rq
        step = fl32(A / 127)
        assert float(dq[e, r, c]) == fl32(Fraction(rq) * Fraction(step))


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------
def test_route_against_stable_sort():
    rng = np.random.default_rng(4)
    T, K, E = 97, 3, 11
    idx = rng.integers(0, E, size=(T, K))
    idx[5, 1] = -1
    idx[8, 2] = E          # out of range: dropped
    counts, offsets, perm = O.route(idx, E)
    flat = idx.reshape(-1)
    valid = [p for p in range(flat.size) if 0 <= flat[p] < E]
    expect = sorted(valid, key=lambda p: flat[p])          # Python's sort is stable
    assert list(perm) == expect
    assert np.array_equal(counts, np.bincount(flat[valid], minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------
def _rand_weights(E, H, I, seed):
    g = torch.Generator().manual_seed(seed)
    gu = (torch.randn((E, 2 * I, H), generator=g) * 0.1).numpy().astype(np.float32)
    dn = (torch.randn((E, H, I), generator=g) * 0.1).numpy().astype(np.float32)
    return gu, dn


def _hidden(T, H, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((T, H), generator=g).to(torch.bfloat16).view(torch.uint16).numpy()


def test_forward_top1_is_one_swiglu_mlp():
    E, H, I, T = 4, 32, 16, 9
    gu, dn = _rand_weights(E, H, I, 0)
    x = _hidden(T, H, 1)
    idx = (np.arange(T) % E).reshape(T, 1)
    w = np.ones((T, 1), np.float32)
    out = O.experts_forward(x, idx, w, gu, dn)
    xt = torch.from_numpy(O.bf16_to_f32(x).astype(np.float64))
    for t in range(T):
        e = idx[t, 0]
        G = torch.from_numpy(gu[e, :I].astype(np.float64))
        U = torch.from_numpy(gu[e, I:].astype(np.float64))
        D = torch.from_numpy(dn[e].astype(np.float64))
        ref = F.linear(F.silu(F.linear(xt[t], G)) * F.linear(xt[t], U), D)
        assert np.allclose(out[t], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_forward_top_all_uniform_is_dense_average():
    E, H, I, T = 5, 24, 8, 6
    gu, dn = _rand_weights(E, H, I, 2)
    x = _hidden(T, H, 3)
    rng = np.random.default_rng(0)
    idx = np.stack([rng.permutation(E) for _ in range(T)])   # every expert once, any order
    w = np.full((T, E), 1.0 / E, np.float32)
    out = O.experts_forward(x, idx, w, gu, dn)
    xt = torch.from_numpy(O.bf16_to_f32(x).astype(np.float64))
    dense = torch.zeros((T, H), dtype=torch.float64)
    for e in range(E):
        G = torch.from_numpy(gu[e, :I].astype(np.float64))
        U = torch.from_numpy(gu[e, I:].astype(np.float64))
        D = torch.from_numpy(dn[e].astype(np.float64))
        dense += F.linear(F.silu(F.linear(xt, G)) * F.linear(xt, U), D)
    dense *= float(np.float32(1.0 / E))
    assert np.allclose(out, dense.numpy(), rtol=1e-10, atol=1e-12)


def test_forward_matches_pure_python_loops():
    E, H, I, T, K = 3, 8, 4, 5, 2
    gu, dn = _rand_weights(E, H, I, 4)
    x = _hidden(T, H, 5)
    rng = np.random.default_rng(6)
    idx = rng.integers(0, E, size=(T, K))
    w = rng.random((T, K)).astype(np.float32)
    out = O.experts_forward(x, idx, w, gu, dn)
    xf = O.bf16_to_f32(x)
    for t in range(T):
        acc = [0.0] * H
        for k in range(K):
            e = int(idx[t, k])
            h = []
            for j in range(I):
                g = sum(float(xf[t, c]) * float(gu[e, j, c]) for c in range(H))
                u = sum(float(xf[t, c]) * float(gu[e, I + j, c]) for c in range(H))
                h.append(g / (1.0 + math.exp(-g)) * u)
            for i in range(H):
                y = sum(h[j] * float(dn[e, i, j]) for j in range(I))
                acc[i] += float(w[t, k]) * y
        assert np.allclose(out[t], acc, rtol=1e-12, atol=1e-14)


def test_forward_gate_is_first_half_on_square_gate_up():
    # square gate_up (2I == H), the orientation the pages warn about
    E, I = 2, 8
    H = 2 * I
    gu = np.zeros((E, 2 * I, H), np.float32)
    gu[:, :I, 0] = 4.0      # gate rows: g = 4 for x = e_0
    gu[:, I:, 0] = 1.0      # up rows:   u = 1
    dn = np.zeros((E, H, I), np.float32)
    for e in range(E):
        dn[e, :I, :] = np.eye(I, dtype=np.float32)
    x = to_bf16_bits(np.eye(1, H, dtype=np.float32))
    out = O.experts_forward(x, np.array([[1]]), np.array([[1.0]], np.float32), gu, dn)
    expect = 4.0 / (1.0 + math.exp(-4.0)) * 1.0     # silu(gate) * up
    assert np.allclose(out[0, :I], expect, rtol=1e-14) and np.all(out[0, I:] == 0)
    assert not np.isclose(expect, 1.0 / (1.0 + math.exp(-1.0)) * 4.0)   # swapped would differ


def test_forward_expert_relabelling_and_dropped_pairs():
    E, H, I, T, K = 6, 16, 8, 20, 3
    gu, dn = _rand_weights(E, H, I, 8)
    x = _hidden(T, H, 9)
    rng = np.random.default_rng(10)
    idx = rng.integers(0, E, size=(T, K))
    w = rng.random((T, K)).astype(np.float32)
    out = O.experts_forward(x, idx, w, gu, dn)
    pi = rng.permutation(E)           # expert e moves to slot pi[e]
    gu2, dn2 = np.empty_like(gu), np.empty_like(dn)
    gu2[pi], dn2[pi] = gu, dn
    out2 = O.experts_forward(x, pi[idx], w, gu2, dn2)
    assert np.allclose(out, out2, rtol=1e-12, atol=1e-14)
    idx3, w3 = idx.copy(), w.copy()
    idx3[4, 1], idx3[7, 0] = -1, E
    w0 = w.copy()
    w0[4, 1], w0[7, 0] = 0.0, 0.0
    assert np.allclose(O.experts_forward(x, idx3, w3, gu, dn), O.experts_forward(x, idx, w0, gu, dn),
                       rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# storage sizes against the footprints printed on the pages
# ---------------------------------------------------------------------------
def test_packed_sizes_against_page_footprints():
    with open(os.path.join(HERE, "golden", "qwen3_30b_a3b_footprint.json")) as f:
        g = json.load(f)
    L, E, H, I = g["layers"], g["num_experts"], g["hidden_size"], g["moe_intermediate_size"]
    elems = L * (E * 2 * I * H + E * H * I)
    bf16_gib = 2 * elems / 2**30
    nf4dq_gib = L * (O.packed_nbytes("nf4_dq", E, 2 * I, H) + O.packed_nbytes("nf4_dq", E, H, I)) / 2**30
    nf4_gib = L * (O.packed_nbytes("nf4", E, 2 * I, H) + O.packed_nbytes("nf4", E, H, I)) / 2**30
    assert bf16_gib < g["footprint_experts_unquantized_gib"]
    assert nf4dq_gib < g["footprint_quantized_gib"] < bf16_gib
    assert nf4dq_gib < nf4_gib
    # the non-expert remainder of the unquantized print is small next to the experts
    assert g["footprint_experts_unquantized_gib"] - bf16_gib < 0.05 * bf16_gib
    assert abs(nf4dq_gib / (elems / 2**30) - (0.5 + 1 / 64 + 4 / (64 * 256))) < 1e-3
