"""GPU parity of the quantizers and the dequantizer (bit-exact against the oracle)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from bit_weight_quantization_moeq_b200 import synth
from tests.helpers import assert_packed_equal, bits, gpu_packed_numpy, oracle_quantize

pytestmark = pytest.mark.gpu

M = None


def moeq():
    global M
    if M is None:
        import bit_weight_quantization_moeq_b200 as m
        M = m
    return M


def quantize(w: torch.Tensor, mode: int):
    m = moeq()
    if mode == 2:
        return m.moeq_quantize_int8_rowwise(w)
    return m.moeq_quantize_nf4(w, double_quant=(mode == 1))


def rand_w(shape, seed, scale=0.02, outliers=False):
    return synth.expert_weights(*shape, seed=seed, outliers=outliers, device="cuda") if scale == 0.02 else \
        (torch.randn(shape, generator=torch.Generator("cuda").manual_seed(seed), device="cuda") * scale).to(torch.bfloat16)


def mantissa_pair_tensor(C=64):
    """Blocks/rows that pair every bf16 divisor mantissa (as the block/row absmax) with
    every bf16 dividend mantissa, at exponent offsets 0..7, both signs, for absmax
    exponents spanning normal numbers and the tiny range that takes the plain-divide
    path."""
    xs = []
    for ex in range(8):
        for man in range(128):
            v = (1.0 + man / 128.0) * 2.0 ** (-ex - 1)
            xs += [v, -v]
    xs = np.array(xs, np.float64)  # |x| < 1
    rows = []
    for a_exp in (-126, -121, -119, -60, -3, 0, 7, 100):
        for am in range(128):
            a = (1.0 + am / 128.0) * 2.0 ** a_exp
            vals = xs * a
            for s in range(0, len(vals), C - 1):
                row = np.zeros(C, np.float64)
                chunk = vals[s:s + C - 1]
                row[:len(chunk)] = chunk
                row[C - 1] = a if (s // (C - 1)) % 2 == 0 else -a
                rows.append(row)
    arr = np.stack(rows).astype(np.float32)
    t = torch.from_numpy(arr).to(torch.bfloat16)
    return t.view(1, -1, C)


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", [(1, 1, 64), (3, 5, 128), (2, 33, 192), (8, 256, 256), (4, 96, 640)])
def test_quantize_parity_random(mode, shape):
    w = rand_w(shape, seed=sum(shape) + 17 * mode, outliers=(mode == 2))
    w[0, 0, :64] = 0.0                      # an all-zero block / zero-prefix row
    if shape[1] > 1:
        w[0, 1, 3] = 7.5                    # a large positive absmax element
        w[0, 1, 9] = -9.0                   # ... and a larger negative one
    p = quantize(w, mode)
    torch.cuda.synchronize()
    assert_packed_equal(gpu_packed_numpy(p), oracle_quantize(bits(w), mode), mode)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_quantize_source_aligned_to_16_bytes_only(mode):
    # a source 16 bytes past a 32-byte boundary takes the 16-byte-load path of the NF4
    # quantizer (32-byte-aligned sources use single 256-bit loads)
    E, R, C = 3, 17, 192
    base = rand_w((1, 1, E * R * C + 64), seed=77 + mode, outliers=(mode == 2)).view(-1)
    w = base[8:8 + E * R * C].view(E, R, C)
    assert w.data_ptr() % 32 == 16
    p = quantize(w, mode)
    torch.cuda.synchronize()
    assert_packed_equal(gpu_packed_numpy(p), oracle_quantize(bits(w), mode), mode)


@pytest.mark.parametrize("mode", [0, 2])
def test_quantize_parity_every_mantissa_pair(mode):
    w = mantissa_pair_tensor(64).cuda()
    p = quantize(w, mode)
    torch.cuda.synchronize()
    assert_packed_equal(gpu_packed_numpy(p), oracle_quantize(bits(w), mode), mode)


def test_double_quant_partial_blocks_and_constant_expert():
    E, R, C = 3, 75, 256            # nb = 300 per expert: a full and a partial 256-block
    w = rand_w((E, R, C), seed=123)
    w[1] = 0.5                       # every block of expert 1 has absmax 0.5: s == 0
    p = quantize(w, 1)
    torch.cuda.synchronize()
    ref = oracle_quantize(bits(w), 1)
    assert_packed_equal(gpu_packed_numpy(p), ref, 1)
    assert np.all(ref["absmax_q"][1] == 0)


def test_double_quant_offset_over_many_chunks():
    # one expert with 1040 chunks of 256 absmax values: the per-expert offset is summed in
    # several staged passes and must still equal the oracle's sequential sum
    w = rand_w((1, 4096, 4160), seed=29)
    p = quantize(w, 1)
    torch.cuda.synchronize()
    assert_packed_equal(gpu_packed_numpy(p), oracle_quantize(bits(w), 1), 1)


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_dequantize_parity(mode, out_dtype):
    m = moeq()
    w = rand_w((4, 96, 640), seed=5 + mode, outliers=(mode == 2))
    p = quantize(w, mode)
    dq = m.moeq_dequantize(p, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = O.dequantize(oracle_quantize(bits(w), mode))
    if out_dtype == torch.float32:
        assert np.array_equal(dq.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    else:
        assert np.array_equal(bits(dq), O.f32_to_bf16(ref))


def test_empty_tensor_is_a_no_op():
    m = moeq()
    w = torch.empty((0, 16, 64), dtype=torch.bfloat16, device="cuda")
    p = m.moeq_quantize_nf4(w)
    assert p.codes.numel() == 0


@pytest.mark.parametrize("name", ["olmoe", "qwen", "mixtral"])
def test_full_size_quantize_sampled(name):
    """Full-size tensors of a workload, quantized on the GPU; sampled experts (NF4) or
    rows (int8) compared bit-exactly with the oracle."""
    wl = synth.WORKLOADS[name]
    s = 1000 * wl.cfg
    rng = np.random.default_rng(wl.cfg)
    for which, (R, C, seed) in {"gate_up": (2 * wl.I, wl.H, s), "down": (wl.H, wl.I, s + 1)}.items():
        w = synth.expert_weights(wl.E, R, C, seed, wl.outliers, device="cuda",
                                 mask_seed=(s + 4 if which == "gate_up" else s + 6))
        p = quantize(w, wl.mode)
        torch.cuda.synchronize()
        g = gpu_packed_numpy(p)
        if wl.mode == 2:
            es = rng.integers(0, wl.E, 2)
            rows = rng.integers(0, R, 512)
            for e in es:
                ref = O.quantize_int8_rowwise(bits(w[e, rows]).reshape(1, len(rows), C))
                assert np.array_equal(g["codes"][e, rows].view(np.uint8), ref["codes"][0].view(np.uint8))
                assert np.array_equal(g["absmax"][e, rows], ref["absmax"][0])
        else:
            for e in rng.choice(wl.E, 2, replace=False):
                ref = oracle_quantize(bits(w[e:e + 1]), wl.mode)
                sub = {k: v[e:e + 1] for k, v in g.items()}
                assert_packed_equal(sub, ref, wl.mode)
        del w, p
