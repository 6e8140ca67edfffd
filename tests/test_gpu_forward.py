"""GPU parity of the routing step (exact) and of the routed experts forward (within
2e-2 * rms of the oracle's output), including ragged tiles, edge cases and the five
workloads at full size on sampled tokens."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from bit_weight_quantization_moeq_b200 import synth
from tests.helpers import check_forward, oracle_forward

pytestmark = pytest.mark.gpu


def moeq():
    import bit_weight_quantization_moeq_b200 as m
    return m


def quantize(w, mode):
    m = moeq()
    if mode == 2:
        return m.moeq_quantize_int8_rowwise(w)
    return m.moeq_quantize_nf4(w, double_quant=(mode == 1))


def make_inputs(E, H, I, T, K, seed, outliers=False, device="cuda"):
    gu = synth.expert_weights(E, 2 * I, H, seed, outliers, device)
    dn = synth.expert_weights(E, H, I, seed + 1, outliers, device, mask_seed=seed + 6)
    x = synth.hidden_states(T, H, seed + 2, device)
    idx, w = synth.routing(T, E, K, seed + 3, 0.0, device)
    return {"gate_up": gu, "down": dn, "hidden": x, "top_k_index": idx, "top_k_weights": w}


def run_forward(inp, mode, **kw):
    """fp32-output forward (the parity subject) and a check that the bf16 output of the
    same call sequence is exactly the round-to-nearest-even of that fp32 output."""
    m = moeq()
    gu = quantize(inp["gate_up"], mode)
    dn = quantize(inp["down"], mode)
    out = m.moeq_experts_forward(inp["hidden"], inp["top_k_index"], inp["top_k_weights"], gu, dn,
                                 out_dtype=torch.float32, **kw)
    out16 = m.moeq_experts_forward(inp["hidden"], inp["top_k_index"], inp["top_k_weights"], gu, dn,
                                   out_dtype=torch.bfloat16, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out16.view(torch.int16), out.to(torch.bfloat16).view(torch.int16))
    return out


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------
# (single-launch routing up to 4096 pairs and 256 experts, the first three cases; the
# chunked three-kernel path beyond)
@pytest.mark.parametrize("T,K,E", [(1, 1, 8), (7, 2, 8), (300, 8, 64), (5000, 8, 128), (32768, 8, 256),
                                   (4096, 2, 1000), (40000, 8, 64), (33000, 8, 256)])
@pytest.mark.parametrize("dtype", [torch.int32, torch.int64])
def test_route_parity(T, K, E, dtype):
    g = torch.Generator().manual_seed(T * 31 + E)
    idx = torch.randint(0, E, (T, K), generator=g).to(dtype)
    counts, offsets, perm = moeq().moeq_route(idx.cuda(), E)
    torch.cuda.synchronize()
    rc, ro, rp = O.route(idx.numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy()[: ro[-1]], rp)


def test_route_drops_bad_indices_and_reports():
    T, K, E = 50, 4, 16
    g = torch.Generator().manual_seed(1)
    idx = torch.randint(0, E, (T, K), generator=g, dtype=torch.int32)
    idx[3, 1] = -1
    idx[10, 0] = E
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    counts, offsets, perm = moeq().moeq_route(idx.cuda(), E, d_status=status)
    torch.cuda.synchronize()
    rc, ro, rp = O.route(idx.numpy(), E)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy()[: ro[-1]], rp)
    assert int(status.item()) == 9  # MOEQ_ERR_INDEX


# ---------------------------------------------------------------------------
# forward parity
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("E,H,I,T,K", [
    (8, 256, 128, 64, 2),       # the tiny workload's shapes
    (6, 384, 192, 700, 2),      # several m-tiles; odd K / 64 in down (a lone last K stage)
    (4, 256, 128, 1500, 2),     # several token tiles per expert (full 192-wide ones, ragged)
    (16, 512, 256, 37, 8),      # few tokens per expert (small UMMA N)
    (4, 128, 64, 300, 2),       # the smallest shapes: one K stage in down, one m-tile
])
def test_forward_parity(mode, E, H, I, T, K):
    inp = make_inputs(E, H, I, T, K, seed=100 * E + T + mode, outliers=(mode == 2))
    out = run_forward(inp, mode)
    check_forward(out, oracle_forward(inp, mode))


def test_forward_single_token_and_empty():
    m = moeq()
    inp = make_inputs(8, 256, 128, 1, 2, seed=7)
    out = run_forward(inp, 0)
    check_forward(out, oracle_forward(inp, 0))
    gu, dn = quantize(inp["gate_up"], 0), quantize(inp["down"], 0)
    empty = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    out0 = m.moeq_experts_forward(empty, inp["top_k_index"][:0], inp["top_k_weights"][:0], gu, dn)
    assert out0.shape == (0, 256)


def test_forward_bad_index_dropped_duplicates_added_and_dtypes():
    inp = make_inputs(8, 256, 128, 40, 4, seed=11)
    idx = inp["top_k_index"].clone()
    idx[2, 1] = -3            # dropped
    idx[5, 0] = 8             # dropped
    idx[7, 1] = idx[7, 0]     # the same expert twice: both terms add
    inp["top_k_index"] = idx.to(torch.int64)
    inp["top_k_weights"] = inp["top_k_weights"].to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_forward(inp, 0, d_status=status)
    check_forward(out, oracle_forward(inp, 0))
    assert int(status.item()) == 9


def test_forward_hidden_beyond_fp16_saturates_and_reports():
    # the tensor cores take fp16 tokens: a hidden value beyond +-65504 saturates and raises
    # MOEQ_ERR_RANGE (11); the other tokens are unaffected
    T = 40
    inp = make_inputs(8, 256, 128, T, 2, seed=13)
    inp["hidden"][3, 5] = 1.0e5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run_forward(inp, 0, d_status=status)
    assert int(status.item()) == 11
    others = [t for t in range(T) if t != 3]
    check_forward(out, oracle_forward(inp, 0, tokens=others), tokens=others)


def test_forward_nf4_absmax_beyond_fp16_reports():
    # an NF4 block whose absmax exceeds the fp16 range cannot be an fp16 tensor-core operand:
    # the GEMM clamps its scale and reports MOEQ_ERR_RANGE (11)
    inp = make_inputs(8, 256, 128, 64, 2, seed=17)
    inp["gate_up"][int(inp["top_k_index"][0, 0]), 5, 9] = 1.0e5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    run_forward(inp, 0, d_status=status)
    assert int(status.item()) == 11


def test_forward_top_all_experts_uniform():
    E, H, I, T = 8, 256, 128, 33
    inp = make_inputs(E, H, I, T, E, seed=21)
    g = torch.Generator().manual_seed(0)
    inp["top_k_index"] = torch.stack([torch.randperm(E, generator=g) for _ in range(T)]).to(torch.int32).cuda()
    inp["top_k_weights"] = torch.full((T, E), 1.0 / E, dtype=torch.float32, device="cuda")
    out = run_forward(inp, 0)
    check_forward(out, oracle_forward(inp, 0))


def test_forward_deterministic_bits():
    inp = make_inputs(16, 512, 256, 900, 4, seed=31)
    m = moeq()
    gu, dn = quantize(inp["gate_up"], 0), quantize(inp["down"], 0)
    a = m.moeq_experts_forward(inp["hidden"], inp["top_k_index"], inp["top_k_weights"], gu, dn)
    b = m.moeq_experts_forward(inp["hidden"], inp["top_k_index"], inp["top_k_weights"], gu, dn)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["tiny", "olmoe", "qwen", "mixtral", "skew1", "skew64", "skew32k"])
def test_forward_full_size_sampled(name):
    wl = synth.WORKLOADS[name]
    inp = synth.workload_inputs(wl, device="cuda")
    out = run_forward(inp, wl.mode)
    n_tok = {"mixtral": 2, "tiny": wl.T, "skew1": 1}.get(name, 4)
    rng = np.random.default_rng(wl.cfg)
    tokens = np.sort(rng.choice(wl.T, n_tok, replace=False))
    check_forward(out, oracle_forward(inp, wl.mode, tokens=tokens), tokens=tokens)
    assert torch.isfinite(out.float()).all()
