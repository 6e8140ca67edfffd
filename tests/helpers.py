"""Helpers for the GPU parity tests: move inputs to numpy for the oracle, run the
oracle on a slice of a workload.  Expected values always come from ``oracle/`` fed
with the seeded inputs, never from the CUDA path."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

MODE_NAME = {0: "nf4", 1: "nf4_dq", 2: "int8"}


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy bit patterns."""
    return t.detach().contiguous().view(torch.uint16).cpu().numpy()


def oracle_quantize(w_bits: np.ndarray, mode: int) -> dict:
    if mode == 2:
        return O.quantize_int8_rowwise(w_bits)
    return O.quantize_nf4(w_bits, double_quant=(mode == 1))


def gpu_packed_numpy(p) -> dict:
    """The buffers of a PackedWeight as numpy arrays (for comparison only)."""
    d = {"codes": p.codes.cpu().numpy()}
    for k in ("absmax", "absmax_q", "absmax_scale", "absmax_offset"):
        v = getattr(p, k)
        if v is not None:
            d[k] = v.cpu().numpy()
    return d


def assert_packed_equal(gpu: dict, ref: dict, mode: int):
    assert np.array_equal(gpu["codes"].view(np.uint8), ref["codes"].view(np.uint8)), "codes differ"
    if mode == 1:
        assert np.array_equal(gpu["absmax_q"], ref["absmax_q"]), "absmax_q differ"
        assert np.array_equal(gpu["absmax_scale"].view(np.uint32),
                              ref["absmax_scale"].astype(np.float32).view(np.uint32)), "scale differ"
        assert np.array_equal(gpu["absmax_offset"].view(np.uint32),
                              ref["absmax_offset"].astype(np.float32).view(np.uint32)), "offset differ"
    else:
        assert np.array_equal(gpu["absmax"].reshape(-1).view(np.uint32),
                              ref["absmax"].astype(np.float32).reshape(-1).view(np.uint32)), "absmax differ"


def oracle_forward(inputs: dict, mode: int, tokens=None) -> np.ndarray:
    """Oracle forward for the listed tokens: quantizes (with the oracle) only the
    experts those tokens use, dequantizes them in fp32 and runs the fp64 forward."""
    idx = inputs["top_k_index"].cpu().numpy().astype(np.int64)
    E = inputs["gate_up"].shape[0]
    t_sel = np.arange(idx.shape[0]) if tokens is None else np.asarray(tokens)
    used = sorted({int(e) for e in idx[t_sel].reshape(-1) if 0 <= e < E})
    gu_full = inputs["gate_up"]
    dn_full = inputs["down"]
    twoI, H = gu_full.shape[1], gu_full.shape[2]
    I = dn_full.shape[2]
    gu = np.zeros((E, twoI, H), np.float32)
    dn = np.zeros((E, H, I), np.float32)
    for e in used:
        gu[e] = O.dequantize(oracle_quantize(bits(gu_full[e:e + 1]), mode))[0]
        dn[e] = O.dequantize(oracle_quantize(bits(dn_full[e:e + 1]), mode))[0]
    w = inputs["top_k_weights"]
    w = w.float().cpu().numpy()
    return O.experts_forward(bits(inputs["hidden"]), idx, w, gu, dn, tokens=t_sel)


def check_forward(out_gpu: torch.Tensor, ref: np.ndarray, tokens=None, tol=2e-2):
    """max |gpu - oracle| <= tol * rms(oracle) over the compared outputs."""
    got = out_gpu.float().cpu().numpy().astype(np.float64)
    if tokens is not None:
        got = got[np.asarray(tokens)]
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(got - ref)))
    assert np.all(np.isfinite(got)), "non-finite output"
    assert err <= tol * rms, f"max|diff| {err:.4g} > {tol} * rms {rms:.4g} (ratio {err / rms:.4g})"
    return err / rms
