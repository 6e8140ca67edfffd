"""The C-ABI library loads, exports every entry point include/moeq.h declares, and
rejects bad arguments on the host before touching the device.  No GPU needed: every
call here either fails validation (so nothing is enqueued) or, on a machine without a
GPU, reaches the device query and reports MOEQ_ERR_CUDA instead of computing anything."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moeq.h")

M = pytest.importorskip("bit_weight_quantization_moeq_b200")
lib = M.lib
OK, NULL, SHAPE, DTYPE, ALIGN, BLOCK, WS, CUDA = 0, 1, 2, 3, 4, 5, 6, 7


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moeq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_entry_point_is_exported():
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/moeq.h but not exported"


def test_packed_bytes_match_closed_form():
    for mode, name in ((0, "nf4"), (1, "nf4_dq"), (2, "int8")):
        for E, R, C in ((1, 1, 64), (8, 256, 256), (64, 2048, 2048), (128, 1536, 2048), (8, 28672, 4096), (3, 75, 256)):
            total, sizes = M.moeq_packed_bytes(mode, E, R, C)
            assert total == O.packed_nbytes(name, E, R, C) == sum(sizes)
    assert M.moeq_packed_bytes(0, 1, 1, 63)[0] == 0
    assert M.moeq_packed_bytes(7, 1, 1, 64)[0] == 0


def test_workspace_sizes():
    assert M.moeq_quantize_workspace(0, 4, 8, 64) == 0
    assert M.moeq_quantize_workspace(2, 4, 8, 64) == 0
    w = M.moeq_quantize_workspace(1, 128, 1536, 2048)
    assert w >= 128 * 1536 * 32 * 4 + 128 * 192 * 8
    T, K, E, H, I = 4096, 8, 64, 2048, 1024
    f = M.moeq_forward_workspace(T, K, E, H, I)
    S = T * K
    assert f >= S * (2 * H + 2 * I + 4 * H) + 4 * S
    assert M.moeq_route_workspace(T, K, E) < f
    assert M.moeq_forward_workspace(T, 0, E, H, I) == 0


def test_status_strings():
    for code in range(12):
        assert M.moeq_status_string(code)
    assert "unknown" in M.moeq_status_string(99)


def packed(mode, E, R, C, base=0x10000):
    p = M._Packed(mode, E, R, C, base, base + 0x1000, base + 0x2000, base + 0x3000, base + 0x4000)
    return p


NOSTREAM = ctypes.c_void_p(0)


def q_nf4(w, E, R, C, dq, out, ws=0, ws_bytes=0):
    return lib.moeq_quantize_nf4(ctypes.c_void_p(w), E, R, C, dq, ctypes.byref(out) if out is not None else None,
                                 ctypes.c_void_p(ws), ws_bytes, NOSTREAM)


def test_quantize_argument_checks():
    l0 = M.moeq_kernel_launches()
    assert lib.moeq_quantize_nf4(ctypes.c_void_p(0x1000), 1, 1, 64, 0, None, None, 0, NOSTREAM) == NULL
    assert q_nf4(0x1000, 1, 1, 96, 0, packed(0, 1, 1, 96)) == BLOCK
    assert q_nf4(0x1000, 1, 1, 64, 1, packed(0, 1, 1, 64)) == DTYPE          # mode vs double_quant
    assert q_nf4(0x1000, 2, 1, 64, 0, packed(0, 1, 1, 64)) == SHAPE          # E mismatch
    assert q_nf4(0x1001, 1, 1, 64, 0, packed(0, 1, 1, 64)) == ALIGN          # misaligned source
    assert q_nf4(0, 1, 1, 64, 0, packed(0, 1, 1, 64)) == NULL
    assert q_nf4(0x1000, 1, 1, 64, 1, packed(1, 1, 1, 64)) == WS            # double quant, no ws
    assert q_nf4(0x1000, 0, 4, 64, 0, packed(0, 0, 4, 64)) == OK            # empty: nothing to do
    bad = packed(0, 1, 1, 64)
    bad.absmax = None
    assert q_nf4(0x1000, 1, 1, 64, 0, bad) == NULL
    assert lib.moeq_quantize_int8_rowwise(ctypes.c_void_p(0x1000), 1, 1, 64, ctypes.byref(packed(0, 1, 1, 64)),
                                          NOSTREAM) == DTYPE
    assert lib.moeq_dequantize(ctypes.byref(packed(0, 1, 1, 64)), ctypes.c_void_p(0x1000), 9, NOSTREAM) == DTYPE
    assert lib.moeq_dequantize(ctypes.byref(packed(0, 1, 1, 64)), None, 0, NOSTREAM) == NULL
    assert M.moeq_kernel_launches() == l0  # nothing was enqueued


def fwd(T, K, gu, dn, idx_dt=2, w_dt=1, out_dt=0, ws=0x800000, ws_bytes=1 << 40, h=0x1000, out=0x2000):
    return lib.moeq_experts_forward(ctypes.c_void_p(h), ctypes.c_void_p(0x3000), idx_dt, ctypes.c_void_p(0x4000),
                                    w_dt, T, K, ctypes.byref(gu), ctypes.byref(dn), ctypes.c_void_p(out), out_dt,
                                    ctypes.c_void_p(ws), ws_bytes, None, NOSTREAM)


def test_forward_argument_checks():
    E, H, I = 8, 256, 128
    gu, dn = packed(0, E, 2 * I, H), packed(0, E, H, I, base=0x20000)
    l0 = M.moeq_kernel_launches()
    assert fwd(4, 2, gu, packed(0, E, H, 192, base=0x20000)) == SHAPE        # gate_up R != 2 * down C
    assert fwd(4, 2, gu, packed(2, E, H, I, base=0x20000)) == DTYPE          # mixed modes
    assert fwd(4, 2, gu, dn, idx_dt=0) == DTYPE
    assert fwd(4, 2, gu, dn, w_dt=3) == DTYPE
    assert fwd(4, 2, gu, dn, out_dt=2) == DTYPE
    assert fwd(4, 0, gu, dn) == SHAPE
    assert fwd(4, 2, gu, dn, ws_bytes=16) == WS
    assert fwd(4, 2, gu, dn, out=0x2008) == ALIGN
    assert fwd(0, 2, gu, dn) == OK                                           # no tokens: no launch
    gu2, dn2 = packed(0, E, 2 * I, 192), packed(0, E, 192, I, base=0x20000)
    assert fwd(4, 2, gu2, dn2) == SHAPE                                      # H % 128 != 0
    assert lib.moeq_route(ctypes.c_void_p(0x3000), 2, 4, 2, 0, ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000),
                          ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1000), 1 << 30, None, NOSTREAM) == SHAPE
    assert M.moeq_kernel_launches() == l0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_a_gpu_fails_loudly():
    # every argument is well formed: the only thing missing is the device
    assert q_nf4(0x1000, 1, 1, 64, 0, packed(0, 1, 1, 64)) in (CUDA, 10)
    E, H, I = 8, 256, 128
    assert fwd(4, 2, packed(0, E, 2 * I, H), packed(0, E, H, I, base=0x20000)) in (CUDA, 10)
