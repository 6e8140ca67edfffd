"""moeq_route_noalloc, the routing step for callers that cannot allocate device memory
(a runtime that owns the whole device through its own pool, or a loop where cudaMalloc
would synchronise the device): called through the C ABI, its counts, offsets and
permutation must equal those of moeq_route, which takes a caller-provided workspace,
on two calls in a row (the second must not see the first one's leftovers in the shared
scratch).  Kept in its own file, collected last."""
from __future__ import annotations

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def _lib():
    import bit_weight_quantization_moeq_b200 as m
    f = m.lib.moeq_route_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return m, f


def _noalloc(f, idx, E, status):
    T, K = idx.shape
    counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((T * K,), -7, dtype=torch.int32, device="cuda")
    dt = 3 if idx.dtype == torch.int64 else 2
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = f(ctypes.c_void_p(idx.data_ptr()), dt, T, K, E, ctypes.c_void_p(counts.data_ptr()),
           ctypes.c_void_p(offsets.data_ptr()), ctypes.c_void_p(perm.data_ptr()),
           ctypes.c_void_p(status.data_ptr()), stream)
    return rc, counts, offsets, perm


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    m, f = _lib()
    g = torch.Generator().manual_seed(5)
    # routing problems up to 4096 pairs and 256 experts take a single launch that keeps its
    # tables in shared memory; larger ones go through the scratch array
    cases = [(40000, 8, 64, torch.int32),     # 625 chunks x 64 experts of scratch
             (3000, 2, 600, torch.int64),     # fewer chunks, more experts: a different layout
             (500, 8, 64, torch.int32)]       # the single-launch form
    for T, K, E, dt in cases:
        idx = torch.randint(0, E, (T, K), generator=g).to(dt).cuda()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc, counts, offsets, perm = _noalloc(f, idx, E, status)
        assert rc == 0, m.moeq_status_string(rc)
        ref_c, ref_o, ref_p = m.moeq_route(idx, E)
        torch.cuda.synchronize()
        assert torch.equal(counts, ref_c)
        assert torch.equal(offsets, ref_o)
        n = int(ref_o[-1].item())
        assert n == T * K
        assert torch.equal(perm[:n], ref_p[:n])
        assert int(status.item()) == 0


def test_route_noalloc_rejects_problems_beyond_its_scratch():
    m, f = _lib()
    idx = torch.zeros((300000, 8), dtype=torch.int32, device="cuda")   # 4688 chunks x 1024 experts
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc, *_ = _noalloc(f, idx, 1024, status)
    assert rc == 6  # MOEQ_ERR_WORKSPACE
