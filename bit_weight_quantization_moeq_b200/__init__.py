"""Python binding of libmoeq (the C ABI in include/moeq.h).

Argument marshalling only: every step runs in the library's sm_100a kernels.  torch
supplies device memory (the binding allocates outputs and workspaces with
``torch.empty`` when the caller does not pass them) and the current CUDA stream.
There is no fallback: if ``libmoeq.so`` is missing or fails to load, importing this
package raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

__all__ = [
    "MOEQ_NF4", "MOEQ_NF4_DQ", "MOEQ_INT8_ROW", "MoeqError", "PackedWeight",
    "moeq_packed_bytes", "moeq_quantize_workspace", "moeq_forward_workspace",
    "moeq_route_workspace", "moeq_quantize_nf4", "moeq_quantize_int8_rowwise",
    "moeq_dequantize", "moeq_experts_forward", "moeq_route", "moeq_kernel_launches",
    "moeq_status_string", "moeq_set_trace_events", "lib", "LIB_PATH",
]

MOEQ_NF4, MOEQ_NF4_DQ, MOEQ_INT8_ROW = 0, 1, 2
MOEQ_BF16, MOEQ_F32, MOEQ_I32, MOEQ_I64 = 0, 1, 2, 3
STATUS = {0: "MOEQ_OK", 1: "MOEQ_ERR_NULL", 2: "MOEQ_ERR_SHAPE", 3: "MOEQ_ERR_DTYPE",
          4: "MOEQ_ERR_ALIGN", 5: "MOEQ_ERR_BLOCKSIZE", 6: "MOEQ_ERR_WORKSPACE",
          7: "MOEQ_ERR_CUDA", 8: "MOEQ_ERR_TIMEOUT", 9: "MOEQ_ERR_INDEX", 10: "MOEQ_ERR_DEVICE",
          11: "MOEQ_ERR_RANGE"}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoeq.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python bit_weight_quantization_moeq_b200/build.py`")
lib = ctypes.CDLL(LIB_PATH)


class _Packed(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("E", ctypes.c_int32), ("R", ctypes.c_int32),
                ("C", ctypes.c_int32), ("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("absmax_q", ctypes.c_void_p), ("absmax_scale", ctypes.c_void_p),
                ("absmax_offset", ctypes.c_void_p)]


_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_P = ctypes.POINTER(_Packed)
_sigs = {
    "moeq_packed_bytes": (_sz, [_i, _i, _i, _i, ctypes.POINTER(_sz)]),
    "moeq_quantize_workspace": (_sz, [_i, _i, _i, _i]),
    "moeq_route_workspace": (_sz, [_i, _i, _i]),
    "moeq_forward_workspace": (_sz, [_i, _i, _i, _i, _i]),
    "moeq_kernel_launches": (ctypes.c_ulonglong, []),
    "moeq_quantize_nf4": (_i, [_vp, _i, _i, _i, _i, _P, _vp, _sz, _vp]),
    "moeq_quantize_int8_rowwise": (_i, [_vp, _i, _i, _i, _P, _vp]),
    "moeq_dequantize": (_i, [_P, _vp, _i, _vp]),
    "moeq_experts_forward": (_i, [_vp, _vp, _i, _vp, _i, _i, _i, _P, _P, _vp, _i, _vp, _sz, _vp, _vp]),
    "moeq_route": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "moeq_status_string": (ctypes.c_char_p, [_i]),
    "moeq_set_trace_events": (None, [ctypes.POINTER(ctypes.c_void_p), _i]),
}
for _name, (_res, _args) in _sigs.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MoeqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} "
                         f"({lib.moeq_status_string(status).decode()})")


def _check(status: int, where: str) -> None:
    if status != 0:
        raise MoeqError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def moeq_status_string(status: int) -> str:
    return lib.moeq_status_string(status).decode()


def moeq_kernel_launches() -> int:
    return int(lib.moeq_kernel_launches())


_trace_keep = None


def moeq_set_trace_events(events) -> None:
    """Record ``events`` (a list of torch.cuda.Event, at least 6) around the kernels of
    every later moeq_experts_forward on this thread; ``None`` stops."""
    global _trace_keep
    if not events:
        _trace_keep = None
        lib.moeq_set_trace_events(None, 0)
        return
    for ev in events:
        if ev.cuda_event == 0:      # torch creates the CUDA event lazily
            ev.record()
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _trace_keep = arr
    lib.moeq_set_trace_events(arr, len(events))


def moeq_packed_bytes(mode: int, E: int, R: int, C: int):
    sizes = (ctypes.c_size_t * 5)()
    total = lib.moeq_packed_bytes(mode, E, R, C, sizes)
    return int(total), [int(s) for s in sizes]


def moeq_quantize_workspace(mode: int, E: int, R: int, C: int) -> int:
    return int(lib.moeq_quantize_workspace(mode, E, R, C))


def moeq_route_workspace(T: int, K: int, E: int) -> int:
    return int(lib.moeq_route_workspace(T, K, E))


def moeq_forward_workspace(T: int, K: int, E: int, H: int, I: int) -> int:
    return int(lib.moeq_forward_workspace(T, K, E, H, I))


@dataclasses.dataclass
class PackedWeight:
    """A packed [E, R, C] expert tensor: the buffers of one ``moeq_packed``."""
    mode: int
    E: int
    R: int
    C: int
    codes: torch.Tensor
    absmax: torch.Tensor | None = None
    absmax_q: torch.Tensor | None = None
    absmax_scale: torch.Tensor | None = None
    absmax_offset: torch.Tensor | None = None

    @staticmethod
    def empty(mode: int, E: int, R: int, C: int, device="cuda") -> "PackedWeight":
        _, sz = moeq_packed_bytes(mode, E, R, C)
        u8, f32, i8 = torch.uint8, torch.float32, torch.int8
        codes = torch.empty(sz[0], dtype=u8 if mode != MOEQ_INT8_ROW else i8, device=device)
        if mode == MOEQ_INT8_ROW:
            codes = codes.view(E, R, C)
        else:
            codes = codes.view(E, R, C // 2)
        p = PackedWeight(mode, E, R, C, codes)
        if mode == MOEQ_NF4:
            p.absmax = torch.empty((E, R, C // 64), dtype=f32, device=device)
        elif mode == MOEQ_INT8_ROW:
            p.absmax = torch.empty((E, R), dtype=f32, device=device)
        else:
            nb = R * C // 64
            p.absmax_q = torch.empty((E, nb), dtype=i8, device=device)
            p.absmax_scale = torch.empty((E, (nb + 255) // 256), dtype=f32, device=device)
            p.absmax_offset = torch.empty((E,), dtype=f32, device=device)
        return p

    def descriptor(self) -> _Packed:
        return _Packed(self.mode, self.E, self.R, self.C, _ptr(self.codes), _ptr(self.absmax),
                       _ptr(self.absmax_q), _ptr(self.absmax_scale), _ptr(self.absmax_offset))

    def tensors(self) -> dict:
        return {k: v for k, v in (("codes", self.codes), ("absmax", self.absmax),
                                  ("absmax_q", self.absmax_q), ("absmax_scale", self.absmax_scale),
                                  ("absmax_offset", self.absmax_offset)) if v is not None}

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.tensors().values())


def moeq_quantize_nf4(w: torch.Tensor, double_quant: bool = False, out: PackedWeight | None = None,
                      ws: torch.Tensor | None = None, stream=None) -> PackedWeight:
    E, R, C = w.shape
    mode = MOEQ_NF4_DQ if double_quant else MOEQ_NF4
    if out is None:
        out = PackedWeight.empty(mode, E, R, C, w.device)
    need = moeq_quantize_workspace(mode, E, R, C)
    if need and ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=w.device)
    d = out.descriptor()
    _check(lib.moeq_quantize_nf4(_ptr(w), E, R, C, int(double_quant), ctypes.byref(d), _ptr(ws),
                                 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "moeq_quantize_nf4")
    return out


def moeq_quantize_int8_rowwise(w: torch.Tensor, out: PackedWeight | None = None, stream=None) -> PackedWeight:
    E, R, C = w.shape
    if out is None:
        out = PackedWeight.empty(MOEQ_INT8_ROW, E, R, C, w.device)
    d = out.descriptor()
    _check(lib.moeq_quantize_int8_rowwise(_ptr(w), E, R, C, ctypes.byref(d), _stream(stream)),
           "moeq_quantize_int8_rowwise")
    return out


def moeq_dequantize(p: PackedWeight, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((p.E, p.R, p.C), dtype=out_dtype, device=p.codes.device)
    code = MOEQ_F32 if out.dtype == torch.float32 else MOEQ_BF16
    d = p.descriptor()
    _check(lib.moeq_dequantize(ctypes.byref(d), _ptr(out), code, _stream(stream)), "moeq_dequantize")
    return out


def moeq_route(top_k_index: torch.Tensor, E: int, ws: torch.Tensor | None = None,
               d_status: torch.Tensor | None = None, stream=None):
    T, K = top_k_index.shape
    dev = top_k_index.device
    idt = MOEQ_I64 if top_k_index.dtype == torch.int64 else MOEQ_I32
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * K, 1), dtype=torch.int32, device=dev)
    if ws is None:
        ws = torch.empty(max(moeq_route_workspace(T, K, E), 16), dtype=torch.uint8, device=dev)
    _check(lib.moeq_route(_ptr(top_k_index), idt, T, K, E, _ptr(counts), _ptr(offsets), _ptr(perm),
                          _ptr(ws), ws.numel(), _ptr(d_status), _stream(stream)), "moeq_route")
    return counts, offsets, perm


def moeq_experts_forward(hidden: torch.Tensor, top_k_index: torch.Tensor, top_k_weights: torch.Tensor,
                         gate_up: PackedWeight, down: PackedWeight, out: torch.Tensor | None = None,
                         ws: torch.Tensor | None = None, d_status: torch.Tensor | None = None,
                         stream=None, out_dtype=torch.bfloat16) -> torch.Tensor:
    T, H = hidden.shape
    K = top_k_index.shape[1]
    I = down.C
    dev = hidden.device
    if out is None:
        out = torch.empty((T, H), dtype=out_dtype, device=dev)
    if ws is None:
        ws = torch.empty(max(moeq_forward_workspace(T, K, gate_up.E, H, I), 16), dtype=torch.uint8, device=dev)
    odt = MOEQ_F32 if out.dtype == torch.float32 else MOEQ_BF16
    idt = MOEQ_I64 if top_k_index.dtype == torch.int64 else MOEQ_I32
    wdt = MOEQ_BF16 if top_k_weights.dtype == torch.bfloat16 else MOEQ_F32
    dg, dd = gate_up.descriptor(), down.descriptor()
    _check(lib.moeq_experts_forward(_ptr(hidden), _ptr(top_k_index), idt, _ptr(top_k_weights), wdt, T, K,
                                    ctypes.byref(dg), ctypes.byref(dd), _ptr(out), odt, _ptr(ws), ws.numel(),
                                    _ptr(d_status), _stream(stream)), "moeq_experts_forward")
    return out
