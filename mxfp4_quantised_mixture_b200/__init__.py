"""Thin Python binding of libmoe_mxfp4.so (the MXFP4 Mixture-of-Experts layer
for NVIDIA B200, sm_100a).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch device tensors (used here for device memory and
streams); their ``data_ptr()`` is handed to the C ABI declared in
``include/moe_mxfp4.h``.  A missing or unloadable library raises at import:
there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_mxfp4.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_SHAPE = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_UNSUPPORTED = 4
MOE_ERR_CUDA = 5
MOE_ERR_NONFINITE = 6
MOE_ERR_TIMEOUT = 7

WS_PERMUTE, WS_EXPERT_MLP, WS_LAYER = 0, 1, 2
WS_EXPERT_MLP_BLOCK_SCALED, WS_EXPERT_MLP_BF16_DECODE = 3, 4
WS_EXPERT_MLP_UNQUANTISED = 5

# GEMM path of moe_expert_mlp_ex
MOE_MLP_PATH_AUTO = 0
MOE_MLP_PATH_BLOCK_SCALED = 1  # tcgen05 block-scaled MMA on the E2M1 codes
MOE_MLP_PATH_BF16_DECODE = 2   # codes decoded to bf16 into tensor memory

MOE_QUANT_RHT = 1  # random-sign Hadamard transform of each 32-block along K
MOE_QUANT_SR = 2   # stochastic rounding


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {moe_status_string(status)} ({status})")
        self.status = status


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32)]

    def __repr__(self):
        return (f"moe_shape(T={self.T}, E={self.E}, k={self.k}, d_model={self.d_model}, "
                f"d_ff={self.d_ff})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python mxfp4_quantised_mixture_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    lib.mxfp4_quantize.argtypes = [vp, i64, i64, vp, vp, vp, vp]
    lib.mxfp4_quantize.restype = st
    lib.mxfp4_quantize_sr_rht.argtypes = [vp, i64, i64, ctypes.c_uint32, vp, ctypes.c_uint64, vp,
                                          vp, vp, vp]
    lib.mxfp4_quantize_sr_rht.restype = st
    lib.moe_route.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    lib.moe_route.restype = st
    lib.moe_router_topk.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.moe_router_topk.restype = st
    lib.moe_permute.argtypes = [vp, vp, moe_shape, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_permute.restype = st
    lib.moe_expert_mlp.argtypes = [vp, vp, moe_shape, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_expert_mlp.restype = st
    lib.moe_expert_mlp_ex.argtypes = [vp, vp, moe_shape, vp, vp, vp, vp, vp, vp, vp, sz, i32, i32,
                                      vp]
    lib.moe_expert_mlp_ex.restype = st
    lib.moe_expert_mlp_unquantised.argtypes = [vp, vp, moe_shape, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_expert_mlp_unquantised.restype = st
    lib.moe_combine.argtypes = [vp, vp, vp, moe_shape, vp, vp]
    lib.moe_combine.restype = st
    lib.moe_layer_forward.argtypes = [vp, vp, moe_shape, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.moe_layer_forward.restype = st
    lib.moe_layer_forward_static.argtypes = [vp, vp, moe_shape, vp, vp, vp, vp, vp, vp]
    lib.moe_layer_forward_static.restype = st
    lib.moe_layer_static_status.argtypes = [vp, vp]
    lib.moe_layer_static_status.restype = st
    lib.moe_workspace_size.argtypes = [moe_shape, ctypes.c_int]
    lib.moe_workspace_size.restype = sz
    lib.moe_status_string.argtypes = [st]
    lib.moe_status_string.restype = ctypes.c_char_p
    return lib


lib = _load()


def _p(t) -> int | None:
    """Device pointer of a tensor argument (None and raw integer addresses
    pass through).  The C ABI reads dense row-major device arrays, so a
    strided view or a host tensor is refused here rather than misread."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous (dense row-major)")
    return t.data_ptr()


def _s(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoeError(fn, status)


def make_shape(T: int, E: int, k: int, d_model: int, d_ff: int) -> moe_shape:
    return moe_shape(T, E, k, d_model, d_ff)


def moe_status_string(status: int) -> str:
    return lib.moe_status_string(int(status)).decode()


def moe_workspace_size(shape: moe_shape, which: int) -> int:
    return int(lib.moe_workspace_size(shape, which))


def mxfp4_quantize(w_bf16, q_packed, scales, d_status=None, stream=None) -> None:
    """w_bf16 [rows][K] bf16 -> q_packed [rows][K/2] u8, scales [rows][K/32] u8."""
    K = w_bf16.shape[-1]
    rows = w_bf16.numel() // K if K else 0
    _check("mxfp4_quantize", lib.mxfp4_quantize(_p(w_bf16), rows, K, _p(q_packed), _p(scales),
                                                _p(d_status), _s(stream)))


def mxfp4_quantize_sr_rht(w_bf16, flags: int, rht_signs, seed: int, q_packed, scales,
                          d_status=None, stream=None) -> None:
    """w_bf16 [rows][K] bf16 -> q_packed [rows][K/2] u8, scales [rows][K/32] u8,
    with the optional transform (MOE_QUANT_RHT; rht_signs [K/32] int32/uint32)
    and stochastic rounding (MOE_QUANT_SR, Philox keyed by ``seed``)."""
    K = w_bf16.shape[-1]
    rows = w_bf16.numel() // K if K else 0
    _check("mxfp4_quantize_sr_rht",
           lib.mxfp4_quantize_sr_rht(_p(w_bf16), rows, K, int(flags) & 0xFFFFFFFF, _p(rht_signs),
                                     int(seed) & 0xFFFFFFFFFFFFFFFF, _p(q_packed), _p(scales),
                                     _p(d_status), _s(stream)))


def moe_route(logits, k: int, topk_idx, topk_w, stream=None) -> None:
    T, E = logits.shape
    _check("moe_route", lib.moe_route(_p(logits), T, E, k, _p(topk_idx), _p(topk_w), _s(stream)))


def moe_router_topk(x, w_router, k: int, topk_idx, topk_w, logits=None, d_status=None,
                    stream=None) -> None:
    """x [T][D] bf16, w_router [E][D] bf16 -> topk_idx [T][k] i32, topk_w [T][k] f32
    (and logits [T][E] f32 when given)."""
    T, D = x.shape
    E = w_router.shape[0]
    _check("moe_router_topk", lib.moe_router_topk(_p(x), _p(w_router), T, D, E, k, _p(logits),
                                                  _p(topk_idx), _p(topk_w), _p(d_status),
                                                  _s(stream)))


def moe_permute(topk_idx, x, shape: moe_shape, counts, offsets, sorted_slot, slot_pos, x_perm,
                ws=None, stream=None) -> None:
    _check("moe_permute", lib.moe_permute(_p(topk_idx), _p(x), shape, _p(counts), _p(offsets),
                                          _p(sorted_slot), _p(slot_pos), _p(x_perm), _p(ws),
                                          _nbytes(ws), _s(stream)))


def moe_expert_mlp(x_perm, offsets, shape: moe_shape, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm, ws,
                   stream=None) -> None:
    _check("moe_expert_mlp", lib.moe_expert_mlp(_p(x_perm), _p(offsets), shape, _p(wgu_q),
                                                _p(wgu_s), _p(wdn_q), _p(wdn_s), _p(h), _p(y_perm),
                                                _p(ws), _nbytes(ws), _s(stream)))


def moe_expert_mlp_ex(x_perm, offsets, shape: moe_shape, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm, ws,
                      path: int = MOE_MLP_PATH_AUTO, test_timeout_cta: int = -1,
                      stream=None) -> None:
    """moe_expert_mlp on a chosen GEMM path (MOE_MLP_PATH_*); ws sized by
    moe_workspace_size(shape, WS_EXPERT_MLP / _BLOCK_SCALED / _BF16_DECODE).
    test_timeout_cta >= 0 is testing support (see the C header)."""
    _check("moe_expert_mlp_ex",
           lib.moe_expert_mlp_ex(_p(x_perm), _p(offsets), shape, _p(wgu_q), _p(wgu_s), _p(wdn_q),
                                 _p(wdn_s), _p(h), _p(y_perm), _p(ws), _nbytes(ws), int(path),
                                 int(test_timeout_cta), _s(stream)))


def moe_expert_mlp_unquantised(x_perm, offsets, shape: moe_shape, w_gu, w_dn, h, y_perm, ws,
                               stream=None) -> None:
    """The grouped expert MLP on unquantised bf16 weights w_gu [E][2F][D] and
    w_dn [E][D][F]; ws sized by moe_workspace_size(shape, WS_EXPERT_MLP_UNQUANTISED)."""
    _check("moe_expert_mlp_unquantised",
           lib.moe_expert_mlp_unquantised(_p(x_perm), _p(offsets), shape, _p(w_gu), _p(w_dn),
                                          _p(h), _p(y_perm), _p(ws), _nbytes(ws), _s(stream)))


def moe_combine(y_perm, slot_pos, topk_w, shape: moe_shape, out, stream=None) -> None:
    _check("moe_combine", lib.moe_combine(_p(y_perm), _p(slot_pos), _p(topk_w), shape, _p(out),
                                          _s(stream)))


def moe_layer_forward(x, logits, shape: moe_shape, wgu_q, wgu_s, wdn_q, wdn_s, out, ws,
                      stream=None) -> None:
    _check("moe_layer_forward", lib.moe_layer_forward(_p(x), _p(logits), shape, _p(wgu_q),
                                                      _p(wgu_s), _p(wdn_q), _p(wdn_s), _p(out),
                                                      _p(ws), _nbytes(ws), _s(stream)))


STATIC_SCRATCH_BYTES = 16 << 20


def moe_layer_forward_static(x, logits, shape: moe_shape, wgu_q, wgu_s, wdn_q, wdn_s, out,
                             stream=None) -> None:
    """moe_layer_forward with the intermediates in the library's own 16 MiB
    device array (for callers that cannot allocate); see the C header."""
    _check("moe_layer_forward_static",
           lib.moe_layer_forward_static(_p(x), _p(logits), shape, _p(wgu_q), _p(wgu_s), _p(wdn_q),
                                        _p(wdn_s), _p(out), _s(stream)))


def moe_layer_static_status(d_status, stream=None) -> None:
    """Copy the device status word of the last moe_layer_forward_static call
    on this device into d_status (a device int32 tensor), on the stream."""
    _check("moe_layer_static_status", lib.moe_layer_static_status(_p(d_status), _s(stream)))


def alloc_workspace(shape: moe_shape, which: int, device="cuda"):
    """A device byte tensor of moe_workspace_size(shape, which) bytes (at least 256)."""
    import torch

    n = max(256, moe_workspace_size(shape, which))
    return torch.empty(n, dtype=torch.uint8, device=device)


__all__ = ["moe_shape", "make_shape", "MoeError", "mxfp4_quantize", "mxfp4_quantize_sr_rht",
           "MOE_QUANT_RHT", "MOE_QUANT_SR", "moe_route",
           "moe_router_topk", "moe_permute",
           "moe_expert_mlp", "moe_expert_mlp_ex", "moe_expert_mlp_unquantised", "moe_combine", "moe_layer_forward",
           "moe_layer_forward_static", "moe_layer_static_status",
           "moe_workspace_size",
           "moe_status_string", "alloc_workspace", "lib", "LIB_PATH"]
