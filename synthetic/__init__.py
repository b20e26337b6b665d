"""Seeded synthetic inputs for the MXFP4 MoE layer.

This package holds none of the layer's arithmetic.  It draws the inputs that
both the CUDA library (through its tests and the benchmark) and the CPU
oracle consume, so that the two sides see the same bytes:

* activations ``x``: bf16 N(0, 1)                       (stream 1)
* router logits: fp32 N(0, 1) [+ per-expert bias]       (stream 2)
* gate/up weights ``w_gu`` [E][2F][D]: bf16 N(0, 0.02)  (stream 3)
* down weights ``w_dn`` [E][D][F]: bf16 N(0, 0.02)      (stream 4)
* outlier masks for the skewed workload                 (streams 5 and 6)

Element i of a tensor is draw i of its stream (counter-based splitmix64, see
``gen.c``), so one expert's weights can be produced without the others.

The five workloads are the layer shapes of a GPT-OSS-style model: a tiny
layer, the 20B-shaped layer (32 experts) at decode and prefill batch sizes,
and the 120B-shaped layer (128 experts) at a decode batch and a skewed
prefill batch whose router logits carry a Zipf(1.1) per-expert bias and
whose weights carry 1% outliers (x20).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsyngen.so")
_SRC = os.path.join(_HERE, "gen.c")

SID_X, SID_LOGITS, SID_WGU, SID_WDN, SID_MASK_GU, SID_MASK_DN = 1, 2, 3, 4, 5, 6


def build(force: bool = False) -> str:
    """Compile gen.c into libsyngen.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _LIB_PATH, _SRC,
                               "-lm", "-lpthread"])
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, dbl, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_int
        vp = ctypes.c_void_p
        lib.syn_normal_bf16.argtypes = [u64, u64, u64, i64, dbl, vp, i32]
        lib.syn_normal_outliers_bf16.argtypes = [u64, u64, u64, u64, i64, dbl, dbl, dbl, vp, i32]
        lib.syn_normal_f64.argtypes = [u64, u64, u64, i64, vp]
        lib.syn_uniform_f64.argtypes = [u64, u64, u64, i64, vp, i32]
        lib.syn_logits_f32.argtypes = [u64, u64, i64, i64, vp, vp]
        lib.syn_bf16_from_double.argtypes = [dbl]
        lib.syn_bf16_from_double.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


@dataclass(frozen=True)
class Workload:
    """One synthetic MoE-layer workload."""

    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    k: int = 4
    seed: int = 0
    zipf_s: float | None = None  # per-expert logit bias 2*ln(p_e), p_e ~ (e+1)^-s
    outlier_p: float = 0.0  # fraction of weight entries multiplied by outlier_factor
    outlier_factor: float = 20.0
    w_sigma: float = 0.02

    @property
    def S(self) -> int:
        return self.T * self.k


WORKLOADS = {
    "tiny": Workload("tiny", T=16, d_model=256, d_ff=256, E=8),
    "20b_decode": Workload("20b_decode", T=64, d_model=2880, d_ff=2880, E=32),
    "20b_prefill": Workload("20b_prefill", T=8192, d_model=2880, d_ff=2880, E=32),
    "120b_decode": Workload("120b_decode", T=128, d_model=2880, d_ff=2880, E=128),
    "120b_skewed_prefill": Workload("120b_skewed_prefill", T=16384, d_model=2880, d_ff=2880,
                                    E=128, zipf_s=1.1, outlier_p=0.01),
}


def expert_bias(wl: Workload) -> np.ndarray | None:
    """Per-expert router-logit bias b_e = 2 ln p_e with p_e = (e+1)^-s / sum."""
    if wl.zipf_s is None:
        return None
    w = np.array([(e + 1.0) ** (-wl.zipf_s) for e in range(wl.E)], dtype=np.float64)
    p = w / w.sum()
    return 2.0 * np.log(p)


def activations(wl: Workload) -> np.ndarray:
    """x [T][D] as bf16 bit patterns (uint16)."""
    out = np.empty((wl.T, wl.d_model), dtype=np.uint16)
    _L().syn_normal_bf16(wl.seed, SID_X, 0, out.size, 1.0, _ptr(out), _threads())
    return out


def logits(wl: Workload) -> np.ndarray:
    """router logits [T][E] fp32."""
    out = np.empty((wl.T, wl.E), dtype=np.float32)
    b = expert_bias(wl)
    bp = None if b is None else _ptr(np.ascontiguousarray(b))
    _L().syn_logits_f32(wl.seed, SID_LOGITS, wl.T, wl.E, bp, _ptr(out))
    return out


def _weights(wl: Workload, sid: int, mask_sid: int, rows: int, K: int,
             experts: list[int] | None) -> np.ndarray:
    experts = list(range(wl.E)) if experts is None else list(experts)
    out = np.empty((len(experts), rows, K), dtype=np.uint16)
    per = rows * K
    for i, e in enumerate(experts):
        dst = out[i]
        if wl.outlier_p > 0:
            _L().syn_normal_outliers_bf16(wl.seed, sid, mask_sid, e * per, per, wl.w_sigma,
                                          wl.outlier_p, wl.outlier_factor, _ptr(dst), _threads())
        else:
            _L().syn_normal_bf16(wl.seed, sid, e * per, per, wl.w_sigma, _ptr(dst), _threads())
    return out


def w_gate_up(wl: Workload, experts: list[int] | None = None) -> np.ndarray:
    """bf16 gate/up weights [len(experts)][2F][D] (rows [0,F) gate, [F,2F) up)."""
    return _weights(wl, SID_WGU, SID_MASK_GU, 2 * wl.d_ff, wl.d_model, experts)


def w_down(wl: Workload, experts: list[int] | None = None) -> np.ndarray:
    """bf16 down weights [len(experts)][D][F]."""
    return _weights(wl, SID_WDN, SID_MASK_DN, wl.d_model, wl.d_ff, experts)


def normal_bf16(seed: int, sid: int, shape, sigma: float = 1.0, offset: int = 0) -> np.ndarray:
    """Generic bf16 normal tensor from an arbitrary stream (for edge-case tests)."""
    out = np.empty(shape, dtype=np.uint16)
    _L().syn_normal_bf16(seed, sid, offset, out.size, sigma, _ptr(out), _threads())
    return out


def logits_custom(seed: int, sid: int, T: int, E: int) -> np.ndarray:
    out = np.empty((T, E), dtype=np.float32)
    _L().syn_logits_f32(seed, sid, T, E, None, _ptr(out))
    return out


def normal_f64(seed: int, sid: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().syn_normal_f64(seed, sid, offset, n, _ptr(out))
    return out


def uniform_f64(seed: int, sid: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _L().syn_uniform_f64(seed, sid, offset, n, _ptr(out), _threads())
    return out


def bf16_from_double(x: float) -> int:
    return int(_L().syn_bf16_from_double(float(x)))


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """View bf16 bit patterns (uint16) as fp32 values (exact)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def expected_tokens_per_expert(wl: Workload) -> float:
    return wl.S / wl.E


__all__ = ["Workload", "WORKLOADS", "activations", "logits", "w_gate_up", "w_down",
           "expert_bias", "normal_bf16", "logits_custom", "normal_f64", "uniform_f64",
           "bf16_from_double", "bf16_bits_to_f32", "build"]
