"""CPU oracle for the MXFP4 Mixture-of-Experts layer -- TEST INFRASTRUCTURE.

A plain, slow, double-precision restatement (``oracle.c``) of what the layer
computes, used only by ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py``.  The CUDA library never imports, links or
calls it, and the two share no code.

Every function cites the page passage it follows (see ``oracle.c``).  All of
them are pinned by ``tests/test_oracle_pins.py`` to facts fixed by the pages
and by mathematics (exhaustive decode table, brute-force encoding,
hand-derived blocks, brute-force top-k, permutation invariants, a dense
per-token restatement, and the single-expert case against fp64
``torch.matmul``), and the training-style quantiser by
``tests/test_oracle_sr_rht_pins.py`` (Philox known answers,
``scipy.linalg.hadamard``, exact counts over all uniforms); no function is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, strict IEEE: no fast-math,
    no FMA contraction, so every fp64 product and sum is rounded once)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-o", _LIB_PATH, _SRC, "-lm", "-lpthread"])
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        path = os.environ.get("ORACLE_LIB_OVERRIDE") or build()
        lib = ctypes.CDLL(path)
        vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_value.restype = dbl
        lib.oracle_bf16_round.argtypes = [dbl]
        lib.oracle_bf16_round.restype = ctypes.c_uint16
        lib.oracle_mxfp4_value.argtypes = [ctypes.c_uint8, ctypes.c_uint8]
        lib.oracle_mxfp4_value.restype = dbl
        lib.oracle_mxfp4_quantize.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_mxfp4_quantize.restype = i64
        lib.oracle_mxfp4_quantize_mt.argtypes = [vp, i64, i64, vp, vp, i32]
        lib.oracle_mxfp4_quantize_mt.restype = i64
        lib.oracle_mxfp4_decode.argtypes = [vp, vp, i64, i64, vp]
        u32, u64 = ctypes.c_uint32, ctypes.c_uint64
        lib.oracle_philox4x32_10.argtypes = [vp, vp, vp]
        lib.oracle_sr_uniform16.argtypes = [u64, u64]
        lib.oracle_sr_uniform16.restype = u32
        lib.oracle_rht32.argtypes = [vp, u32, vp]
        lib.oracle_sr_code.argtypes = [dbl, u32]
        lib.oracle_sr_code.restype = ctypes.c_uint8
        lib.oracle_mxfp4_quantize_sr_rht.argtypes = [vp, i64, i64, u32, vp, u64, vp, vp, i32]
        lib.oracle_mxfp4_quantize_sr_rht.restype = i64
        lib.oracle_route.argtypes = [vp, i64, i32, i32, vp, vp]
        lib.oracle_router_logits.argtypes = [vp, vp, i64, i32, i32, vp]
        lib.oracle_permute.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
        lib.oracle_gather.argtypes = [vp, vp, i64, i32, i32, vp]
        lib.oracle_expert_mlp.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, i32]
        lib.oracle_expert_mlp.restype = i32
        lib.oracle_expert_mlp_bf16.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, i32]
        lib.oracle_expert_mlp_bf16.restype = i32
        lib.oracle_combine.argtypes = [vp, vp, vp, i64, i32, i32, vp]
        lib.oracle_layer_forward.argtypes = [vp, vp, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32]
        lib.oracle_layer_forward.restype = i32
        lib.oracle_layer_tokens.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, i64, vp,
                                            vp, i32]
        lib.oracle_layer_tokens.restype = i32
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


# ------------------------------------------------------------------ scalars

def bf16_value(bits: int) -> float:
    return float(_L().oracle_bf16_value(int(bits)))


def bf16_round(x: float) -> int:
    return int(_L().oracle_bf16_round(float(x)))


def mxfp4_value(code: int, scale_byte: int) -> float:
    return float(_L().oracle_mxfp4_value(int(code), int(scale_byte)))


# ------------------------------------------------------------------- MXFP4

def mxfp4_quantize(w_bf16: np.ndarray) -> tuple[np.ndarray, np.ndarray, int]:
    """bf16 bits [..., K] -> (codes [..., K/2] u8, scales [..., K/32] u8, #non-finite blocks)."""
    w = _c(w_bf16, np.uint16)
    K = w.shape[-1]
    rows = w.size // K if K else 0
    q = np.empty(w.shape[:-1] + (K // 2,), dtype=np.uint8)
    s = np.empty(w.shape[:-1] + (K // 32,), dtype=np.uint8)
    bad = _L().oracle_mxfp4_quantize_mt(_p(w), rows, K, _p(q), _p(s), _threads())
    return q, s, int(bad)


# flags of the training-style quantiser ("MXFP4-based MoE technical review",
# sections 2 and 4): a random-sign Hadamard transform of each 32-block along K,
# and stochastic rounding
QUANT_RHT = 1
QUANT_SR = 2


def philox4x32_10(ctr, key) -> tuple[int, int, int, int]:
    """Philox4x32-10 (Salmon et al., SC 2011) of a 4-word counter and 2-word key."""
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    _L().oracle_philox4x32_10(_p(c), _p(k), _p(out))
    return tuple(int(v) for v in out)


def sr_uniform16(seed: int, n: int) -> int:
    """16-bit uniform that element n of a call keyed by ``seed`` draws."""
    return int(_L().oracle_sr_uniform16(int(seed), int(n)))


def rht32(x: np.ndarray, sign_word: int) -> np.ndarray:
    """y = H (s . x) of one 32-element block (unnormalised Sylvester H)."""
    xv = _c(x, np.float64)
    assert xv.shape == (32,)
    y = np.empty(32, dtype=np.float64)
    _L().oracle_rht32(_p(xv), int(sign_word) & 0xFFFFFFFF, _p(y))
    return y


def sr_code(v: float, u: int) -> int:
    """Stochastic rounding of v >= 0 onto the E2M1 magnitudes, 16-bit uniform u."""
    return int(_L().oracle_sr_code(float(v), int(u)))


def mxfp4_quantize_sr_rht(w_bf16: np.ndarray, flags: int, signs: np.ndarray | None,
                          seed: int) -> tuple[np.ndarray, np.ndarray, int]:
    """bf16 bits [..., K] -> (codes, scales, #non-finite blocks) with the
    optional transform (``signs`` [K/32] uint32) and stochastic rounding."""
    w = _c(w_bf16, np.uint16)
    K = w.shape[-1]
    rows = w.size // K if K else 0
    q = np.empty(w.shape[:-1] + (K // 2,), dtype=np.uint8)
    s = np.empty(w.shape[:-1] + (K // 32,), dtype=np.uint8)
    if signs is None:
        sg = np.zeros(max(1, K // 32), dtype=np.uint32)
    else:
        sg = _c(signs, np.uint32)
        assert sg.shape == (K // 32,)
    bad = _L().oracle_mxfp4_quantize_sr_rht(_p(w), rows, K, int(flags), _p(sg), int(seed), _p(q),
                                            _p(s), _threads())
    return q, s, int(bad)


def mxfp4_decode(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = _c(q, np.uint8)
    s = _c(s, np.uint8)
    K = q.shape[-1] * 2
    rows = q.size // (K // 2) if K else 0
    out = np.empty(q.shape[:-1] + (K,), dtype=np.float64)
    _L().oracle_mxfp4_decode(_p(q), _p(s), rows, K, _p(out))
    return out


# ---------------------------------------------------------------- routing

def route(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    lg = _c(logits, np.float32)
    T, E = lg.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _L().oracle_route(_p(lg), T, E, k, _p(idx), _p(w))
    return idx, w


def router_logits(x_bf16: np.ndarray, w_bf16: np.ndarray) -> np.ndarray:
    """x [T][D] and w [E][D] as bf16 bit patterns (uint16) -> fp64 [T][E]
    scores x . w^T (the router before routing)."""
    x = _c(x_bf16, np.uint16)
    w = _c(w_bf16, np.uint16)
    T, D = x.shape
    E = w.shape[0]
    assert w.shape[1] == D
    out = np.empty((T, E), dtype=np.float64)
    _L().oracle_router_logits(_p(x), _p(w), T, D, E, _p(out))
    return out


def permute(idx: np.ndarray, E: int):
    ix = _c(idx, np.int32)
    T, k = ix.shape
    S = T * k
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    sorted_slot = np.empty(S, dtype=np.int32)
    slot_pos = np.empty(S, dtype=np.int32)
    _L().oracle_permute(_p(ix), T, E, k, _p(counts), _p(offsets), _p(sorted_slot), _p(slot_pos))
    return counts, offsets, sorted_slot, slot_pos


def gather(x: np.ndarray, sorted_slot: np.ndarray, k: int) -> np.ndarray:
    xx = _c(x, np.uint16)
    ss = _c(sorted_slot, np.int32)
    D = xx.shape[1]
    out = np.empty((ss.size, D), dtype=np.uint16)
    _L().oracle_gather(_p(xx), _p(ss), ss.size, k, D, _p(out))
    return out


def expert_mlp(x_perm, offsets, wgu_q, wgu_s, wdn_q, wdn_s, want_h: bool = True):
    """Grouped SwiGLU MLP over permuted rows -> (h [S][F] or None, y [S][D])."""
    xp = _c(x_perm, np.uint16)
    off = _c(offsets, np.int32)
    E = off.size - 1
    S, D = xp.shape
    F = wdn_q.shape[-1] * 2
    gq, gs, dq, ds = (_c(a, np.uint8) for a in (wgu_q, wgu_s, wdn_q, wdn_s))
    h = np.empty((S, F), dtype=np.uint16) if want_h else None
    y = np.empty((S, D), dtype=np.uint16)
    rc = _L().oracle_expert_mlp(_p(xp), _p(off), E, D, F, _p(gq), _p(gs), _p(dq), _p(ds),
                                _p(h) if want_h else None, _p(y), _threads())
    if rc != 0:
        raise MemoryError("oracle_expert_mlp: allocation failed")
    return h, y


def expert_mlp_bf16(x_perm, offsets, wgu_bf16, wdn_bf16, want_h: bool = True):
    """The grouped expert MLP with unquantised bf16 weights (bit patterns):
    wgu [E][2F][D], wdn [E][D][F] -> (h [S][F] or None, y [S][D])."""
    xp = _c(x_perm, np.uint16)
    off = _c(offsets, np.int32)
    E = off.size - 1
    S, D = xp.shape
    F = wdn_bf16.shape[-1]
    gu = _c(wgu_bf16, np.uint16)
    dn = _c(wdn_bf16, np.uint16)
    assert gu.shape == (E, 2 * F, D) and dn.shape == (E, D, F)
    h = np.empty((S, F), dtype=np.uint16) if want_h else None
    y = np.empty((S, D), dtype=np.uint16)
    rc = _L().oracle_expert_mlp_bf16(_p(xp), _p(off), E, D, F, _p(gu), _p(dn),
                                     _p(h) if want_h else None, _p(y), _threads())
    if rc != 0:
        raise MemoryError("oracle_expert_mlp_bf16: allocation failed")
    return h, y


def combine(y_perm, slot_pos, w, k: int) -> np.ndarray:
    yp = _c(y_perm, np.uint16)
    sp = _c(slot_pos, np.int32)
    ww = _c(w, np.float64)
    T = ww.shape[0]
    D = yp.shape[1]
    out = np.empty((T, D), dtype=np.uint16)
    _L().oracle_combine(_p(yp), _p(sp), _p(ww), T, k, D, _p(out))
    return out


def layer_forward(x, logits, k, wgu_q, wgu_s, wdn_q, wdn_s) -> np.ndarray:
    xx = _c(x, np.uint16)
    lg = _c(logits, np.float32)
    T, D = xx.shape
    E = lg.shape[1]
    F = wdn_q.shape[-1] * 2
    gq, gs, dq, ds = (_c(a, np.uint8) for a in (wgu_q, wgu_s, wdn_q, wdn_s))
    out = np.empty((T, D), dtype=np.uint16)
    rc = _L().oracle_layer_forward(_p(xx), _p(lg), T, E, k, D, F, _p(gq), _p(gs), _p(dq), _p(ds),
                                   _p(out), _threads())
    if rc != 0:
        raise MemoryError("oracle_layer_forward: allocation failed")
    return out


def layer_tokens(x, logits, k, wgu_q, wgu_s, wdn_q, wdn_s, tokens, want_y: bool = False):
    """Output rows of the selected tokens, computed per token (no permutation);
    with want_y also the bf16 expert outputs [len(tokens)][k][D]."""
    xx = _c(x, np.uint16)
    lg = _c(logits, np.float32)
    T, D = xx.shape
    E = lg.shape[1]
    F = wdn_q.shape[-1] * 2
    tk = _c(np.asarray(tokens), np.int64)
    gq, gs, dq, ds = (_c(a, np.uint8) for a in (wgu_q, wgu_s, wdn_q, wdn_s))
    out = np.empty((tk.size, D), dtype=np.uint16)
    y = np.empty((tk.size, k, D), dtype=np.uint16) if want_y else None
    rc = _L().oracle_layer_tokens(_p(xx), _p(lg), E, k, D, F, _p(gq), _p(gs), _p(dq), _p(ds),
                                  _p(tk), tk.size, _p(out), _p(y) if want_y else None, _threads())
    if rc != 0:
        raise MemoryError("oracle_layer_tokens: allocation failed")
    return (out, y) if want_y else out


def quantize_experts(w_bf16: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    q, s, bad = mxfp4_quantize(w_bf16)
    if bad:
        raise ValueError(f"{bad} non-finite blocks in expert weights")
    return q, s
