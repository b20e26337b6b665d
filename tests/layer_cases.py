"""Shared set-up for the GPU parity tests: seeded inputs on the device, the
library's quantised weights, and the oracle's view of the same inputs."""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn

# layer-output tolerance: relative Frobenius error and max-abs relative to rms(ref)
REL_FRO = 5e-3
MAX_ABS_RMS = 1e-2
ROUTE_W_ATOL = 1e-6


def to_dev_u16(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(bits: np.ndarray) -> np.ndarray:
    return syn.bf16_bits_to_f32(bits).astype(np.float64)


def layer_error(got_bits: np.ndarray, ref_bits: np.ndarray) -> tuple[float, float, float]:
    g, r = f64(got_bits), f64(ref_bits)
    rms = float(np.sqrt(np.mean(r * r)))
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    mx = float(np.max(np.abs(g - r))) if g.size else 0.0
    return rel, mx, rms


def bf16_ulp(bits: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at each element: 2^(exponent - 7) (2^-133 for
    zero and subnormals)."""
    e = ((bits.astype(np.int64) >> 7) & 0xFF)
    return np.ldexp(1.0, (np.maximum(e, 1) - 127 - 7).astype(np.int64))


def assert_layer_close(got_bits, ref_bits, what="", y_ulp=None):
    """Relative Frobenius error <= 5e-3, and per element
    |got - ref| <= 1e-2 * rms(ref) + ulp(ref) + y_ulp.

    The two ulp terms are the reading of the max-abs bar for a layer whose
    intermediates and output are bf16: each bf16 rounding point may land on
    the other neighbour when the library (fp32 accumulation) and the oracle
    (fp64) see a sum within fp32 error of a rounding boundary.  ulp(ref)
    covers the final rounding of the output; y_ulp (the largest bf16 ulp of
    the k expert outputs y_j mixed into the element, whose weights sum to 1)
    covers a flip of one y_j.  Outputs above ~2.6 rms already have one ulp
    above 1e-2 * rms, so without these terms the bar would reject any
    fp32-accumulating implementation.  Differences beyond one ulp of the
    output must also stay rare (<= 1% of elements)."""
    got_bits = np.asarray(got_bits, dtype=np.uint16)
    ref_bits = np.asarray(ref_bits, dtype=np.uint16)
    rel, mx, rms = layer_error(got_bits, ref_bits)
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    g, r = f64(got_bits), f64(ref_bits)
    ulp = bf16_ulp(ref_bits)
    extra = 0.0 if y_ulp is None else np.asarray(y_ulp, dtype=np.float64)
    excess = np.abs(g - r) - (MAX_ABS_RMS * rms + ulp + extra)
    worst = int(np.argmax(excess)) if excess.size else 0
    assert excess.size == 0 or excess.flat[worst] <= 0, (
        f"{what}: |diff| {abs(g.flat[worst] - r.flat[worst]):.3e} at {worst} exceeds "
        f"{MAX_ABS_RMS} * rms {rms:.3e} + ulp {ulp.flat[worst]:.3e} (max abs {mx:.3e})")
    beyond_ulp = float(np.mean(np.abs(g - r) > ulp)) if g.size else 0.0
    assert beyond_ulp <= 0.01, f"{what}: {beyond_ulp:.2%} of elements differ by more than one ulp"
    return rel, mx, rms


@dataclass
class DeviceLayer:
    wl: syn.Workload
    x: torch.Tensor
    logits: torch.Tensor
    wgu_q: torch.Tensor
    wgu_s: torch.Tensor
    wdn_q: torch.Tensor
    wdn_s: torch.Tensor
    shape: moe.moe_shape
    host: dict = field(default_factory=dict)


def device_layer(wl: syn.Workload, dev, keep_host_weights: bool = False) -> DeviceLayer:
    """Inputs on the device; weights generated expert by expert and quantised
    by the library's mxfp4_quantize."""
    D, F, E = wl.d_model, wl.d_ff, wl.E
    x_np = syn.activations(wl)
    lg_np = syn.logits(wl)
    wgu_q = torch.empty((E, 2 * F, D // 2), dtype=torch.uint8, device=dev)
    wgu_s = torch.empty((E, 2 * F, D // 32), dtype=torch.uint8, device=dev)
    wdn_q = torch.empty((E, D, F // 2), dtype=torch.uint8, device=dev)
    wdn_s = torch.empty((E, D, F // 32), dtype=torch.uint8, device=dev)
    host = {"x": x_np, "logits": lg_np}
    chunk = max(1, min(E, (1 << 28) // (2 * F * D)))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for e0 in range(0, E, chunk):
        ex = list(range(e0, min(E, e0 + chunk)))
        gu = syn.w_gate_up(wl, ex)
        dn = syn.w_down(wl, ex)
        if keep_host_weights:
            host.setdefault("w_gu", []).append(gu)
            host.setdefault("w_dn", []).append(dn)
        gu_d = to_dev_u16(gu, dev)
        dn_d = to_dev_u16(dn, dev)
        moe.mxfp4_quantize(gu_d, wgu_q[e0:e0 + len(ex)], wgu_s[e0:e0 + len(ex)], status)
        moe.mxfp4_quantize(dn_d, wdn_q[e0:e0 + len(ex)], wdn_s[e0:e0 + len(ex)], status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.MOE_OK
    if keep_host_weights:
        host["w_gu"] = np.concatenate(host["w_gu"])
        host["w_dn"] = np.concatenate(host["w_dn"])
    return DeviceLayer(wl, to_dev_u16(x_np, dev), torch.from_numpy(lg_np).to(dev), wgu_q, wgu_s,
                       wdn_q, wdn_s, moe.make_shape(wl.T, E, wl.k, D, F), host)


def oracle_weights_for(wl: syn.Workload, experts) -> tuple[np.ndarray, ...]:
    """Oracle-quantised weights [E][...] with only `experts` filled (others 0)."""
    D, F, E = wl.d_model, wl.d_ff, wl.E
    gq = np.zeros((E, 2 * F, D // 2), np.uint8)
    gs = np.zeros((E, 2 * F, D // 32), np.uint8)
    dq = np.zeros((E, D, F // 2), np.uint8)
    ds = np.zeros((E, D, F // 32), np.uint8)
    for e in sorted(set(int(v) for v in experts)):
        q, s = oracle.quantize_experts(syn.w_gate_up(wl, [e]))
        gq[e], gs[e] = q[0], s[0]
        q, s = oracle.quantize_experts(syn.w_down(wl, [e]))
        dq[e], ds[e] = q[0], s[0]
    return gq, gs, dq, ds


def oracle_layer_with_y(x, lg, k, gq, gs, dq, ds):
    """The oracle's layer in its step order, returning the output and, per
    output element, the largest bf16 ulp among the k expert outputs mixed
    into it."""
    E = lg.shape[1]
    idx, w = oracle.route(lg, k)
    _, offsets, ss, sp = oracle.permute(idx, E)
    xp = oracle.gather(x, ss, k)
    _, y = oracle.expert_mlp(xp, offsets, gq, gs, dq, ds, want_h=False)
    out = oracle.combine(y, sp, w, k)
    T = x.shape[0]
    yt = y[sp].reshape(T, k, -1)
    return out, bf16_ulp(yt).max(axis=1)


def h_flip_bound(h_bits, offsets, w_dn) -> np.ndarray:
    """Per element of y [S][D]: how far one bf16 h value rounded to its other
    neighbour moves it, max_n |w_dn[e][d][n]| * ulp(h[r][n]) with e the
    expert of row r (bounded by max_n |w| times max_n ulp(h)).  h is a
    rounding point of the method: where the library (fp32 accumulation) and
    the oracle (fp64) see g or u within fp32 error of a bf16 rounding
    boundary, their h differ by one ulp, and y = h . w_dn^T carries it.
    w_dn: the down weights as values, [E][D][F] (decoded MXFP4 or bf16)."""
    S, F = h_bits.shape
    hul = bf16_ulp(h_bits).max(axis=1) if S else np.zeros(0)
    out = np.zeros((S, w_dn.shape[1]))
    for e in range(len(offsets) - 1):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            wmax = np.abs(w_dn[e]).max(axis=1)
            out[r0:r1] = hul[r0:r1, None] * wmax[None, :]
    return out


def decoded_down(dq, ds) -> np.ndarray:
    """The oracle's decoded down weights [E][D][F] (fp64)."""
    return oracle.mxfp4_decode(dq, ds)


def oracle_tokens_with_y(x, lg, k, gq, gs, dq, ds, tokens):
    out, y = oracle.layer_tokens(x, lg, k, gq, gs, dq, ds, tokens, want_y=True)
    return out, bf16_ulp(y).max(axis=1)


def run_layer(L: DeviceLayer) -> torch.Tensor:
    dev = L.x.device
    out = torch.empty((L.wl.T, L.wl.d_model), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(L.shape, moe.WS_LAYER, dev)
    moe.moe_layer_forward(L.x, L.logits, L.shape, L.wgu_q, L.wgu_s, L.wdn_q, L.wdn_s, out, ws)
    torch.cuda.synchronize()
    status = int(ws[:4].view(torch.int32).item())
    assert status == moe.MOE_OK, moe.moe_status_string(status)
    return out
