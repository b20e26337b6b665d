"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Bit-exact: quantised bytes, top-k indices, counts, offsets, permutation,
gathered rows.  Within tolerance: routing weights (abs 1e-6, fp32 vs fp64)
and layer outputs (relative Frobenius error <= 5e-3 and max abs error
<= 1e-2 * rms of the oracle's output).
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import (ROUTE_W_ATOL, assert_layer_close, bf16_np, device_layer,
                         oracle_layer_with_y, oracle_tokens_with_y, oracle_weights_for, run_layer,
                         to_dev_u16)

pytestmark = pytest.mark.gpu

FULL = ["tiny", "20b_decode", "20b_prefill", "120b_decode", "120b_skewed_prefill"]


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


# ---------------------------------------------------------------- quantiser


def _gpu_quantize(w_np, dev):
    w = to_dev_u16(w_np, dev)
    R, K = w_np.reshape(-1, w_np.shape[-1]).shape
    q = torch.empty(w_np.shape[:-1] + (K // 2,), dtype=torch.uint8, device=dev)
    s = torch.empty(w_np.shape[:-1] + (K // 32,), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    moe.mxfp4_quantize(w, q, s, st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), int(st.item())


def test_quantize_every_bf16_value(dev):
    # every finite bf16 pattern, in blocks whose maximum fixes several scales
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (allbits & 0x7F80) != 0x7F80
    vals = allbits[finite]
    n = vals.size
    blocks = np.zeros(((n + 31) // 32, 32), dtype=np.uint16)
    blocks.reshape(-1)[:n] = vals
    q, s, st = _gpu_quantize(blocks, dev)
    oq, os_, bad = oracle.mxfp4_quantize(blocks)
    assert bad == 0 and st == moe.MOE_OK
    assert np.array_equal(q, oq) and np.array_equal(s, os_)


@pytest.mark.parametrize("rows,K,sigma", [(1, 32, 1.0), (3, 96, 1e-30), (7, 2880, 0.02),
                                          (129, 256, 3e4), (5, 4096, 1e-38)])
def test_quantize_random_shapes(dev, rows, K, sigma):
    w = syn.normal_bf16(9, 200 + K, (rows, K), sigma=sigma)
    q, s, st = _gpu_quantize(w, dev)
    oq, os_, _ = oracle.mxfp4_quantize(w)
    assert st == moe.MOE_OK
    assert np.array_equal(q, oq) and np.array_equal(s, os_)


def test_quantize_flags_nonfinite(dev):
    w = syn.normal_bf16(1, 300, (4, 64))
    w[2, 37] = 0x7FC0
    _, _, st = _gpu_quantize(w, dev)
    assert st == moe.MOE_ERR_NONFINITE


@pytest.mark.parametrize("name", ["20b_decode", "120b_skewed_prefill"])
def test_quantize_workload_experts(dev, name):
    wl = syn.WORKLOADS[name]
    for e in (0, wl.E - 1):
        for w in (syn.w_gate_up(wl, [e]), syn.w_down(wl, [e])):
            q, s, st = _gpu_quantize(w, dev)
            oq, os_, _ = oracle.mxfp4_quantize(w)
            assert st == moe.MOE_OK
            assert np.array_equal(q, oq) and np.array_equal(s, os_)


# ------------------------------------------------------------------ routing


def _gpu_route(lg_np, k, dev):
    lg = torch.from_numpy(lg_np).to(dev)
    T = lg_np.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    moe.moe_route(lg, k, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name", FULL)
def test_route_workloads(dev, name):
    wl = syn.WORKLOADS[name]
    lg = syn.logits(wl)
    idx, w = _gpu_route(lg, wl.k, dev)
    oi, ow = oracle.route(lg, wl.k)
    assert np.array_equal(idx, oi)
    assert np.max(np.abs(w - ow)) <= ROUTE_W_ATOL


@pytest.mark.parametrize("T,E,k", [(1, 4, 4), (3, 7, 2), (33, 256, 8), (100, 64, 1), (5, 33, 4)])
def test_route_odd_shapes_and_ties(dev, T, E, k):
    lg = syn.logits_custom(4, 500 + E, T, E)
    lg[0, :] = 0.0
    lg[0, ::2] = -0.0  # +0 and -0 tie: lowest index wins
    if T > 1:
        lg[1, :] = np.float32(1.25)
    idx, w = _gpu_route(lg, k, dev)
    oi, ow = oracle.route(lg, k)
    assert np.array_equal(idx, oi)
    assert np.max(np.abs(w - ow)) <= ROUTE_W_ATOL


# ------------------------------------------------------------------ permute


def _gpu_permute(idx_np, x_np, E, D, dev):
    T, k = idx_np.shape
    S = T * k
    sh = moe.make_shape(T, E, k, D, 128)
    idx = torch.from_numpy(idx_np).to(dev)
    x = to_dev_u16(x_np, dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ss = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    sp = torch.empty(max(S, 1), dtype=torch.int32, device=dev)
    xp = torch.empty((max(S, 1), D), dtype=torch.bfloat16, device=dev)
    moe.moe_permute(idx, x, sh, counts, offsets, ss, sp, xp)
    torch.cuda.synchronize()
    return (counts.cpu().numpy(), offsets.cpu().numpy(), ss.cpu().numpy()[:S], sp.cpu().numpy()[:S],
            bf16_np(xp)[:S])


@pytest.mark.parametrize("name", FULL)
def test_permute_workloads(dev, name):
    wl = syn.WORKLOADS[name]
    oi, _ = oracle.route(syn.logits(wl), wl.k)
    x = syn.activations(wl)
    got = _gpu_permute(oi, x, wl.E, wl.d_model, dev)
    want = oracle.permute(oi, wl.E)
    for g, w_ in zip(got[:4], want):
        assert np.array_equal(g, w_)
    assert np.array_equal(got[4], oracle.gather(x, want[2], wl.k))


@pytest.mark.parametrize("T,E,k,mode", [(1, 4, 4, "rand"), (3, 8, 2, "rand"), (50, 16, 4, "one_hot"),
                                         (257, 64, 8, "rand"), (4096, 128, 4, "skew")])
def test_permute_edge_cases(dev, T, E, k, mode):
    rng = np.random.default_rng(T + E)
    if mode == "one_hot":  # every token's first choice is expert 5; 15 experts empty-ish
        idx = np.stack([[5] + list(rng.choice([e for e in range(E) if e != 5], k - 1, replace=False))
                        for _ in range(T)]).astype(np.int32)
    elif mode == "skew":
        p = 1.0 / (np.arange(E) + 1.0) ** 2
        p /= p.sum()
        idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    else:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    x = syn.normal_bf16(2, 600, (T, 128))
    got = _gpu_permute(idx, x, E, 128, dev)
    want = oracle.permute(idx, E)
    for g, w_ in zip(got[:4], want):
        assert np.array_equal(g, w_)
    assert np.array_equal(got[4], oracle.gather(x, want[2], k))


# ------------------------------------------------- expert MLP and combine


def test_expert_mlp_and_combine_tiny(dev):
    wl = syn.WORKLOADS["tiny"]
    L = device_layer(wl, dev)
    lg = syn.logits(wl)
    oi, ow = oracle.route(lg, wl.k)
    counts, offsets, ss, sp = oracle.permute(oi, wl.E)
    x = syn.activations(wl)
    xp = oracle.gather(x, ss, wl.k)
    gq, gs, dq, ds = oracle_weights_for(wl, range(wl.E))
    oh, oy = oracle.expert_mlp(xp, offsets, gq, gs, dq, ds)
    S = wl.S
    h = torch.empty((S, wl.d_ff), dtype=torch.bfloat16, device=dev)
    y = torch.empty((S, wl.d_model), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(L.shape, moe.WS_EXPERT_MLP, dev)
    ws[:4].fill_(0xFF)  # the call clears its status word
    moe.moe_expert_mlp(to_dev_u16(xp, dev), torch.from_numpy(offsets).to(dev), L.shape, L.wgu_q,
                       L.wgu_s, L.wdn_q, L.wdn_s, h, y, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
    assert_layer_close(bf16_np(h), oh, "h")
    # y mixes bf16 h values: a flip of one h moves y by far less than an ulp
    assert_layer_close(bf16_np(y), oy, "y")
    # combine of the oracle's y with fp32 routing weights
    out = torch.empty((wl.T, wl.d_model), dtype=torch.bfloat16, device=dev)
    moe.moe_combine(to_dev_u16(oy, dev), torch.from_numpy(sp).to(dev),
                    torch.from_numpy(ow.astype(np.float32)).to(dev), L.shape, out)
    torch.cuda.synchronize()
    want = oracle.combine(oy, sp, ow, wl.k)
    assert_layer_close(bf16_np(out), want, "combine")


# -------------------------------------------------------------------- layer


@pytest.mark.parametrize("name", ["tiny", "20b_decode", "120b_decode"])
def test_layer_full_output(dev, name):
    wl = syn.WORKLOADS[name]
    L = device_layer(wl, dev)
    out = bf16_np(run_layer(L))
    gq, gs, dq, ds = oracle_weights_for(wl, range(wl.E))
    want, y_ulp = oracle_layer_with_y(L.host["x"], L.host["logits"], wl.k, gq, gs, dq, ds)
    assert_layer_close(out, want, name, y_ulp)


@pytest.mark.parametrize("name", ["20b_prefill", "120b_skewed_prefill"])
def test_layer_sampled_tokens(dev, name):
    wl = syn.WORKLOADS[name]
    L = device_layer(wl, dev)
    out = bf16_np(run_layer(L))
    rng = np.random.default_rng(7)
    tokens = np.unique(np.concatenate([[0, wl.T - 1], rng.integers(0, wl.T, 10)]))
    oi, _ = oracle.route(L.host["logits"][tokens], wl.k)
    gq, gs, dq, ds = oracle_weights_for(wl, oi.ravel())
    want, y_ulp = oracle_tokens_with_y(L.host["x"], L.host["logits"], wl.k, gq, gs, dq, ds, tokens)
    assert_layer_close(out[tokens], want, name, y_ulp)
    # properties that hold at any size: finite, and the scale of the output
    o = out.view(np.uint16)
    assert ((o & 0x7F80) != 0x7F80).all()


@pytest.mark.parametrize("T,D,F,E,k", [(1, 128, 128, 4, 4), (3, 192, 320, 8, 2), (33, 256, 128, 16, 4),
                                        (70, 128, 256, 64, 8), (17, 2880, 2880, 4, 1)])
def test_layer_odd_shapes(dev, T, D, F, E, k):
    wl = syn.Workload("odd", T=T, d_model=D, d_ff=F, E=E, k=k, seed=3)
    L = device_layer(wl, dev)
    out = bf16_np(run_layer(L))
    gq, gs, dq, ds = oracle_weights_for(wl, range(E))
    want, y_ulp = oracle_layer_with_y(L.host["x"], L.host["logits"], k, gq, gs, dq, ds)
    assert_layer_close(out, want, f"{T},{D},{F},{E},{k}", y_ulp)


def test_layer_all_tokens_on_few_experts(dev):
    # logits pushed so that every token picks experts 0..3: the rest get none
    wl = syn.Workload("hot", T=300, d_model=256, d_ff=256, E=32, k=4, seed=6)
    L = device_layer(wl, dev)
    lg = L.host["logits"].copy()
    lg[:, :4] += 100.0
    L.logits = torch.from_numpy(lg).to(dev)
    L.host["logits"] = lg
    out = bf16_np(run_layer(L))
    gq, gs, dq, ds = oracle_weights_for(wl, range(4))
    want, y_ulp = oracle_layer_with_y(L.host["x"], lg, 4, gq, gs, dq, ds)
    assert_layer_close(out, want, "hot", y_ulp)


@pytest.mark.parametrize("gu_sigma,dn_sigma,x_sigma", [(3e-39, 0.02, 1e36), (0.02, 1e3, 1.0)])
def test_layer_extreme_scales(dev, gu_sigma, dn_sigma, x_sigma):
    # scale byte 0 (gate/up weights at the bottom of the bf16 range, decoded
    # values subnormal) and scale bytes above 128 (large down weights)
    T, D, F, E, k = 24, 256, 256, 8, 4
    wl = syn.Workload("scales", T=T, d_model=D, d_ff=F, E=E, k=k, seed=12)
    x_np = syn.normal_bf16(12, 701, (T, D), sigma=x_sigma)
    lg_np = syn.logits_custom(12, 702, T, E)
    gu = syn.normal_bf16(12, 703, (E, 2 * F, D), sigma=gu_sigma)
    dn = syn.normal_bf16(12, 704, (E, D, F), sigma=dn_sigma)
    gq, gs, _ = oracle.mxfp4_quantize(gu)
    dq, ds, _ = oracle.mxfp4_quantize(dn)
    if gu_sigma < 1e-30:
        assert (gs == 0).mean() > 0.5
    else:
        assert (ds > 128).all()
    shape = moe.make_shape(T, E, k, D, F)
    wgu_q = torch.from_numpy(gq).to(dev)
    wgu_s = torch.from_numpy(gs).to(dev)
    wdn_q = torch.from_numpy(dq).to(dev)
    wdn_s = torch.from_numpy(ds).to(dev)
    out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(shape, moe.WS_LAYER, dev)
    moe.moe_layer_forward(to_dev_u16(x_np, dev), torch.from_numpy(lg_np).to(dev), shape, wgu_q,
                          wgu_s, wdn_q, wdn_s, out, ws)
    torch.cuda.synchronize()
    want, y_ulp = oracle_layer_with_y(x_np, lg_np, k, gq, gs, dq, ds)
    assert_layer_close(bf16_np(out), want, f"scales {gu_sigma} {dn_sigma}", y_ulp)


@pytest.mark.parametrize("name", ["20b_decode", "20b_prefill"])
def test_layer_is_deterministic(dev, name):
    # every output element is summed in a fixed order (no atomics, no
    # split-K races), so repeated calls agree bit for bit; outputs are
    # prefilled with NaN so a row no kernel wrote shows up
    wl = syn.WORKLOADS[name]
    L = device_layer(wl, dev)
    ws = moe.alloc_workspace(L.shape, moe.WS_LAYER, dev)
    first = None
    for _ in range(6):
        out = torch.full((wl.T, wl.d_model), float("nan"), dtype=torch.bfloat16, device=dev)
        moe.moe_layer_forward(L.x, L.logits, L.shape, L.wgu_q, L.wgu_s, L.wdn_q, L.wdn_s, out, ws)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
        got = bf16_np(out)
        if first is None:
            first = got
        assert np.array_equal(got, first)
