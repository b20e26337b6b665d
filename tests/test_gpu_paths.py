"""Both GEMM paths of the grouped expert MLP against the oracle, on every
output element (h and y), and against each other on the same inputs.

moe_expert_mlp_ex picks the path: the block-scaled one (tcgen05 block-scaled
MMA on the E2M1 codes, each bf16 row split exactly into two E4M3 pieces) and
the decode-to-bf16 one (codes decoded to exact bf16 into tensor memory, bf16
MMA).  Both take exact products of the bf16 rows and the MXFP4 weights and
differ only in the fp32 accumulation order (and, on the block-scaled path,
in bits of an activation more than 2^13 below its 32-block's largest), so
both must meet the layer tolerance against the oracle; "Tricks from OpenAI
gpt-oss ..." (summary), section 8 (GEMMs that read the MXFP4 blocks and their
scales); "Welcome GPT OSS ..." (summary), section 4 (SwiGLU experts).
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import (assert_layer_close, bf16_np, bf16_ulp, decoded_down, device_layer, f64,
                         h_flip_bound, oracle_layer_with_y, oracle_weights_for, run_layer,
                         to_dev_u16)

pytestmark = pytest.mark.gpu

BS, BF = moe.MOE_MLP_PATH_BLOCK_SCALED, moe.MOE_MLP_PATH_BF16_DECODE
WS_OF = {moe.MOE_MLP_PATH_AUTO: moe.WS_EXPERT_MLP, BS: moe.WS_EXPERT_MLP_BLOCK_SCALED,
         BF: moe.WS_EXPERT_MLP_BF16_DECODE}


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


def _weights(gu, dn, dev):
    """bf16 weights -> oracle-quantised MXFP4 (host) and the same bytes on the device."""
    gq, gs, bad1 = oracle.mxfp4_quantize(gu)
    dq, ds, bad2 = oracle.mxfp4_quantize(dn)
    assert bad1 == 0 and bad2 == 0
    host = (gq, gs, dq, ds)
    return host, tuple(torch.from_numpy(a).to(dev) for a in host)


def _mlp(dev, shape, xp_np, offsets_np, wdev, path):
    S = xp_np.shape[0]
    h = torch.empty((S, shape.d_ff), dtype=torch.bfloat16, device=dev)
    y = torch.empty((S, shape.d_model), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(shape, WS_OF[path], dev)
    ws[:4].fill_(0x7F)  # the call clears its status word
    moe.moe_expert_mlp_ex(to_dev_u16(xp_np, dev), torch.from_numpy(offsets_np).to(dev), shape,
                          *wdev, h, y, ws, path=path)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
    return bf16_np(h), bf16_np(y)


def _permuted(x_np, lg_np, k, E):
    idx, _ = oracle.route(lg_np, k)
    counts, offsets, ss, _ = oracle.permute(idx, E)
    return oracle.gather(x_np, ss, k), offsets, counts


def _case(T, D, F, E, k, seed, x_sigma=1.0, gu_sigma=0.02, dn_sigma=0.02):
    x = syn.normal_bf16(seed, 801, (T, D), sigma=x_sigma)
    lg = syn.logits_custom(seed, 802, T, E)
    gu = syn.normal_bf16(seed, 803, (E, 2 * F, D), sigma=gu_sigma)
    dn = syn.normal_bf16(seed, 804, (E, D, F), sigma=dn_sigma)
    return x, lg, gu, dn


# ------------------------------------------------ the decode-to-bf16 path


@pytest.mark.parametrize("T,D,F,E,k,path", [
    (512, 192, 320, 8, 4, 0),     # d_model != d_ff, both with K % 128 = 64; tiles of 256 rows
    (300, 256, 128, 16, 4, 0),    # ragged last tiles of every expert
    (1000, 128, 256, 64, 8, 0),   # k = 8, 64 experts
    (64, 2880, 2880, 32, 4, BF),  # the 20B decode batch forced onto this path: tiles of 32 rows
    (128, 384, 256, 16, 4, BF),   # tiles of 64 rows
    (37, 256, 192, 8, 2, BF),     # a few rows per expert
])
def test_bf16_decode_path_every_element(dev, T, D, F, E, k, path):
    shape = moe.make_shape(T, E, k, D, F)
    x, lg, gu, dn = _case(T, D, F, E, k, seed=T + D + F)
    host, wdev = _weights(gu, dn, dev)
    xp, offsets, _ = _permuted(x, lg, k, E)
    if path == 0:  # the shape itself selects this path
        assert 2 * -(-T * k // E) > 64
    h, y = _mlp(dev, shape, xp, offsets, wdev, path if path else moe.MOE_MLP_PATH_AUTO)
    oh, oy = oracle.expert_mlp(xp, offsets, *host)
    assert_layer_close(h, oh, f"h {T},{D},{F},{E},{k}")
    # y compared directly: one flipped h per element is within the reading
    assert_layer_close(y, oy, f"y {T},{D},{F},{E},{k}",
                       h_flip_bound(oh, offsets, decoded_down(host[2], host[3])))


@pytest.mark.parametrize("gu_sigma,dn_sigma,x_sigma", [(3e-39, 0.02, 1e36), (0.02, 1e3, 1.0)])
def test_bf16_decode_path_extreme_scales(dev, gu_sigma, dn_sigma, x_sigma):
    # scale byte 0 (decoded gate/up weights are bf16 subnormals) and scale
    # bytes above 128 (the decode's two-step scaling), on a token-heavy layer
    # that takes this path by itself
    T, D, F, E, k = 512, 256, 256, 8, 4
    x, lg, gu, dn = _case(T, D, F, E, k, 21, x_sigma, gu_sigma, dn_sigma)
    host, wdev = _weights(gu, dn, dev)
    if gu_sigma < 1e-30:
        assert (host[1] == 0).mean() > 0.5
    else:
        assert (host[3] > 128).all()
    shape = moe.make_shape(T, E, k, D, F)
    out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(shape, moe.WS_LAYER, dev)
    moe.moe_layer_forward(to_dev_u16(x, dev), torch.from_numpy(lg).to(dev), shape, *wdev, out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
    want, y_ulp = oracle_layer_with_y(x, lg, k, *host)
    assert_layer_close(bf16_np(out), want, f"scales {gu_sigma} {dn_sigma}", y_ulp)
    # the same inputs on the other path, through the standalone call
    xp, offsets, _ = _permuted(x, lg, k, E)
    oh, oy = oracle.expert_mlp(xp, offsets, *host)
    hflip = h_flip_bound(oh, offsets, decoded_down(host[2], host[3]))
    for path in (BS, BF):
        h, y = _mlp(dev, shape, xp, offsets, wdev, path)
        assert_layer_close(h, oh, f"h path {path}")
        assert_layer_close(y, oy, f"y path {path}", hflip)


@pytest.mark.parametrize("name", ["20b_prefill", "120b_skewed_prefill"])
def test_prefill_experts_every_row(dev, name):
    # the full-size prefill batch through moe_expert_mlp in the launch
    # configuration the layer uses; every h and y row of the hottest and the
    # coldest touched expert (20B), or of the coldest touched expert and the
    # one closest to 600 rows (skewed 120B, whose hottest expert holds ~16K
    # rows), against the oracle
    wl = syn.WORKLOADS[name]
    L = device_layer(wl, dev)
    xp, offsets, counts = _permuted(L.host["x"], L.host["logits"], wl.k, wl.E)
    S = wl.S
    h = torch.empty((S, wl.d_ff), dtype=torch.bfloat16, device=dev)
    y = torch.empty((S, wl.d_model), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(L.shape, moe.WS_EXPERT_MLP, dev)
    moe.moe_expert_mlp(to_dev_u16(xp, dev), torch.from_numpy(offsets).to(dev), L.shape, L.wgu_q,
                       L.wgu_s, L.wdn_q, L.wdn_s, h, y, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
    touched = np.nonzero(counts)[0]
    cold = int(touched[np.argmin(counts[touched])])
    if name == "20b_prefill":
        other = int(np.argmax(counts))
    else:
        other = int(touched[np.argmin(np.abs(counts[touched] - 600))])
    experts = sorted({cold, other})
    gq, gs, dq, ds = oracle_weights_for(wl, experts)
    rows = np.concatenate([np.arange(offsets[e], offsets[e + 1]) for e in experts])
    sub_off = np.concatenate([[0], np.cumsum([counts[e] for e in experts])]).astype(np.int32)
    oh, oy = oracle.expert_mlp(xp[rows], sub_off, gq[experts], gs[experts], dq[experts],
                               ds[experts])
    hb, yb = bf16_np(h), bf16_np(y)
    assert_layer_close(hb[rows], oh, f"{name} h experts {experts}")
    assert_layer_close(yb[rows], oy, f"{name} y experts {experts}",
                       h_flip_bound(oh, sub_off, decoded_down(dq[experts], ds[experts])))


# --------------------------------------------------- the block-scaled path


def test_block_scaled_wide_dynamic_range(dev):
    # activations spanning far more than 2^13 inside a 32-element block: one
    # element per block is 2^15 times larger, so the small ones lose their low
    # bits in the two-piece split (bits below 2^-20 of the block's largest)
    T, D, F, E, k = 48, 256, 256, 8, 4
    x = syn.normal_bf16(31, 811, (T, D)).copy()
    xv = syn.bf16_bits_to_f32(x)
    xv[:, ::32] *= np.float32(2.0 ** 15)
    x = (xv.view(np.uint32) >> 16).astype(np.uint16)  # exact: a power-of-two scaling
    lg = syn.logits_custom(31, 812, T, E)
    gu = syn.normal_bf16(31, 813, (E, 2 * F, D), sigma=0.02)
    dn = syn.normal_bf16(31, 814, (E, D, F), sigma=0.02)
    host, wdev = _weights(gu, dn, dev)
    xp, offsets, _ = _permuted(x, lg, k, E)
    blk = f64(xp).reshape(xp.shape[0], -1, 32)
    span = np.abs(blk).max(axis=2) / np.maximum(np.abs(np.where(blk == 0, np.inf, blk)).min(axis=2),
                                                1e-300)
    assert (span > 2.0 ** 13).mean() > 0.9  # the case the split truncates
    shape = moe.make_shape(T, E, k, D, F)
    oh, oy = oracle.expert_mlp(xp, offsets, *host)
    hflip = h_flip_bound(oh, offsets, decoded_down(host[2], host[3]))
    for path in (moe.MOE_MLP_PATH_AUTO, BF):
        h, y = _mlp(dev, shape, xp, offsets, wdev, path)
        assert_layer_close(h, oh, f"h path {path}")
        assert_layer_close(y, oy, f"y path {path}", hflip)
    # h = silu(g) * u itself spans a wide range inside its blocks (many
    # elements near zero): the down GEMM's split of h meets that case too
    hb = f64(oh).reshape(oh.shape[0], -1, 32)
    nz = np.where(hb == 0, np.inf, np.abs(hb))
    assert (np.abs(hb).max(axis=2) / nz.min(axis=2) > 2.0 ** 13).any()


# ------------------------------------------------- both paths, same inputs


@pytest.mark.parametrize("T,D,F,E,k", [(16, 256, 256, 8, 4), (64, 2880, 2880, 32, 4),
                                       (512, 256, 384, 8, 4), (200, 2880, 2880, 32, 4)])
def test_both_paths_on_one_shape(dev, T, D, F, E, k):
    shape = moe.make_shape(T, E, k, D, F)
    x, lg, gu, dn = _case(T, D, F, E, k, seed=5 + T)
    host, wdev = _weights(gu, dn, dev)
    xp, offsets, _ = _permuted(x, lg, k, E)
    oh, oy = oracle.expert_mlp(xp, offsets, *host)
    hs, ys = _mlp(dev, shape, xp, offsets, wdev, BS)
    hf, yf = _mlp(dev, shape, xp, offsets, wdev, BF)
    hflip = h_flip_bound(oh, offsets, decoded_down(host[2], host[3]))
    for got, want, what, extra in ((hs, oh, "h block-scaled", None), (hf, oh, "h bf16", None),
                                   (ys, oy, "y block-scaled", hflip), (yf, oy, "y bf16", hflip)):
        assert_layer_close(got, want, what, extra)
    # the two paths against each other: the same exact products summed in
    # another fp32 order, so the bf16 results may land on neighbouring values
    # where a sum sits within fp32 error of a rounding boundary
    for a, b, what in ((hs, hf, "h"), (ys, yf, "y")):
        d = np.abs(f64(a) - f64(b))
        ulp = bf16_ulp(b)
        rms = float(np.sqrt(np.mean(f64(b) ** 2)))
        frac_equal = float(np.mean(a == b))
        beyond = float(np.mean(d > ulp))
        print(f"{what} {T},{D},{F},{E},{k}: bit-identical {frac_equal:.4%}, "
              f"max |diff| {d.max() / rms:.3e} rms, beyond one ulp {beyond:.4%}")
        assert frac_equal > 0.95
        assert beyond <= 0.01
        # each path may carry one flipped h against the exact result
        assert_layer_close(a, b, f"{what} paths", 2 * hflip if what == "y" else None)


# ------------------------------------------------------ repeated calls


@pytest.mark.parametrize("T,D,F,E,k,path", [
    (200, 2880, 2880, 32, 4, BF),  # tiles of 64 rows (one MMA issuer, two CTAs per SM)
    (64, 2880, 2880, 32, 4, BF),   # tiles of 32 rows (two issuers, two CTAs per SM)
    (400, 1024, 1024, 32, 4, BF),  # tiles of 128 rows (two issuers, one CTA per SM)
    (2000, 512, 768, 16, 4, BF),   # tiles of 256 rows
    (64, 2880, 2880, 32, 4, BS),   # the block-scaled path at the 20B decode batch
])
def test_paths_repeatable(dev, T, D, F, E, k, path):
    # Every output element is one fixed-order sum, so repeated calls agree
    # bit for bit; outputs are prefilled with NaN so an element that no
    # kernel wrote, or one that read a ring slot out of turn, shows up.
    shape = moe.make_shape(T, E, k, D, F)
    x, lg, gu, dn = _case(T, D, F, E, k, seed=11 + T)
    host, wdev = _weights(gu, dn, dev)
    xp, offsets, _ = _permuted(x, lg, k, E)
    S = xp.shape[0]
    ws = moe.alloc_workspace(shape, WS_OF[path], dev)
    xd, od = to_dev_u16(xp, dev), torch.from_numpy(offsets).to(dev)
    first = None
    for rep in range(8):
        h = torch.full((S, F), float("nan"), dtype=torch.bfloat16, device=dev)
        y = torch.full((S, D), float("nan"), dtype=torch.bfloat16, device=dev)
        moe.moe_expert_mlp_ex(xd, od, shape, *wdev, h, y, ws, path=path)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
        got = (bf16_np(h), bf16_np(y))
        if first is None:
            first = got
            oh, oy = oracle.expert_mlp(xp, offsets, *host)
            assert_layer_close(got[0], oh, f"h {T},{D},{F},{E},{k}")
            assert_layer_close(got[1], oy, f"y {T},{D},{F},{E},{k}",
                               h_flip_bound(oh, offsets, decoded_down(host[2], host[3])))
        else:
            assert np.array_equal(got[0], first[0]), f"h differs on call {rep}"
            assert np.array_equal(got[1], first[1]), f"y differs on call {rep}"
