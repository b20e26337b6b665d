"""The grouped expert MLP on unquantised bf16 weights (moe_expert_mlp_unquantised)
against the oracle's bf16 expert MLP (oracle.expert_mlp_bf16, pinned), on
every element of h and y.

"Tricks from OpenAI gpt-oss you can use with transformers" (summary),
section 7, and agentlenshq "Transformers ... GPT-OSS" (ja), "What is MXFP4":
without MXFP4 the experts are held in bf16; this path is the comparison point.
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import assert_layer_close, bf16_np, f64, h_flip_bound, to_dev_u16

pytestmark = pytest.mark.gpu


def _run(dev, T, D, F, E, k, seed, wl=None):
    if wl is None:
        x = syn.normal_bf16(seed, 821, (T, D))
        lg = syn.logits_custom(seed, 822, T, E)
        gu = syn.normal_bf16(seed, 823, (E, 2 * F, D), sigma=0.02)
        dn = syn.normal_bf16(seed, 824, (E, D, F), sigma=0.02)
    else:
        x, lg, gu, dn = syn.activations(wl), syn.logits(wl), syn.w_gate_up(wl), syn.w_down(wl)
    idx, _ = oracle.route(lg, k)
    _, offsets, ss, _ = oracle.permute(idx, E)
    xp = oracle.gather(x, ss, k)
    shape = moe.make_shape(T, E, k, D, F)
    S = T * k
    h = torch.empty((S, F), dtype=torch.bfloat16, device=dev)
    y = torch.empty((S, D), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(shape, moe.WS_EXPERT_MLP_UNQUANTISED, dev)
    ws[:4].fill_(0x7F)  # the call clears its status word
    moe.moe_expert_mlp_unquantised(to_dev_u16(xp, dev), torch.from_numpy(offsets).to(dev), shape,
                                   to_dev_u16(gu, dev), to_dev_u16(dn, dev), h, y, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
    oh, oy = oracle.expert_mlp_bf16(xp, offsets, gu, dn)
    # y compared directly: one flipped h per element is within the reading
    hflip = h_flip_bound(oh, offsets, f64(dn))
    return bf16_np(h), bf16_np(y), oh, oy, hflip


@pytest.mark.parametrize("T,D,F,E,k", [
    (16, 256, 256, 8, 4),      # the tiny layer's shape, tiles of 32 rows
    (37, 256, 192, 8, 2),      # d_model != d_ff, ragged tiles
    (128, 384, 256, 16, 4),    # tiles of 64 rows
    (300, 256, 128, 8, 4),     # tiles of 256 rows, ragged last tiles
    (600, 192, 320, 16, 4),    # tiles of 256 rows, K % 128 = 64 on both GEMMs
    (1, 128, 128, 4, 4),       # one token
])
def test_unquantised_mlp_every_element(cuda_device, T, D, F, E, k):
    h, y, oh, oy, hflip = _run(cuda_device, T, D, F, E, k, seed=T + D)
    assert_layer_close(h, oh, f"h {T},{D},{F},{E},{k}")
    assert_layer_close(y, oy, f"y {T},{D},{F},{E},{k}", hflip)


def test_unquantised_mlp_20b_decode(cuda_device):
    # the 20B decode batch with the workload's own (unquantised) weights
    wl = syn.WORKLOADS["20b_decode"]
    h, y, oh, oy, hflip = _run(cuda_device, wl.T, wl.d_model, wl.d_ff, wl.E, wl.k, 0, wl)
    assert_layer_close(h, oh, "h 20b_decode")
    assert_layer_close(y, oy, "y 20b_decode", hflip)
