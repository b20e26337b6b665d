"""moe_router_topk (router scores on the tensor core fused with the top-k and
the softmax over the chosen experts) against the CPU oracle.

"Welcome GPT OSS ..." (summary), section 4: token-choice routing over router
scores, softmax after the top-k.  The scores are checked against the oracle's
fp64 dot products within the fp32-accumulation bound; the routing decided on
them (an integer decision taken in the kernel's precision) is checked exactly
against the oracle's top-k of the kernel's own fp32 scores, and bit for bit
against moe_route applied to them.
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import ROUTE_W_ATOL, to_dev_u16

pytestmark = pytest.mark.gpu


def _run(x_np, w_np, k, dev):
    T, D = x_np.shape
    E = w_np.shape[0]
    x = to_dev_u16(x_np, dev)
    w = to_dev_u16(w_np, dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, k), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    moe.moe_router_topk(x, w, k, idx, tw, logits, status)
    # the same scores through moe_route
    idx2 = torch.empty_like(idx)
    tw2 = torch.empty_like(tw)
    moe.moe_route(logits, k, idx2, tw2)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.MOE_OK
    return (logits.cpu().numpy(), idx.cpu().numpy(), tw.cpu().numpy(), idx2.cpu().numpy(),
            tw2.cpu().numpy())


def _check(x_np, w_np, k, dev):
    lg, idx, tw, idx2, tw2 = _run(x_np, w_np, k, dev)
    ref = oracle.router_logits(x_np, w_np)
    # fp32 accumulation of exact products: |error| <= ~D * 2^-24 * sum |x w|
    xf = syn.bf16_bits_to_f32(x_np).astype(np.float64)
    wf = syn.bf16_bits_to_f32(w_np).astype(np.float64)
    bound = np.abs(xf) @ np.abs(wf).T * (x_np.shape[1] * 2.0 ** -24) + 1e-30
    assert np.all(np.abs(lg - ref) <= bound)
    oi, ow = oracle.route(lg, k)
    assert np.array_equal(idx, oi)
    assert np.max(np.abs(tw - ow)) <= ROUTE_W_ATOL
    assert np.array_equal(idx, idx2) and np.array_equal(tw.view(np.uint32), tw2.view(np.uint32))


# T * E <= 16384 runs the small-batch kernel (a cluster of two CTAs per token
# while 2 T fits the SMs, one CTA per token above; one or two router rows per
# warp and pass), larger batches the tensor-core kernel; all kinds are here
@pytest.mark.parametrize("T,D,E,k", [(64, 2880, 32, 4), (128, 2880, 128, 4), (1, 64, 8, 4),
                                     (40, 320, 65, 3), (74, 2880, 32, 4), (75, 2880, 32, 4),
                                     (200, 256, 33, 2), (17, 192, 16, 1), (1, 16384, 256, 8),
                                     (300, 512, 256, 8), (600, 512, 32, 4), (1000, 128, 64, 8),
                                     (2048, 2880, 128, 4)])
def test_router_topk(cuda_device, T, D, E, k):
    x = syn.normal_bf16(30, 910 + E, (T, D))
    w = syn.normal_bf16(30, 911 + E, (E, D), sigma=1.0 / np.sqrt(D))
    _check(x, w, k, cuda_device)


@pytest.mark.parametrize("T", [50, 130, 1000])
def test_router_ties_go_to_the_lower_index(cuda_device, T):
    D, E, k = 128, 24, 4
    x = syn.normal_bf16(31, 920, (T, D))
    w = syn.normal_bf16(31, 921, (E, D), sigma=0.1)
    w[5] = w[2]    # experts 2 and 5 always score the same
    w[17] = w[11]
    _, idx, _, _, _ = _run(x, w, k, cuda_device)
    for t in range(T):
        row = list(idx[t])
        if 5 in row:
            assert 2 in row and row.index(2) < row.index(5)
        if 17 in row:
            assert 11 in row and row.index(11) < row.index(17)
    _check(x, w, k, cuda_device)


def test_router_rejects_bad_shapes(cuda_device):
    x = torch.zeros((4, 96), dtype=torch.bfloat16, device=cuda_device)  # D not a multiple of 64
    w = torch.zeros((8, 96), dtype=torch.bfloat16, device=cuda_device)
    idx = torch.empty((4, 4), dtype=torch.int32, device=cuda_device)
    tw = torch.empty((4, 4), dtype=torch.float32, device=cuda_device)
    with pytest.raises(moe.MoeError) as err:
        moe.moe_router_topk(x, w, 4, idx, tw)
    assert err.value.status == moe.MOE_ERR_SHAPE
