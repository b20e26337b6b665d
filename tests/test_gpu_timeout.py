"""The bounded-wait failure path of both grouped GEMMs, without a GPU fault.

moe_expert_mlp_ex(test_timeout_cta=0) makes the first pipeline wait of the
MMA issuer in CTA 0 of the (first) GEMM launch wait on a barrier that nothing
completes, with a short limit, so it gives up as a real timeout would: the
CTA records MOE_ERR_TIMEOUT in the device status word, every role leaves its
loop, the CTA waits for its own copies and MMAs to finish (the drains do not
look at the abort flag), frees its tensor memory and exits.  The other CTAs
finish their work; on the block-scaled path, where one launch runs both
GEMMs, a CTA whose down item needs a gate/up item that CTA 0 took and left
undone gives up the same way after the wait limit.  The host reads the status
after a sync and the context stays usable: the next normal call gives the
earlier result bit for bit.
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import bf16_np, to_dev_u16

pytestmark = pytest.mark.gpu

WS_OF = {moe.MOE_MLP_PATH_BLOCK_SCALED: moe.WS_EXPERT_MLP_BLOCK_SCALED,
         moe.MOE_MLP_PATH_BF16_DECODE: moe.WS_EXPERT_MLP_BF16_DECODE}


@pytest.mark.parametrize("path,T,D,F,E,k", [
    (moe.MOE_MLP_PATH_BLOCK_SCALED, 64, 2880, 2880, 32, 4),
    (moe.MOE_MLP_PATH_BLOCK_SCALED, 24, 256, 192, 8, 4),
    (moe.MOE_MLP_PATH_BF16_DECODE, 512, 256, 256, 8, 4),
    (moe.MOE_MLP_PATH_BF16_DECODE, 64, 2880, 2880, 32, 4),
])
def test_timeout_is_reported_and_the_next_call_is_exact(cuda_device, path, T, D, F, E, k):
    dev = cuda_device
    x = syn.normal_bf16(41, 901, (T, D))
    lg = syn.logits_custom(41, 902, T, E)
    gq, gs, _ = oracle.mxfp4_quantize(syn.normal_bf16(41, 903, (E, 2 * F, D), sigma=0.02))
    dq, ds, _ = oracle.mxfp4_quantize(syn.normal_bf16(41, 904, (E, D, F), sigma=0.02))
    w = [torch.from_numpy(a).to(dev) for a in (gq, gs, dq, ds)]
    idx, _ = oracle.route(lg, k)
    _, offsets, ss, _ = oracle.permute(idx, E)
    xp = to_dev_u16(oracle.gather(x, ss, k), dev)
    off = torch.from_numpy(offsets).to(dev)
    shape = moe.make_shape(T, E, k, D, F)
    S = T * k
    ws = moe.alloc_workspace(shape, WS_OF[path], dev)

    def call(fail):
        h = torch.zeros((S, F), dtype=torch.bfloat16, device=dev)
        y = torch.zeros((S, D), dtype=torch.bfloat16, device=dev)
        moe.moe_expert_mlp_ex(xp, off, shape, *w, h, y, ws, path=path, test_timeout_cta=fail)
        torch.cuda.synchronize()
        return int(ws[:4].view(torch.int32).item()), bf16_np(y)

    st0, y0 = call(-1)
    assert st0 == moe.MOE_OK
    st1, _ = call(0)
    assert st1 == moe.MOE_ERR_TIMEOUT
    st2, y2 = call(-1)
    assert st2 == moe.MOE_OK
    assert np.array_equal(y0, y2)
