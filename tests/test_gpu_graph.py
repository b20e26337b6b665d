"""The library's calls inside a CUDA graph: a call captured once and replayed
gives, bit for bit, what the same call gives when launched directly, also
after the input buffers are refilled between replays (the graph keeps the
addresses, not the contents).  A serving loop runs the layer this way, so the
calls must do no host synchronisation and no allocation while enqueueing."""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import synthetic as syn
from layer_cases import bf16_np, device_layer

pytestmark = pytest.mark.gpu


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream())
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("name", ["20b_decode", "tiny", "20b_prefill"])
def test_layer_graph_replay_matches_eager(cuda_device, name):
    wl = syn.WORKLOADS[name]
    L = device_layer(wl, cuda_device)
    out = torch.empty((wl.T, wl.d_model), dtype=torch.bfloat16, device=cuda_device)
    ws = moe.alloc_workspace(L.shape, moe.WS_LAYER, cuda_device)
    call = lambda s: moe.moe_layer_forward(L.x, L.logits, L.shape, L.wgu_q, L.wgu_s, L.wdn_q,
                                           L.wdn_s, out, ws, s)
    g = _capture(call)
    x0, lg0 = L.x.clone(), L.logits.clone()
    gen = torch.Generator(device=cuda_device).manual_seed(7)
    for rep in range(3):
        if rep > 0:  # new inputs in the same buffers
            L.x.copy_(torch.randn(L.x.shape, generator=gen, device=cuda_device).to(torch.bfloat16))
            L.logits.copy_(torch.randn(L.logits.shape, generator=gen, device=cuda_device))
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == moe.MOE_OK
        replayed = bf16_np(out)
        out.fill_(float("nan"))
        call(torch.cuda.current_stream())
        torch.cuda.synchronize()
        assert np.array_equal(replayed, bf16_np(out)), f"replay {rep}"
    L.x.copy_(x0)
    L.logits.copy_(lg0)
