"""The expert-parallel layer on the CUDA library with one NCCL rank: the
exchange degenerates to copies; the output must meet the layer tolerance
against the oracle and equal the one-GPU layer bit for bit (the rows reach
the grouped GEMM in the same expert groups and the same order, and every
kernel is deterministic).  The several-rank
exchange is covered on CPU ranks in ``test_ep_gloo.py``; agentlenshq
"Transformers ... GPT-OSS" (ja), section "Expert parallel (EP)"."""
import datetime

import numpy as np
import pytest
import torch
import torch.distributed as dist

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import assert_layer_close, bf16_np, oracle_layer_with_y, oracle_weights_for
from mxfp4_quantised_mixture_b200 import ep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_one_rank(cuda_device):
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=cuda_device)
    yield cuda_device
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["tiny", "20b_decode"])
def test_one_rank_ep_equals_layer(nccl_one_rank, name):
    dev = nccl_one_rank
    wl = syn.WORKLOADS[name]
    D, F, E, T, k = wl.d_model, wl.d_ff, wl.E, wl.T, wl.k

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    x_np, lg_np = syn.activations(wl), syn.logits(wl)
    x = bf16(x_np)
    logits = torch.from_numpy(lg_np).to(dev)
    wgu_q = torch.empty((E, 2 * F, D // 2), dtype=torch.uint8, device=dev)
    wgu_s = torch.empty((E, 2 * F, D // 32), dtype=torch.uint8, device=dev)
    wdn_q = torch.empty((E, D, F // 2), dtype=torch.uint8, device=dev)
    wdn_s = torch.empty((E, D, F // 32), dtype=torch.uint8, device=dev)
    moe.mxfp4_quantize(bf16(syn.w_gate_up(wl)), wgu_q, wgu_s)
    moe.mxfp4_quantize(bf16(syn.w_down(wl)), wdn_q, wdn_s)

    shape = moe.make_shape(T, E, k, D, F)
    ref = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(shape, moe.WS_LAYER, dev)
    moe.moe_layer_forward(x, logits, shape, wgu_q, wgu_s, wdn_q, wdn_s, ref, ws)

    local = ep.LocalExperts(0, E, wgu_q, wgu_s, wdn_q, wdn_s)
    out = ep.ep_layer_forward(x, logits, k, E, F, local)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # and against the oracle's one-process layer
    gq, gs, dq, ds = oracle_weights_for(wl, range(E))
    want, y_ulp = oracle_layer_with_y(x_np, lg_np, k, gq, gs, dq, ds)
    assert_layer_close(bf16_np(out), want, f"ep {name}", y_ulp)
