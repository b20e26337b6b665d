"""The allocation-free layer entry point (moe_layer_forward_static).

For callers that cannot allocate device memory, the library offers the whole
layer with its intermediates in a 16 MiB device array of its own.  These
tests call it through the C ABI and compare it with moe_layer_forward on a
caller-owned workspace, on two different layers called back to back (the
second call must not see anything left over from the first), and check that
a shape needing more than the array is refused before anything runs.
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import synthetic as syn
from layer_cases import assert_layer_close, bf16_np, device_layer, run_layer

pytestmark = pytest.mark.gpu


def _static(L):
    out = torch.empty((L.wl.T, L.wl.d_model), dtype=torch.bfloat16, device=L.x.device)
    moe.moe_layer_forward_static(L.x, L.logits, L.shape, L.wgu_q, L.wgu_s, L.wdn_q, L.wdn_s, out)
    torch.cuda.synchronize()
    return bf16_np(out)


def test_static_matches_workspace_entry_on_two_calls(cuda_device):
    a = device_layer(syn.WORKLOADS["20b_decode"], cuda_device)
    b = device_layer(syn.Workload("odd", T=37, d_model=256, d_ff=192, E=8, k=2, seed=9), cuda_device)
    want_a = bf16_np(run_layer(a))
    want_b = bf16_np(run_layer(b))
    got_a = _static(a)  # first call: the library resolves its array on this device
    got_b = _static(b)  # second call reuses the array left over from the first
    assert_layer_close(got_a, want_a, "static 20b_decode")
    assert_layer_close(got_b, want_b, "static odd shape")
    # the same kernels run in the same order, so the results are in fact equal
    assert np.array_equal(got_a, want_a) and np.array_equal(got_b, want_b)


def test_static_rejects_shapes_beyond_its_array(cuda_device):
    sh = moe.make_shape(8192, 32, 4, 2880, 2880)  # the 20B prefill batch: ~570 MB of intermediates
    assert moe.moe_workspace_size(sh, moe.WS_LAYER) > moe.STATIC_SCRATCH_BYTES
    st = moe.lib.moe_layer_forward_static(16, 16, sh, 16, 16, 16, 16, 16, None)
    assert st == moe.MOE_ERR_WORKSPACE
