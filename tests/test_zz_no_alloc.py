"""The allocation-free layer entry point (moe_layer_forward_static).

For callers that cannot allocate device memory, the library offers the whole
layer with its intermediates in a 16 MiB device array of its own.  These
tests call it through the C ABI and compare it with moe_layer_forward on a
caller-owned workspace, on three different layers called back to back (each
call must not see anything left over from the one before; the third takes the
other GEMM path, whose workspace lies differently in the array), read the
device status word it leaves in the array, and check that a shape needing
more than the array is refused before anything runs.
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
    # token-heavy (2 * ceil(T k / E) > 64): the decode-to-bf16 GEMM path
    c = device_layer(syn.Workload("heavy", T=1024, d_model=256, d_ff=256, E=8, k=4, seed=10),
                     cuda_device)
    assert moe.moe_workspace_size(c.shape, moe.WS_LAYER) <= moe.STATIC_SCRATCH_BYTES
    want_a = bf16_np(run_layer(a))
    want_b = bf16_np(run_layer(b))
    want_c = bf16_np(run_layer(c))
    got_a = _static(a)  # first call: the library resolves its array on this device
    got_b = _static(b)  # the next calls reuse the array left over from the one before
    got_c = _static(c)
    assert_layer_close(got_a, want_a, "static 20b_decode")
    assert_layer_close(got_b, want_b, "static odd shape")
    assert_layer_close(got_c, want_c, "static token-heavy shape")
    # the same kernels run in the same order, so the results are in fact equal
    assert np.array_equal(got_a, want_a) and np.array_equal(got_b, want_b)
    assert np.array_equal(got_c, want_c)
    # the last call's device status word, copied out of the array
    st = torch.full((1,), -1, dtype=torch.int32, device=cuda_device)
    moe.moe_layer_static_status(st)
    torch.cuda.synchronize()
    assert int(st.item()) == moe.MOE_OK


def test_static_rejects_shapes_beyond_its_array(cuda_device):
    sh = moe.make_shape(8192, 32, 4, 2880, 2880)  # the 20B prefill batch: ~570 MB of intermediates
    assert moe.moe_workspace_size(sh, moe.WS_LAYER) > moe.STATIC_SCRATCH_BYTES
    st = moe.lib.moe_layer_forward_static(16, 16, sh, 16, 16, 16, 16, 16, None)
    assert st == moe.MOE_ERR_WORKSPACE
