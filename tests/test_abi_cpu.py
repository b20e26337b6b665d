"""The C-ABI library loads on a machine without a GPU, exports every symbol
that include/*.h declares, and rejects bad arguments on the host before it
touches the device (no compute calls here)."""
import ctypes
import glob
import os
import re

import pytest

import mxfp4_quantised_mixture_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)
    return names


def test_header_declares_the_six_calls_and_helpers():
    names = declared_functions()
    for n in ["mxfp4_quantize", "mxfp4_quantize_sr_rht", "moe_route", "moe_permute",
              "moe_expert_mlp", "moe_expert_mlp_ex", "moe_combine", "moe_layer_static_status",
              "moe_layer_forward", "moe_workspace_size", "moe_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_library_needs_no_cuda_shared_library():
    # cudart is linked statically and the driver is reached at run time, so
    # the library loads where no GPU driver is installed
    with open("/proc/self/maps") as f:
        maps = f.read()
    assert moe.LIB_PATH in maps


def test_status_strings():
    assert moe.moe_status_string(0) == "MOE_OK"
    assert moe.moe_status_string(3) == "MOE_ERR_WORKSPACE"
    assert moe.moe_status_string(7) == "MOE_ERR_TIMEOUT"
    assert moe.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_size_is_host_only_and_monotone():
    small = moe.make_shape(64, 32, 4, 2880, 2880)
    big = moe.make_shape(8192, 32, 4, 2880, 2880)
    a = moe.moe_workspace_size(small, moe.WS_LAYER)
    b = moe.moe_workspace_size(big, moe.WS_LAYER)
    assert 0 < a < b
    S = 8192 * 4
    # the layer workspace holds at least x_perm, h and y_perm (bf16)
    assert b >= S * 2880 * 2 * 3
    assert moe.moe_workspace_size(small, 9) == 0
    # the standalone expert MLP's workspace starts with a 256-byte status head
    assert moe.moe_workspace_size(small, moe.WS_EXPERT_MLP) >= 256
    assert moe.moe_workspace_size(moe.make_shape(64, 300, 4, 2880, 2880), moe.WS_LAYER) == 0


@pytest.mark.parametrize("shape", [
    (64, 0, 4, 2880, 2880),      # E = 0
    (64, 32, 9, 2880, 2880),     # k > 8
    (64, 4, 5, 2880, 2880),      # k > E
    (64, 32, 4, 2880, 2890),     # F not a multiple of 64
    (64, 32, 4, 32, 2880),       # D too small
    (64, 32, 4, 64, 2880),       # D below the 128-code weight window
    (64, 32, 4, 2880, 64),       # F below the 128-code weight window
    (-1, 32, 4, 2880, 2880),     # T < 0
])
def test_bad_shapes_rejected_before_the_device(shape):
    sh = moe.make_shape(*shape)
    st = moe.lib.moe_layer_forward(16, 16, sh, 16, 16, 16, 16, 16, 16, 1 << 30, None)
    assert st == moe.MOE_ERR_SHAPE
    st = moe.lib.moe_expert_mlp(16, 16, sh, 16, 16, 16, 16, 16, 16, 16, 1 << 30, None)
    assert st == moe.MOE_ERR_SHAPE


def test_bad_arguments_rejected_before_the_device():
    L = moe.lib
    assert L.mxfp4_quantize(16, 4, 48, 16, 16, None, None) == moe.MOE_ERR_SHAPE  # K % 32
    assert L.mxfp4_quantize(None, 4, 64, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize(24, 4, 64, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG  # misaligned
    assert L.mxfp4_quantize(16, 0, 64, 16, 16, None, None) == moe.MOE_OK  # empty: no-op
    assert L.moe_route(16, 4, 300, 4, 16, 16, None) == moe.MOE_ERR_SHAPE
    assert L.moe_route(None, 4, 32, 4, 16, 16, None) == moe.MOE_ERR_INVALID_ARG
    sh = moe.make_shape(64, 32, 4, 2880, 2880)
    need = moe.moe_workspace_size(sh, moe.WS_LAYER)
    # weight code arrays at 32-byte addresses, everything else at 16
    assert L.moe_layer_forward(16, 16, sh, 32, 16, 32, 16, 16, 16, need - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_layer_forward(16, 16, sh, 32, 16, 32, 16, 16, None, need, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_layer_forward(16, None, sh, 32, 16, 32, 16, 16, 16, need, None) == moe.MOE_ERR_INVALID_ARG
    # a code array only 16-byte aligned is refused
    assert L.moe_layer_forward(16, 16, sh, 48, 16, 32, 16, 16, 16, need, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_forward(16, 16, sh, 32, 16, 48, 16, 16, 16, need, None) == moe.MOE_ERR_INVALID_ARG
    mlp = moe.moe_workspace_size(sh, moe.WS_EXPERT_MLP)
    assert L.moe_expert_mlp(16, 16, sh, 48, 16, 32, 16, 16, 16, 16, mlp, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_mlp(16, 16, sh, 32, 16, 32, 16, 16, 16, 16, mlp - 1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_combine(16, 16, 16, sh, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_permute(16, 16, sh, None, 16, 16, 16, 16, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_static_status(None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_layer_static_status(18, None) == moe.MOE_ERR_INVALID_ARG  # not 4-byte aligned


def test_expert_mlp_ex_path_and_workspace_checked_before_the_device():
    L = moe.lib
    sh = moe.make_shape(64, 32, 4, 2880, 2880)  # decode-sized: auto = block-scaled
    bs = moe.moe_workspace_size(sh, moe.WS_EXPERT_MLP_BLOCK_SCALED)
    bf = moe.moe_workspace_size(sh, moe.WS_EXPERT_MLP_BF16_DECODE)
    auto = moe.moe_workspace_size(sh, moe.WS_EXPERT_MLP)
    assert auto == bs and bs > bf >= 256
    pre = moe.make_shape(8192, 32, 4, 2880, 2880)  # token-heavy: auto = bf16 decode
    assert moe.moe_workspace_size(pre, moe.WS_EXPERT_MLP) == \
        moe.moe_workspace_size(pre, moe.WS_EXPERT_MLP_BF16_DECODE)
    # (x_perm, offsets, shape, wgu_q, wgu_s, wdn_q, wdn_s, h, y_perm, ws, ws_bytes, path, fail, stream)
    for bad_path in (-1, 3, 99):
        assert L.moe_expert_mlp_ex(16, 16, sh, 32, 16, 32, 16, 16, 16, 256, bs, bad_path, -1,
                                   None) == moe.MOE_ERR_INVALID_ARG
    # a workspace that fits one path is too small for the other
    assert L.moe_expert_mlp_ex(16, 16, sh, 32, 16, 32, 16, 16, 16, 256, bf,
                               moe.MOE_MLP_PATH_BLOCK_SCALED, -1, None) == moe.MOE_ERR_WORKSPACE
    assert L.moe_expert_mlp_ex(16, 16, sh, 32, 16, 32, 16, None, 16, 256, bs,
                               moe.MOE_MLP_PATH_BF16_DECODE, -1, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_expert_mlp_ex(16, 16, moe.make_shape(64, 32, 4, 2880, 2890), 32, 16, 32, 16, 16,
                               16, 256, bs, 0, -1, None) == moe.MOE_ERR_SHAPE


def test_router_arguments_rejected_before_the_device():
    L = moe.lib
    # (x, w_router, T, D, E, k, logits, idx, w, d_status, stream)
    assert L.moe_router_topk(16, 16, 4, 96, 8, 4, None, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.moe_router_topk(16, 16, 4, 32, 8, 4, None, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.moe_router_topk(16, 16, 4, 128, 0, 1, None, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.moe_router_topk(16, 16, 4, 128, 300, 4, None, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.moe_router_topk(16, 16, 4, 128, 4, 5, None, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.moe_router_topk(16, 16, 0, 128, 8, 4, None, 16, 16, None, None) == moe.MOE_OK
    assert L.moe_router_topk(None, 16, 4, 128, 8, 4, None, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(16, 24, 4, 128, 8, 4, None, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(16, 16, 4, 128, 8, 4, 40, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG


def test_sr_rht_quantiser_arguments_rejected_before_the_device():
    L = moe.lib
    RHT, SR = moe.MOE_QUANT_RHT, moe.MOE_QUANT_SR
    # (w, rows, K, flags, signs, seed, q, s, d_status, stream)
    assert L.mxfp4_quantize_sr_rht(16, 4, 64, 4, 16, 0, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize_sr_rht(16, 4, 48, SR, None, 0, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.mxfp4_quantize_sr_rht(16, -1, 64, SR, None, 0, 16, 16, None, None) == moe.MOE_ERR_SHAPE
    assert L.mxfp4_quantize_sr_rht(16, 4, 64, RHT, None, 0, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize_sr_rht(16, 4, 64, RHT, 18, 0, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize_sr_rht(24, 4, 64, SR, None, 0, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize_sr_rht(16, 4, 64, SR, None, 0, 16, 16, 18, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize_sr_rht(None, 4, 64, 0, None, 0, 16, 16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.mxfp4_quantize_sr_rht(16, 0, 64, RHT | SR, 16, 7, 16, 16, None, None) == moe.MOE_OK


def _no_gpu_here() -> bool:
    import torch

    return not torch.cuda.is_available() and not os.path.exists("/dev/nvidiactl")


@pytest.mark.skipif(not _no_gpu_here(), reason="its placeholder pointers must never reach a device")
def test_well_formed_calls_fail_cleanly_without_a_device():
    # host-side failure injection: every argument passes validation, the
    # device probe finds no usable GPU, and the call returns a status with
    # nothing launched (no crash, no fallback)
    L = moe.lib
    sh = moe.make_shape(64, 32, 4, 2880, 2880)
    need = moe.moe_workspace_size(sh, moe.WS_LAYER)
    mlp = moe.moe_workspace_size(sh, moe.WS_EXPERT_MLP)
    no_device = (moe.MOE_ERR_CUDA, moe.MOE_ERR_UNSUPPORTED)
    assert L.mxfp4_quantize(16, 4, 64, 16, 16, None, None) in no_device
    assert L.mxfp4_quantize_sr_rht(16, 4, 64, moe.MOE_QUANT_SR, None, 1, 16, 16, None, None) in no_device
    assert L.moe_route(16, 4, 32, 4, 16, 16, None) in no_device
    assert L.moe_router_topk(16, 16, 4, 128, 8, 4, None, 16, 16, None, None) in no_device
    assert L.moe_permute(16, 16, sh, 16, 16, 16, 16, 16, None, 0, None) in no_device
    assert L.moe_expert_mlp(16, 16, sh, 32, 16, 32, 16, 16, 16, 256, mlp, None) in no_device
    assert L.moe_combine(16, 16, 16, sh, 16, None) in no_device
    assert L.moe_layer_forward(16, 16, sh, 32, 16, 32, 16, 16, 256, need, None) in no_device
    for path in (moe.MOE_MLP_PATH_BLOCK_SCALED, moe.MOE_MLP_PATH_BF16_DECODE):
        assert L.moe_expert_mlp_ex(16, 16, sh, 32, 16, 32, 16, 16, 16, 256, 1 << 30, path, -1,
                                   None) in no_device
    assert L.moe_layer_forward_static(16, 16, sh, 32, 16, 32, 16, 16, None) in no_device
    assert L.moe_layer_static_status(16, None) in no_device


def test_binding_refuses_host_and_strided_tensors():
    import torch

    sh = moe.make_shape(4, 8, 4, 128, 128)
    host = torch.zeros((4, 8), dtype=torch.float32)
    with pytest.raises(ValueError):
        moe.moe_route(host, 4, host, host)
    with pytest.raises(ValueError):
        moe.moe_combine(host, host, host, sh, host)
    if torch.cuda.is_available():  # a strided device view is refused as well
        dev = torch.zeros((8, 4), dtype=torch.float32, device="cuda").t()
        with pytest.raises(ValueError):
            moe.moe_route(dev, 4, dev, dev)
