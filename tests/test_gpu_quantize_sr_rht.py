"""Parity of the training-style quantiser (mxfp4_quantize_sr_rht, through the
C ABI) with the CPU oracle: codes and scale bytes bit for bit, for every flag
combination ("MXFP4-based MoE technical review", sections 2 and 4: stochastic
rounding and a random Hadamard transform).

Both sides take each rounding decision on the exact transformed value (fp64,
exact for blocks whose exponents span under 40 binades, which every input here
keeps) and draw the same Philox4x32-10 uniforms, so nothing but bytes is
compared.
"""
import numpy as np
import pytest
import torch

import mxfp4_quantised_mixture_b200 as moe
import oracle
import synthetic as syn
from layer_cases import to_dev_u16

pytestmark = pytest.mark.gpu

FLAGS = [0, moe.MOE_QUANT_RHT, moe.MOE_QUANT_SR, moe.MOE_QUANT_RHT | moe.MOE_QUANT_SR]


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


def random_signs(seed: int, K: int) -> np.ndarray:
    return np.random.default_rng(seed).integers(0, 1 << 32, size=K // 32,
                                                dtype=np.uint64).astype(np.uint32)


def gpu_quantize(w_np, flags, signs, seed, dev):
    w = to_dev_u16(w_np, dev)
    K = w_np.shape[-1]
    q = torch.empty(w_np.shape[:-1] + (K // 2,), dtype=torch.uint8, device=dev)
    s = torch.empty(w_np.shape[:-1] + (K // 32,), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    sg = None if signs is None else torch.from_numpy(signs.view(np.int32)).to(dev)
    moe.mxfp4_quantize_sr_rht(w, flags, sg, seed, q, s, st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), int(st.item())


def assert_parity(w, flags, seed, dev, signs=None):
    K = w.shape[-1]
    if signs is None:
        signs = random_signs(seed ^ 0x5EED, K)
    q, s, st = gpu_quantize(w, flags, signs, seed, dev)
    oq, os_, bad = oracle.mxfp4_quantize_sr_rht(w, flags, signs, seed)
    assert bad == 0 and st == moe.MOE_OK
    assert np.array_equal(s, os_), np.argwhere(s != os_)[:5]
    assert np.array_equal(q, oq), np.argwhere(q != oq)[:5]
    return q, s


@pytest.mark.parametrize("flags", FLAGS)
def test_every_bf16_value(dev, flags):
    # every finite bf16 pattern, 32 consecutive patterns to a block (so each
    # block spans at most a binade or two), positive and negative halves
    pos = np.arange(0x0000, 0x7F80, dtype=np.uint32).astype(np.uint16)
    neg = pos | np.uint16(0x8000)
    blocks = np.concatenate([pos, neg]).reshape(-1, 32)
    # rows of 4 blocks in shuffled order, so rows mix signs and magnitudes
    order = np.random.default_rng(1).permutation(blocks.shape[0])
    w = blocks[order].reshape(-1, 128)
    assert_parity(w, flags, seed=0xC0FFEE, dev=dev)


def test_no_flags_equals_deterministic_quantiser(dev):
    w = syn.normal_bf16(3, 510, (77, 2880), sigma=0.02)
    q, s, _ = gpu_quantize(w, 0, None, 0, dev)
    oq, os_, _ = oracle.mxfp4_quantize(w)
    assert np.array_equal(q, oq) and np.array_equal(s, os_)


@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("rows,K,sigma", [(1, 32, 1.0), (3, 96, 1e-30), (7, 2880, 0.02),
                                          (129, 256, 3e4), (1000, 2880, 0.02), (33, 4096, 1e-38)])
def test_random_shapes(dev, flags, rows, K, sigma):
    w = syn.normal_bf16(11, 600 + K, (rows, K), sigma=sigma)
    assert_parity(w, flags, seed=rows * 7919 + K, dev=dev)


@pytest.mark.parametrize("flags", FLAGS[1:])
@pytest.mark.parametrize("name", ["20b_decode", "120b_skewed_prefill"])
def test_workload_experts(dev, flags, name):
    # whole expert matrices at the workloads' sizes: the gate/up matrix
    # (5760 x 2880, 518,400 blocks) runs two grid-stride passes, and
    # K / 32 = 90 does not divide the pass, so the column index wraps
    wl = syn.WORKLOADS[name]
    e = wl.E - 1
    for w in (syn.w_gate_up(wl, [e]), syn.w_down(wl, [e])):
        assert_parity(w.reshape(-1, w.shape[-1]), flags, seed=1234 + e, dev=dev)


def test_same_seed_same_bytes_other_seed_other_bytes(dev):
    w = syn.normal_bf16(5, 700, (64, 1024), sigma=0.02)
    flags = moe.MOE_QUANT_RHT | moe.MOE_QUANT_SR
    signs = random_signs(2, 1024)
    a = gpu_quantize(w, flags, signs, 42, dev)
    b = gpu_quantize(w, flags, signs, 42, dev)
    c = gpu_quantize(w, flags, signs, 43, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0])
    assert np.array_equal(a[1], c[1])  # the scale does not depend on the draw


def test_zero_subnormal_and_saturating_blocks(dev):
    K = 128
    w = np.zeros((5, K), dtype=np.uint16)
    w[1, :] = 0x8000
    w[2, :] = 0x7F7F
    w[3, :] = 0x0001
    w[4, ::2] = 0x7F7F
    w[4, 1::2] = 0xFF7F
    for flags in FLAGS:
        assert_parity(w, flags, seed=9, dev=dev)


def test_nonfinite_input_is_flagged(dev):
    w = syn.normal_bf16(1, 300, (4, 64))
    w[2, 37] = 0x7F80
    for flags in FLAGS:
        _, _, st = gpu_quantize(w, flags, random_signs(0, 64), 1, dev)
        assert st == moe.MOE_ERR_NONFINITE
