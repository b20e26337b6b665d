"""Pins of the oracle's training-style quantiser (CPU only).

"MXFP4-based MoE technical review", sections 2 and 4: MXFP4 training keeps
its quality with stochastic rounding and a random Hadamard transform.  The
oracle's readings of those two words are checked here against facts that do
not come from the oracle itself:

* Philox4x32-10 against the published known-answer vectors of its authors'
  reference implementation (Random123, Salmon et al., SC 2011);
* the transform against ``scipy.linalg.hadamard`` (Sylvester construction)
  and against orthogonality (a product of two transformed operands is 32x the
  plain product, exactly, for small integers);
* stochastic rounding against exact rational counts over all 65536 uniforms
  (how many round up, and the mean, which is the unbiasedness closed form);
* the scale rules against exact rational logarithms of the block maximum;
* no flags against the deterministic quantiser, which is pinned elsewhere.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle
import synthetic as syn

GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
        Fraction(4), Fraction(6)]
H32 = scipy.linalg.hadamard(32).astype(np.float64)


def bits_to_f64(b):
    with np.errstate(invalid="ignore"):
        return syn.bf16_bits_to_f32(np.asarray(b, dtype=np.uint16)).astype(np.float64)


def signs_vector(word: int) -> np.ndarray:
    return np.array([-1.0 if (word >> j) & 1 else 1.0 for j in range(32)])


def decode_codes(q: np.ndarray) -> np.ndarray:
    """E2M1 codes [..., K] from packed bytes (element 2i in the low nibble)."""
    lo = q & 15
    hi = q >> 4
    return np.stack([lo, hi], axis=-1).reshape(q.shape[:-1] + (q.shape[-1] * 2,))


E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])


def code_values(q: np.ndarray) -> np.ndarray:
    return E2M1[decode_codes(q)]


def test_philox_known_answers():
    # philox4x32, 10 rounds: counter, key -> output (Random123 known-answer vectors)
    kat = [
        ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for ctr, key, want in kat:
        assert oracle.philox4x32_10(ctr, key) == want


def test_uniform_stream_covers_each_philox_output_once():
    seed = 0x0123456789ABCDEF
    for m in [0, 1, 7, 123456, (1 << 32) + 5]:
        words = oracle.philox4x32_10([m & 0xFFFFFFFF, m >> 32, 0, 0],
                                     [seed & 0xFFFFFFFF, seed >> 32])
        u = [oracle.sr_uniform16(seed, 8 * m + j) for j in range(8)]
        assert [u[2 * i] | (u[2 * i + 1] << 16) for i in range(4)] == list(words)


def test_uniform_stream_is_roughly_uniform():
    u = np.array([oracle.sr_uniform16(7, n) for n in range(1 << 14)], dtype=np.float64)
    # mean and variance of a uniform on {0..65535}: 5 standard errors
    n = u.size
    assert abs(u.mean() - 32767.5) < 5 * 18918.6 / math.sqrt(n)
    hist = np.bincount((u // 4096).astype(int), minlength=16)
    chi2 = ((hist - n / 16) ** 2 / (n / 16)).sum()
    assert chi2 < 50.0  # 15 degrees of freedom; p ~ 1e-5


@pytest.mark.parametrize("word", [0, 0xFFFFFFFF, 0x8000_0001, 0x5A5A_1234])
def test_transform_matches_scipy_hadamard(word):
    rng = np.random.default_rng(word & 0xFFFF)
    x = rng.integers(-100, 100, size=32).astype(np.float64)
    y = oracle.rht32(x, word)
    np.testing.assert_array_equal(y, H32 @ (signs_vector(word) * x))
    for j in range(32):
        e = np.zeros(32)
        e[j] = 1.0
        np.testing.assert_array_equal(oracle.rht32(e, word), H32[:, j] * signs_vector(word)[j])


def test_transform_preserves_products_up_to_32():
    rng = np.random.default_rng(3)
    for _ in range(50):
        word = int(rng.integers(0, 1 << 32))
        x = rng.integers(-1000, 1000, size=32).astype(np.float64)
        w = rng.integers(-1000, 1000, size=32).astype(np.float64)
        assert float(oracle.rht32(x, word) @ oracle.rht32(w, word)) == 32.0 * float(x @ w)
        # and the unsigned transform is its own inverse up to 32
        np.testing.assert_array_equal(oracle.rht32(oracle.rht32(x, 0), 0), 32.0 * x)


def _neighbours(v: Fraction):
    if v >= 6:
        return 7, 7
    c = max(i for i, g in enumerate(GRID) if g <= v)
    return c, c + 1


def _sr_values():
    vals = [Fraction(0), Fraction(6), Fraction(1, 4), Fraction(3, 4), Fraction(5, 4), Fraction(5, 2),
            Fraction(7, 2), Fraction(5), Fraction(1, 3), Fraction(1, 65536), Fraction(1, 131072),
            Fraction(65535, 65536) * 6, Fraction(4) + Fraction(1, 1 << 20)]
    vals += [g for g in GRID]
    rng = np.random.default_rng(11)
    vals += [Fraction(float(v)) for v in rng.uniform(0, 6, size=12)]
    return vals


@pytest.mark.parametrize("v", _sr_values())
def test_sr_counts_over_all_uniforms(v):
    """Over all 65536 uniforms the upper neighbour is taken exactly
    ceil(frac * 2^16) times, and the mean value is within a 2^-16 step of v."""
    lo, hi = _neighbours(v)
    codes = np.array([oracle.sr_code(float(v), u) for u in range(65536)])
    assert set(np.unique(codes)) <= {lo, hi}
    n_up = int((codes == hi).sum()) if hi != lo else 0
    if hi == lo:
        assert (codes == lo).all()
        return
    frac = (v - GRID[lo]) / (GRID[hi] - GRID[lo])
    want = math.ceil(frac * 65536)
    assert n_up == want
    # rounding up happens for the smallest uniforms (u < frac 2^16)
    assert (codes[:want] == hi).all() and (codes[want:] == lo).all()
    mean = GRID[lo] + (GRID[hi] - GRID[lo]) * Fraction(n_up, 65536)
    assert abs(mean - v) < (GRID[hi] - GRID[lo]) / 65536


def _ceil_log2(q: Fraction) -> int:
    e = math.floor(math.log2(q))
    while Fraction(2) ** e < q:
        e += 1
    while e > -2000 and Fraction(2) ** (e - 1) >= q:
        e -= 1
    return e


def _floor_log2(q: Fraction) -> int:
    e = math.floor(math.log2(q))
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    return e


def _rows(seed, rows, K, outliers=True):
    w = syn.normal_bf16(seed, 90, (rows, K), sigma=0.02)
    if outliers:
        f = bits_to_f64(w)
        mask = np.random.default_rng(seed).random((rows, K)) < 0.01
        f[mask] *= 20.0
        w = np.array([oracle.bf16_round(float(v)) for v in f.ravel()], dtype=np.uint16).reshape(rows, K)
    return w


def _transformed(w, signs):
    x = bits_to_f64(w)
    rows, K = x.shape
    y = np.empty_like(x)
    for b in range(K // 32):
        y[:, 32 * b:32 * b + 32] = (x[:, 32 * b:32 * b + 32] * signs_vector(int(signs[b]))) @ H32.T
    return y


@pytest.mark.parametrize("flags", [0, oracle.QUANT_RHT, oracle.QUANT_SR, oracle.QUANT_RHT | oracle.QUANT_SR])
def test_scale_rules(flags):
    rows, K = 24, 256
    w = _rows(5, rows, K)
    signs = np.random.default_rng(1).integers(0, 1 << 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    q, s, bad = oracle.mxfp4_quantize_sr_rht(w, flags, signs, seed=99)
    assert bad == 0
    y = _transformed(w, signs) if flags & oracle.QUANT_RHT else bits_to_f64(w)
    for r in range(rows):
        for b in range(K // 32):
            amax = Fraction(float(np.abs(y[r, 32 * b:32 * b + 32]).max()))
            if amax == 0:
                want = 0
            elif flags & oracle.QUANT_SR:
                want = 127 + _ceil_log2(amax / 6)  # smallest scale with amax / scale <= 6
            else:
                want = 127 + _floor_log2(amax) - 2
            want = min(max(want, 0), 254)
            assert int(s[r, b]) == want, (r, b, amax)


def test_no_flags_equals_deterministic_quantiser():
    rows, K = 40, 320
    w = _rows(8, rows, K)
    special = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x0080, 0x7F7F, 0xFF7F, 0x3E80,
                        0xBE80, 0x3F40, 0x4040], dtype=np.uint16)
    w[0, :special.size] = special
    w[1, :32] = 0x8000
    q0, s0, bad0 = oracle.mxfp4_quantize(w)
    q1, s1, bad1 = oracle.mxfp4_quantize_sr_rht(w, 0, None, seed=12345)
    np.testing.assert_array_equal(q0, q1)
    np.testing.assert_array_equal(s0, s1)
    assert bad0 == bad1 == 0


@pytest.mark.parametrize("flags", [oracle.QUANT_SR, oracle.QUANT_RHT | oracle.QUANT_SR])
def test_sr_codes_are_grid_neighbours_drawn_by_the_stream(flags):
    rows, K = 6, 128
    seed = 0xDEADBEEF12345678
    w = _rows(21, rows, K)
    signs = np.random.default_rng(4).integers(0, 1 << 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    q, s, _ = oracle.mxfp4_quantize_sr_rht(w, flags, signs, seed=seed)
    y = _transformed(w, signs) if flags & oracle.QUANT_RHT else bits_to_f64(w)
    codes = decode_codes(q)
    for r in range(rows):
        for c in range(K):
            scale = Fraction(2) ** (int(s[r, c // 32]) - 127)
            v = abs(Fraction(float(y[r, c]))) / scale
            lo, hi = _neighbours(v)
            mag = int(codes[r, c]) & 7
            u = oracle.sr_uniform16(seed, r * K + c)
            if lo == hi:
                assert mag == lo
            else:
                frac = (v - GRID[lo]) / (GRID[hi] - GRID[lo])
                assert mag == (hi if Fraction(u, 65536) < frac else lo), (r, c)
            assert v <= 6  # no element clips under stochastic rounding


def test_sr_is_unbiased_over_seeds():
    """The mean of the dequantised block over many seeds approaches the
    transformed input (then, inverted, the input): the error of the mean stays
    within 5 standard errors of a variable bounded by half a grid gap."""
    K = 64
    w = _rows(31, 1, K)
    signs = np.array([0x13579BDF, 0x2468ACE0], dtype=np.uint32)
    y = _transformed(w, signs)[0]
    n = 400
    acc = np.zeros(K)
    for sd in range(n):
        q, s, _ = oracle.mxfp4_quantize_sr_rht(w, oracle.QUANT_RHT | oracle.QUANT_SR, signs, seed=sd)
        scale = np.repeat(2.0 ** (s[0].astype(np.float64) - 127), 32)
        acc += code_values(q)[0] * scale
    mean = acc / n
    scale = np.repeat(2.0 ** (s[0].astype(np.float64) - 127), 32)
    gap = 2.0 * scale  # the widest E2M1 gap
    assert (np.abs(mean - y) <= 5 * (gap / 2) / math.sqrt(n)).all()
    # the deterministic variant is biased on the same block (sanity of the test)
    qd, sd_, _ = oracle.mxfp4_quantize_sr_rht(w, oracle.QUANT_RHT, signs, seed=0)
    assert not np.allclose(code_values(qd)[0] * np.repeat(2.0 ** (sd_[0] - 127.0), 32), y, atol=0, rtol=1e-3)


def test_rht_round_to_nearest_error_bound_and_inverse():
    rows, K = 16, 256
    w = _rows(41, rows, K)
    signs = np.random.default_rng(9).integers(0, 1 << 32, size=K // 32, dtype=np.uint64).astype(np.uint32)
    q, s, _ = oracle.mxfp4_quantize_sr_rht(w, oracle.QUANT_RHT, signs, seed=0)
    y = _transformed(w, signs)
    scale = np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=1)
    yq = code_values(q) * scale
    # round to nearest: within half the local gap up to 6; above 6 (amax in
    # [4, 8) scale under this scale rule) the element clips to 6 exactly
    v = np.abs(y) / scale
    gap = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0)) * scale
    bound = np.where(v <= 6, gap / 2, (v - 6) * scale)
    assert (np.abs(yq - y) <= bound).all()
    assert (v > 6).any()  # the clipping branch is exercised
    # inverting the (orthogonal up to 32) transform gives back x with the
    # error norm divided by sqrt(32)
    x = bits_to_f64(w)
    for b in range(K // 32):
        sl = slice(32 * b, 32 * b + 32)
        xr = (yq[:, sl] @ H32) * signs_vector(int(signs[b])) / 32.0
        err_x = np.linalg.norm(xr - x[:, sl], axis=1)
        err_y = np.linalg.norm(yq[:, sl] - y[:, sl], axis=1)
        np.testing.assert_allclose(err_x, err_y / math.sqrt(32), rtol=1e-12, atol=1e-300)


def test_zero_and_saturating_blocks():
    K = 64
    w = np.zeros((4, K), dtype=np.uint16)
    w[1, :] = 0x8000                       # all -0
    w[2, :] = 0x7F7F                       # largest finite bf16, all positive
    w[3, :32] = 0x0001                     # one block of the smallest subnormal
    w[3, 32:] = 0x8001
    signs = np.array([0xFFFF0000, 0x0000FFFF], dtype=np.uint32)
    for flags in [oracle.QUANT_RHT, oracle.QUANT_RHT | oracle.QUANT_SR]:
        q, s, bad = oracle.mxfp4_quantize_sr_rht(w, flags, signs, seed=3)
        assert bad == 0
        codes = decode_codes(q)
        assert (codes[0] == 0).all() and (s[0] == 0).all()
        assert (codes[1] == 0).all()       # a transformed zero is +0
        assert (s[2] == 254).all()         # y reaches 32 x 3.39e38: the clamped scale
        # block 0 of row 2: y_0 = sum of the signed terms; the saturated
        # elements take the top magnitude
        y = _transformed(w[2:3], signs)[0]
        big = np.abs(y) / 2.0 ** 127 >= 6
        assert big.any() and ((codes[2][big] & 7) == 7).all()
        assert (s[3] == 0).all()
    # without the transform -0 keeps its sign bit, as in the deterministic quantiser
    q, s, _ = oracle.mxfp4_quantize_sr_rht(w, oracle.QUANT_SR, None, seed=3)
    assert (decode_codes(q)[1] == 8).all()


def test_nonfinite_blocks_are_counted():
    w = np.zeros((2, 96), dtype=np.uint16)
    w[0, 5] = 0x7F80   # +inf
    w[1, 70] = 0x7FC1  # nan
    for flags in range(4):
        _, _, bad = oracle.mxfp4_quantize_sr_rht(w, flags, np.zeros(3, np.uint32), seed=1)
        assert bad == 2
