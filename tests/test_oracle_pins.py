"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something the pages or mathematics fix,
never against a retyped copy of its own formula:

* the E2M1 bit layout (1 sign, 2 exponent, 1 mantissa bit) and the shared
  32-element power-of-two scale ["Tricks from OpenAI gpt-oss ...", section 6;
  agentlenshq (ja), "What is MXFP4"; "MXFP4-based MoE technical review",
  section 1 for the OCP MX / E8M0 reading];
* brute-force nearest-value search for the element encoding;
* hand-derived blocks (the pages print no worked example);
* brute-force sorting for the token-choice top-k and a direct softmax
  ["Welcome GPT OSS ...", section 4];
* the permutation's defining invariants;
* a dense per-token restatement, the single-expert layer as fp64
  torch.matmul, and a full restatement of the layer in torch fp64;
* expert independence [aitrends.kr talk summary, "Q&A"].
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic as syn

# ---------------------------------------------------------------- helpers


def bits_to_f64(b):
    with np.errstate(invalid="ignore"):
        return syn.bf16_bits_to_f32(np.asarray(b, dtype=np.uint16)).astype(np.float64)


def e2m1_from_bits(code: int) -> float:
    """E2M1 value from its bit fields: 1 sign, 2 exponent (bias 1), 1 mantissa;
    exponent field 0 is the subnormal range (0 or 0.5)."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        mag = m * 0.5
    else:
        mag = 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


def rne_bf16_exact(x: float) -> int:
    """bf16 bits of x rounded to nearest even, by exact rational arithmetic."""
    if x == 0.0:
        return 0x8000 if math.copysign(1.0, x) < 0 else 0
    sign = 0x8000 if x < 0 else 0
    a = Fraction(abs(x))
    # find exponent e with 2^e <= a < 2^(e+1)
    e = math.floor(math.log2(abs(x)))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = max(e - 7, -133)
    m = a / Fraction(2) ** q
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = Fraction(fl) * Fraction(2) ** q
    if v >= Fraction(2) ** 128:
        return sign | 0x7F80
    f = np.float32(float(v))
    return sign | int((f.view(np.uint32) >> 16) & 0x7FFF)


def decode_by_bitfields(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Independent MXFP4 decode: nibble order low-first, value from bit fields."""
    lut = np.array([e2m1_from_bits(c) for c in range(16)], dtype=np.float64)
    lo = q & 15
    hi = q >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(q.shape[:-1] + (q.shape[-1] * 2,))
    vals = lut[codes]
    scale = np.power(2.0, s.astype(np.float64) - 127.0)
    scale = np.repeat(scale, 32, axis=-1)
    return vals * scale


def np_round_bf16(x: np.ndarray) -> np.ndarray:
    """Vectorised RNE to bf16 (values), for normal-range inputs."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, |m| in [0.5, 1)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)  # np.rint: ties to even
    return r


# ------------------------------------------------------------ E2M1 / E8M0


def test_decode_table_exhaustive():
    for b in (0, 1, 100, 119, 125, 127, 130, 200, 254):
        for code in range(16):
            want = e2m1_from_bits(code) * 2.0 ** (b - 127)
            got = oracle.mxfp4_value(code, b)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, b)


def test_bf16_round_matches_exact_rational():
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000))
    # exact ties at several magnitudes, subnormals and the overflow edge
    for e in (-140, -133, -130, -126, -1, 0, 5, 100, 127):
        for mant in (0x101, 0x103, 0x1FF, 0x180):
            xs.append(math.ldexp(mant / 256.0, e))
            xs.append(-math.ldexp(mant / 256.0, e))
    xs += [0.0, -0.0, 2.0 ** -134, 3 * 2.0 ** -135, (2 - 2 ** -8) * 2.0 ** 127, 2.0 ** 128 * 0.999]
    for x in xs:
        assert oracle.bf16_round(x) == rne_bf16_exact(x), x


def _block_with(values_bits, first_bits):
    blk = np.zeros(32, dtype=np.uint16)
    blk[0] = first_bits
    blk[1:1 + len(values_bits)] = values_bits
    return blk


def test_scale_byte_is_floor_log2_amax_minus_2():
    rng = np.random.default_rng(2)
    for _ in range(3000):
        exp = int(rng.integers(-135, 128))
        amax = float(np.float32(rng.uniform(1.0, 2.0) * 2.0 ** exp))
        if not math.isfinite(amax) or amax >= 3.3e38:
            continue
        ab = rne_bf16_exact(amax)
        av = float(bits_to_f64(ab))
        blk = syn.normal_bf16(7, 99, (32,), sigma=1.0, offset=int(rng.integers(0, 1 << 30)))
        # scale the other elements well below amax
        others = np.array([rne_bf16_exact(float(v) * av / 16.0) if av > 0 else 0 for v in bits_to_f64(blk)],
                          dtype=np.uint16)
        others[int(rng.integers(0, 32))] = ab | (0x8000 if rng.integers(0, 2) else 0)
        q, s, bad = oracle.mxfp4_quantize(others.reshape(1, 32))
        assert bad == 0
        amax_true = float(np.max(np.abs(bits_to_f64(others))))
        if amax_true == 0.0:
            want = 0
        else:
            _, e = math.frexp(amax_true)  # amax in [2^(e-1), 2^e)
            want = min(max((e - 1) + 127 - 2, 0), 254)
        assert int(s[0, 0]) == want, (amax_true, int(s[0, 0]), want)


def test_zero_block_scale_byte_is_zero():
    q, s, bad = oracle.mxfp4_quantize(np.zeros((2, 64), dtype=np.uint16))
    assert bad == 0 and (s == 0).all() and (q == 0).all()
    neg0 = np.full((1, 32), 0x8000, dtype=np.uint16)
    q, s, _ = oracle.mxfp4_quantize(neg0)
    assert (s == 0).all() and (q == 0x88).all()


def _brute_force_code(v: float, scale: float) -> int:
    """nearest of the 8 magnitudes to |v|/scale, ties to even code, sign kept"""
    r = abs(v) / scale  # exact: scale is a power of two
    mags = [abs(e2m1_from_bits(c)) for c in range(8)]
    best = min(range(8), key=lambda c: (abs(r - mags[c]), c & 1))
    if math.copysign(1.0, v) < 0:
        best |= 8
    return best


@pytest.mark.parametrize("b", [3, 60, 119, 124, 127, 130, 200, 252])
def test_encode_brute_force_all_bf16(b):
    scale = 2.0 ** (b - 127)
    # the block maximum 7.75*scale (bf16-exact) fixes the scale byte to b
    first = rne_bf16_exact(7.75 * scale)
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits_to_f64(allbits)
    ok = np.isfinite(vals) & (np.abs(vals) <= 7.75 * scale)
    cand = allbits[ok]
    n = cand.size
    nblk = (n + 30) // 31
    blocks = np.zeros((nblk, 32), dtype=np.uint16)
    blocks[:, 0] = first
    flat = np.zeros(nblk * 31, dtype=np.uint16)
    flat[:n] = cand
    blocks[:, 1:] = flat.reshape(nblk, 31)
    q, s, bad = oracle.mxfp4_quantize(blocks)
    assert bad == 0
    assert (s == b).all()
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(nblk, 32)
    lut_codes = {}
    for bits in np.unique(blocks):
        v = float(bits_to_f64(bits))
        lut_codes[int(bits)] = _brute_force_code(v, scale)
    want = np.vectorize(lambda x: lut_codes[int(x)])(blocks)
    assert (codes == want).all()


def test_hand_derived_blocks():
    # (1) a block of 1.0: amax 1 -> floor(log2 1) - 2 = -2 -> byte 125, scale
    #     1/4, 1.0/0.25 = 4 -> code 6, two per byte -> 0x66
    q, s, _ = oracle.mxfp4_quantize(np.full((1, 32), 0x3F80, dtype=np.uint16))
    assert int(s[0, 0]) == 125 and (q == 0x66).all()
    # (2) amax 6: floor(log2 6) = 2 -> byte 127, scale 1.  Elements
    #     6 -> 6.0 (code 7); -3 -> code 8|5 = 0xD; 0.7 (bf16 0.69921875) -> 0.5
    #     (code 1); 0.2 -> 0 (code 0); 0.25 ties 0/0.5 -> 0 (even); 0.75 ties
    #     0.5/1 -> 1 (code 2); 5 ties 4/6 -> 4 (code 6); 2.5 ties 2/3 -> 2 (code 4)
    vals = [6.0, -3.0, 0.7, 0.2, 0.25, 0.75, 5.0, 2.5] + [0.0] * 24
    bits = np.array([rne_bf16_exact(v) for v in vals], dtype=np.uint16).reshape(1, 32)
    q, s, _ = oracle.mxfp4_quantize(bits)
    assert int(s[0, 0]) == 127
    assert list(q[0, :4]) == [0xD7, 0x01, 0x20, 0x46]
    # (3) amax 0.02: floor(log2 0.02) = -6 -> byte 119, scale 2^-8;
    #     bf16(0.02) = 0.02001953125 -> /2^-8 = 5.125 > 5 -> 6.0 (code 7)
    bits = np.zeros((1, 32), dtype=np.uint16)
    bits[0, 5] = rne_bf16_exact(0.02)
    q, s, _ = oracle.mxfp4_quantize(bits)
    assert int(s[0, 0]) == 119 and int(q[0, 2]) == 0x70


def test_round_trip_on_grid_values():
    rng = np.random.default_rng(3)
    for b in (10, 119, 127, 240):
        scale = 2.0 ** (b - 127)
        codes = rng.integers(0, 16, size=(64, 32))
        codes[:, 0] = 7  # one 6.0 per block keeps the scale at b
        vals = np.vectorize(e2m1_from_bits)(codes) * scale
        bits = np.vectorize(rne_bf16_exact)(vals).astype(np.uint16)
        q, s, _ = oracle.mxfp4_quantize(bits)
        assert (s == b).all()
        back = oracle.mxfp4_decode(q, s)
        assert np.array_equal(back, vals)


def test_block_invariants_and_byte_ratio():
    wl = syn.WORKLOADS["120b_skewed_prefill"]  # N(0,0.02) with 1% x20 outliers
    w = syn.w_down(wl, [5])[0][:256]
    q, s, bad = oracle.mxfp4_quantize(w)
    assert bad == 0
    R, K = w.shape
    assert q.shape == (R, K // 2) and s.shape == (R, K // 32)
    # bytes: 16 code bytes + 1 scale byte per 32 bf16 (64 bytes) -> 17/64,
    # i.e. 3.76x smaller than bf16 ("~4x" in the pages)
    assert (q.nbytes + s.nbytes) * 64 == w.nbytes * 17
    vals = bits_to_f64(w).reshape(R, K // 32, 32)
    dec = oracle.mxfp4_decode(q, s).reshape(R, K // 32, 32)
    codes = np.stack([q & 15, q >> 4], -1).reshape(R, K // 32, 32)
    amax = np.abs(vals).max(-1)
    nz = amax > 0
    maxmag = (codes & 7).max(-1)
    assert np.isin(maxmag[nz], [6, 7]).all()  # amax/scale in [4, 8)
    assert (np.abs(dec) <= 1.5 * amax[..., None] + 0).all()
    # every element decodes to its nearest representable value (so the error
    # is at most half a grid step, or the distance beyond 6*scale when the
    # element saturates)
    scale = np.power(2.0, s.astype(np.float64) - 127)[..., None]
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    nearest = np.abs(np.abs(vals / scale)[..., None] - mags).min(-1)
    err = np.abs(dec - vals) / scale
    assert np.array_equal(err, nearest)


def test_nonfinite_blocks_are_counted():
    w = np.zeros((1, 96), dtype=np.uint16)
    w[0, 40] = 0x7FC0  # NaN in block 1
    w[0, 70] = 0xFF80  # -Inf in block 2
    _, _, bad = oracle.mxfp4_quantize(w)
    assert bad == 2


# ------------------------------------------------------------------ routing


def _brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


@pytest.mark.parametrize("T,E,k", [(16, 8, 4), (33, 32, 4), (5, 128, 4), (7, 4, 4), (9, 64, 1), (3, 256, 8)])
def test_route_brute_force(T, E, k):
    lg = syn.logits_custom(11, 40 + E, T, E)
    idx, w = oracle.route(lg, k)
    for t in range(T):
        want = _brute_topk(lg[t], k)
        assert list(idx[t]) == want
        ex = [math.exp(float(lg[t, e]) - float(lg[t, want[0]])) for e in want]
        z = sum(ex)
        assert np.allclose(w[t], [v / z for v in ex], rtol=0, atol=1e-15)
        assert abs(w[t].sum() - 1.0) < 1e-12
        assert (np.diff(w[t]) <= 0).all()
        assert len(set(idx[t])) == k
    if k == 1:
        assert (w == 1.0).all()


def test_route_ties_go_to_lowest_index():
    lg = np.zeros((3, 16), dtype=np.float32)
    lg[0, [3, 7, 9, 12, 15]] = 1.5  # five-way tie for four places
    lg[1, :] = -0.0
    lg[1, [2, 5]] = 0.0  # +0 and -0 compare equal
    lg[2, :] = np.float32(-1e30)
    lg[2, 10] = 3.0
    idx, w = oracle.route(lg, 4)
    assert list(idx[0]) == [3, 7, 9, 12]
    assert list(idx[1]) == [0, 1, 2, 3]
    assert list(idx[2]) == [10, 0, 1, 2]
    assert np.allclose(w[0], 0.25) and np.allclose(w[1], 0.25)
    assert w[2, 0] == 1.0 and (w[2, 1:] == 0.0).all()


# ------------------------------------------------------------------ permute


@pytest.mark.parametrize("T,E,k", [(16, 8, 4), (1, 4, 4), (100, 64, 4), (50, 3, 2)])
def test_permute_invariants(T, E, k):
    rng = np.random.default_rng(T * 31 + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    if T > 10:
        idx[: T // 2, 0] = 0  # a hot expert
    counts, offsets, sorted_slot, slot_pos = oracle.permute(idx, E)
    S = T * k
    assert counts.sum() == S
    assert offsets[0] == 0 and offsets[-1] == S and (np.diff(offsets) == counts).all()
    assert sorted(sorted_slot.tolist()) == list(range(S))
    assert (sorted_slot[slot_pos] == np.arange(S)).all()
    flat = idx.ravel()
    # brute force: stable sort of slots by expert
    want = sorted(range(S), key=lambda s: (int(flat[s]), s))
    assert sorted_slot.tolist() == want
    for e in range(E):
        seg = sorted_slot[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()
    x = syn.normal_bf16(3, 77, (T, 64))
    xp = oracle.gather(x, sorted_slot, k)
    assert (xp == x[sorted_slot // k]).all()


# -------------------------------------------------------------------- layer


def _tiny_quantised(wl):
    gu = syn.w_gate_up(wl)
    dn = syn.w_down(wl)
    gq, gs = oracle.quantize_experts(gu)
    dq, ds = oracle.quantize_experts(dn)
    return gq, gs, dq, ds


@pytest.mark.parametrize("shape", [(16, 256, 256, 8, 4), (7, 64, 128, 4, 2), (33, 128, 64, 16, 4)])
def test_dense_per_token_equals_permuted_pipeline(shape):
    T, D, F, E, k = shape
    wl = syn.Workload("t", T=T, d_model=D, d_ff=F, E=E, k=k, seed=5)
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs, dq, ds = _tiny_quantised(wl)
    a = oracle.layer_forward(x, lg, k, gq, gs, dq, ds)
    b = oracle.layer_tokens(x, lg, k, gq, gs, dq, ds, list(range(T)))
    assert np.array_equal(a, b)


def _torch_layer(x_bits, lg, k, gq, gs, dq, ds):
    """The layer restated with torch fp64 matmuls on independently decoded
    weights, python sorting for top-k and math.exp for the softmax."""
    T, D = x_bits.shape
    E = lg.shape[1]
    Wgu = torch.from_numpy(decode_by_bitfields(gq, gs))  # [E][2F][D]
    Wdn = torch.from_numpy(decode_by_bitfields(dq, ds))  # [E][D][F]
    F = Wdn.shape[2]
    x = torch.from_numpy(bits_to_f64(x_bits))
    out = np.zeros((T, D))
    hs = {}
    for t in range(T):
        top = _brute_topk(lg[t], k)
        ex = [math.exp(float(lg[t, e]) - float(lg[t, top[0]])) for e in top]
        z = sum(ex)
        acc = torch.zeros(D, dtype=torch.float64)
        for j, e in enumerate(top):
            gu = Wgu[e] @ x[t]
            g, u = gu[:F], gu[F:]
            h = torch.from_numpy(np_round_bf16((g * torch.sigmoid(g) * u).numpy()))
            y = torch.from_numpy(np_round_bf16((Wdn[e] @ h).numpy()))
            hs[(t, e)] = h
            acc = acc + (ex[j] / z) * y
        out[t] = np_round_bf16(acc.numpy())
    return out


def test_layer_matches_torch_fp64_restatement():
    wl = syn.WORKLOADS["tiny"]
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs, dq, ds = _tiny_quantised(wl)
    got = bits_to_f64(oracle.layer_forward(x, lg, wl.k, gq, gs, dq, ds))
    want = _torch_layer(x, lg, wl.k, gq, gs, dq, ds)
    # both sides are fp64 up to summation order; bf16 roundings of h, y, out
    # may differ by one ulp only where the fp64 value sits on a rounding tie
    ulp = np.abs(want) * 2.0 ** -7 + 1e-30
    diff = np.abs(got - want)
    assert (diff <= ulp).all()
    assert (diff == 0).mean() > 0.999


def test_single_expert_layer_is_dense_mlp():
    # k = E = 1: routing weight is exactly 1, the layer is one dense SwiGLU MLP
    T, D, F = 9, 128, 192
    wl = syn.Workload("one", T=T, d_model=D, d_ff=F, E=1, k=1, seed=8)
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs, dq, ds = _tiny_quantised(wl)
    _, w = oracle.route(lg, 1)
    assert (w == 1.0).all()
    got = bits_to_f64(oracle.layer_forward(x, lg, 1, gq, gs, dq, ds))
    Wg = torch.from_numpy(decode_by_bitfields(gq, gs))[0]
    Wd = torch.from_numpy(decode_by_bitfields(dq, ds))[0]
    X = torch.from_numpy(bits_to_f64(x))
    G = X @ Wg[:F].T
    U = X @ Wg[F:].T
    H = torch.from_numpy(np_round_bf16((torch.nn.functional.silu(G) * U).numpy()))
    Y = np_round_bf16((H @ Wd.T).numpy())
    assert np.array_equal(got, Y)


def test_unchosen_experts_do_not_affect_output():
    wl = syn.Workload("ind", T=6, d_model=64, d_ff=64, E=16, k=4, seed=4)
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs, dq, ds = _tiny_quantised(wl)
    idx, _ = oracle.route(lg, 4)
    unused = sorted(set(range(16)) - set(idx.ravel().tolist()))
    assert unused
    a = oracle.layer_forward(x, lg, 4, gq, gs, dq, ds)
    gq2, dq2, gs2 = gq.copy(), dq.copy(), gs.copy()
    rng = np.random.default_rng(0)
    for e in unused:
        gq2[e] = rng.integers(0, 256, gq2[e].shape)
        dq2[e] = rng.integers(0, 256, dq2[e].shape)
        gs2[e] = rng.integers(100, 140, gs2[e].shape)
    b = oracle.layer_forward(x, lg, 4, gq2, gs2, dq2, ds)
    assert np.array_equal(a, b)
    # and perturbing a chosen expert does change it
    e0 = int(idx[0, 0])
    gq2[e0] ^= 0x11
    c = oracle.layer_forward(x, lg, 4, gq2, gs2, dq2, ds)
    assert not np.array_equal(a, c)


def test_golden_digest_of_tiny_workload():
    """Regression fixture written by tests/golden/make_golden.py (oracle only)."""
    import hashlib
    import os

    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_digest.txt")
    want = dict(line.split() for line in open(path) if line.strip() and not line.startswith("#"))
    wl = syn.WORKLOADS["tiny"]
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs, dq, ds = _tiny_quantised(wl)
    idx, _ = oracle.route(lg, wl.k)
    out = oracle.layer_forward(x, lg, wl.k, gq, gs, dq, ds)
    got = {
        "w_gu_codes": hashlib.sha256(gq.tobytes()).hexdigest(),
        "w_gu_scales": hashlib.sha256(gs.tobytes()).hexdigest(),
        "w_dn_codes": hashlib.sha256(dq.tobytes()).hexdigest(),
        "w_dn_scales": hashlib.sha256(ds.tobytes()).hexdigest(),
        "topk_idx": hashlib.sha256(idx.tobytes()).hexdigest(),
        "out": hashlib.sha256(out.tobytes()).hexdigest(),
    }
    assert got == want


# ------------------------------------------------------------------- router
# "Welcome GPT OSS ..." (summary), section 4: a router scores every token
# against every expert; the scores are a plain dot product of the token's
# activations with the expert's router row.


def _bits_value(b: int) -> Fraction:
    """Exact rational value of a finite bf16 bit pattern, decoded from its
    fields (sign, 8-bit exponent, 7-bit mantissa) without the oracle."""
    sign = -1 if b & 0x8000 else 1
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    if e == 0:
        return sign * Fraction(m, 128) * Fraction(2) ** -126
    return sign * (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)


def test_router_one_hot_rows_select_activations():
    # a router row with a single 1.0 at column d(e) scores x[t][d(e)] exactly
    T, D, E = 5, 64, 7
    x = syn.normal_bf16(21, 900, (T, D))
    w = np.zeros((E, D), np.uint16)
    cols = [3, 0, 63, 17, 17, 40, 9]
    for e, d in enumerate(cols):
        w[e, d] = 0x3F80  # 1.0
    got = oracle.router_logits(x, w)
    want = syn.bf16_bits_to_f32(x[:, cols]).astype(np.float64)
    assert np.array_equal(got, want)


def test_router_matches_exact_rational_sums():
    # small exponent range: every partial sum is exact in fp64, so the oracle
    # must equal the exact rational dot product
    T, D, E = 3, 16, 4
    x = syn.normal_bf16(22, 901, (T, D))
    w = syn.normal_bf16(22, 902, (E, D), sigma=0.5)
    got = oracle.router_logits(x, w)
    for t in range(T):
        for e in range(E):
            exact = sum(_bits_value(int(x[t, d])) * _bits_value(int(w[e, d])) for d in range(D))
            assert got[t, e] == float(exact)


def test_router_row_permutation_permutes_columns():
    T, D, E = 4, 128, 9
    x = syn.normal_bf16(23, 903, (T, D))
    w = syn.normal_bf16(23, 904, (E, D), sigma=0.05)
    perm = np.array([4, 8, 0, 3, 1, 7, 2, 6, 5])
    assert np.array_equal(oracle.router_logits(x, w[perm]), oracle.router_logits(x, w)[:, perm])


# ------------------------------------------------ bf16 expert path (comparison)


def _bf16_bits_exact(v: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of values known to be bf16-representable."""
    f32 = v.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), v)
    bits = (f32.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(bits_to_f64(bits), v)  # nothing below bf16 precision was dropped
    return bits


def test_bf16_expert_mlp_equals_mxfp4_on_decoded_weights():
    # every MXFP4 value at these scales is a bf16 value, so the bf16 path fed
    # the decoded weights must give the MXFP4 path's h and y bit for bit
    wl = syn.Workload("cmp", T=21, d_model=128, d_ff=192, E=4, k=2, seed=12)
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs, dq, ds = _tiny_quantised(wl)
    idx, _ = oracle.route(lg, wl.k)
    _, offsets, sorted_slot, _ = oracle.permute(idx, wl.E)
    xp = oracle.gather(x, sorted_slot, wl.k)
    h1, y1 = oracle.expert_mlp(xp, offsets, gq, gs, dq, ds)
    gu16 = _bf16_bits_exact(oracle.mxfp4_decode(gq, gs))
    dn16 = _bf16_bits_exact(oracle.mxfp4_decode(dq, ds))
    h2, y2 = oracle.expert_mlp_bf16(xp, offsets, gu16, dn16)
    assert np.array_equal(h1, h2) and np.array_equal(y1, y2)


def test_bf16_single_expert_is_dense_mlp():
    # unquantised bf16 weights (not MXFP4 values): one expert against a dense
    # fp64 torch restatement, up to ties of the bf16 roundings
    T, D, F = 11, 128, 64
    x = syn.normal_bf16(31, 1, (T, D), sigma=1.0)
    gu = syn.normal_bf16(31, 3, (1, 2 * F, D), sigma=0.05)
    dn = syn.normal_bf16(31, 4, (1, D, F), sigma=0.05)
    offsets = np.array([0, T], dtype=np.int32)
    h, y = oracle.expert_mlp_bf16(x, offsets, gu, dn)
    X = torch.from_numpy(bits_to_f64(x))
    Wg = torch.from_numpy(bits_to_f64(gu[0]))
    Wd = torch.from_numpy(bits_to_f64(dn[0]))
    G = X @ Wg[:F].T
    U = X @ Wg[F:].T
    H = np_round_bf16((torch.nn.functional.silu(G) * U).numpy())
    Y = np_round_bf16((torch.from_numpy(H) @ Wd.T).numpy())
    assert np.array_equal(bits_to_f64(h), H)
    assert np.array_equal(bits_to_f64(y), Y)
    # a planted sign error in one weight changes the output
    gu2 = gu.copy()
    gu2[0, 0, 0] ^= 0x8000
    _, y_bad = oracle.expert_mlp_bf16(x, offsets, gu2, dn)
    assert not np.array_equal(y_bad, y)


@pytest.mark.parametrize("T,E,k", [(64, 32, 4), (128, 128, 4), (50, 8, 8), (20, 3, 1)])
def test_route_invariants(T, E, k):
    # token-choice top-k with the softmax over the chosen k ("Welcome GPT OSS
    # ...", section 4): k distinct experts per token, weights in (0, 1]
    # summing to 1 and ordered like their logits
    lg = np.random.default_rng(T * E + k).standard_normal((T, E)).astype(np.float32)
    idx, w = oracle.route(lg, k)
    for t in range(T):
        assert len(set(idx[t].tolist())) == k
        assert abs(w[t].sum() - 1.0) <= 1e-15
        assert (w[t] > 0).all() and (np.diff(w[t]) <= 0).all()
        assert (np.diff(lg[t, idx[t]].astype(np.float64)) <= 0).all()
        # every unchosen logit is at most the smallest chosen one
        rest = np.setdiff1d(np.arange(E), idx[t])
        if rest.size:
            assert lg[t, rest].max() <= lg[t, idx[t]].min()
