"""Pins for the CPU oracle: each check ties the oracle to something other
than itself -- values printed on the pages (tests/golden), closed forms,
invariants, and brute force on tiny inputs.  No GPU."""
from __future__ import annotations

import os
from fractions import Fraction
import itertools

import numpy as np
import pytest
import torch

from oracle import bitlinear as O
from ternary_weight_linear_int8_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals):
    """Exact bf16 bit patterns for values that bf16 represents exactly."""
    f = np.asarray(vals, dtype=np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), f)
    return bits


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _golden_comment(name, key):
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            if line.startswith("# " + key + ":"):
                return [int(t) for t in line.split(":", 1)[1].split()]
    raise KeyError(key)


# --------------------------------------------------------------------------
# exact rounding helpers
# --------------------------------------------------------------------------
def _is_nearest_f32(r: np.float32, x: Fraction) -> bool:
    """Brute-force check that fp32 r is a nearest fp32 to x, ties to even."""
    r = np.float32(r)
    lo = np.nextafter(r, np.float32(-np.inf))
    hi = np.nextafter(r, np.float32(np.inf))
    d = abs(Fraction(float(r)) - x)
    for nb in (lo, hi):
        if np.isinf(nb):
            continue
        dn = abs(Fraction(float(nb)) - x)
        if dn < d:
            return False
        if dn == d:   # tie: r must have an even significand
            if int(np.float32(r).view(np.uint32)) & 1:
                return False
    return True


def test_round_rational_ties_and_edges():
    R = O.round_rational_to_f32
    assert R(1, 1) == np.float32(1.0)
    # midpoint between 1 and 1+2^-23 -> even (1.0)
    assert R(2**24 + 1, 2**24) == np.float32(1.0)
    # midpoint between 1+2^-23 and 1+2^-22 -> even (1+2^-22)
    assert R(2**24 + 3, 2**24) == np.float32(1 + 2.0**-22)
    # just above the first midpoint rounds up
    assert R(2**25 + 3, 2**25) == np.float32(1 + 2.0**-23)
    # subnormals: 2^-149 exactly, half of it ties to 0, 1.5x ties to 2^-148
    assert R(1, 2**149) == np.float32(2.0**-149)
    assert R(1, 2**150) == np.float32(0.0)
    assert R(3, 2**150) == np.float32(2.0**-148)
    # largest finite and overflow
    assert R((2**24 - 1) * 2**104, 1) == np.finfo(np.float32).max
    assert np.isinf(R(2**128, 1))
    assert R(1, 3) == np.float32(1.0) / np.float32(3.0)     # IEEE division
    rng = np.random.default_rng(7)
    for _ in range(2000):
        num = int(rng.integers(1, 2**62)) * 2 ** int(rng.integers(0, 40))
        den = int(rng.integers(1, 2**62))
        assert _is_nearest_f32(R(num, den), Fraction(num, den))


def test_gamma_constant_and_known_means():
    for c in (0.02, 1.0, 3.0e-41, 1.5e30, -0.75):
        W = np.full((7, 12), c, dtype=np.float32)
        assert O.absmean_gamma(W) == abs(np.float32(c))
    assert O.absmean_gamma(np.array([[1, -2, 4, -8]], np.float32)) == np.float32(3.75)
    assert O.absmean_gamma(np.zeros((3, 4), np.float32)) == np.float32(0.0)
    # mean of {1, 2^-24}: exact value 0.5 + 2^-25 rounds to 0.5 (below the midpoint)
    assert O.absmean_gamma(np.array([[1.0, 2.0**-24]], np.float32)) == np.float32(0.5)
    # mean of {1, 1+2^-23, 1+2^-23, 1+2^-23} = 1 + 0.75*2^-23 -> 1+2^-23
    w = np.array([[1.0, 1 + 2.0**-23, 1 + 2.0**-23, 1 + 2.0**-23]], np.float32)
    assert O.absmean_gamma(w) == np.float32(1 + 2.0**-23)


def test_gamma_matches_exact_rational_and_is_order_free():
    rng = np.random.default_rng(3)
    for shape in [(1, 1), (3, 5), (17, 33), (64, 64)]:
        W = (rng.standard_normal(shape) * 10.0 ** rng.integers(-30, 30, size=shape)).astype(np.float32)
        exact = sum(Fraction(float(abs(v))) for v in W.ravel()) / W.size
        g = O.absmean_gamma(W)
        assert _is_nearest_f32(g, exact)
        perm = rng.permutation(W.size)
        assert O.absmean_gamma(W.ravel()[perm].reshape(shape)) == g
    with pytest.raises(ValueError):
        O.absmean_gamma(np.array([[1.0, np.inf]], np.float32))


# --------------------------------------------------------------------------
# bf16
# --------------------------------------------------------------------------
def test_bf16_rounding_pins():
    f = O.f32_to_bf16_bits
    assert f(np.float32(1 + 2.0**-8)) == 0x3F80          # tie -> even
    assert f(np.float32(1 + 3 * 2.0**-8)) == 0x3F82      # tie -> even (up)
    assert f(np.float32(1 + 2.0**-8 + 2.0**-20)) == 0x3F81
    assert f(np.float32(-2.5)) == 0xC020
    assert f(np.float32(0.0)) == 0 and f(np.float32(-0.0)) == 0x8000
    # every finite bf16 pattern survives widen -> round
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    fin = np.isfinite(O.bf16_bits_to_f32(allbits))
    assert np.array_equal(f(O.bf16_bits_to_f32(allbits[fin])), allbits[fin])
    # agrees with torch's bf16 cast (a library routine) on random fp32
    x = (np.random.default_rng(1).standard_normal(100000) * 1e3).astype(np.float32)
    tb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f(x), tb)


# --------------------------------------------------------------------------
# step 1: activation quantisation
# --------------------------------------------------------------------------
def test_act_quant_hand_computed_rows():
    x = _bf16([[1.0, -2.0, 0.5, 0.25, -0.125],
               [3.0, 1.0, -1.0, 0.0, 0.75]])
    q, s, rs = O.act_quant(x)
    # row 0: s = 127/2 = 63.5 exactly; 63.5 ties to 64
    assert s[0] == np.float32(63.5)
    assert q[0].tolist() == [64, -127, 32, 16, -8]
    assert rs[0] == -23
    # row 1: s = fp32(127/3); products 127-, 42.33, -42.33, 0, 31.75- -> 127, 42, -42, 0, 32
    assert q[1].tolist() == [127, 42, -42, 0, 32]
    assert rs[1] == 159


def test_act_quant_invariants():
    rng = np.random.default_rng(11)
    x = inputs.activations((33, 640), rng=rng, outliers=True)
    q, s, rs = O.act_quant(x)
    xf = O.bf16_bits_to_f32(x)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    amax_idx = np.abs(xf).argmax(axis=1)
    pick = q[np.arange(33), amax_idx].astype(np.int32)
    assert np.array_equal(np.abs(pick), np.full(33, 127))
    assert np.array_equal(np.sign(pick), np.sign(xf[np.arange(33), amax_idx]).astype(np.int32))
    assert np.array_equal(rs, q.astype(np.int32).sum(axis=1))
    # negation symmetry (rint is odd, the scale is unchanged)
    qn, sn, _ = O.act_quant(x ^ np.uint16(0x8000))
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    # scaling by 2^k keeps the codes (exact multiply, scale moves by 2^-k)
    for k in (-7, 3, 20):
        q2, s2, _ = O.act_quant_f32(xf * np.float32(2.0**k))
        assert np.array_equal(q2, q)
        assert np.array_equal(s2, s * np.float32(2.0**-k))
    # all-zero token: q = 0 and s = 127/1e-5
    q0, s0, r0 = O.act_quant(np.zeros((2, 8), np.uint16))
    assert not q0.any() and not r0.any()
    assert s0[0] == np.float32(127.0) / np.float32(1e-5)


def test_act_quant_is_nearest_integer_of_scaled_value():
    rng = np.random.default_rng(5)
    x = inputs.activations((8, 512), rng=rng)
    q, s, _ = O.act_quant(x)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    ideal = xf * (127.0 / np.abs(xf).max(axis=1, keepdims=True))
    # the fp32 pipeline may only differ from exact rounding at near-ties
    diff = np.abs(q - np.rint(ideal))
    near_tie = np.abs(np.abs(ideal - np.floor(ideal)) - 0.5) < 1e-4
    assert np.all((diff == 0) | near_tie)


# --------------------------------------------------------------------------
# step 2: ternarisation and packing
# --------------------------------------------------------------------------
def test_i2s_code_map_golden():
    rows = _read_table("i2s_code_map.txt")
    cmap = {int(r[0]): int(r[1], 2) for r in rows[:3]}
    for w, code in cmap.items():
        p = O.pack_i2s(np.full((1, 4), w, np.int8))
        assert p[0, 0] == code * 0x55      # same code in all four slots
    # one weight per slot, LSB first: [-1, 0, 1, -1] -> 00 | 01<<2 | 10<<4 | 00<<6
    assert O.pack_i2s(np.array([[-1, 0, 1, -1]], np.int8))[0, 0] == 0b00100100
    # size facts: 8 weights -> 16 bits, 16 weights -> one 32-bit word
    for nw, nbits in ([int(a), int(b)] for a, b in rows[3:]):
        assert O.pack_i2s(np.zeros((1, nw), np.int8)).nbytes * 8 == nbits
    # 100B weights at 2 bits -> 25e9 bytes
    assert 100e9 * 2 / 8 == 25e9


def test_pack_round_trip_and_no_code_3():
    rng = np.random.default_rng(2)
    w = rng.integers(-1, 2, size=(37, 96)).astype(np.int8)
    p = O.pack_i2s(w)
    assert p.shape == (37, 24)
    assert np.array_equal(O.unpack_i2s(p, 96), w)
    codes = np.stack([(p >> (2 * i)) & 3 for i in range(4)])
    assert not np.any(codes == 3)
    with pytest.raises(ValueError):
        O.unpack_i2s(np.array([[0xFF]], np.uint8), 4)


def test_ternarize_closed_forms():
    # all-zero W: gamma 0, every code 01, byte 0x55
    p, g = O.pack_weights(np.zeros((5, 8), np.float32))
    assert g == 0 and np.all(p == 0x55)
    # constant +c: gamma = c, W/(c+1e-5) < 1 rounds to 1 -> 0xAA ; -c -> 0x00
    for c in (0.02, 1.0, 7.5):
        p, g = O.pack_weights(np.full((3, 16), c, np.float32))
        assert g == np.float32(c) and np.all(p == 0xAA)
        p, g = O.pack_weights(np.full((3, 16), -c, np.float32))
        assert np.all(p == 0x00)
    # thresholds: with gamma fixed, |W| just below / above 0.5*(gamma+eps)
    g = np.float32(1.0)
    den = g + O.EPS_F32
    half = np.float32(0.5) * den
    W = np.array([[np.nextafter(half, np.float32(0)), np.nextafter(half, np.float32(1)),
                   -np.nextafter(half, np.float32(1)), 1.49 * den]], np.float32)
    assert O.ternarize(W, g).tolist() == [[0, 1, -1, 1]]


def test_ternary_statistics_gaussian():
    W = inputs.weights(512, 2048, seed=1234)
    p, g = O.pack_weights(W)
    w = O.unpack_i2s(p, 2048)
    # gamma ~= sigma * sqrt(2/pi); zero iff |W| < gamma/2 -> P ~= 2*Phi(0.399)-1 ~= 0.310
    assert abs(float(g) - 0.02 * np.sqrt(2 / np.pi)) < 2e-4
    assert abs((w == 0).mean() - 0.310) < 0.01
    assert abs((w == 1).mean() - 0.345) < 0.01
    assert abs((w == -1).mean() - 0.345) < 0.01


# --------------------------------------------------------------------------
# step 3: the integer matmul
# --------------------------------------------------------------------------
def _brute_acc(xq, w):
    M, K = xq.shape
    N = w.shape[0]
    out = np.zeros((M, N), np.int64)
    for m in range(M):
        for n in range(N):
            t = 0
            for k in range(K):
                t += int(xq[m, k]) * int(w[n, k])
            out[m, n] = t
    return out


def test_matmul_brute_force_tiny_shapes():
    rng = np.random.default_rng(9)
    for M, N, K in itertools.product([1, 2, 5], [1, 3, 8], [4, 8, 20]):
        xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
        w = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        assert np.array_equal(O.ternary_matmul(xq, w), _brute_acc(xq, w))


def test_matmul_all_81_ternary_rows_k4():
    w = np.array(list(itertools.product([-1, 0, 1], repeat=4)), np.int8)
    xq = np.random.default_rng(4).integers(-128, 128, size=(6, 4)).astype(np.int8)
    assert np.array_equal(O.ternary_matmul(xq, w), _brute_acc(xq, w))


def test_matmul_is_sum_pos_minus_sum_neg():
    """dashen-tech.com "BitNet.cpp 深度解析" section 3.1: Y = sum_pos - sum_neg."""
    rng = np.random.default_rng(10)
    xq = rng.integers(-127, 128, size=(4, 1024)).astype(np.int8)
    w = O.ternarize(inputs.weights(64, 1024, seed=5), np.float32(0.016))
    acc = O.ternary_matmul(xq, w)
    x64 = xq.astype(np.int64)
    pos = np.stack([(x64 * (w[n] == 1)).sum(axis=1) for n in range(64)], axis=1)
    neg = np.stack([(x64 * (w[n] == -1)).sum(axis=1) for n in range(64)], axis=1)
    assert np.array_equal(acc, pos - neg)
    # offset form used by integer kernels: dot(x_q, code) - sum(x_q)
    code = (w.astype(np.int64) + 1)
    assert np.array_equal(acc, x64 @ code.T - x64.sum(axis=1, keepdims=True))


def test_matmul_equals_tl2_pair_lookup():
    """youngju.dev section "I2_Sカーネルの内部動作": pair index + 9-entry LUT."""
    table = {int(r[0]): (int(r[1]), int(r[2])) for r in _read_table("tl2_pair_table.txt")}
    wts = _golden_comment("tl2_pair_table.txt", "weights")
    idx = _golden_comment("tl2_pair_table.txt", "indices")
    enc = [(wts[i] + 1) * 3 + (wts[i + 1] + 1) for i in range(0, len(wts), 2)]
    assert enc == idx
    for i, (c0, c1) in table.items():      # the table is the encoding's inverse
        assert (c0 + 1) * 3 + (c1 + 1) == i

    def tl2_dot(a, w):
        total = 0
        for i in range(0, len(a), 2):
            lut = [table[j][0] * int(a[i]) + table[j][1] * int(a[i + 1]) for j in range(9)]
            total += lut[(int(w[i]) + 1) * 3 + (int(w[i + 1]) + 1)]
        return total

    rng = np.random.default_rng(42)
    a = rng.integers(-127, 128, size=8).astype(np.int8)
    w = np.array(wts, np.int8)
    assert O.ternary_matmul(a[None], w[None])[0, 0] == tl2_dot(a, w)
    xq = rng.integers(-128, 128, size=(3, 64)).astype(np.int8)
    W = rng.integers(-1, 2, size=(5, 64)).astype(np.int8)
    acc = O.ternary_matmul(xq, W)
    for m in range(3):
        for n in range(5):
            assert acc[m, n] == tl2_dot(xq[m], W[n])


# --------------------------------------------------------------------------
# step 4 and the composed linear
# --------------------------------------------------------------------------
def test_linear_all_zero_weights_give_zero():
    x = inputs.activations((4, 64), seed=3)
    out = O.linear_from_float(np.zeros((9, 64), np.float32), x)
    assert not out["acc"].any()
    assert np.all(out["y32"] == 0) and np.all((out["y"] & 0x7FFF) == 0)


def test_linear_all_plus_one_weights_closed_form():
    x = inputs.activations((4, 64), seed=3)
    c = np.float32(0.03)
    out = O.linear_from_float(np.full((6, 64), c, np.float32), x)
    q, s, rs = O.act_quant(x)
    assert out["gamma"] == c
    assert np.array_equal(out["acc"], np.repeat(rs[:, None].astype(np.int64), 6, axis=1))
    expect = rs.astype(np.float32) * (c / s)
    assert np.array_equal(out["y32"], np.repeat(expect[:, None], 6, axis=1))


def test_linear_dequant_exact_cases_and_odd_symmetry():
    # gamma = s gives d = 1 exactly, y32 = acc
    b, y32 = O.dequant(np.array([[5, -7, 0, 2**20]]), np.float32(2.5), np.array([2.5], np.float32))
    assert y32.tolist() == [[5.0, -7.0, 0.0, 2.0**20]]
    x = inputs.activations((3, 128), seed=8)
    W = inputs.weights(10, 128, seed=9)
    a = O.linear_from_float(W, x)
    b = O.linear_from_float(W, x ^ np.uint16(0x8000))
    assert np.array_equal(b["y32"], -a["y32"])


def test_linear_matches_float64_reference_within_bound():
    """The integer path equals F.linear on the dequantised operands: with exact
    integer acc the only error is the two fp32 roundings of the dequant."""
    x, W = inputs.single_layer()
    out = O.linear_from_float(W, x)
    w = O.unpack_i2s(out["packed"], 512).astype(np.float64)
    xq = out["xq"].astype(np.float64)
    ref = (xq @ w.T) * (float(out["gamma"]) / out["s"].astype(np.float64))[:, None]
    rel = np.abs(out["y32"] - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= 2 * 2.0**-24 + 1e-12
    assert out["y"].shape == (8, 400)


# --------------------------------------------------------------------------
# step 5: the FFN block
# --------------------------------------------------------------------------
def _ffn_literal_f64(x_bits, Wg, Wu, Wd, n1, n2, eps):
    """Unfolded float64 form: RMSNorm -> quant -> BitLinear -> ReLU^2*up ->
    RMSNorm -> quant -> BitLinear, quantising the normalised values."""
    xf = O.bf16_bits_to_f32(x_bits).astype(np.float64)

    def rms(v, g):
        return v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + eps) * g

    def quant(v):
        s = 127.0 / np.maximum(np.abs(v).max(axis=1, keepdims=True), 1e-5)
        return np.clip(np.rint(v * s), -128, 127), s

    def bitlin(v, W):
        p, g = O.pack_weights(W)
        w = O.unpack_i2s(p, W.shape[1]).astype(np.float64)
        q, s = quant(v)
        return (q @ w.T) * float(g) / s, q

    xn = rms(xf, n1)
    g, q1 = bitlin(xn, Wg)
    u, _ = bitlin(xn, Wu)
    h = np.maximum(g, 0) ** 2 * u
    y, q2 = bitlin(rms(h, n2), Wd)
    return y, q1, q2


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_ffn_fold_matches_literal_float64(seed):
    H, I = 64, 128
    rng = np.random.default_rng(seed)
    x = inputs.activations((3, H), rng=rng)
    Wg, Wu, Wd = (inputs.weights(I, H, rng=rng), inputs.weights(I, H, rng=rng),
                  inputs.weights(H, I, rng=rng))
    n1 = (1 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    n2 = (1 + 0.1 * rng.standard_normal(I)).astype(np.float32)
    out = O.ffn(x, O.pack_weights(Wg), O.pack_weights(Wu), O.pack_weights(Wd), n1, n2, 1e-5)
    y, q1, q2 = _ffn_literal_f64(x, Wg, Wu, Wd, n1.astype(np.float64),
                                 n2.astype(np.float64), float(np.float32(1e-5)))
    assert np.array_equal(q1, out["q1"])
    assert np.array_equal(q2, out["q2"])
    rel = np.abs(out["y32"] - y) / np.maximum(np.abs(y), 1e-30)
    assert rel[np.abs(y) > 0].max() < 1e-5
    assert np.array_equal(out["y32"] == 0, y == 0)


def test_ffn_scale_invariances_and_zero_cases():
    H, I = 64, 96
    rng = np.random.default_rng(21)
    x = inputs.activations((4, H), rng=rng)
    G, U, D = (O.pack_weights(inputs.weights(I, H, rng=rng)),
               O.pack_weights(inputs.weights(I, H, rng=rng)),
               O.pack_weights(inputs.weights(H, I, rng=rng)))
    # with eps = 0 RMSNorm removes any positive per-token scale exactly, so a
    # 2^k scale of x and a constant first-norm gain must both cancel
    base = O.ffn(x, G, U, D, eps=0.0)
    xs = O.f32_to_bf16_bits(O.bf16_bits_to_f32(x) * np.float32(8.0))
    for other in (O.ffn(xs, G, U, D, eps=0.0),
                  O.ffn(x, G, U, D, norm1_w=np.full(H, 2.0, np.float32), eps=0.0)):
        rel = np.abs(other["y32"] - base["y32"]) / np.maximum(np.abs(base["y32"]), 1e-30)
        assert rel.max() < 1e-5
    # the second norm's statistic is taken before its gain, so a constant gain
    # c = 4 leaves the codes alone and scales y by exactly 4 (s2 moves by 2^-2)
    o2 = O.ffn(x, G, U, D, norm2_w=np.full(I, 4.0, np.float32), eps=0.0)
    assert np.array_equal(o2["q2"], base["q2"])
    assert np.array_equal(o2["y32"], base["y32"] * np.float32(4.0))
    # all -1 gate with a non-negative token: acc_g <= 0 -> relu 0 -> y == 0
    xpos = O.f32_to_bf16_bits(np.abs(O.bf16_bits_to_f32(x)))
    Gneg = O.pack_weights(np.full((I, H), -0.02, np.float32))
    assert not O.ffn(xpos, Gneg, U, D)["y32"].any()
    # all-zero down projection -> y == 0
    Dz = O.pack_weights(np.zeros((H, I), np.float32))
    assert not O.ffn(x, G, U, Dz)["y32"].any()
