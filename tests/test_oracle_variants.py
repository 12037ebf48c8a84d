"""Pins of the variant oracles (oracle/variants.py) to what the pages and the
mathematics fix, independent of the oracle's own code paths:

BitNet v1 W1A8 (youngju.dev "BitNet論文分析", section "BitNet v1：BitLinearの誕生"):
  the sign rule with W = 0 -> +1, a hand-packed byte, alpha = mean |W|, the
  identity x.W_b = 2 sum_{+1} x - sum x, brute force on tiny shapes, the
  all-positive / all-negative closed forms, and the cross-check that a +-1
  matrix stored as I2_S ternary codes gives the same result through the
  W1.58A8 oracle.

BitNet a4.8 (same page, section "BitNet a4.8：ハイブリッド量子化戦略"):
  a hand-computed token (including two .5 ties), the n_out = K case that
  reduces exactly to the 8-bit W1.58A8 path, selection by brute force
  (every outlier at least as large as every inlier, ties to the lower index),
  disjoint supports, power-of-two scale invariance and the all-(+1)
  closed form.
"""
from __future__ import annotations

import itertools

import numpy as np
import pytest

from oracle import bitlinear as O
from oracle import variants as V
from ternary_weight_linear_int8_b200 import inputs


def _bf16(vals):
    return O.f32_to_bf16_bits(np.asarray(vals, np.float32))


# ------------------------------------------------------------- BitNet v1
def test_sign_rule_zero_is_plus_one():
    W = np.array([[0.0, -0.0, 1e-30, -1e-30, 3.0, -2.0, 0.5, -0.5]], np.float32)
    assert V.sign_binarize(W).tolist() == [[1, 1, 1, -1, 1, -1, 1, -1]]


def test_w1_hand_packed_byte_and_round_trip():
    wb = np.array([[1, -1, -1, 1, 1, 1, -1, -1]], np.int8)
    # bit k = weight k, 1 for +1: 0b00111001
    assert V.pack_w1(wb).tolist() == [[0x39]]
    rng = np.random.default_rng(1)
    wb = np.where(rng.random((7, 64)) < 0.5, 1, -1).astype(np.int8)
    p = V.pack_w1(wb)
    assert p.shape == (7, 8)
    assert np.array_equal(V.unpack_w1(p, 64), wb)
    assert np.array_equal(V.pack_w1(np.ones((2, 16), np.int8)), np.full((2, 2), 0xFF, np.uint8))
    assert np.array_equal(V.pack_w1(-np.ones((2, 16), np.int8)), np.zeros((2, 2), np.uint8))


def test_w1_alpha_is_mean_abs():
    W = np.full((4, 16), -0.25, np.float32)
    assert V.pack_weights_w1(W)[1] == np.float32(0.25)
    W = np.array([[1.0, -3.0, 0.5, 0.5, -1.0, 2.0, 0.0, 0.0]], np.float32)
    assert V.pack_weights_w1(W)[1] == np.float32(1.0)          # 8 / 8


def _dot64(xq, wb):
    return np.array([[sum(int(a) * int(b) for a, b in zip(xr, wr)) for wr in wb] for xr in xq])


def test_w1_matmul_brute_force_and_sum_identity():
    rng = np.random.default_rng(2)
    for M, N, K in [(1, 1, 8), (3, 5, 16), (2, 7, 24)]:
        x = inputs.activations((M, K), rng=rng)
        W = rng.standard_normal((N, K)).astype(np.float32)
        p, a = V.pack_weights_w1(W)
        out = V.linear_w1(p, a, x)
        wb = np.where(W >= 0, 1, -1)
        assert np.array_equal(out["acc"], _dot64(out["xq"], wb))
        pos = np.array([[int(out["xq"][m][wb[n] == 1].astype(np.int64).sum()) for n in range(N)]
                        for m in range(M)])
        assert np.array_equal(out["acc"], 2 * pos - out["rowsum"][:, None])


def test_w1_all_eight_sign_patterns_k8():
    xq_rows = inputs.activations((4, 8), seed=3)
    for signs in itertools.product((-1.0, 1.0), repeat=8):
        W = np.array([signs], np.float32)
        out = V.linear_w1(*V.pack_weights_w1(W), xq_rows)
        assert np.array_equal(out["acc"][:, 0], out["xq"].astype(np.int64) @ np.array(signs, np.int64))


def test_w1_closed_forms():
    x = inputs.activations((3, 64), seed=4)
    c = np.float32(0.02)
    pos = V.linear_w1(*V.pack_weights_w1(np.full((5, 64), c, np.float32)), x)
    assert np.array_equal(pos["acc"], np.repeat(pos["rowsum"][:, None], 5, axis=1))
    want = (pos["rowsum"].astype(np.float32) * (c / pos["s"]))[:, None]
    assert np.array_equal(pos["y32"], np.repeat(want, 5, axis=1))
    neg = V.linear_w1(*V.pack_weights_w1(np.full((5, 64), -c, np.float32)), x)
    assert np.array_equal(neg["acc"], -pos["acc"])


def test_w1_equals_ternary_path_on_the_same_signs():
    """A +-1 matrix is a ternary matrix: stored as I2_S codes with gamma = alpha
    it must give the W1.58A8 oracle's result bit for bit."""
    rng = np.random.default_rng(5)
    x = inputs.activations((4, 256), rng=rng, outliers=True)
    W = inputs.weights(33, 256, rng=rng)
    p1, alpha = V.pack_weights_w1(W)
    w1 = V.linear_w1(p1, alpha, x)
    t = O.linear(O.pack_i2s(V.sign_binarize(W)), alpha, x)
    for k in ("acc", "y32", "y"):
        assert np.array_equal(w1[k], t[k])


# ------------------------------------------------------------- BitNet a4.8
def test_a48_hand_computed_token():
    x = _bf16([[0.5, -4.0, 1.0, 3.5, -0.25, 2.0, 0.0, 8.0]])
    q4, s4, q8, s8, mask = V.act_quant_a48(x, 2)
    assert mask.tolist() == [[False, True, False, False, False, False, False, True]]
    # inlier max 3.5 -> s4 = 2: 0.5->1, 1->2, 3.5->7, -0.25 -> -0.5 -> tie -> 0, 2->4
    assert s4[0] == np.float32(2.0)
    assert q4.tolist() == [[1, 0, 2, 7, 0, 4, 0, 0]]
    # outlier max 8 -> s8 = 15.875: 8 -> 127, -4 -> -63.5 -> tie -> -64
    assert s8[0] == np.float32(15.875)
    assert q8.tolist() == [[0, -64, 0, 0, 0, 0, 0, 127]]


def test_a48_all_outliers_is_the_8bit_path():
    rng = np.random.default_rng(6)
    x = inputs.activations((3, 128), rng=rng, outliers=True)
    W = inputs.weights(40, 128, rng=rng)
    p, g = O.pack_weights(W)
    out = V.linear_a48(p, g, x, 128)
    ref = O.linear(p, g, x)
    assert not out["q4"].any()
    assert np.array_equal(out["q8"], ref["xq"])
    assert np.array_equal(out["acc8"], ref["acc"])
    assert np.array_equal(out["y32"], ref["y32"])


def test_a48_no_outliers_uses_seven_levels():
    x = inputs.activations((4, 64), seed=7)
    q4, s4, q8, s8, mask = V.act_quant_a48(x, 0)
    assert not q8.any() and not mask.any()
    xf = O.bf16_bits_to_f32(x)
    for t in range(4):
        i = int(np.argmax(np.abs(xf[t])))
        assert abs(int(q4[t, i])) == 7
    assert np.abs(q4).max() <= 7


@pytest.mark.parametrize("n_out", [1, 3, 5])
def test_a48_selection_by_brute_force(n_out):
    # magnitudes with ties: equal |x| must go to the lower index
    x = _bf16([[1.0, -2.0, 2.0, 0.5, -2.0, 3.0, 1.0, -0.25],
               [4.0, 4.0, -4.0, 4.0, 1.0, 1.0, 1.0, 1.0]])
    mask = V.outlier_mask(x, n_out)
    ax = np.abs(O.bf16_bits_to_f32(x))
    for t in range(2):
        assert mask[t].sum() == n_out
        sel, rest = ax[t][mask[t]], ax[t][~mask[t]]
        assert sel.min() >= rest.max()
        thr = sel.min()
        ties = np.flatnonzero(ax[t] == thr)
        chosen = [i for i in ties if mask[t, i]]
        assert chosen == sorted(ties)[: len(chosen)]
    assert V.outlier_mask(x, 3)[1].tolist() == [True, True, True, False, False, False, False, False]


def test_a48_supports_disjoint_and_scale_invariant():
    x = inputs.activations((5, 256), seed=8, outliers=True)
    q4, s4, q8, s8, mask = V.act_quant_a48(x, 3)
    assert not np.any((q4 != 0) & mask) and not np.any((q8 != 0) & ~mask)
    xs = O.f32_to_bf16_bits(O.bf16_bits_to_f32(x) * np.float32(0.125))
    q4b, _, q8b, _, maskb = V.act_quant_a48(xs, 3)
    assert np.array_equal(q4, q4b) and np.array_equal(q8, q8b) and np.array_equal(mask, maskb)


def test_a48_all_plus_one_closed_form():
    x = inputs.activations((3, 64), seed=9, outliers=True)
    c = np.float32(0.02)
    p, g = O.pack_weights(np.full((6, 64), c, np.float32))
    out = V.linear_a48(p, g, x, 2)
    assert np.array_equal(out["acc4"], np.repeat(out["rowsum4"][:, None], 6, axis=1))
    assert np.array_equal(out["acc8"], np.repeat(out["rowsum8"][:, None], 6, axis=1))
    want = (out["rowsum4"].astype(np.float32) * (g / out["s4"])) + \
           (out["rowsum8"].astype(np.float32) * (g / out["s8"]))
    assert np.array_equal(out["y32"], np.repeat(want[:, None], 6, axis=1))
