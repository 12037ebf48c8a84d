"""Plant plausible mistakes in the oracle (on the CPU, via monkeypatch) and
check that the pins catch each one.  This guards the pins themselves."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import bitlinear as O
from tests import test_oracle_pins as P


def _act_quant_qb128(xf):
    xf = np.asarray(xf, dtype=np.float32)
    a = np.abs(xf).max(axis=1)
    s = np.float32(128.0) / np.maximum(a, O.EPS_F32)
    q = np.clip(np.rint(xf * s[:, None]), -128, 127).astype(np.int8)
    return q, s, q.astype(np.int64).sum(axis=1).astype(np.int32)


def _act_quant_trunc(xf):
    xf = np.asarray(xf, dtype=np.float32)
    s = O.QMAX_F32 / np.maximum(np.abs(xf).max(axis=1), O.EPS_F32)
    q = np.clip(np.trunc(xf * s[:, None]), -128, 127).astype(np.int8)
    return q, s, q.astype(np.int64).sum(axis=1).astype(np.int32)


def _ternarize_no_eps(W, gamma):
    return np.clip(np.rint(np.asarray(W, np.float32) / np.float32(gamma)), -1, 1).astype(np.int8)


def _pack_msb_first(w):
    w = np.asarray(w, dtype=np.int8)
    N, K = w.shape
    c = (w.astype(np.int16) + 1).astype(np.uint8).reshape(N, K // 4, 4)
    return (c[..., 3] | (c[..., 2] << 2) | (c[..., 1] << 4) | (c[..., 0] << 6)).astype(np.uint8)


def _code_map_shifted(w):
    w = np.asarray(w, dtype=np.int8)
    N, K = w.shape
    c = (w.astype(np.int16) + 2).astype(np.uint8) & 3
    c = c.reshape(N, K // 4, 4)
    return (c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)).astype(np.uint8)


def _dequant_mul(acc, gamma, s):
    d = np.float32(gamma) * np.asarray(s, np.float32)
    y32 = np.asarray(acc).astype(np.float32) * d[:, None]
    return O.f32_to_bf16_bits(y32), y32


def _gamma_mean_sq(W):
    a = np.asarray(W, np.float64)
    return np.float32(np.sqrt(np.mean(a * a)))


_ORIG_MATMUL = O.ternary_matmul


def _matmul_drop_neg(xq, w):
    return _ORIG_MATMUL(xq, np.maximum(w, 0))


def _bf16_truncate(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _ffn_r1_squared(*a, **k):
    out = _ORIG_FFN(*a, **k)
    # emulate a dropped power of r1 in the folded scale
    out = dict(out)
    out["y32"] = out["y32"] * (1.0 / out["r1"]).astype(np.float32)[:, None]
    return out


def _ffn_no_relu(x_bits, gate, up, down, norm1_w=None, norm2_w=None, eps=1e-5):
    xf = O.bf16_bits_to_f32(x_bits)
    H = xf.shape[1]
    I = gate[0].shape[0]
    n1 = np.ones(H, np.float32) if norm1_w is None else np.asarray(norm1_w, np.float32)
    n2 = np.ones(I, np.float32) if norm2_w is None else np.asarray(norm2_w, np.float32)
    e = float(np.float32(eps))
    r1 = 1.0 / np.sqrt(np.mean(xf.astype(np.float64) ** 2, axis=1) + e)
    q1, s1, rs1 = O.act_quant_f32(xf * n1)
    g = O.ternary_matmul(q1, O.unpack_i2s(gate[0], H)).astype(np.float32) * (np.float32(gate[1]) / s1)[:, None]
    u = O.ternary_matmul(q1, O.unpack_i2s(up[0], H)).astype(np.float32) * (np.float32(up[1]) / s1)[:, None]
    h = (g * g) * u
    q2, s2, rs2 = O.act_quant_f32(h * n2)
    acc = O.ternary_matmul(q2, O.unpack_i2s(down[0], I))
    r2 = 1.0 / np.sqrt(r1 ** 6 * np.mean(h.astype(np.float64) ** 2, axis=1) + e)
    f = (r1 ** 3 * r2).astype(np.float32)
    y32 = (acc.astype(np.float32) * (np.float32(down[1]) / s2)[:, None]) * f[:, None]
    return {"q1": q1, "q2": q2, "y32": y32, "r1": r1, "h": h}


_ORIG_FFN = O.ffn

MUTATIONS = [
    ("act_quant_f32", _act_quant_qb128, [P.test_act_quant_hand_computed_rows]),
    ("act_quant_f32", _act_quant_trunc, [P.test_act_quant_hand_computed_rows]),
    ("ternarize", _ternarize_no_eps, [P.test_ternarize_closed_forms]),
    ("pack_i2s", _pack_msb_first, [P.test_i2s_code_map_golden]),
    ("pack_i2s", _code_map_shifted, [P.test_i2s_code_map_golden]),
    ("dequant", _dequant_mul, [P.test_linear_all_plus_one_weights_closed_form]),
    ("absmean_gamma", _gamma_mean_sq, [P.test_gamma_constant_and_known_means]),
    ("ternary_matmul", _matmul_drop_neg, [P.test_matmul_is_sum_pos_minus_sum_neg]),
    ("f32_to_bf16_bits", _bf16_truncate, [P.test_bf16_rounding_pins]),
    ("ffn", _ffn_r1_squared, [lambda: P.test_ffn_fold_matches_literal_float64(0)]),
    ("ffn", _ffn_no_relu, [lambda: P.test_ffn_fold_matches_literal_float64(0)]),
]


@pytest.mark.parametrize("name,mutant,pins", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(O, name, mutant)
    caught = False
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, KeyError):
            caught = True
    assert caught, f"no pin failed with the mutant {mutant.__name__} in {name}"
