"""Plant plausible mistakes in the variant oracles (on the CPU, via
monkeypatch) and check that the pins in test_oracle_variants catch each."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import bitlinear as O
from oracle import variants as V
from tests import test_oracle_variants as P


def _sign_strict(W):                       # 0 -> -1 instead of +1
    return np.where(np.asarray(W, np.float32) > 0, 1, -1).astype(np.int8)


def _pack_w1_msb_first(wb):
    wb = np.asarray(wb, dtype=np.int8)
    N, K = wb.shape
    bits = (wb == 1).astype(np.uint8).reshape(N, K // 8, 8)
    out = np.zeros((N, K // 8), np.uint8)
    for i in range(8):
        out |= (bits[..., i] << (7 - i)).astype(np.uint8)
    return out


def _mask_ties_high(x_bits, n_out):        # equal |x| go to the higher index
    xf = O.bf16_bits_to_f32(x_bits)
    M, K = xf.shape
    mask = np.zeros((M, K), bool)
    for t in range(M):
        order = np.argsort(-np.abs(xf[t][::-1]).astype(np.float64), kind="stable")
        mask[t, (K - 1 - order)[:n_out]] = True
    return mask


_ORIG_A48 = V.act_quant_a48


def _a48_qb8(x_bits, n_out):               # 4-bit scale 8/a instead of 7/a
    q4, s4, q8, s8, mask = _ORIG_A48(x_bits, n_out)
    xf = O.bf16_bits_to_f32(x_bits)
    a4 = np.where(mask, np.float32(0), np.abs(xf)).max(axis=1)
    s4 = (np.float32(8.0) / np.maximum(a4, O.EPS_F32)).astype(np.float32)
    q4 = np.clip(np.rint(xf * s4[:, None]), -8, 7).astype(np.int8)
    q4[mask] = 0
    return q4, s4, q8, s8, mask


_ORIG_LINEAR_A48 = V.linear_a48


def _a48_one_scale(packed, gamma, x_bits, n_out):   # dequantises both parts with d8
    out = dict(_ORIG_LINEAR_A48(packed, gamma, x_bits, n_out))
    d8 = np.float32(gamma) / out["s8"]
    out["y32"] = ((out["acc4"] + out["acc8"]).astype(np.float32) * d8[:, None]).astype(np.float32)
    return out


MUTATIONS = [
    ("sign_binarize", _sign_strict, [P.test_sign_rule_zero_is_plus_one]),
    ("pack_w1", _pack_w1_msb_first, [P.test_w1_hand_packed_byte_and_round_trip]),
    ("outlier_mask", _mask_ties_high, [lambda: P.test_a48_selection_by_brute_force(3)]),
    ("act_quant_a48", _a48_qb8, [P.test_a48_hand_computed_token]),
    ("linear_a48", _a48_one_scale, [P.test_a48_all_plus_one_closed_form]),
]


@pytest.mark.parametrize("name,mutant,pins", MUTATIONS,
                         ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, mutant, pins):
    monkeypatch.setattr(V, name, mutant)
    caught = False
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, KeyError):
            caught = True
    assert caught, f"no pin failed with the mutant {mutant.__name__} in {name}"
