"""CPU oracle for two variants of BitLinear that the pages describe next to
W1.58A8: BitNet v1 (1-bit sign weights, W1A8) and BitNet a4.8 (4-bit
activations with an 8-bit split for the largest values).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import this module.  It shares no code with the CUDA library
and imports nothing from it; it reuses the W1.58A8 oracle's steps
(``oracle.bitlinear``) where the variants share them.

BitNet v1 -- youngju.dev "BitNet論文分析：1-Bit LLMの時代", section
"BitNet v1：BitLinearの誕生" > "1-Bit重みとSign関数":
  * W_b = +1 where W >= 0 and -1 where W < 0 (the page's formula; its listing
    calls ``sign()``, which would map 0 to 0 and is not a 1-bit code, so the
    formula is taken);
  * alpha = (1/nm) * sum |W_ij| (the same mean as gamma of b1.58, computed the
    same exact way);
  * activations: absmax quantisation to 8-bit integers.  The v1 listing takes
    the absmax over the whole tensor; this library keeps one activation
    quantiser for every weight format, the per-token one of b1.58 (the two
    agree for a single token, the decode case);
  * output = (x_q . W_b) * alpha / s, i.e. d = alpha / s and y32 = fp32(acc) * d,
    the same dequantisation order as W1.58A8.
  * storage (not on the pages): 8 weights per byte along K, weight k at bit
    k % 8 of byte k // 8 (least significant bit first, like I2_S), bit 1 for
    +1 and 0 for -1.

BitNet a4.8 -- same youngju.dev page, section "BitNet a4.8：ハイブリッド量子化戦略":
ternary (1.58-bit) weights; per token the largest-magnitude values are split
off and quantised at 8 bits, the rest at 4 bits.  The pages give neither the
fraction nor the scales, so the plainest reading is taken:
  * outliers = the ``n_out`` values of largest |x| in the token (ties between
    equal |x| go to the lower channel index); ``n_out`` is an argument;
  * inliers: s4 = 7 / max(max |x_inlier|, 1e-5), q4 = clamp(rint(x * s4), -8, 7),
    zero at outlier channels;
  * outliers: s8 = 127 / max(max |x_outlier|, 1e-5), q8 = clamp(rint(x * s8),
    -128, 127), zero at inlier channels;
  * acc4 = q4 . W_q, acc8 = q8 . W_q (exact integers), d4 = gamma / s4,
    d8 = gamma / s8 (fp32 divisions), y32 = fp32(fp32(acc4) * d4) + fp32(fp32(acc8) * d8)
    (two fp32 products, then one fp32 sum), y = bf16(y32).
  The page's second technique, per-channel scaling, is given without any
  formula and is not applied.
"""
from __future__ import annotations

import numpy as np

from . import bitlinear as O

Q4_MAX = np.float32(7.0)


# --------------------------------------------------------------------------
# BitNet v1: sign weights, 1 bit each
# --------------------------------------------------------------------------
def sign_binarize(W: np.ndarray) -> np.ndarray:
    """W_b = +1 where W >= 0 (including -0.0), -1 where W < 0; int8."""
    W = np.asarray(W, dtype=np.float32)
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    return np.where(W >= np.float32(0.0), 1, -1).astype(np.int8)


def pack_w1(wb: np.ndarray) -> np.ndarray:
    """Pack +-1 weights [N, K] (K % 8 == 0): bit k % 8 of byte k // 8 is 1 for +1."""
    wb = np.asarray(wb, dtype=np.int8)
    N, K = wb.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    if not np.all((wb == 1) | (wb == -1)):
        raise ValueError("weights must be +-1")
    bits = (wb == 1).astype(np.uint8).reshape(N, K // 8, 8)
    out = np.zeros((N, K // 8), np.uint8)
    for i in range(8):
        out |= (bits[..., i] << i).astype(np.uint8)
    return out


def unpack_w1(packed: np.ndarray, K: int) -> np.ndarray:
    """Inverse of pack_w1: int8 +-1 [N, K]."""
    p = np.asarray(packed, dtype=np.uint8)
    N = p.shape[0]
    bits = np.stack([(p >> i) & 1 for i in range(8)], axis=-1).reshape(N, K)
    return (2 * bits.astype(np.int8) - 1).astype(np.int8)


def pack_weights_w1(W: np.ndarray):
    """(packed uint8 [N, K/8], alpha fp32): alpha = mean |W| (exact, one rounding)."""
    return pack_w1(sign_binarize(W)), O.absmean_gamma(W)


def linear_w1(packed: np.ndarray, alpha: np.float32, x_bits: np.ndarray):
    """W1A8 forward: per-token int8 activations, +-1 weights, y = acc * alpha / s."""
    K = np.asarray(x_bits).shape[1]
    xq, s, rowsum = O.act_quant(x_bits)
    acc = O.ternary_matmul(xq, unpack_w1(packed, K))
    y_bits, y32 = O.dequant(acc, alpha, s)
    return {"xq": xq, "s": s, "rowsum": rowsum, "acc": acc, "y32": y32, "y": y_bits}


# --------------------------------------------------------------------------
# BitNet a4.8: 4-bit activations with the largest values at 8 bits
# --------------------------------------------------------------------------
def outlier_mask(x_bits: np.ndarray, n_out: int) -> np.ndarray:
    """Boolean [M, K]: per token the n_out channels of largest |x|, ties to the
    lower channel index (a stable sort on -|x|)."""
    xf = O.bf16_bits_to_f32(x_bits)
    M, K = xf.shape
    if not 0 <= n_out <= K:
        raise ValueError("n_out must be in [0, K]")
    mask = np.zeros((M, K), bool)
    for t in range(M):
        order = np.argsort(-np.abs(xf[t]).astype(np.float64), kind="stable")
        mask[t, order[:n_out]] = True
    return mask


def act_quant_a48(x_bits: np.ndarray, n_out: int):
    """Returns q4 int8 [M,K], s4 fp32 [M], q8 int8 [M,K], s8 fp32 [M], mask."""
    xf = O.bf16_bits_to_f32(x_bits)
    M, K = xf.shape
    mask = outlier_mask(x_bits, n_out)
    ax = np.abs(xf)
    a4 = np.where(mask, np.float32(0.0), ax).max(axis=1) if K else np.zeros(M, np.float32)
    a8 = np.where(mask, ax, np.float32(0.0)).max(axis=1) if K else np.zeros(M, np.float32)
    s4 = (Q4_MAX / np.maximum(a4, O.EPS_F32)).astype(np.float32)
    s8 = (O.QMAX_F32 / np.maximum(a8, O.EPS_F32)).astype(np.float32)
    q4 = np.clip(np.rint(xf * s4[:, None]), -8, 7).astype(np.int8)
    q8 = np.clip(np.rint(xf * s8[:, None]), -128, 127).astype(np.int8)
    q4[mask] = 0
    q8[~mask] = 0
    return q4, s4, q8, s8, mask


def linear_a48(packed: np.ndarray, gamma: np.float32, x_bits: np.ndarray, n_out: int):
    """a4.8 forward on I2_S ternary weights; returns every stage."""
    K = np.asarray(x_bits).shape[1]
    q4, s4, q8, s8, mask = act_quant_a48(x_bits, n_out)
    w = O.unpack_i2s(packed, K)
    acc4 = O.ternary_matmul(q4, w)
    acc8 = O.ternary_matmul(q8, w)
    g = np.float32(gamma)
    d4 = g / s4                                                   # fp32 divide
    d8 = g / s8
    y32 = (acc4.astype(np.float32) * d4[:, None]) + (acc8.astype(np.float32) * d8[:, None])
    return {"q4": q4, "s4": s4, "q8": q8, "s8": s8, "mask": mask, "acc4": acc4, "acc8": acc8,
            "rowsum4": q4.astype(np.int64).sum(axis=1), "rowsum8": q8.astype(np.int64).sum(axis=1),
            "y32": y32.astype(np.float32), "y": O.f32_to_bf16_bits(y32)}
