"""CPU oracle for the BitNet b1.58 BitLinear forward pass (W1.58A8).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import this module.  It shares no code with the CUDA library
and imports nothing from it.

Plain, slow and written to be checked by eye against the pages:

* act quant     -- youngju.dev "BitNet論文分析：1-Bit LLMの時代", section
                   "Absmean量子化関数", method ``activation_quant`` of
                   ``BitLinear_b158`` (per-token absmax, round, clamp); the
                   8-bit absmax reading of reinforz.co.jp "BitNet b1.58 2B4T",
                   section "積極的量子化と三値化がもたらす学習効率の革新".
* absmean ternary quant -- same youngju.dev page and section, function
                   ``weight_quant_ternary`` (gamma = mean|W|, round(W/(gamma+eps)),
                   clamp to [-1, 1]).
* I2_S packing  -- youngju.dev page, section "bitnet.cpp推論フレームワーク" >
                   "アーキテクチャ概要" (codes 00=-1, 01=0, 10=+1, 16 weights per
                   32-bit register); dashen-tech.com "BitNet.cpp 深度解析",
                   section "2.3 I2_S 形式：実際の保存は 2-bit" (8 weights in 16 bits).
* ternary matmul -- dashen-tech.com page, section "3.1 計算コア：整数行列乗算"
                   (Y = sum_pos - sum_neg); youngju.dev ``F.linear(x_q, w_q)``.
* dequant       -- youngju.dev ``BitLinear_b158.forward`` (scale restore).
* FFN block     -- abeam.tech review of "BitNet: 1-bit Pre-training for Large
                   Language Models", sections "モデル構造" (LLaMA-like, RMSNorm,
                   SwiGLU-shaped FFN) and "正規化で分散を安定させる" (subln
                   before BitLinear); reinforz.co.jp page, section
                   "BitNetが実現したCPU上での高効率AI処理" (ReLU^2).

Readings taken where the pages are silent or disagree (each one is listed
with its reason in the design notes):

* activation scale s = 127 / max(max|x|, 1e-5) (the youngju.dev listing uses
  Qb=128 and (gamma+1e-5); we take the 127 / max form), codes clamped to
  [-128, 127];
* rounding is round-half-to-even everywhere (``torch.round`` semantics);
* gamma is the fp32 value nearest (ties to even) to the exact real mean of
  |W| -- one rounding, no summation-order dependence;
* dequant: d = gamma / s (fp32 division, once per token), y32 = fp32(acc) * d,
  y = bf16(y32) rounded to nearest even;
* bit order inside a packed byte: weight k sits at bits 2*(k mod 4) of byte
  k // 4 (LSB first); code 11 is never produced;
* FFN: h = ReLU(gate)^2 * up, no residual, RMSNorm gains default 1.  The
  RMSNorm factor r is a positive per-token scale and absmax quantisation is
  invariant to it, so the token is quantised before multiplying by r and r is
  carried into the dequant scale ("fold").

Floating point: every fp32 step below is a single correctly rounded numpy
float32 operation (numpy never contracts a*b+c into an FMA); RMSNorm
statistics are taken in fp64.  Integer accumulators are exact.
"""
from __future__ import annotations

import numpy as np

EPS_F32 = np.float32(1e-5)      # the fp32 value nearest to 1e-5
QMAX_F32 = np.float32(127.0)


# --------------------------------------------------------------------------
# bf16 <-> fp32 (the oracle's own conversion, independent of the input module)
# --------------------------------------------------------------------------
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32: exact, the bits move up 16."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest with ties to even; returns uint16 bits.

    Adding 0x7FFF plus the lowest kept bit to the fp32 bit pattern and
    truncating implements round-to-nearest-even for finite values.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


# --------------------------------------------------------------------------
# Step 1: per-token absmax int8 activation quantisation
# --------------------------------------------------------------------------
def act_quant_f32(xf: np.ndarray):
    """Quantise fp32 rows: returns (x_q int8 [M,K], s fp32 [M], rowsum int32 [M]).

    a_t = max_k |x|;  s_t = 127 / max(a_t, 1e-5)  (fp32 division);
    x_q = clamp(rint(x * s_t), -128, 127)  (one fp32 multiply, ties to even).
    """
    xf = np.asarray(xf, dtype=np.float32)
    M, K = xf.shape
    a = np.abs(xf).max(axis=1) if K > 0 else np.zeros(M, np.float32)
    s = QMAX_F32 / np.maximum(a, EPS_F32)                      # fp32 / fp32
    prod = xf * s[:, None]                                     # fp32 * fp32
    q = np.clip(np.rint(prod), -128, 127).astype(np.int8)
    rowsum = q.astype(np.int64).sum(axis=1).astype(np.int32)
    return q, s.astype(np.float32), rowsum


def act_quant(x_bits: np.ndarray):
    """Quantise bf16 activations given as uint16 bits, shape [M, K]."""
    return act_quant_f32(bf16_bits_to_f32(x_bits))


# --------------------------------------------------------------------------
# Step 2: absmean ternary quantisation and I2_S 2-bit packing
# --------------------------------------------------------------------------
def round_rational_to_f32(num: int, den: int) -> np.float32:
    """The fp32 value nearest to num/den (num >= 0, den > 0), ties to even.

    Exact integer arithmetic: find the binade, take a 24-bit quotient (or the
    subnormal grid 2^-149), round on the remainder.
    """
    if num < 0 or den <= 0:
        raise ValueError("round_rational_to_f32 needs num >= 0, den > 0")
    if num == 0:
        return np.float32(0.0)
    # e such that 2^e <= num/den < 2^(e+1)
    e = num.bit_length() - den.bit_length()
    if (num << max(0, -e)) < (den << max(0, e)):
        e -= 1
    e = max(e, -126)                       # below 2^-126 use the subnormal grid
    shift = 23 - e                         # quotient scaled to 2^23..2^24
    if shift >= 0:
        q, rem = divmod(num << shift, den)
        rden = den
    else:
        q, rem = divmod(num, den << (-shift))
        rden = den << (-shift)
    twice = 2 * rem
    if twice > rden or (twice == rden and (q & 1)):
        q += 1
    if q >= (1 << 24):                     # rounding carried into next binade
        q >>= 1
        e += 1
    if e > 127:
        return np.float32(np.inf)
    val = float(q) * (2.0 ** (e - 23))     # exact in fp64 (q < 2^25)
    out = np.float32(val)
    if float(out) != val:
        raise AssertionError("internal: value not representable in fp32")
    return out


def absmean_gamma(W: np.ndarray) -> np.float32:
    """gamma = mean|W| as the fp32 nearest to the exact real mean.

    Each fp32 |w| equals m * 2^(e-150) with an integer mantissa m (hidden bit
    included) and biased exponent e (e=1 for subnormals), so the exact sum is
    an integer multiple of 2^-149; it is built with Python integers and
    divided by N*K with one rounding.
    """
    a = np.abs(np.asarray(W, dtype=np.float32)).ravel()
    count = a.size
    if count == 0:
        raise ValueError("empty weight matrix")
    bits = a.view(np.uint32)
    exp = (bits >> np.uint32(23)) & np.uint32(0xFF)
    if np.any(exp == 0xFF):
        raise ValueError("non-finite weight")
    total = 0                              # exact sum, in units of 2^-149
    chunk = 1 << 26
    for c0 in range(0, count, chunk):
        b = bits[c0:c0 + chunk]
        e = exp[c0:c0 + chunk]
        man = (b & np.uint32(0x7FFFFF)) | np.where(e > 0, np.uint32(0x800000), np.uint32(0))
        eb = np.maximum(e, np.uint32(1))
        # per-exponent mantissa sums: every partial sum is an integer below
        # 2^26 * 2^24 = 2^50, so the float64 accumulation is exact
        sums = np.bincount(eb, weights=man.astype(np.float64), minlength=256)
        for k in np.flatnonzero(sums):
            total += int(sums[k]) << int(k - 1)
    return round_rational_to_f32(total, count << 149)


def ternarize(W: np.ndarray, gamma: np.float32) -> np.ndarray:
    """w = clamp(rint(W / (gamma + 1e-5)), -1, 1), all fp32 steps; int8 out."""
    W = np.asarray(W, dtype=np.float32)
    den = np.float32(gamma) + EPS_F32                          # fp32 add
    t = W / den                                                # fp32 divide
    return np.clip(np.rint(t), -1, 1).astype(np.int8)


def pack_i2s(w: np.ndarray) -> np.ndarray:
    """Pack ternary w [N,K] (K % 4 == 0) as codes w+1, 4 per byte, LSB first."""
    w = np.asarray(w, dtype=np.int8)
    N, K = w.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    code = (w.astype(np.int16) + 1).astype(np.uint8)
    if np.any(code > 2):
        raise ValueError("weights must be ternary")
    c = code.reshape(N, K // 4, 4)
    return (c[..., 0] | (c[..., 1] << 2) | (c[..., 2] << 4) | (c[..., 3] << 6)).astype(np.uint8)


def unpack_i2s(packed: np.ndarray, K: int) -> np.ndarray:
    """Inverse of pack_i2s: int8 ternary [N, K].  Code 3 is rejected."""
    p = np.asarray(packed, dtype=np.uint8)
    N = p.shape[0]
    codes = np.stack([(p >> (2 * i)) & 3 for i in range(4)], axis=-1).reshape(N, K)
    if np.any(codes == 3):
        raise ValueError("invalid code 11")
    return (codes.astype(np.int8) - 1).astype(np.int8)


def pack_weights(W: np.ndarray):
    """Full step 2: (packed uint8 [N, K/4], gamma fp32)."""
    g = absmean_gamma(W)
    return pack_i2s(ternarize(W, g)), g


# --------------------------------------------------------------------------
# Step 3: ternary integer matmul
# --------------------------------------------------------------------------
def ternary_matmul(xq: np.ndarray, w: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k x_q[m, k] * w[n, k], exact, int64 [M, N].

    A floating-point matrix product is used as a library step: every product
    and every partial sum is an integer of magnitude at most 128*K, below
    2^24 (fp32) or 2^53 (fp64), so any summation order gives the exact
    integer result.
    """
    xq = np.asarray(xq, dtype=np.int8)
    w = np.asarray(w, dtype=np.int8)
    K = xq.shape[1]
    if 128 * K >= 2 ** 53:
        raise ValueError("K too large for an exact floating-point product")
    # fp32 when every partial sum is an integer below 2^24 (then also exact)
    ft = np.float32 if 128 * K < 2 ** 24 else np.float64
    acc = xq.astype(ft) @ w.astype(ft).T
    return acc.astype(np.int64)


# --------------------------------------------------------------------------
# Step 4: dequantisation and bf16 store
# --------------------------------------------------------------------------
def dequant(acc: np.ndarray, gamma: np.float32, s: np.ndarray):
    """d_t = gamma / s_t (fp32); y32 = fp32(acc) * d_t; y = bf16_rne(y32)."""
    d = np.float32(gamma) / np.asarray(s, dtype=np.float32)     # fp32 divide
    accf = np.asarray(acc).astype(np.float32)                   # nearest fp32
    y32 = accf * d[:, None]                                     # fp32 multiply
    return f32_to_bf16_bits(y32), y32


def linear(packed: np.ndarray, gamma: np.float32, x_bits: np.ndarray):
    """BitLinear forward on packed weights: returns dict of every stage."""
    K = np.asarray(x_bits).shape[1]
    xq, s, rowsum = act_quant(x_bits)
    w = unpack_i2s(packed, K)
    acc = ternary_matmul(xq, w)
    y_bits, y32 = dequant(acc, gamma, s)
    return {"xq": xq, "s": s, "rowsum": rowsum, "acc": acc,
            "y32": y32, "y": y_bits}


def linear_from_float(W: np.ndarray, x_bits: np.ndarray):
    packed, g = pack_weights(W)
    out = linear(packed, g, x_bits)
    out["packed"], out["gamma"] = packed, g
    return out


# --------------------------------------------------------------------------
# Step 5: the FFN block (RMSNorm -> gate/up -> ReLU^2(gate)*up -> RMSNorm -> down)
# --------------------------------------------------------------------------
def ffn(x_bits, gate, up, down, norm1_w=None, norm2_w=None, eps=1e-5):
    """Fused-block oracle in folded form.  ``gate``/``up``/``down`` are
    (packed, gamma) pairs; gate/up are [I, H], down is [H, I].

    r1 = 1/sqrt(mean(x^2) + eps) (fp64); u = x * n1 (fp32); quantise u;
    g' = fp32(acc_g) * (gamma_g/s1); u' likewise; h' = (relu(g')*relu(g'))*u';
    v = h' * n2; quantise v; acc_d; r2 = 1/sqrt(r1^6 * mean(h'^2) + eps) (fp64);
    f = fp32(r1^3 * r2); y32 = (fp32(acc_d) * (gamma_d/s2)) * f; y = bf16(y32).
    True activations are g = g' r1, u = u' r1, h = h' r1^3.
    """
    xf = bf16_bits_to_f32(x_bits)
    M, H = xf.shape
    g_packed, g_gamma = gate
    u_packed, u_gamma = up
    d_packed, d_gamma = down
    I = g_packed.shape[0]
    n1 = np.ones(H, np.float32) if norm1_w is None else np.asarray(norm1_w, np.float32)
    n2 = np.ones(I, np.float32) if norm2_w is None else np.asarray(norm2_w, np.float32)
    eps64 = float(np.float32(eps))

    ms1 = np.mean(xf.astype(np.float64) ** 2, axis=1)
    r1 = 1.0 / np.sqrt(ms1 + eps64)
    u = xf * n1[None, :]
    q1, s1, rs1 = act_quant_f32(u)
    acc_g = ternary_matmul(q1, unpack_i2s(g_packed, H))
    acc_u = ternary_matmul(q1, unpack_i2s(u_packed, H))
    gq = acc_g.astype(np.float32) * (np.float32(g_gamma) / s1)[:, None]
    uq = acc_u.astype(np.float32) * (np.float32(u_gamma) / s1)[:, None]
    rg = np.maximum(gq, np.float32(0.0))
    h = (rg * rg) * uq
    v = h * n2[None, :]
    q2, s2, rs2 = act_quant_f32(v)
    acc_d = ternary_matmul(q2, unpack_i2s(d_packed, I))
    ms2 = np.mean(h.astype(np.float64) ** 2, axis=1)
    r2 = 1.0 / np.sqrt(r1 ** 6 * ms2 + eps64)
    f = (r1 ** 3 * r2).astype(np.float32)
    d = np.float32(d_gamma) / s2
    y32 = (acc_d.astype(np.float32) * d[:, None]) * f[:, None]
    return {"q1": q1, "s1": s1, "rowsum1": rs1, "acc_gate": acc_g, "acc_up": acc_u,
            "h": h, "q2": q2, "s2": s2, "rowsum2": rs2, "acc_down": acc_d,
            "r1": r1, "r2": r2, "f": f, "y32": y32, "y": f32_to_bf16_bits(y32)}
