"""Count the quantised codes on which the folded FFN evaluation differs from
the literal one, at the 100B-class shapes (hidden 8192, intermediate 28672).

The FFN normalises before each activation quantiser (abeam.tech review of
"BitNet: 1-bit Pre-training for Large Language Models", section
"正規化で分散を安定させる": subln before BitLinear; reinforz.co.jp, section
"積極的量子化と三値化がもたらす学習効率の革新").  The oracle and the GPU
library quantise x * n1 and carry the RMS factor r1 into the dequant scale
("fold"): absmax quantisation is invariant to a positive per-token factor, so
in real arithmetic the codes are those of the literal form, which quantises
the fp32 RMSNorm output itself.  In fp32 the two can differ where a scaled
value lands within rounding error of a .5 tie.  This script evaluates the
literal fp32 form (the RMSNorm as an fp32 framework computes it: r rounded to
fp32, x * r, then the gain) beside oracle.ffn on the first 32 tokens of the
M = 2048 workload and writes the counts of differing codes q1 (first
quantiser) and q2 (second quantiser).

Run from the repository root:  python tests/golden/fold_vs_literal.py
It calls only the oracle and the input generator; the output file is read by
tests/test_oracle_pins.py.
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import bitlinear as O  # noqa: E402
from ternary_weight_linear_int8_b200 import inputs  # noqa: E402

H, I, TOKENS, EPS = 8192, 28672, 32, 1e-5
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fold_vs_literal_100b.txt")


def literal_ffn_codes(x_bits, gate, up, norm1_w, norm2_w, eps):
    """Literal form: quantise fp32 RMSNorm outputs.  Returns (q1, q2)."""
    xf = O.bf16_bits_to_f32(x_bits)
    eps64 = float(np.float32(eps))
    r1 = (1.0 / np.sqrt(np.mean(xf.astype(np.float64) ** 2, axis=1) + eps64)).astype(np.float32)
    xn = (xf * r1[:, None]) * norm1_w[None, :]
    q1, s1, _ = O.act_quant_f32(xn)
    g = O.ternary_matmul(q1, O.unpack_i2s(gate[0], H)).astype(np.float32) * (np.float32(gate[1]) / s1)[:, None]
    u = O.ternary_matmul(q1, O.unpack_i2s(up[0], H)).astype(np.float32) * (np.float32(up[1]) / s1)[:, None]
    rg = np.maximum(g, np.float32(0.0))
    h = (rg * rg) * u
    r2 = (1.0 / np.sqrt(np.mean(h.astype(np.float64) ** 2, axis=1) + eps64)).astype(np.float32)
    hn = (h * r2[:, None]) * norm2_w[None, :]
    q2, _, _ = O.act_quant_f32(hn)
    return q1, q2


def main():
    t0 = time.time()
    x = inputs.activations((TOKENS, H), seed=0)      # the first 32 tokens of the M=2048 input
    packs = []
    for n, k, seed in ((I, H, 2000), (I, H, 2001), (H, I, 2002)):
        W = inputs.weights(n, k, seed=seed)
        packs.append(O.pack_weights(W))
        del W
    ones_h, ones_i = np.ones(H, np.float32), np.ones(I, np.float32)
    fold = O.ffn(x, packs[0], packs[1], packs[2], None, None, EPS)
    q1l, q2l = literal_ffn_codes(x, packs[0], packs[1], ones_h, ones_i, EPS)
    d1 = int(np.count_nonzero(fold["q1"] != q1l))
    d2 = int(np.count_nonzero(fold["q2"] != q2l))
    with open(OUT, "w") as fh:
        fh.write("# Codes on which the folded FFN quantisers differ from the literal fp32\n")
        fh.write("# RMSNorm-then-quantise form; written by tests/golden/fold_vs_literal.py\n")
        fh.write(f"# H={H} I={I} tokens={TOKENS} (first tokens of the M=2048 input, seed 0);\n")
        fh.write("# weights seeds 2000/2001/2002; norm gains 1; eps 1e-5\n")
        fh.write(f"q1_codes_total {TOKENS * H}\n")
        fh.write(f"q1_codes_differing {d1}\n")
        fh.write(f"q2_codes_total {TOKENS * I}\n")
        fh.write(f"q2_codes_differing {d2}\n")
    print(open(OUT).read(), f"({time.time() - t0:.0f} s)")


if __name__ == "__main__":
    main()
