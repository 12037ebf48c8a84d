"""GPU parity of the BitLinear variants against the CPU oracle:

* BitNet v1 W1A8 (sign weights, 1 bit each): bitnet_pack_weights_w1 and
  bitnet_linear_w1 through both of its paths (the decode kernel on the sign
  bits, and the sign bits expanded to I2_S codes for the other kernels);
* the pair-lookup-table inner loop, bitnet_linear_tl2 (one token).

Integer results (packed bits, alpha bits, accumulators) bit-exact; fp32 and
bf16 outputs bit-exact (the same IEEE steps as the oracle); every output
inside guard bands."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import bitlinear as O
from oracle import variants as V
from ternary_weight_linear_int8_b200 import bitnet as B
from ternary_weight_linear_int8_b200 import inputs
from tests.gpu_util import dev_bits, dev_f32, f32_bits, guarded, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert B.bitnet_last_device_status() == 0


@pytest.mark.parametrize("N,K,seed", [(400, 512, 1), (7, 64, 2), (1, 8, 3), (6912, 2560, 4),
                                      (2560, 6912, 5)])
def test_pack_w1_matches_oracle(N, K, seed):
    W = inputs.weights(N, K, seed=seed)
    W.ravel()[:: max(1, W.size // 7)] = 0.0          # zeros pack as +1
    W.ravel()[1:: max(1, W.size // 5)] = -0.0
    p_ref, a_ref = V.pack_weights_w1(W)
    pg, ag = guarded((N, K // 8), torch.uint8), guarded((1,), torch.float32)
    p, a = B.bitnet_pack_weights_w1(dev_f32(W), packed=pg.t, alpha=ag.t)
    assert f32_bits(a.cpu().numpy())[0] == f32_bits(a_ref)
    assert np.array_equal(p.cpu().numpy(), p_ref)
    pg.check()
    ag.check()


# (M, N, K): decode kernel on the sign bits (1-3 tokens, K % 128 == 0), and
# the expansion to I2_S codes (K % 128 != 0, more tokens, ragged K)
W1_SHAPES = [(1, 6912, 2560), (1, 2560, 6912), (2, 400, 512), (3, 257, 1024), (1, 7, 128),
             (1, 64, 192), (8, 400, 512), (64, 300, 1024), (5, 33, 104), (2, 2560, 6912)]


@pytest.mark.parametrize("M,N,K", W1_SHAPES)
def test_linear_w1_matches_oracle(M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    x = inputs.activations((M, K), rng=rng, outliers=K >= 100)
    W = inputs.weights(N, K, rng=rng)
    p_ref, a_ref = V.pack_weights_w1(W)
    ref = V.linear_w1(p_ref, a_ref, x)
    p, a = B.bitnet_pack_weights_w1(dev_f32(W))
    outs = [guarded((M, N), torch.bfloat16), guarded((M, N), torch.float32),
            guarded((M, N), torch.int32)]
    y, y32, acc = B.bitnet_linear_w1(p, a, dev_bits(x), y=outs[0].t, y_f32=outs[1].t,
                                     acc=outs[2].t)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y), ref["y"])
    for o in outs:
        o.check()


def test_linear_w1_chain_of_2b_layers():
    """Four 2B-class W1A8 layers back to back, each fed the previous output."""
    x = inputs.activations((1, 2560), seed=0)
    cur_ref, cur = x, dev_bits(x)
    for layer in range(4):
        N, K = (6912, 2560) if layer % 2 == 0 else (2560, 6912)
        W = inputs.weights(N, K, seed=inputs.layer_seed(layer))
        ref = V.linear_w1(*V.pack_weights_w1(W), cur_ref)
        p, a = B.bitnet_pack_weights_w1(dev_f32(W))
        y, _, _ = B.bitnet_linear_w1(p, a, cur)
        assert np.array_equal(host_bits(y), ref["y"]), f"layer {layer}"
        cur_ref, cur = ref["y"], y


@pytest.mark.parametrize("N,K", [(6912, 2560), (2560, 6912), (400, 512), (7, 64), (257, 1024)])
def test_linear_tl2_matches_oracle(N, K):
    rng = np.random.default_rng(N + K)
    x = inputs.activations((1, K), rng=rng, outliers=True)
    W = inputs.weights(N, K, rng=rng)
    ref = O.linear_from_float(W, x)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    outs = [guarded((1, N), torch.bfloat16), guarded((1, N), torch.float32),
            guarded((1, N), torch.int32)]
    y, y32, acc = B.bitnet_linear_tl2(p, g, dev_bits(x), y=outs[0].t, y_f32=outs[1].t,
                                      acc=outs[2].t)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y), ref["y"])
    for o in outs:
        o.check()


# ------------------------------------------------------------------- a4.8
def _a48_tokens(M, K, seed):
    """Outlier-channel activations, plus a token with many equal magnitudes
    (ties at the selection threshold must go to the lower channels)."""
    x = inputs.activations((M, K), seed=seed, outliers=True)
    if M > 1:
        xf = np.tile(np.array([4.0, -4.0, 4.0, 1.0, -2.0, 2.0, 2.0, -2.0], np.float32), K // 8)
        x[1] = O.f32_to_bf16_bits(xf)
    return x


@pytest.mark.parametrize("M,K,n_out", [(1, 2560, 26), (4, 6912, 69), (3, 512, 0), (2, 512, 512),
                                       (5, 64, 3), (2, 1024, 257), (8, 2560, 1)])
def test_quant_act_a48_matches_oracle(M, K, n_out):
    x = _a48_tokens(M, K, seed=M + K + n_out)
    q4r, s4r, q8r, s8r, _ = V.act_quant_a48(x, n_out)
    q4, s4, q8, s8 = B.bitnet_quant_act_a48(dev_bits(x), n_out)
    assert np.array_equal(q4.cpu().numpy(), q4r)
    assert np.array_equal(q8.cpu().numpy(), q8r)
    assert np.array_equal(f32_bits(s4.cpu().numpy()), f32_bits(s4r))
    assert np.array_equal(f32_bits(s8.cpu().numpy()), f32_bits(s8r))


@pytest.mark.parametrize("M,N,K,n_out", [(1, 6912, 2560, 26), (1, 2560, 6912, 69),
                                         (4, 400, 512, 5), (16, 300, 1024, 10),
                                         (64, 2560, 6912, 69), (3, 257, 128, 0), (2, 100, 128, 128)])
def test_linear_a48_matches_oracle(M, N, K, n_out):
    x = _a48_tokens(M, K, seed=N + K)
    W = inputs.weights(N, K, seed=K + 3)
    p_ref, g_ref = O.pack_weights(W)
    ref = V.linear_a48(p_ref, g_ref, x, n_out)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    outs = [guarded((M, N), torch.bfloat16), guarded((M, N), torch.float32),
            guarded((M, N), torch.int32), guarded((M, N), torch.int32)]
    y, y32, a4, a8 = B.bitnet_linear_a48(p, g, dev_bits(x), n_out, y=outs[0].t, y_f32=outs[1].t,
                                         acc4=outs[2].t, acc8=outs[3].t)
    assert np.array_equal(a4.cpu().numpy(), ref["acc4"].astype(np.int32))
    assert np.array_equal(a8.cpu().numpy(), ref["acc8"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y), ref["y"])
    for o in outs:
        o.check()
