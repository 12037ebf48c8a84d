"""GPU parity: every kernel, called through the C ABI, against the CPU oracle on
the same seeded inputs.  Integer results (x_q, packed codes, gamma bits,
int32 accumulators) must be bit-exact; fp32 outputs of bitnet_linear are
bit-exact by construction (same IEEE steps), fp32 FFN outputs within 1e-5
relative (their RMS factors are reductions in another order)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import bitlinear as O
from ternary_weight_linear_int8_b200 import bitnet as B
from ternary_weight_linear_int8_b200 import inputs
from tests.gpu_util import (assert_bf16_close, assert_f32_rel, dev_bits, dev_f32, dev_u8,
                            f32_bits, host_bits)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert B.bitnet_last_device_status() == 0


# --------------------------------------------------------------- packing
PACK_SHAPES = [(400, 512, 1000), (7, 68, 1), (1, 4, 2), (33, 1024, 3), (6912, 2560, 1000),
               (2560, 6912, 1001)]


@pytest.mark.parametrize("N,K,seed", PACK_SHAPES)
def test_pack_matches_oracle(N, K, seed):
    W = inputs.weights(N, K, seed=seed)
    p_ref, g_ref = O.pack_weights(W)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    assert f32_bits(g.cpu().numpy())[0] == f32_bits(g_ref)
    assert np.array_equal(p.cpu().numpy(), p_ref)


@pytest.mark.parametrize("kind", ["zero", "plus", "minus", "tiny", "huge", "mixed_exp"])
def test_pack_special_values(kind):
    rng = np.random.default_rng(5)
    if kind == "zero":
        W = np.zeros((16, 64), np.float32)
    elif kind == "plus":
        W = np.full((16, 64), 0.02, np.float32)
    elif kind == "minus":
        W = np.full((16, 64), -3.5, np.float32)
    elif kind == "tiny":     # subnormal weights: the exact-sum path on its smallest grid
        W = (rng.standard_normal((16, 64)) * 1e-39).astype(np.float32)
    elif kind == "huge":
        W = (rng.standard_normal((16, 64)) * 1e37).astype(np.float32)
    else:                    # exponents spread over the whole fp32 range
        W = (rng.standard_normal((64, 256)) * 10.0 ** rng.integers(-40, 38, size=(64, 256))).astype(np.float32)
    p_ref, g_ref = O.pack_weights(W)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    assert f32_bits(g.cpu().numpy())[0] == f32_bits(g_ref)
    assert np.array_equal(p.cpu().numpy(), p_ref)


def test_pack_nonfinite_is_reported():
    W = np.ones((4, 8), np.float32)
    W[2, 3] = np.inf
    p, g = B.bitnet_pack_weights(dev_f32(W))
    assert B.bitnet_last_device_status() == 8
    assert np.isnan(g.cpu().numpy()[0])


# ------------------------------------------------------ activation quant
# few tokens or long rows: a CTA per token; many short rows: a warp per token
QUANT_SHAPES = [(1, 2560, False), (8, 512, False), (3, 68, False), (17, 4, False),
                (64, 6912, True), (5, 28672, True), (300, 1024, True), (600, 6912, True),
                (297, 2560, False), (1000, 400, True), (260, 68, False)]


@pytest.mark.parametrize("M,K,outl", QUANT_SHAPES)
def test_quant_act_matches_oracle(M, K, outl):
    x = inputs.activations((M, K), seed=M * 7 + K, outliers=outl)
    x[0, : min(K, 8)] = 0          # partial zeros
    if M > 2:
        x[2, :] = 0                # an all-zero token
    q_ref, s_ref, r_ref = O.act_quant(x)
    q, s, r = B.bitnet_quant_act(dev_bits(x))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


# ------------------------------------------------------------- BitLinear
# (M, N, K): decode kernel (M <= 8, K % 64 == 0), tensor-core kernel (with and
# without split-K), and the ragged-K kernel.
LINEAR_SHAPES = [
    (1, 6912, 2560), (1, 2560, 6912), (8, 400, 512), (2, 7, 64), (3, 1, 128), (5, 33, 1024),
    (4, 6912, 2560), (1, 257, 8192),
    (9, 400, 512), (16, 6912, 2560), (64, 2560, 6912), (65, 257, 640), (17, 1, 256),
    (300, 1000, 1024), (129, 128, 128), (256, 300, 2560),
    (8, 400, 68), (3, 5, 4), (1, 9, 20), (70, 13, 36),
]


def _linear_case(M, N, K, seed=0, outliers=True):
    rng = np.random.default_rng(seed + 31 * M + 7 * N + K)
    x = inputs.activations((M, K), rng=rng, outliers=outliers and K >= 100)
    W = inputs.weights(N, K, rng=rng)
    return x, W


@pytest.mark.parametrize("M,N,K", LINEAR_SHAPES)
def test_linear_matches_oracle(M, N, K):
    x, W = _linear_case(M, N, K)
    ref = O.linear_from_float(W, x)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    y, y32, acc = B.bitnet_linear(p, g, dev_bits(x), want_f32=True, want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y), ref["y"])


def test_linear_output_only_call_matches():
    """The plain call (no debug outputs) writes the same y."""
    x, W = _linear_case(16, 1000, 2560)
    ref = O.linear_from_float(W, x)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    for M in (1, 16):
        y, _, _ = B.bitnet_linear(p, g, dev_bits(x[:M]))
        assert np.array_equal(host_bits(y), ref["y"][:M])


@pytest.mark.parametrize("M", [1, 4, 64])
def test_linear_closed_forms(M):
    K, N = 512, 96
    x = inputs.activations((M, K), seed=9)
    if M > 1:
        x[1] = 0                                   # zero token -> zero outputs
    xd = dev_bits(x)
    q, s, rs = O.act_quant(x)
    # all-zero weights -> y == 0
    p, g = B.bitnet_pack_weights(dev_f32(np.zeros((N, K), np.float32)))
    y, y32, acc = B.bitnet_linear(p, g, xd, want_f32=True, want_acc=True)
    assert not acc.cpu().numpy().any() and not y32.cpu().numpy().any()
    # all +1 weights -> y32 = fp32(rowsum) * (gamma / s) in every column
    c = np.float32(0.02)
    p, g = B.bitnet_pack_weights(dev_f32(np.full((N, K), c, np.float32)))
    y, y32, acc = B.bitnet_linear(p, g, xd, want_f32=True, want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), np.repeat(rs[:, None], N, axis=1))
    want = (rs.astype(np.float32) * (c / s))[:, None]
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(np.repeat(want, N, axis=1)))


def test_linear_under_cuda_graph_replay():
    """A captured chain of calls (as the benchmark runs it) replays to the same
    result as eager calls."""
    K1, K2 = 2560, 6912
    x = inputs.activations((1, K1), seed=0)
    Ws = [inputs.weights(K2, K1, seed=1000), inputs.weights(K1, K2, seed=1001)]
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    xd = dev_bits(x)
    ys = [torch.empty((1, K2), dtype=torch.bfloat16, device="cuda"),
          torch.empty((1, K1), dtype=torch.bfloat16, device="cuda")]
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        B.bitnet_linear(*packs[0], xd, y=ys[0])
        B.bitnet_linear(*packs[1], ys[0], y=ys[1])
    s.synchronize()
    eager = host_bits(ys[1]).copy()
    ys[1].zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        B.bitnet_linear(*packs[0], xd, y=ys[0])
        B.bitnet_linear(*packs[1], ys[0], y=ys[1])
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(ys[1]), eager)
    # and both equal the oracle chain
    r1 = O.linear_from_float(Ws[0], x)
    r2 = O.linear_from_float(Ws[1], r1["y"])
    assert np.array_equal(eager, r2["y"])


# ------------------------------------------------------------------- FFN
FFN_SHAPES = [(1, 256, 512), (2, 512, 1024), (1, 2560, 6912), (5, 256, 512), (8, 512, 1024),
              (9, 256, 512), (64, 512, 1024), (130, 256, 768), (300, 128, 320)]


def _ffn_case(M, H, I, seed=0, gains=True):
    rng = np.random.default_rng(seed + 17 * M + H + 3 * I)
    x = inputs.activations((M, H), rng=rng, outliers=True)
    Wg, Wu = inputs.weights(I, H, rng=rng), inputs.weights(I, H, rng=rng)
    Wd = inputs.weights(H, I, rng=rng)
    n1 = (1 + 0.2 * rng.standard_normal(H)).astype(np.float32) if gains else None
    n2 = (1 + 0.2 * rng.standard_normal(I)).astype(np.float32) if gains else None
    return x, Wg, Wu, Wd, n1, n2


def _run_ffn(x, Wg, Wu, Wd, n1, n2, eps=1e-5):
    pg, gg = B.bitnet_pack_weights(dev_f32(Wg))
    pu, gu = B.bitnet_pack_weights(dev_f32(Wu))
    pd, gd = B.bitnet_pack_weights(dev_f32(Wd))
    w = B.FfnWeights(pg, gg, pu, gu, pd, gd,
                     None if n1 is None else dev_f32(n1), None if n2 is None else dev_f32(n2))
    return B.bitnet_ffn(dev_bits(x), w, eps=eps, debug=True)


def _check_ffn(ref, y, dbg, rows=None):
    sel = slice(None) if rows is None else rows
    got = {k: v.cpu().numpy()[sel] for k, v in dbg.items()}
    assert np.array_equal(got["xq1"], ref["q1"])
    assert np.array_equal(got["acc_gate"], ref["acc_gate"].astype(np.int32))
    assert np.array_equal(got["acc_up"], ref["acc_up"].astype(np.int32))
    assert np.array_equal(f32_bits(got["h"]), f32_bits(ref["h"]))
    assert np.array_equal(got["xq2"], ref["q2"])
    assert np.array_equal(got["acc_down"], ref["acc_down"].astype(np.int32))
    assert_f32_rel(got["y_f32"], ref["y32"], 1e-5)
    assert_bf16_close(host_bits(y)[sel], ref["y"], got["y_f32"], ref["y32"])


@pytest.mark.parametrize("M,H,I", FFN_SHAPES)
def test_ffn_matches_oracle(M, H, I):
    x, Wg, Wu, Wd, n1, n2 = _ffn_case(M, H, I)
    ref = O.ffn(x, O.pack_weights(Wg), O.pack_weights(Wu), O.pack_weights(Wd), n1, n2, 1e-5)
    y, dbg = _run_ffn(x, Wg, Wu, Wd, n1, n2)
    _check_ffn(ref, y, dbg)


def test_ffn_default_gains_and_plain_call():
    x, Wg, Wu, Wd, _, _ = _ffn_case(4, 256, 512, gains=False)
    ref = O.ffn(x, O.pack_weights(Wg), O.pack_weights(Wu), O.pack_weights(Wd), None, None, 1e-5)
    y, dbg = _run_ffn(x, Wg, Wu, Wd, None, None)
    _check_ffn(ref, y, dbg)
    # the call without debug outputs gives the same y
    pg, gg = B.bitnet_pack_weights(dev_f32(Wg))
    pu, gu = B.bitnet_pack_weights(dev_f32(Wu))
    pd, gd = B.bitnet_pack_weights(dev_f32(Wd))
    y2, _ = B.bitnet_ffn(dev_bits(x), B.FfnWeights(pg, gg, pu, gu, pd, gd))
    assert np.array_equal(host_bits(y2), host_bits(y))


# ------------------------------------------------- full-size workloads
def test_fullsize_decode_chain_2b():
    """2B-class decode: x[1,2560] -> up [6912,2560] -> down [2560,6912] -> ...,
    four distinct layers, every intermediate bit-exact (the launch
    configuration the benchmark times, minus the graph)."""
    x = inputs.activations((1, 2560), seed=0)
    cur_ref = x
    cur = dev_bits(x)
    for layer in range(4):
        N, K = (6912, 2560) if layer % 2 == 0 else (2560, 6912)
        W = inputs.weights(N, K, seed=inputs.layer_seed(layer))
        ref = O.linear_from_float(W, cur_ref)
        p, g = B.bitnet_pack_weights(dev_f32(W))
        y, y32, acc = B.bitnet_linear(p, g, cur, want_f32=True, want_acc=True)
        assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
        assert np.array_equal(host_bits(y), ref["y"])
        cur_ref, cur = ref["y"], y


@pytest.mark.parametrize("N,K", [(6912, 2560), (2560, 6912)])
def test_fullsize_prefill_sampled_rows(N, K):
    """Prefill M=4096 on the tensor-core kernel; the oracle checks 48
    seed-chosen tokens (tokens are independent)."""
    M = 4096
    x = inputs.activations((M, K), seed=0)
    W = inputs.weights(N, K, seed=1000)
    rows = np.sort(np.random.default_rng(123).choice(M, 48, replace=False))
    rows[-1] = M - 1
    ref = O.linear_from_float(W, x[rows])
    p, g = B.bitnet_pack_weights(dev_f32(W))
    y, y32, acc = B.bitnet_linear(p, g, dev_bits(x), want_f32=True, want_acc=True)
    assert np.array_equal(acc.cpu().numpy()[rows], ref["acc"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()[rows]), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y)[rows], ref["y"])


@pytest.mark.parametrize("M", [16, 64])
def test_fullsize_batched_decode(M):
    for N, K in [(6912, 2560), (2560, 6912)]:
        x = inputs.activations((M, K), seed=0, outliers=True)
        W = inputs.weights(N, K, seed=1002)
        ref = O.linear_from_float(W, x)
        p, g = B.bitnet_pack_weights(dev_f32(W))
        y, y32, acc = B.bitnet_linear(p, g, dev_bits(x), want_f32=True, want_acc=True)
        assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
        assert np.array_equal(host_bits(y), ref["y"])


@pytest.fixture(scope="module")
def ffn_100b():
    H, I = 8192, 28672
    Wg = inputs.weights(I, H, seed=2000)
    Wu = inputs.weights(I, H, seed=2001)
    Wd = inputs.weights(H, I, seed=2002)
    return Wg, Wu, Wd, (O.pack_weights(Wg), O.pack_weights(Wu), O.pack_weights(Wd))


@pytest.mark.parametrize("M", [1, 2048])
def test_fullsize_ffn_100b(M, ffn_100b):
    """100B-class FFN block, hidden 8192, intermediate 28672.  M=1 is checked
    whole; M=2048 on 8 seed-chosen tokens."""
    H = 8192
    Wg, Wu, Wd, packed = ffn_100b
    x = inputs.activations((M, H), seed=0)
    rows = np.arange(M) if M == 1 else np.sort(np.random.default_rng(7).choice(M, 8, replace=False))
    ref = O.ffn(x[rows], *packed, None, None, 1e-5)
    y, dbg = _run_ffn(x, Wg, Wu, Wd, None, None)
    _check_ffn(ref, y, dbg, rows=rows)
