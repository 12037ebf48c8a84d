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
                            f32_bits, guarded, host_bits)

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
    pg, gg = guarded((N, K // 4), torch.uint8), guarded((1,), torch.float32)
    p, g = B.bitnet_pack_weights(dev_f32(W), packed=pg.t, gamma=gg.t)
    assert f32_bits(g.cpu().numpy())[0] == f32_bits(g_ref)
    assert np.array_equal(p.cpu().numpy(), p_ref)
    pg.check()
    gg.check()


def _threshold_weights(N, K, seed):
    """Gaussian weights with 48 entries placed exactly on the ternary
    rounding thresholds of their own matrix: +-0.5*(gamma+1e-5), the fp32
    neighbours of those, and +-1.5*(gamma+1e-5).  gamma depends on the
    placed values, so the placement is repeated until gamma stops moving."""
    rng = np.random.default_rng(seed)
    W = inputs.weights(N, K, rng=rng)
    pos = rng.choice(N * K, 48, replace=False)
    for _ in range(20):
        den = np.float32(O.absmean_gamma(W)) + O.EPS_F32
        half = np.float32(den * np.float32(0.5))
        up, dn = np.nextafter(half, np.float32(1)), np.nextafter(half, np.float32(0))
        th = np.float32(den * np.float32(1.5))
        vals = np.array([half, -half, up, -up, dn, -dn, th, -th], np.float32)
        W2 = W.copy()
        W2.ravel()[pos] = vals[np.arange(48) % 8]
        if np.array_equal(W2, W):
            break
        W = W2
    else:
        raise AssertionError("threshold placement did not settle")
    return W, pos


@pytest.mark.parametrize("N,K", [(64, 256), (6912, 2560)])
def test_pack_threshold_weights(N, K):
    """Weights exactly on +-0.5 (gamma + 1e-5) round half to even (to 0),
    their fp32 neighbours go wherever the fp32 quotient lands, and
    +-1.5 (gamma + 1e-5) clamps to +-1: GPU codes and gamma equal the
    oracle's, and the oracle confirms the placed values sit on the
    thresholds of the final gamma."""
    W, pos = _threshold_weights(N, K, seed=N + K)
    g_ref = O.absmean_gamma(W)
    den = np.float32(g_ref) + O.EPS_F32
    q = (W.ravel()[pos] / den).astype(np.float32)
    assert np.all(np.abs(q[0::8]) == 0.5) and np.all(np.abs(q[1::8]) == 0.5)
    w_ref = O.ternarize(W, g_ref).ravel()[pos]
    assert np.all(w_ref[0::8] == 0) and np.all(w_ref[1::8] == 0)
    assert np.all(w_ref[6::8] == 1) and np.all(w_ref[7::8] == -1)
    p_ref, _ = O.pack_weights(W)
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
                (297, 2560, False), (1000, 400, True), (260, 68, False),
                # the persistent quantiser's edges: longest row it takes, one
                # group of 16, a row one group past a whole warp, and many
                # short rows per CTA
                (2000, 8192, True), (40, 16, False), (33, 1040, True), (6000, 400, False)]


@pytest.mark.parametrize("M,K,outl", QUANT_SHAPES)
def test_quant_act_matches_oracle(M, K, outl):
    x = inputs.activations((M, K), seed=M * 7 + K, outliers=outl)
    x[0, : min(K, 8)] = 0          # partial zeros
    if M > 2:
        x[2, :] = 0                # an all-zero token
    q_ref, s_ref, r_ref = O.act_quant(x)
    outs = [guarded((M, K), torch.int8), guarded((M,), torch.float32), guarded((M,), torch.int32)]
    q, s, r = B.bitnet_quant_act(dev_bits(x), xq=outs[0].t, scale=outs[1].t, rowsum=outs[2].t)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)
    for o in outs:
        o.check()


# ------------------------------------------------------------- BitLinear
# (M, N, K): resident decode kernel (M <= 3), streaming decode kernel (M <= 8),
# batched decode kernel (9 <= M <= 32, with and without split K, ragged row
# groups), tensor-core kernel (with and without split-K, ragged last token
# tiles), and the ragged-K kernel.
LINEAR_SHAPES = [
    (512, 1000, 1024), (777, 400, 2560), (1000, 2560, 6912), (600, 257, 640),
    (24, 300, 2560), (32, 1000, 2560), (9, 6912, 64), (31, 5, 6912), (12, 4096, 4096),
    (20, 257, 640), (13, 2560, 2560), (7, 129, 192), (33, 1000, 2560), (48, 6912, 64),
    (1, 6912, 2560), (1, 2560, 6912), (8, 400, 512), (2, 7, 64), (3, 1, 128), (5, 33, 1024),
    (4, 6912, 2560), (1, 257, 8192), (4, 2560, 6912), (8, 2560, 6912), (8, 6912, 2560),
    (2, 2560, 6912), (3, 6912, 2560),
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
    outs = [guarded((M, N), torch.bfloat16), guarded((M, N), torch.float32),
            guarded((M, N), torch.int32)]
    y, y32, acc = B.bitnet_linear(p, g, dev_bits(x), y=outs[0].t, y_f32=outs[1].t, acc=outs[2].t)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y), ref["y"])
    for o in outs:
        o.check()


def _edge_tokens(M, K, seed):
    """Tokens that pin the quantiser's definition on the GPU:
    0: max |x| = 2 (s = 63.5 exactly) with +-1.0 entries, x*s = +-63.5, a tie
       that rounds to the even +-64;
    1: max |x| = 63.5 (s = 2) with +-0.25, 0.75, 1.25: ties at 0.5, 1.5,
       2.5 -> 0, 2, 2;
    2: a non-zero token whose max |x| is below the 1e-5 floor (s = 127/1e-5,
       not 127/(a + 1e-5));
    3: all zeros; the rest ~N(0,1)."""
    rng = np.random.default_rng(seed)
    xf = rng.standard_normal((M, K)).astype(np.float32)
    rows = []
    r0 = (rng.standard_normal(K) * 0.4).clip(-1.9, 1.9).astype(np.float32)
    r0[: K // 8] = np.where(np.arange(K // 8) % 2 == 0, 1.0, -1.0)
    r0[K // 8] = 2.0
    rows.append(r0)
    r1 = (rng.standard_normal(K) * 3).clip(-60, 60).astype(np.float32)
    r1[: 3 * (K // 16)] = np.tile(np.array([0.25, 0.75, 1.25], np.float32), K // 16)
    r1[K // 2] = -63.5
    rows.append(r1)
    rows.append((rng.standard_normal(K) * 2e-6).clip(-9e-6, 9e-6).astype(np.float32))
    rows.append(np.zeros(K, np.float32))
    for i, r in enumerate(rows[:M]):
        xf[i] = r
    return inputs.to_bf16_bits(xf)


@pytest.mark.parametrize("M", [1, 2, 4, 8, 9, 64])
@pytest.mark.parametrize("K", [512, 2560])
def test_linear_edge_activations(M, K):
    """Rounding ties, a sub-floor absmax and a zero token, through the
    standalone quantiser and every BitLinear path (decode, tensor-core)."""
    N = 300
    x = _edge_tokens(M, K, seed=M * 131 + K)
    ref_q, ref_s, _ = O.act_quant(x)
    if M >= 2:
        assert ref_q[0][np.flatnonzero(O.bf16_bits_to_f32(x[0]) == 1.0)].min() == 64
        assert ref_q[1][np.flatnonzero(O.bf16_bits_to_f32(x[1]) == 0.75)].min() == 2
    if M >= 3:
        xs = O.bf16_bits_to_f32(x[2])
        assert 0 < np.abs(xs).max() < 1e-5 and ref_s[2] == np.float32(127.0) / np.float32(1e-5)
    q, s, _ = B.bitnet_quant_act(dev_bits(x))
    assert np.array_equal(q.cpu().numpy(), ref_q)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(ref_s))
    W = inputs.weights(N, K, seed=K + 5)
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
    """The FFN with every output (y and the debug intermediates) allocated
    inside guard bands, which are checked after the call."""
    pg, gg = B.bitnet_pack_weights(dev_f32(Wg))
    pu, gu = B.bitnet_pack_weights(dev_f32(Wu))
    pd, gd = B.bitnet_pack_weights(dev_f32(Wd))
    w = B.FfnWeights(pg, gg, pu, gu, pd, gd,
                     None if n1 is None else dev_f32(n1), None if n2 is None else dev_f32(n2))
    M, H = x.shape
    I = Wg.shape[0]
    specs = {"xq1": ((M, H), torch.int8), "acc_gate": ((M, I), torch.int32),
             "acc_up": ((M, I), torch.int32), "h": ((M, I), torch.float32),
             "xq2": ((M, I), torch.int8), "acc_down": ((M, H), torch.int32),
             "y_f32": ((M, H), torch.float32)}
    g = {k: guarded(*v) for k, v in specs.items()}
    gy = guarded((M, H), torch.bfloat16)
    y, dbg = B.bitnet_ffn(dev_bits(x), w, eps=eps, y=gy.t, debug={k: v.t for k, v in g.items()})
    torch.cuda.synchronize()
    for v in list(g.values()) + [gy]:
        v.check()
    return y, dbg


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
def test_fullsize_prefill_all_rows(N, K):
    """Prefill M=4096 on the tensor-core kernel, every token checked against
    the oracle, outputs inside guard bands."""
    M = 4096
    x = inputs.activations((M, K), seed=0)
    W = inputs.weights(N, K, seed=1000)
    ref = O.linear_from_float(W, x)
    p, g = B.bitnet_pack_weights(dev_f32(W))
    outs = [guarded((M, N), torch.bfloat16), guarded((M, N), torch.float32),
            guarded((M, N), torch.int32)]
    y, y32, acc = B.bitnet_linear(p, g, dev_bits(x), y=outs[0].t, y_f32=outs[1].t, acc=outs[2].t)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
    assert np.array_equal(host_bits(y), ref["y"])
    for o in outs:
        o.check()


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 64])
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
    whole; M=2048 on the first and last token of every 64-token block (so
    every token tile of the tensor-core kernel, 64, 128, 192 or 256 wide,
    has its edges checked) plus 16 seed-chosen tokens."""
    H = 8192
    Wg, Wu, Wd, packed = ffn_100b
    x = inputs.activations((M, H), seed=0)
    if M == 1:
        rows = np.arange(1)
    else:
        edges = np.concatenate([np.arange(0, M, 64), np.arange(63, M, 64)])
        extra = np.random.default_rng(7).choice(M, 16, replace=False)
        rows = np.unique(np.concatenate([edges, extra]))
    ref = O.ffn(x[rows], *packed, None, None, 1e-5)
    y, dbg = _run_ffn(x, Wg, Wu, Wd, None, None)
    _check_ffn(ref, y, dbg, rows=rows)
