"""The batched decode kernel (9..32 tokens, weights resident in shared
memory, int8 mma.sync, split K through bulk reductions into a scratch that
each layer leaves zero) against the oracle: chains that hand each layer's
per-token absmax to the next, repeated calls and graph replays on one
workspace, and a workspace shared by layers of different widths.  Every
integer and every bf16 output must equal the oracle's bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import bitlinear as O
from ternary_weight_linear_int8_b200 import bitnet as B
from ternary_weight_linear_int8_b200 import inputs
from tests.gpu_util import dev_bits, dev_f32, f32_bits, guarded, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert B.bitnet_last_device_status() == 0


def _oracle_chain(Ws, x):
    outs, cur = [], x
    for W in Ws:
        cur = O.linear_from_float(W, cur)["y"]
        outs.append(cur)
    return outs


@pytest.mark.parametrize("M", [9, 13, 16, 24, 32])
def test_batched_chain_small_layers(M):
    """Nine layers of mixed widths (K a multiple of 64 throughout), so every
    layer after the first takes its scales from the hand-over ring."""
    dims = [512, 1024, 256, 768, 64, 320, 2048, 128, 640, 512]
    rng = np.random.default_rng(40 + M)
    x = inputs.activations((M, dims[0]), rng=rng, outliers=True)
    Ws = [inputs.weights(dims[l + 1], dims[l], rng=rng) for l in range(len(dims) - 1)]
    want = _oracle_chain(Ws, x)
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    outs = [guarded((M, W.shape[0]), torch.bfloat16) for W in Ws]
    B.bitnet_linear_chain([p for p, _ in packs], [g for _, g in packs], dev_bits(x),
                          ys=[o.t for o in outs])
    torch.cuda.synchronize()
    for l in range(len(Ws)):
        assert np.array_equal(host_bits(outs[l].t), want[l]), f"layer {l}"
        outs[l].check()


@pytest.mark.parametrize("M", [16, 32, 11])
def test_batched_chain_2b_shapes_and_graph(M):
    """2B-class layers, up [6912,2560] then down [2560,6912], six of them,
    into two ping-pong buffers: eager twice, then three CUDA-graph replays
    on the same workspace, all equal to the oracle (the split-K scratch and
    the counters are clean again after every layer)."""
    L = 6
    x = inputs.activations((M, 2560), seed=M, outliers=True)
    Ws = [inputs.weights(*((6912, 2560) if l % 2 == 0 else (2560, 6912)),
                         seed=inputs.layer_seed(l)) for l in range(L)]
    want = _oracle_chain(Ws, x)
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    P, G = [p for p, _ in packs], [g for _, g in packs]
    bufs = [torch.empty((M, 6912), dtype=torch.bfloat16, device="cuda"),
            torch.empty((M, 2560), dtype=torch.bfloat16, device="cuda")]
    ys = [bufs[l % 2] for l in range(L)]
    xd = dev_bits(x)
    ws = torch.empty(B.bitnet_linear_chain_workspace_size([6912, 2560] * (L // 2),
                                                          [2560, 6912] * (L // 2), M),
                     dtype=torch.uint8, device="cuda")
    for _ in range(2):
        bufs[0].zero_()
        bufs[1].zero_()
        B.bitnet_linear_chain(P, G, xd, ys=ys, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(bufs[1]), want[-1])
        assert np.array_equal(host_bits(bufs[0]), want[-2])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        B.bitnet_linear_chain(P, G, xd, ys=ys, workspace=ws)
    torch.cuda.synchronize()
    for _ in range(3):
        bufs[0].zero_()
        bufs[1].zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(bufs[1]), want[-1])
        assert np.array_equal(host_bits(bufs[0]), want[-2])
    del graph


def test_batched_workspace_reused_across_shapes():
    """One workspace, sized for the largest call, used in turn by layers of
    different widths and token counts, twice over: every result equal to the
    oracle's (a scratch left dirty by one call would corrupt the next)."""
    cases = [(16, 6912, 2560), (32, 2560, 6912), (9, 1000, 2560), (32, 300, 2560),
             (4, 2560, 6912), (64, 2560, 6912), (20, 2560, 6912)]
    nb = max(B.bitnet_linear_workspace_size(*c) for c in cases)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    data = []
    for i, (M, N, K) in enumerate(cases):
        x = inputs.activations((M, K), seed=100 + i, outliers=True)
        W = inputs.weights(N, K, seed=200 + i)
        p, g = B.bitnet_pack_weights(dev_f32(W))
        data.append((dev_bits(x), p, g, O.linear_from_float(W, x)))
    for _ in range(2):
        for xd, p, g, ref in data:
            y, y32, acc = B.bitnet_linear(p, g, xd, want_f32=True, want_acc=True, workspace=ws)
            assert np.array_equal(acc.cpu().numpy(), ref["acc"].astype(np.int32))
            assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(ref["y32"]))
            assert np.array_equal(host_bits(y), ref["y"])


def test_batched_handover_matches_quantiser():
    """The absmax a layer hands over equals what the standalone quantiser
    finds in that layer's bf16 output: a two-layer chain's second output
    equals the oracle run on the first output as stored."""
    M, dims = 32, [2560, 6912, 2560]
    x = inputs.activations((M, dims[0]), seed=7, outliers=True)
    Ws = [inputs.weights(dims[1], dims[0], seed=8), inputs.weights(dims[2], dims[1], seed=9)]
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    ys = B.bitnet_linear_chain([p for p, _ in packs], [g for _, g in packs], dev_bits(x))
    y0 = host_bits(ys[0])
    ref1 = O.linear_from_float(Ws[1], y0)
    assert np.array_equal(host_bits(ys[1]), ref1["y"])
    q, s, _ = B.bitnet_quant_act(ys[0])
    q_ref, s_ref, _ = O.act_quant(y0)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
