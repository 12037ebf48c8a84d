"""GPU parity of bitnet_linear_chain: a chain of BitLinear layers, each fed
the previous one's output (one launch per layer, programmatic dependent
launch between them), must give, layer for layer, exactly the oracle's bf16
outputs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import bitlinear as O
from ternary_weight_linear_int8_b200 import bitnet as B
from ternary_weight_linear_int8_b200 import inputs
from tests.gpu_util import dev_bits, dev_f32, guarded, host_bits

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


def _chain_case(dims, M, seed):
    """dims = [K0, N0, N1, ...]: layer l maps dims[l] -> dims[l+1]."""
    rng = np.random.default_rng(seed)
    x = inputs.activations((M, dims[0]), rng=rng, outliers=dims[0] >= 100)
    Ws = [inputs.weights(dims[l + 1], dims[l], rng=rng) for l in range(len(dims) - 1)]
    return x, Ws


def _run_chain(Ws, x, ys=None):
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    return B.bitnet_linear_chain([p for p, _ in packs], [g for _, g in packs], dev_bits(x), ys=ys)


@pytest.mark.parametrize("M", [1, 2, 3, 8])
def test_chain_small_layers_match_oracle(M):
    """Nine decode-range layers of mixed widths."""
    dims = [512, 1024, 256, 768, 64, 320, 2048, 128, 640, 512]
    x, Ws = _chain_case(dims, M, seed=11 + M)
    ys = _run_chain(Ws, x)
    for l, want in enumerate(_oracle_chain(Ws, x)):
        assert np.array_equal(host_bits(ys[l]), want), f"layer {l}"


@pytest.mark.parametrize("M", [2, 4, 8])
def test_chain_2b_shapes_batched(M):
    """2B-class layers, up [6912,2560] then down [2560,6912], twice, with M
    tokens carrying outlier channels: every layer's output equals the
    oracle's, and no layer writes outside its output."""
    L = 4
    x = inputs.activations((M, 2560), seed=M, outliers=True)
    Ws = [inputs.weights(*((6912, 2560) if l % 2 == 0 else (2560, 6912)),
                         seed=inputs.layer_seed(l)) for l in range(L)]
    want = _oracle_chain(Ws, x)
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    outs = [guarded((M, W.shape[0]), torch.bfloat16) for W in Ws]
    B.bitnet_linear_chain([p for p, _ in packs], [g for _, g in packs], dev_bits(x),
                          ys=[o.t for o in outs])
    torch.cuda.synchronize()
    for l in range(L):
        assert np.array_equal(host_bits(outs[l].t), want[l]), f"layer {l}"
        outs[l].check()


def test_chain_of_70_layers():
    """70 layers of mixed widths back to back."""
    rng = np.random.default_rng(3)
    dims = [256] + [int(v) for v in rng.choice([128, 192, 256, 384], size=70)]
    x, Ws = _chain_case(dims, 1, seed=5)
    ys = _run_chain(Ws, x)
    want = _oracle_chain(Ws, x)
    for l in (0, 1, 62, 63, 64, 65, 69):
        assert np.array_equal(host_bits(ys[l]), want[l]), f"layer {l}"


def test_chain_with_layers_outside_the_decode_range():
    """K % 64 != 0 (400) takes the scalar path between decode-kernel layers."""
    dims = [512, 400, 256, 320, 128, 400, 64]
    x, Ws = _chain_case(dims, 4, seed=21)
    ys = _run_chain(Ws, x)
    for l, want in enumerate(_oracle_chain(Ws, x)):
        assert np.array_equal(host_bits(ys[l]), want), f"layer {l}"


def test_chain_many_tokens_uses_tensor_cores():
    dims = [2560, 1024, 512, 2560]
    x, Ws = _chain_case(dims, 40, seed=8)
    ys = _run_chain(Ws, x)
    for l, want in enumerate(_oracle_chain(Ws, x)):
        assert np.array_equal(host_bits(ys[l]), want), f"layer {l}"


def test_chain_fullsize_2b_ping_pong_and_graph():
    """2B-class decode, x[1,2560] -> up [6912,2560] -> down [2560,6912] -> ...,
    eight distinct layers into two ping-pong buffers (as the benchmark runs
    it); eager and CUDA-graph replays equal the oracle."""
    L = 8
    x = inputs.activations((1, 2560), seed=0)
    Ws = [inputs.weights(*((6912, 2560) if l % 2 == 0 else (2560, 6912)),
                         seed=inputs.layer_seed(l)) for l in range(L)]
    want = _oracle_chain(Ws, x)
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    P, G = [p for p, _ in packs], [g for _, g in packs]
    bufs = [torch.empty((1, 6912), dtype=torch.bfloat16, device="cuda"),
            torch.empty((1, 2560), dtype=torch.bfloat16, device="cuda")]
    ys = [bufs[l % 2] for l in range(L)]
    xd = dev_bits(x)
    ws = torch.empty(B.bitnet_linear_chain_workspace_size([p.shape[0] for p in P],
                                                          [p.shape[1] * 4 for p in P], 1),
                     dtype=torch.uint8, device="cuda")
    # eager, one layer at a time checked through single-layer chains
    cur = xd
    for l in range(L):
        out = B.bitnet_linear_chain([P[l]], [G[l]], cur, ys=[bufs[l % 2]], workspace=ws)[0]
        assert np.array_equal(host_bits(out), want[l]), f"layer {l}"
        cur = out
    # the whole chain in one call, eager then captured
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
    bufs[0].zero_()
    bufs[1].zero_()
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(bufs[1]), want[-1])
    assert np.array_equal(host_bits(bufs[0]), want[-2])


@pytest.mark.parametrize("M", [1, 16])
def test_prepared_chain_graph_replay(M):
    """PreparedChain.capture: the chain recorded once as a CUDA graph on a
    fixed input buffer, replayed for two different inputs written into that
    buffer; every replay's output equals the oracle's."""
    dims = [512, 1024, 256, 768, 512]
    rng = np.random.default_rng(70 + M)
    Ws = [inputs.weights(dims[l + 1], dims[l], rng=rng) for l in range(len(dims) - 1)]
    xs = [inputs.activations((M, dims[0]), rng=rng, outliers=True) for _ in range(2)]
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    ys = [torch.empty((M, W.shape[0]), dtype=torch.bfloat16, device="cuda") for W in Ws]
    prog = B.PreparedChain([p for p, _ in packs], [g for _, g in packs], ys)
    xd = dev_bits(xs[0]).clone()
    replay = prog.capture(xd)
    for x in xs * 2:
        xd.copy_(dev_bits(x))
        replay()
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(ys[-1]), _oracle_chain(Ws, x)[-1])
