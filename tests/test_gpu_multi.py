"""GPU parity of bitnet_linear_multi: several BitLinear matrices applied to
one input (query/key/value, or gate/up) must each give exactly the oracle's
bf16 outputs for that matrix, on every path (decode kernels, batched decode,
tensor-core GEMMs sharing one quantisation of x, ragged K), and write
nothing outside their outputs."""
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


@pytest.mark.parametrize("M,K,Ns", [
    (1, 2560, (2560, 640, 640)),        # resident decode kernel, one launch per matrix
    (6, 2048, (512, 128, 400)),         # streaming decode kernel
    (16, 2560, (2560, 640, 640)),       # batched decode kernel
    (40, 2560, (2560, 640, 400)),       # tensor core, split K, one region per matrix
    (300, 1024, (1000, 256, 256)),      # tensor core, ragged token tile and N
    (1024, 2560, (6912, 6912)),         # gate/up at prefill size
    (40, 260, (200, 72)),               # K % 64 != 0: generic kernel
])
def test_multi_matches_oracle(M, K, Ns):
    rng = np.random.default_rng(M * 7 + K)
    x = inputs.activations((M, K), rng=rng, outliers=True)
    Ws = [inputs.weights(n, K, rng=rng) for n in Ns]
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    outs = [guarded((M, n), torch.bfloat16) for n in Ns]
    B.bitnet_linear_multi([p for p, _ in packs], [g for _, g in packs], dev_bits(x),
                          ys=[o.t for o in outs])
    torch.cuda.synchronize()
    for l, W in enumerate(Ws):
        want = O.linear_from_float(W, x)["y"]
        assert np.array_equal(host_bits(outs[l].t), want), f"matrix {l}"
        outs[l].check()


def test_multi_equals_separate_calls_and_reuses_workspace():
    """Two calls through one workspace (the split-K regions must start from
    zero again) equal bitnet_linear on each matrix."""
    M, K, Ns = 64, 2560, (2560, 512, 512)
    rng = np.random.default_rng(5)
    Ws = [inputs.weights(n, K, rng=rng) for n in Ns]
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    P, G = [p for p, _ in packs], [g for _, g in packs]
    ws = torch.empty(B.bitnet_linear_multi_workspace_size(list(Ns), K, M), dtype=torch.uint8,
                     device="cuda")
    for seed in (1, 2):
        x = dev_bits(inputs.activations((M, K), seed=seed, outliers=True))
        ys = B.bitnet_linear_multi(P, G, x, workspace=ws)
        for l in range(len(Ns)):
            ref = B.bitnet_linear(P[l], G[l], x)[0]
            assert torch.equal(ys[l].view(torch.int16), ref.view(torch.int16)), (seed, l)
