"""bitnet_linear_noalloc: the workspace-free BitLinear entry point for callers
that cannot allocate device memory.  Through the C ABI it must give the same
output as bitnet_linear on two calls in a row (the shared scratch array keeps
the previous call's contents, so the second call checks that nothing stale
leaks into the result), and refuse shapes whose scratch exceeds the array.

This file is collected last on purpose."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from ternary_weight_linear_int8_b200 import bitnet as B
from ternary_weight_linear_int8_b200 import inputs
from tests.gpu_util import guarded

SCRATCH_BYTES = 32 * 1024 * 1024


def _dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [
    (1, 6912, 2560),       # decode kernel (needs no scratch)
    (64, 2560, 6912),      # tensor-core kernel with split-K accumulators in the scratch
    (300, 1000, 1024),     # tensor-core kernel, one K range
    (8, 400, 68),          # ragged K
    (4096, 2560, 2048),    # large prefill: 8 MiB of quantised activations
])
def test_noalloc_matches_linear_two_calls_in_a_row(M, N, K):
    assert B.bitnet_linear_workspace_size(M, N, K) <= SCRATCH_BYTES
    rng = np.random.default_rng(M + N + K)
    W = torch.from_numpy(inputs.weights(N, K, rng=rng)).cuda()
    xs = [_dev_bits(inputs.activations((M, K), rng=rng, outliers=True)) for _ in range(2)]
    p, g = B.bitnet_pack_weights(W)
    refs = [_bits(B.bitnet_linear(p, g, x)[0]) for x in xs]
    assert not np.array_equal(refs[0], refs[1])
    for x, ref in zip(xs, refs):            # two calls in a row, different inputs
        out = guarded((M, N), torch.bfloat16)
        y = B.bitnet_linear_noalloc(p, g, x, y=out.t)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(y), ref)
        out.check()
    assert B.bitnet_last_device_status() == 0


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_the_array():
    M, N, K = 4096, 2560, 16384            # 64 MiB of quantised activations
    assert B.bitnet_linear_workspace_size(M, N, K) > SCRATCH_BYTES
    p = torch.zeros((N, K // 4), dtype=torch.uint8, device="cuda")
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    st = B.lib().bitnet_linear_noalloc(ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(g.data_ptr()),
                                       N, K, ctypes.c_void_p(x.data_ptr()), M,
                                       ctypes.c_void_p(y.data_ptr()), None)
    assert st == 4                          # BITNET_ERR_WORKSPACE, nothing enqueued
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
