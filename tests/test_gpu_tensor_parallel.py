"""The tensor-parallel FFN steps (bitnet_ffn_tp_*) on the GPU.

Two shards of one block run one after the other on one GPU, the two
all-reduces done between them by the test (the ranks never wait on one
another): every shard's h', the all-reduced integer accumulators and the
codes must equal the single-device bitnet_ffn's bit for bit, and y32 the
oracle's within 1e-5.  Then the orchestration module with a one-rank NCCL
group (the collectives as calls, on the GPU tensors)."""
from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from oracle import bitlinear as O
from ternary_weight_linear_int8_b200 import bitnet as B
from ternary_weight_linear_int8_b200 import inputs
from ternary_weight_linear_int8_b200 import tensor_parallel as TP
from tests.gpu_util import assert_bf16_close, assert_f32_rel, dev_bits, dev_f32, host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert B.bitnet_last_device_status() == 0


def _block(M, H, I, seed):
    rng = np.random.default_rng(seed)
    x = inputs.activations((M, H), rng=rng, outliers=True)
    Ws = [inputs.weights(I, H, rng=rng), inputs.weights(I, H, rng=rng), inputs.weights(H, I, rng=rng)]
    n1 = (1 + 0.2 * rng.standard_normal(H)).astype(np.float32)
    n2 = (1 + 0.2 * rng.standard_normal(I)).astype(np.float32)
    return x, Ws, n1, n2


@pytest.mark.parametrize("M,H,I,world", [(1, 512, 1024, 2), (4, 2560, 6912, 2), (64, 256, 512, 2),
                                         (3, 256, 768, 3)])
def test_tp_shards_on_one_gpu_match_single_device(M, H, I, world):
    x, Ws, n1, n2 = _block(M, H, I, seed=M + H + I)
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    full = B.FfnWeights(packs[0][0], packs[0][1], packs[1][0], packs[1][1], packs[2][0],
                        packs[2][1], dev_f32(n1), dev_f32(n2))
    xd = dev_bits(x)
    y_ref, dbg = B.bitnet_ffn(xd, full, eps=1e-5, debug=True)
    shards = [TP.shard_packed_ffn(packs[0][0], packs[0][1], packs[1][0], packs[1][1],
                                  packs[2][0], packs[2][1], I, world, r, norm1_w=full.norm1_w,
                                  norm2_w=full.norm2_w) for r in range(world)]
    ops = TP.GpuFfnOps(B)
    parts = [ops.gate_up(xd, s) for s in shards]
    for s, (h, _, _, ssx) in zip(shards, parts):
        assert torch.equal(h, dbg["h"][:, s.i0:s.i1])
        assert torch.equal(ssx, parts[0][3])
    amax2 = parts[0][1].clone()
    ssh = parts[0][2].clone()
    for _, a2, sh, _ in parts[1:]:
        amax2 = torch.maximum(amax2, a2)
        ssh = ssh + sh
    acc = sum(ops.down(h, s, amax2) for s, (h, _, _, _) in zip(shards, parts))
    assert torch.equal(acc, dbg["acc_down"])
    y, y32 = ops.finish(acc, shards[0], amax2, parts[0][3], ssh, 1e-5)
    ref = O.ffn(x, O.pack_weights(Ws[0]), O.pack_weights(Ws[1]), O.pack_weights(Ws[2]), n1, n2,
                1e-5)
    assert np.array_equal(acc.cpu().numpy(), ref["acc_down"].astype(np.int32))
    assert_f32_rel(y32.cpu().numpy(), ref["y32"], 1e-5)
    assert_bf16_close(host_bits(y), ref["y"], y32.cpu().numpy(), ref["y32"])
    assert_bf16_close(host_bits(y), host_bits(y_ref), y32.cpu().numpy(),
                      dbg["y_f32"].cpu().numpy())


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def test_tp_orchestration_one_rank_nccl():
    M, H, I = 2, 512, 1024
    x, Ws, n1, n2 = _block(M, H, I, seed=5)
    packs = [B.bitnet_pack_weights(dev_f32(W)) for W in Ws]
    full = B.FfnWeights(packs[0][0], packs[0][1], packs[1][0], packs[1][1], packs[2][0],
                        packs[2][1], dev_f32(n1), dev_f32(n2))
    xd = dev_bits(x)
    _, dbg = B.bitnet_ffn(xd, full, eps=1e-5, debug=True)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        shard = TP.shard_packed_ffn(packs[0][0], packs[0][1], packs[1][0], packs[1][1],
                                    packs[2][0], packs[2][1], I, 1, 0, norm1_w=full.norm1_w,
                                    norm2_w=full.norm2_w)
        y, y32 = TP.tp_ffn(xd, shard, TP.GpuFfnOps(B), eps=1e-5)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert_f32_rel(y32.cpu().numpy(), dbg["y_f32"].cpu().numpy(), 1e-5)
