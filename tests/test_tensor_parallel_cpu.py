"""The tensor-parallel FFN orchestration (ternary_weight_linear_int8_b200.
tensor_parallel) as world_size-2 gloo process groups on the CPU.  The
per-shard steps are computed by oracle arithmetic (test code), so the test
checks the split and the collectives: every code and the all-reduced integer
accumulators must equal the unsharded oracle's bit for bit, and y32 must
agree within 1e-5 relative (the fp64 sum of squares is added in another
order)."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import bitlinear as O
from ternary_weight_linear_int8_b200 import inputs
from ternary_weight_linear_int8_b200 import tensor_parallel as TP


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The three per-shard steps in oracle arithmetic on CPU tensors."""

    def gate_up(self, x, s):
        xb = x.numpy().view(np.uint16)
        xf = O.bf16_bits_to_f32(xb)
        M, H = xf.shape
        n1 = np.ones(H, np.float32) if s.norm1_w is None else s.norm1_w.numpy()
        q1, s1, _ = O.act_quant_f32(xf * n1[None, :])
        ag = O.ternary_matmul(q1, O.unpack_i2s(s.gate.numpy(), H))
        au = O.ternary_matmul(q1, O.unpack_i2s(s.up.numpy(), H))
        g = ag.astype(np.float32) * (np.float32(s.gamma_gate.item()) / s1)[:, None]
        u = au.astype(np.float32) * (np.float32(s.gamma_up.item()) / s1)[:, None]
        rg = np.maximum(g, np.float32(0))
        h = (rg * rg) * u
        n2 = np.ones(h.shape[1], np.float32) if s.norm2_w is None else s.norm2_w.numpy()
        amax2 = np.abs(h * n2[None, :]).max(axis=1).astype(np.float32)
        ssh = (h.astype(np.float64) ** 2).sum(axis=1)
        ssx = (xf.astype(np.float64) ** 2).sum(axis=1)
        return (torch.from_numpy(h), torch.from_numpy(amax2), torch.from_numpy(ssh),
                torch.from_numpy(ssx))

    def down(self, h, s, amax2):
        hf = h.numpy()
        n2 = np.ones(hf.shape[1], np.float32) if s.norm2_w is None else s.norm2_w.numpy()
        v = hf * n2[None, :]
        s2 = O.QMAX_F32 / np.maximum(amax2.numpy(), O.EPS_F32)
        q2 = np.clip(np.rint(v * s2[:, None]), -128, 127).astype(np.int8)
        acc = O.ternary_matmul(q2, O.unpack_i2s(s.down.numpy(), hf.shape[1]))
        return torch.from_numpy(acc.astype(np.int32))

    def finish(self, acc, s, amax2, ssx, ssh, eps):
        H = acc.shape[1]
        e = float(np.float32(eps))
        r1 = 1.0 / np.sqrt(ssx.numpy() / H + e)
        r2 = 1.0 / np.sqrt(r1 ** 6 * (ssh.numpy() / s.I) + e)
        f = (r1 ** 3 * r2).astype(np.float32)
        s2 = O.QMAX_F32 / np.maximum(amax2.numpy(), O.EPS_F32)
        d = np.float32(s.gamma_down.item()) / s2
        y32 = (acc.numpy().astype(np.float32) * d[:, None]) * f[:, None]
        return torch.from_numpy(O.f32_to_bf16_bits(y32).view(np.int16)), torch.from_numpy(y32)


def _case(M=3, H=128, I=256, seed=0):
    rng = np.random.default_rng(seed)
    x = inputs.activations((M, H), rng=rng, outliers=True)
    Wg, Wu = inputs.weights(I, H, rng=rng), inputs.weights(I, H, rng=rng)
    Wd = inputs.weights(H, I, rng=rng)
    n1 = (1 + 0.2 * rng.standard_normal(H)).astype(np.float32)
    n2 = (1 + 0.2 * rng.standard_normal(I)).astype(np.float32)
    return x, O.pack_weights(Wg), O.pack_weights(Wu), O.pack_weights(Wd), n1, n2


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, (pg, gg), (pu, gu), (pd, gd), n1, n2 = _case()
        I = pg.shape[0]
        t = torch.from_numpy
        shard = TP.shard_packed_ffn(t(pg), t(np.array([gg])), t(pu), t(np.array([gu])), t(pd),
                                    t(np.array([gd])), I, world, rank, norm1_w=t(n1),
                                    norm2_w=t(n2))
        ops = OracleOps()
        xt = torch.from_numpy(x.view(np.int16))
        h, amax2, ssh, ssx = ops.gate_up(xt, shard)
        local_amax = amax2.clone()
        y, y32 = TP.tp_ffn(xt, shard, ops, eps=1e-5)
        out[rank] = (y.numpy().copy(), y32.numpy().copy(), local_amax.numpy().copy(),
                     (shard.i0, shard.i1))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_ffn_gloo_world2_matches_unsharded_oracle():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    x, G, U, D, n1, n2 = _case()
    ref = O.ffn(x, G, U, D, n1, n2, 1e-5)
    assert res[0][3] == (0, 128) and res[1][3] == (128, 256)
    # each rank saw only part of h'; the all-reduced max is the whole token's
    assert not np.array_equal(res[0][2], res[1][2])
    v = ref["h"] * n2[None, :]
    assert np.array_equal(np.maximum(res[0][2], res[1][2]), np.abs(v).max(axis=1))
    for r in range(world):
        y, y32 = res[r][0].view(np.uint16), res[r][1]
        rel = np.abs(y32.astype(np.float64) - ref["y32"]) / np.maximum(np.abs(ref["y32"]), 1e-30)
        assert rel[ref["y32"] != 0].max() < 1e-5
        same = y32.view(np.uint32) == ref["y32"].view(np.uint32)
        assert np.array_equal(y[same], ref["y"][same])
    # both ranks hold the identical result
    assert np.array_equal(res[0][1], res[1][1])


def test_shard_bounds():
    assert TP.shard_bounds(28672, 8, 0) == (0, 3584)
    assert TP.shard_bounds(28672, 8, 7) == (25088, 28672)
    assert TP.shard_bounds(320, 3, 1) == (64, 192)
    with pytest.raises(ValueError):
        TP.shard_bounds(100, 2, 0)
    with pytest.raises(ValueError):
        TP.shard_bounds(128, 4, 0)
