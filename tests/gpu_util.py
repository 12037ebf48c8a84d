"""Helpers for GPU parity tests: host numpy <-> device tensors, oracle runs.
Imports no kernel code; the CUDA path is reached only through the binding."""
from __future__ import annotations

import numpy as np
import torch

from oracle import bitlinear as O


def dev_bits(x_bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA int16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def f32_bits(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def assert_f32_rel(got: np.ndarray, want: np.ndarray, tol: float = 1e-5):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape
    nz = want != 0
    assert np.all(got[~nz] == 0), "expected zeros differ"
    if nz.any():
        rel = np.abs(got[nz] - want[nz]) / np.abs(want[nz])
        assert rel.max() <= tol, f"max rel err {rel.max():.3e} > {tol}"


def assert_bf16_close(got_bits: np.ndarray, want_bits: np.ndarray, got32, want32):
    """bf16 outputs: identical wherever the fp32 values are identical, else at
    most one bf16 ulp apart (the fp32 values straddle a rounding boundary)."""
    same32 = f32_bits(got32) == f32_bits(want32)
    assert np.array_equal(got_bits[same32], want_bits[same32])
    d = np.abs(got_bits.astype(np.int64) - want_bits.astype(np.int64))
    assert d[~same32].max(initial=0) <= 1


def oracle_pack(W: np.ndarray):
    return O.pack_weights(W)


class Guarded:
    """A device output with guard bands: the tensor `t` sits inside a larger
    allocation whose 256 bytes before it and 4 KB after it hold a sentinel
    byte pattern.  check() asserts that no kernel wrote outside `t` (the
    bounds check that stands in for a memory checker)."""

    HEAD = 256
    TAIL = 4096
    SENTINEL = 0xA5

    def __init__(self, shape, dtype):
        es = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape))
        self.head = self.HEAD // es
        self.full = torch.empty(self.head + self.n + self.TAIL // es, dtype=dtype, device="cuda")
        self.full.view(torch.uint8).fill_(self.SENTINEL)
        self.t = self.full[self.head:self.head + self.n].view(shape)
        self.es = es

    def check(self):
        raw = self.full.view(torch.uint8)
        lo = self.head * self.es
        hi = lo + self.n * self.es
        assert bool((raw[:lo] == self.SENTINEL).all()), "write before the start of an output"
        assert bool((raw[hi:] == self.SENTINEL).all()), "write past the end of an output"


def guarded(shape, dtype):
    return Guarded(shape, dtype)
