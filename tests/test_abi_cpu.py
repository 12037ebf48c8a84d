"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/bitnet.h declares, and rejects bad arguments on the host
before touching CUDA (the pointers below are never dereferenced)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from ternary_weight_linear_int8_b200 import bitnet as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    return B.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    # and the binding knows every one of them
    assert set(names) <= set(B.SIGNATURES)


def test_status_strings_and_version(L):
    assert B.bitnet_version() == 100
    for code, name in B.STATUS.items():
        assert B.bitnet_status_string(code) == name
    assert B.bitnet_status_string(99) == "BITNET_ERR_UNKNOWN"


def test_workspace_sizes_are_host_only(L):
    assert L.bitnet_pack_workspace_size(400, 512) >= 2052
    assert L.bitnet_linear_workspace_size(1, 6912, 2560) == 0          # fused decode kernel
    assert L.bitnet_linear_workspace_size(4096, 6912, 2560) >= 4096 * 2560
    assert L.bitnet_linear_workspace_size(64, 2560, 6912) >= 64 * 6912 + 64 * 2560 * 4
    assert L.bitnet_linear_workspace_size(8, 400, 68) >= 8 * 68        # ragged K
    assert L.bitnet_ffn_workspace_size(1, 8192, 28672) == 28672 * 4     # h' between the launches
    assert L.bitnet_ffn_workspace_size(2048, 8192, 28672) > 2048 * 28672 * 4


FAKE = 0x10000          # 16-byte aligned, never dereferenced
MIS = 0x10001           # misaligned


def test_linear_validation(L):
    lin = L.bitnet_linear
    ok_args = dict(packed=FAKE, gamma=FAKE, N=400, K=512, x=FAKE, M=8, y=FAKE, y32=None,
                   acc=None, ws=None, nb=0, stream=None)

    def call(**kw):
        a = dict(ok_args, **kw)
        return lin(a["packed"], a["gamma"], a["N"], a["K"], a["x"], a["M"], a["y"], a["y32"],
                   a["acc"], a["ws"], a["nb"], a["stream"])

    assert call(packed=None) == 1
    assert call(y=None) == 1
    assert call(K=510) == 2
    assert call(K=0) == 2
    assert call(M=0) == 2
    assert call(N=-1) == 2
    assert call(x=MIS) == 3
    assert call(packed=MIS) == 3
    assert call(y32=FAKE + 2) == 3
    # tensor-core shapes need a workspace
    assert call(M=4096, K=2560, N=6912) == 4
    assert call(M=4096, K=2560, N=6912, ws=FAKE, nb=16) == 4


def test_pack_quant_ffn_validation(L):
    assert L.bitnet_pack_weights(None, 4, 4, FAKE, FAKE, FAKE, 4096, None) == 1
    assert L.bitnet_pack_weights(FAKE, 4, 6, FAKE, FAKE, FAKE, 4096, None) == 2
    assert L.bitnet_pack_weights(MIS, 4, 8, FAKE, FAKE, FAKE, 4096, None) == 3
    assert L.bitnet_pack_weights(FAKE, 4, 8, FAKE, FAKE, FAKE, 16, None) == 4
    assert L.bitnet_pack_weights(FAKE, 4, 8, FAKE, FAKE, None, 4096, None) == 4
    assert L.bitnet_quant_act(None, 1, 8, FAKE, FAKE, None, None) == 1
    assert L.bitnet_quant_act(FAKE, 1, 6, FAKE, FAKE, None, None) == 2
    assert L.bitnet_quant_act(FAKE, 1, 8, MIS, FAKE, None, None) == 3
    f = L.bitnet_ffn
    args = [FAKE, 1, 256, 512, None, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1e-5, FAKE, None,
            FAKE, 1 << 20, None]
    a = list(args); a[5] = None
    assert f(*a) == 1
    a = list(args); a[12] = -1.0
    assert f(*a) == 1
    a = list(args); a[2] = 200
    assert f(*a) == 2
    a = list(args); a[0] = MIS
    assert f(*a) == 3
    a = list(args); a[16] = 16
    assert f(*a) == 4


def _chain_args(Ns, Ks, ys, x=FAKE):
    n = len(Ns)
    I64 = ctypes.c_int64 * n
    VP = ctypes.c_void_p * n
    return (n, VP(*([FAKE] * n)), VP(*([FAKE] * n)), I64(*Ns), I64(*Ks), x, VP(*ys))


def test_chain_workspace_and_validation(L):
    I64 = ctypes.c_int64 * 2
    # decode-range layers need no scratch; others reuse the largest layer's
    assert L.bitnet_linear_chain_workspace_size(2, I64(6912, 2560), I64(2560, 6912), 1) == 0
    big = L.bitnet_linear_chain_workspace_size(2, I64(6912, 2560), I64(2560, 6912), 4096)
    assert big == max(L.bitnet_linear_workspace_size(4096, 6912, 2560),
                      L.bitnet_linear_workspace_size(4096, 2560, 6912))
    assert L.bitnet_linear_chain_workspace_size(0, I64(1, 1), I64(4, 4), 1) == 0
    y0, y1 = 0x100000, 0x200000
    n, P, G, N, K, x, Y = _chain_args([6912, 2560], [2560, 6912], [y0, y1])
    ws, nb = None, 0

    def call(**kw):
        a = dict(n=n, P=P, G=G, N=N, K=K, x=x, M=1, Y=Y, ws=ws, nb=nb)
        a.update(kw)
        return L.bitnet_linear_chain(a["n"], a["P"], a["G"], a["N"], a["K"], a["x"], a["M"],
                                     a["Y"], a["ws"], a["nb"], None)

    assert call(n=0) == 1
    assert call(P=None) == 1
    assert call(x=None) == 1
    assert call(M=0) == 2
    # layer 1's K must equal layer 0's N
    _, _, _, N2, K2, _, _ = _chain_args([6912, 2560], [2560, 6000], [y0, y1])
    assert call(N=N2, K=K2) == 2
    assert call(x=MIS) == 3
    _, _, _, _, _, _, Ymis = _chain_args([6912, 2560], [2560, 6912], [y0, MIS])
    assert call(Y=Ymis) == 3
    # a layer's output overlapping its own input
    _, _, _, _, _, _, Yal = _chain_args([6912, 2560], [2560, 6912], [FAKE + 64, y1])
    assert call(Y=Yal) == 1
    _, _, _, _, _, _, Yal2 = _chain_args([6912, 2560], [2560, 6912], [y0, y0 + 16])
    assert call(Y=Yal2) == 1
    # ping-pong (y[2] == y[0]) is allowed by the aliasing rule; here it fails
    # only on the missing workspace that M = 64 needs
    n3, P3, G3, N3, K3, x3, Y3 = _chain_args([6912, 2560, 6912], [2560, 6912, 2560],
                                             [y0, y1, y0])
    assert L.bitnet_linear_chain(n3, P3, G3, N3, K3, x3, 64, Y3, None, 0, None) == 4
    need = L.bitnet_linear_chain_workspace_size(2, I64(6912, 2560), I64(2560, 6912), 64)
    assert call(M=64, ws=FAKE, nb=need - 1) == 4
    assert call(M=64, ws=MIS, nb=need) == 3


def test_multi_workspace_and_validation(L):
    I64 = ctypes.c_int64 * 3
    Ns = I64(2560, 512, 512)          # e.g. query, key and value projections
    # decode-range token counts quantise inside their kernels: no scratch
    assert L.bitnet_linear_multi_workspace_size(3, Ns, 2560, 1) == 0
    # tensor-core path: the codes, scales and row sums once (plus split-K
    # regions per matrix for <= 256 tokens), less than one scratch per matrix
    big = L.bitnet_linear_multi_workspace_size(3, Ns, 2560, 4096)
    assert 4096 * 2560 + 2 * 4096 * 4 <= big < 3 * L.bitnet_linear_workspace_size(4096, 2560, 2560)
    mid = L.bitnet_linear_multi_workspace_size(3, Ns, 2560, 64)
    assert mid >= 64 * 2560 + sum(64 * n * 4 for n in (2560, 512, 512))
    # 9..32 tokens may run the batched decode kernel: the largest single scratch
    assert L.bitnet_linear_multi_workspace_size(3, Ns, 2560, 16) == max(
        L.bitnet_linear_workspace_size(16, n, 2560) for n in (2560, 512, 512))
    assert L.bitnet_linear_multi_workspace_size(0, Ns, 2560, 1) == 0
    y = [0x100000, 0x200000, 0x300000]
    VP = ctypes.c_void_p * 3
    P, G, Y = VP(FAKE, FAKE, FAKE), VP(FAKE, FAKE, FAKE), VP(*y)

    def call(**kw):
        a = dict(n=3, P=P, G=G, N=Ns, K=2560, x=FAKE, M=1, Y=Y, ws=None, nb=0)
        a.update(kw)
        return L.bitnet_linear_multi(a["n"], a["P"], a["G"], a["N"], a["K"], a["x"], a["M"],
                                     a["Y"], a["ws"], a["nb"], None)

    assert call(n=0) == 1
    assert call(G=None) == 1
    assert call(Y=VP(y[0], None, y[2])) == 1
    assert call(M=0) == 2
    assert call(K=2562) == 2
    assert call(N=I64(2560, 0, 512)) == 2
    assert call(x=MIS) == 3
    assert call(Y=VP(y[0], MIS, y[2])) == 3
    # an output overlapping the input, or another output
    assert call(Y=VP(y[0], FAKE + 64, y[2])) == 1
    assert call(Y=VP(y[0], y[0] + 16, y[2])) == 1
    need = L.bitnet_linear_multi_workspace_size(3, Ns, 2560, 64)
    assert call(M=64) == 4
    assert call(M=64, ws=FAKE, nb=need - 1) == 4
    assert call(M=64, ws=MIS, nb=need) == 3


def test_binding_rejects_host_tensors_before_any_call():
    """The Python binding only marshals: tensors that are not on a GPU are
    refused before anything reaches the library."""
    import torch
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    p = torch.zeros((8, 16), dtype=torch.uint8)
    g = torch.ones((1,), dtype=torch.float32)
    for fn, args in ((B.bitnet_linear, (p, g, x)),
                     (B.bitnet_linear_multi, ([p], [g], x)),
                     (B.bitnet_linear_chain, ([p], [g], x)),
                     (B.bitnet_quant_act, (x,))):
        with pytest.raises(ValueError):
            fn(*args)
    with pytest.raises(ValueError):
        B.bitnet_linear_multi([], [], x)
    with pytest.raises(ValueError):
        B.bitnet_linear_multi([p, p], [g], x)
