"""Thin Python binding of the C ABI in include/bitnet.h.

Argument marshalling only: PyTorch provides device memory and the current
stream; every step of the computation runs in the library's CUDA kernels.
The binding refuses to run when the shared library is missing (there is no
fallback of any kind).

Function names match the C entry points.  Tensors must live on the CUDA
device; bf16 arrays may be passed as torch.bfloat16 or as 16-bit integer
tensors holding the bit patterns.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet_b200.so")

STATUS = {
    0: "BITNET_OK", 1: "BITNET_ERR_INVALID_ARG", 2: "BITNET_ERR_SHAPE", 3: "BITNET_ERR_ALIGN",
    4: "BITNET_ERR_WORKSPACE", 5: "BITNET_ERR_UNSUPPORTED", 6: "BITNET_ERR_CUDA",
    7: "BITNET_ERR_TIMEOUT", 8: "BITNET_ERR_NONFINITE",
}

# name -> (restype, argtypes)
_P, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "bitnet_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bitnet_version": (ctypes.c_int, []),
    "bitnet_pack_workspace_size": (_SZ, [_I64, _I64]),
    "bitnet_pack_weights": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "bitnet_quant_act": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P]),
    "bitnet_linear_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitnet_linear": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bitnet_ffn_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitnet_ffn": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _F,
                                  _P, _P, _P, _SZ, _P]),
    "bitnet_last_device_status": (ctypes.c_int, [_P]),
    "bitnet_linear_noalloc": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _I64, _P, _P]),
    "bitnet_linear_chain_workspace_size": (_SZ, [_I64, _P, _P, _I64]),
    "bitnet_linear_chain": (ctypes.c_int, [_I64, _P, _P, _P, _P, _P, _I64, _P, _P, _SZ, _P]),
    "bitnet_linear_multi_workspace_size": (_SZ, [_I64, _P, _I64, _I64]),
    "bitnet_linear_multi": (ctypes.c_int, [_I64, _P, _P, _P, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "bitnet_pack_w1_workspace_size": (_SZ, [_I64, _I64]),
    "bitnet_pack_weights_w1": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "bitnet_linear_w1_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitnet_linear_w1": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bitnet_linear_tl2": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _P, _P, _P, _P]),
    "bitnet_quant_act_a48": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "bitnet_linear_a48_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitnet_linear_a48": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _I64, _I64, _P, _P, _P, _P, _P,
                                         _SZ, _P]),
    "bitnet_ffn_tp_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bitnet_ffn_tp_gate_up": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _P,
                                             _P, _P, _P, _SZ, _P]),
    "bitnet_ffn_tp_down": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _SZ, _P]),
    "bitnet_ffn_tp_finish": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _F, _P, _P,
                                            _P]),
}


class FfnDebug(ctypes.Structure):
    _fields_ = [("xq1", _P), ("acc_gate", _P), ("acc_up", _P), ("h", _P), ("xq2", _P),
                ("acc_down", _P), ("y_f32", _P)]


class BitnetError(RuntimeError):
    def __init__(self, func: str, status: int):
        super().__init__(f"{func} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "ternary_weight_linear_int8_b200/build.py (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(name, st):
    if st != 0:
        raise BitnetError(name, st)


def _dev(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _bits16(t, name):
    _dev(t, name)
    if t.element_size() != 2:
        raise ValueError(f"{name} must hold 16-bit (bf16) elements")
    return t


def _workspace(nbytes, device, ws=None):
    if nbytes == 0:
        return None
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


def bitnet_status_string(status: int) -> str:
    return lib().bitnet_status_string(status).decode()


def bitnet_version() -> int:
    return lib().bitnet_version()


def bitnet_pack_weights(W: torch.Tensor, packed=None, gamma=None, workspace=None):
    """W fp32 [N,K] -> (packed uint8 [N,K/4], gamma fp32 [1])."""
    _dev(W, "W")
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device) if packed is None else packed
    gamma = torch.empty(1, dtype=torch.float32, device=W.device) if gamma is None else gamma
    nb = lib().bitnet_pack_workspace_size(N, K)
    ws = _workspace(nb, W.device, workspace)
    st = lib().bitnet_pack_weights(_ptr(W), N, K, _ptr(packed), _ptr(gamma), _ptr(ws), nb, _stream())
    _check("bitnet_pack_weights", st)
    return packed, gamma


def bitnet_quant_act(x: torch.Tensor, with_rowsum: bool = True, xq=None, scale=None,
                     rowsum=None):
    """x bf16 [M,K] -> (x_q int8 [M,K], scale fp32 [M], rowsum int32 [M] or None).
    The outputs may be given as preallocated tensors."""
    _bits16(x, "x")
    M, K = x.shape
    xq = torch.empty((M, K), dtype=torch.int8, device=x.device) if xq is None else _dev(xq, "xq")
    s = torch.empty(M, dtype=torch.float32, device=x.device) if scale is None else _dev(scale, "scale")
    rs = rowsum if rowsum is not None else (
        torch.empty(M, dtype=torch.int32, device=x.device) if with_rowsum else None)
    st = lib().bitnet_quant_act(_ptr(x), M, K, _ptr(xq), _ptr(s), _ptr(rs), _stream())
    _check("bitnet_quant_act", st)
    return xq, s, rs


def bitnet_linear_workspace_size(M: int, N: int, K: int) -> int:
    return lib().bitnet_linear_workspace_size(M, N, K)


def bitnet_linear(packed: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor, y=None,
                  want_f32: bool = False, want_acc: bool = False, workspace=None,
                  y_f32=None, acc=None):
    """y = BitLinear(x) on packed weights.  Returns (y bf16 [M,N], y_f32, acc).
    `y`, `y_f32` and `acc` may be given as preallocated [M,N] tensors."""
    _dev(packed, "packed")
    _dev(gamma, "gamma")
    _bits16(x, "x")
    N, Kb = packed.shape
    M, K = x.shape
    if K != 4 * Kb:
        raise ValueError("x and packed disagree on K")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    y32 = y_f32 if y_f32 is not None else (
        torch.empty((M, N), dtype=torch.float32, device=x.device) if want_f32 else None)
    acc = acc if acc is not None else (
        torch.empty((M, N), dtype=torch.int32, device=x.device) if want_acc else None)
    for t, name in ((y, "y"), (y32, "y_f32"), (acc, "acc")):
        if t is not None:
            _dev(t, name)
            if tuple(t.shape) != (M, N):
                raise ValueError(f"{name} must have shape [M, N]")
    nb = lib().bitnet_linear_workspace_size(M, N, K)
    ws = _workspace(nb, x.device, workspace)
    st = lib().bitnet_linear(_ptr(packed), _ptr(gamma), N, K, _ptr(x), M, _ptr(y), _ptr(y32),
                             _ptr(acc), _ptr(ws), nb, _stream())
    _check("bitnet_linear", st)
    return y, y32, acc


def bitnet_ffn_workspace_size(M: int, H: int, I: int) -> int:
    return lib().bitnet_ffn_workspace_size(M, H, I)


@dataclass
class FfnWeights:
    gate: torch.Tensor
    gamma_gate: torch.Tensor
    up: torch.Tensor
    gamma_up: torch.Tensor
    down: torch.Tensor
    gamma_down: torch.Tensor
    norm1_w: torch.Tensor | None = None
    norm2_w: torch.Tensor | None = None


def bitnet_ffn(x: torch.Tensor, w: FfnWeights, eps: float = 1e-5, y=None, debug=False,
               workspace=None):
    """Fused FFN block.  Returns (y bf16 [M,H], dict of debug outputs or None).
    `debug` is False, True (the binding allocates the debug outputs) or a dict
    of preallocated tensors with the keys below."""
    _bits16(x, "x")
    M, H = x.shape
    I = w.gate.shape[0]
    dev = x.device
    y = torch.empty((M, H), dtype=torch.bfloat16, device=dev) if y is None else y
    dbg = None
    dstruct = None
    if isinstance(debug, dict):
        dbg = debug
    elif debug:
        dbg = {
            "xq1": torch.empty((M, H), dtype=torch.int8, device=dev),
            "acc_gate": torch.empty((M, I), dtype=torch.int32, device=dev),
            "acc_up": torch.empty((M, I), dtype=torch.int32, device=dev),
            "h": torch.empty((M, I), dtype=torch.float32, device=dev),
            "xq2": torch.empty((M, I), dtype=torch.int8, device=dev),
            "acc_down": torch.empty((M, H), dtype=torch.int32, device=dev),
            "y_f32": torch.empty((M, H), dtype=torch.float32, device=dev),
        }
    if dbg is not None:
        dstruct = FfnDebug(*[_ptr(dbg[k]) for k in
                             ("xq1", "acc_gate", "acc_up", "h", "xq2", "acc_down", "y_f32")])
    nb = lib().bitnet_ffn_workspace_size(M, H, I)
    ws = _workspace(nb, dev, workspace)
    st = lib().bitnet_ffn(_ptr(x), M, H, I, _ptr(w.norm1_w), _ptr(w.gate), _ptr(w.gamma_gate),
                          _ptr(w.up), _ptr(w.gamma_up), _ptr(w.norm2_w), _ptr(w.down),
                          _ptr(w.gamma_down), float(eps), _ptr(y),
                          ctypes.byref(dstruct) if dstruct is not None else None,
                          _ptr(ws), nb, _stream())
    _check("bitnet_ffn", st)
    return y, dbg


def _host_arrays(packs, gammas, ys, x):
    L = len(packs)
    Ns = (ctypes.c_int64 * L)(*[int(p.shape[0]) for p in packs])
    Ks = (ctypes.c_int64 * L)(*[int(p.shape[1]) * 4 for p in packs])
    P = (ctypes.c_void_p * L)(*[p.data_ptr() for p in packs])
    G = (ctypes.c_void_p * L)(*[g.data_ptr() for g in gammas])
    Y = (ctypes.c_void_p * L)(*[y.data_ptr() for y in ys])
    return L, Ns, Ks, P, G, Y


def bitnet_linear_chain_workspace_size(Ns, Ks, M: int) -> int:
    L = len(Ns)
    n = (ctypes.c_int64 * L)(*Ns)
    k = (ctypes.c_int64 * L)(*Ks)
    return lib().bitnet_linear_chain_workspace_size(L, n, k, M)


def bitnet_linear_chain(packs, gammas, x: torch.Tensor, ys=None, workspace=None):
    """Layers l = 0..L-1: y[l] = BitLinear(packs[l], gammas[l])(y[l-1]), y[-1] = x.
    `ys` (optional) are the output tensors, one per layer; a layer's output
    may not be its own input (ping-pong buffers are fine).  Returns ys."""
    _bits16(x, "x")
    if len(packs) != len(gammas) or not packs:
        raise ValueError("packs and gammas must be non-empty lists of equal length")
    M = x.shape[0]
    for p, g in zip(packs, gammas):
        _dev(p, "packed")
        _dev(g, "gamma")
    if ys is None:
        ys = [torch.empty((M, p.shape[0]), dtype=torch.bfloat16, device=x.device) for p in packs]
    for y in ys:
        _bits16(y, "y")
    L, Ns, Ks, P, G, Y = _host_arrays(packs, gammas, ys, x)
    nb = lib().bitnet_linear_chain_workspace_size(L, Ns, Ks, M)
    ws = _workspace(nb, x.device, workspace)
    st = lib().bitnet_linear_chain(L, P, G, Ns, Ks, _ptr(x), M, Y, _ptr(ws), nb, _stream())
    _check("bitnet_linear_chain", st)
    return ys


def bitnet_linear_multi_workspace_size(Ns, K: int, M: int) -> int:
    L = len(Ns)
    n = (ctypes.c_int64 * L)(*Ns)
    return lib().bitnet_linear_multi_workspace_size(L, n, K, M)


def bitnet_linear_multi(packs, gammas, x: torch.Tensor, ys=None, workspace=None):
    """Matrices l = 0..L-1 on one input: y[l] = BitLinear(packs[l], gammas[l])(x)
    (e.g. query/key/value or gate/up projections).  All matrices share K;
    `ys` (optional) are the output tensors, one per matrix, none overlapping
    x or each other.  Returns ys."""
    _bits16(x, "x")
    if len(packs) != len(gammas) or not packs:
        raise ValueError("packs and gammas must be non-empty lists of equal length")
    M, K = x.shape
    for p, g in zip(packs, gammas):
        _dev(p, "packed")
        _dev(g, "gamma")
        if int(p.shape[1]) * 4 != K:
            raise ValueError("every packed matrix must have K/4 columns")
    if ys is None:
        ys = [torch.empty((M, p.shape[0]), dtype=torch.bfloat16, device=x.device) for p in packs]
    for y in ys:
        _bits16(y, "y")
    L, Ns, _, P, G, Y = _host_arrays(packs, gammas, ys, x)
    nb = lib().bitnet_linear_multi_workspace_size(L, Ns, K, M)
    ws = _workspace(nb, x.device, workspace)
    st = lib().bitnet_linear_multi(L, P, G, Ns, K, _ptr(x), M, Y, _ptr(ws), nb, _stream())
    _check("bitnet_linear_multi", st)
    return ys


class PreparedChain:
    """bitnet_linear_chain with its argument arrays and workspace built once:
    calling it enqueues the whole chain with one C call (the layers' device
    pointers, shapes and output buffers are fixed; only x and the stream
    change from call to call)."""

    def __init__(self, packs, gammas, ys, workspace=None):
        if len(packs) != len(gammas) or len(packs) != len(ys) or not packs:
            raise ValueError("packs, gammas and ys must be non-empty lists of equal length")
        for p, g, y in zip(packs, gammas, ys):
            _dev(p, "packed")
            _dev(g, "gamma")
            _bits16(y, "y")
        self.M = ys[0].shape[0]
        self.K0 = packs[0].shape[1] * 4
        self._keep = (list(packs), list(gammas), list(ys))
        self.L, self.Ns, self.Ks, self.P, self.G, self.Y = _host_arrays(packs, gammas, ys, None)
        nb = lib().bitnet_linear_chain_workspace_size(self.L, self.Ns, self.Ks, self.M)
        self.nb = nb
        self.ws = _workspace(nb, ys[0].device, workspace)
        self.ys = ys
        self._fn = lib().bitnet_linear_chain
        self._ws_ptr = _ptr(self.ws)

    def __call__(self, x: torch.Tensor):
        if x.shape[0] != self.M or x.shape[1] != self.K0:
            raise ValueError("x does not match the prepared chain")
        st = self._fn(self.L, self.P, self.G, self.Ns, self.Ks, ctypes.c_void_p(x.data_ptr()),
                      self.M, self.Y, self._ws_ptr, self.nb, _stream())
        _check("bitnet_linear_chain", st)
        return self.ys[-1]

    def capture(self, x: torch.Tensor):
        """Record the chain on the input buffer x into a CUDA graph (one
        eager call first, so that every kernel is loaded) and return a
        function that replays it on the current stream: one launch for the
        whole chain.  New inputs are written into x between replays; the
        result is self.ys[-1].  The graph holds the buffers it was recorded
        on (x, the outputs, the workspace)."""
        if x.shape[0] != self.M or x.shape[1] != self.K0:
            raise ValueError("x does not match the prepared chain")
        side = torch.cuda.Stream(device=x.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self(x)
        side.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self(x)
        self._graph = graph
        self._graph_x = x
        return graph.replay


def bitnet_linear_noalloc(packed: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor, y=None):
    """BitLinear using the library's fixed device scratch array instead of a
    workspace (for callers that cannot allocate).  Returns y bf16 [M,N]."""
    _dev(packed, "packed")
    _dev(gamma, "gamma")
    _bits16(x, "x")
    N, Kb = packed.shape
    M, K = x.shape
    if K != 4 * Kb:
        raise ValueError("x and packed disagree on K")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    st = lib().bitnet_linear_noalloc(_ptr(packed), _ptr(gamma), N, K, _ptr(x), M, _ptr(y),
                                     _stream())
    _check("bitnet_linear_noalloc", st)
    return y


def bitnet_linear_w1_workspace_size(M: int, N: int, K: int) -> int:
    return lib().bitnet_linear_w1_workspace_size(M, N, K)


def bitnet_pack_weights_w1(W: torch.Tensor, packed=None, alpha=None, workspace=None):
    """BitNet v1 sign weights: W fp32 [N,K] -> (packed uint8 [N,K/8], alpha fp32 [1])."""
    _dev(W, "W")
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    packed = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device) if packed is None else packed
    alpha = torch.empty(1, dtype=torch.float32, device=W.device) if alpha is None else alpha
    nb = lib().bitnet_pack_w1_workspace_size(N, K)
    ws = _workspace(nb, W.device, workspace)
    st = lib().bitnet_pack_weights_w1(_ptr(W), N, K, _ptr(packed), _ptr(alpha), _ptr(ws), nb,
                                      _stream())
    _check("bitnet_pack_weights_w1", st)
    return packed, alpha


def bitnet_linear_w1(packed: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, y=None,
                     want_f32: bool = False, want_acc: bool = False, workspace=None,
                     y_f32=None, acc=None):
    """W1A8 BitLinear on sign-packed weights.  Returns (y bf16 [M,N], y_f32, acc)."""
    _dev(packed, "packed")
    _dev(alpha, "alpha")
    _bits16(x, "x")
    N, Kb = packed.shape
    M, K = x.shape
    if K != 8 * Kb:
        raise ValueError("x and packed disagree on K")
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    y32 = y_f32 if y_f32 is not None else (
        torch.empty((M, N), dtype=torch.float32, device=x.device) if want_f32 else None)
    acc = acc if acc is not None else (
        torch.empty((M, N), dtype=torch.int32, device=x.device) if want_acc else None)
    nb = lib().bitnet_linear_w1_workspace_size(M, N, K)
    ws = _workspace(nb, x.device, workspace)
    st = lib().bitnet_linear_w1(_ptr(packed), _ptr(alpha), N, K, _ptr(x), M, _ptr(y), _ptr(y32),
                                _ptr(acc), _ptr(ws), nb, _stream())
    _check("bitnet_linear_w1", st)
    return y, y32, acc


def bitnet_linear_tl2(packed: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor, y=None,
                      want_f32: bool = False, want_acc: bool = False, y_f32=None, acc=None):
    """One-token BitLinear through pair lookup tables (same result as bitnet_linear)."""
    _dev(packed, "packed")
    _dev(gamma, "gamma")
    _bits16(x, "x")
    N, Kb = packed.shape
    M, K = x.shape
    if M != 1 or K != 4 * Kb:
        raise ValueError("x must be [1, K] with K = 4 * packed.shape[1]")
    y = torch.empty((1, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    y32 = y_f32 if y_f32 is not None else (
        torch.empty((1, N), dtype=torch.float32, device=x.device) if want_f32 else None)
    acc = acc if acc is not None else (
        torch.empty((1, N), dtype=torch.int32, device=x.device) if want_acc else None)
    st = lib().bitnet_linear_tl2(_ptr(packed), _ptr(gamma), N, K, _ptr(x), _ptr(y), _ptr(y32),
                                 _ptr(acc), _stream())
    _check("bitnet_linear_tl2", st)
    return y, y32, acc


def bitnet_quant_act_a48(x: torch.Tensor, n_out: int):
    """a4.8 activations: x bf16 [M,K] -> (q4 int8 [M,K], s4 [M], q8 int8 [M,K], s8 [M])."""
    _bits16(x, "x")
    M, K = x.shape
    q4 = torch.empty((M, K), dtype=torch.int8, device=x.device)
    q8 = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s4 = torch.empty(M, dtype=torch.float32, device=x.device)
    s8 = torch.empty(M, dtype=torch.float32, device=x.device)
    st = lib().bitnet_quant_act_a48(_ptr(x), M, K, int(n_out), _ptr(q4), _ptr(s4), _ptr(q8),
                                    _ptr(s8), _stream())
    _check("bitnet_quant_act_a48", st)
    return q4, s4, q8, s8


def bitnet_linear_a48_workspace_size(M: int, N: int, K: int) -> int:
    return lib().bitnet_linear_a48_workspace_size(M, N, K)


def bitnet_linear_a48(packed: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor, n_out: int,
                      y=None, want_f32: bool = False, want_acc: bool = False, workspace=None,
                      y_f32=None, acc4=None, acc8=None):
    """a4.8 BitLinear.  Returns (y bf16 [M,N], y_f32, acc4, acc8)."""
    _dev(packed, "packed")
    _dev(gamma, "gamma")
    _bits16(x, "x")
    N, Kb = packed.shape
    M, K = x.shape
    if K != 4 * Kb:
        raise ValueError("x and packed disagree on K")
    dev = x.device
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    y32 = y_f32 if y_f32 is not None else (
        torch.empty((M, N), dtype=torch.float32, device=dev) if want_f32 else None)
    if want_acc:
        acc4 = torch.empty((M, N), dtype=torch.int32, device=dev) if acc4 is None else acc4
        acc8 = torch.empty((M, N), dtype=torch.int32, device=dev) if acc8 is None else acc8
    nb = lib().bitnet_linear_a48_workspace_size(M, N, K)
    ws = _workspace(nb, dev, workspace)
    st = lib().bitnet_linear_a48(_ptr(packed), _ptr(gamma), N, K, _ptr(x), M, int(n_out), _ptr(y),
                                 _ptr(y32), _ptr(acc4), _ptr(acc8), _ptr(ws), nb, _stream())
    _check("bitnet_linear_a48", st)
    return y, y32, acc4, acc8


def bitnet_ffn_tp_workspace_size(M: int, H: int, Ir: int) -> int:
    return lib().bitnet_ffn_tp_workspace_size(M, H, Ir)


def bitnet_ffn_tp_gate_up(x, gate, gamma_gate, up, gamma_up, norm1_w=None, norm2_w=None,
                          workspace=None):
    """Tensor-parallel FFN step 1 on this shard.  Returns (h [M,Ir] fp32,
    amax2 [M] fp32, sumsq_h [M] fp64, sumsq_x [M] fp64)."""
    _bits16(x, "x")
    M, H = x.shape
    Ir = gate.shape[0]
    dev = x.device
    h = torch.empty((M, Ir), dtype=torch.float32, device=dev)
    amax2 = torch.empty(M, dtype=torch.float32, device=dev)
    ssh = torch.empty(M, dtype=torch.float64, device=dev)
    ssx = torch.empty(M, dtype=torch.float64, device=dev)
    nb = lib().bitnet_ffn_tp_workspace_size(M, H, Ir)
    ws = _workspace(nb, dev, workspace)
    st = lib().bitnet_ffn_tp_gate_up(_ptr(x), M, H, Ir, _ptr(norm1_w), _ptr(gate), _ptr(gamma_gate),
                                     _ptr(up), _ptr(gamma_up), _ptr(norm2_w), _ptr(h), _ptr(amax2),
                                     _ptr(ssh), _ptr(ssx), _ptr(ws), nb, _stream())
    _check("bitnet_ffn_tp_gate_up", st)
    return h, amax2, ssh, ssx


def bitnet_ffn_tp_down(h, down, amax2, norm2_w=None, workspace=None):
    """Tensor-parallel FFN step 3 on this shard: partial int32 accumulators [M,H]."""
    _dev(h, "h")
    M, Ir = h.shape
    H = down.shape[0]
    acc = torch.empty((M, H), dtype=torch.int32, device=h.device)
    nb = lib().bitnet_ffn_tp_workspace_size(M, H, Ir)
    ws = _workspace(nb, h.device, workspace)
    st = lib().bitnet_ffn_tp_down(_ptr(h), M, H, Ir, _ptr(norm2_w), _ptr(down), _ptr(amax2),
                                  _ptr(acc), _ptr(ws), nb, _stream())
    _check("bitnet_ffn_tp_down", st)
    return acc


def bitnet_ffn_tp_finish(acc, I, gamma_down, amax2, sumsq_x, sumsq_h, eps=1e-5, y=None,
                         want_f32=False):
    """Tensor-parallel FFN step 5: y bf16 [M,H] (and y_f32) from the all-reduced values."""
    _dev(acc, "acc")
    M, H = acc.shape
    y = torch.empty((M, H), dtype=torch.bfloat16, device=acc.device) if y is None else y
    y32 = torch.empty((M, H), dtype=torch.float32, device=acc.device) if want_f32 else None
    st = lib().bitnet_ffn_tp_finish(_ptr(acc), M, H, int(I), _ptr(gamma_down), _ptr(amax2),
                                    _ptr(sumsq_x), _ptr(sumsq_h), float(eps), _ptr(y), _ptr(y32),
                                    _stream())
    _check("bitnet_ffn_tp_finish", st)
    return y, y32


def bitnet_last_device_status() -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    return lib().bitnet_last_device_status(_stream())
