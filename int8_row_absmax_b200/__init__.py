"""Python binding of the B200 BitLinear library (ctypes over libbitlinear.so).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI (include/bitlinear.h).  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library was
not built, or no GPU is visible, every call raises.

    import int8_row_absmax_b200 as bl
    Wp, beta = bl.quantize_weights_pack5(W)          # W [N,K] float32 on cuda
    Y = bl.linear(X, Wp, bl.PACK5, N=W.shape[0], K=W.shape[1], beta=beta)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libbitlinear.so")

I8, PACK5 = 0, 1                       # bl_wfmt
PATH_AUTO, PATH_SIMT, PATH_GEMV, PATH_TC = 0, 1, 2, 3   # bl_path
FLAG_STATIC_WEIGHTS = 0x100            # BL_FLAG_STATIC_WEIGHTS

STATUS = {0: "BL_OK", 1: "BL_ERR_INVALID_ARG", 2: "BL_ERR_ALIGNMENT", 3: "BL_ERR_UNSUPPORTED",
          4: "BL_ERR_WORKSPACE", 5: "BL_ERR_CUDA", 6: "BL_ERR_DEVICE_TIMEOUT",
          7: "BL_ERR_NONFINITE", 8: "BL_ERR_IO"}

# Every symbol the header declares, with (restype, argtypes).
_P, _I64, _SZ, _F, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_int


class LinearCall(ctypes.Structure):
    """bl_linear_call: one call of bl_linear_group (field order and types as in the header)."""
    _fields_ = [("X", _P), ("M", _I64), ("K", _I64), ("W", _P), ("N", _I64), ("ldw", _I64),
                ("f", _I), ("eps", _F), ("beta_dev", _P), ("bias", _P), ("Y", _P)]


_CALLS = ctypes.POINTER(LinearCall)


class HostIO(ctypes.Structure):
    """bl_host_io: the host buffers of one call of bl_linear_group_host (as in the header)."""
    _fields_ = [("X_host", _P), ("Y_host", _P)]


_IOS = ctypes.POINTER(HostIO)


class DeployedLayer(ctypes.Structure):
    """bl_deployed_layer: one layer for bl_save_deployed (as in the header)."""
    _fields_ = [("name", ctypes.c_char_p), ("N", _I64), ("K", _I64), ("Wp", _P), ("ldp", _I64),
                ("beta_dev", _P), ("bias_dev", _P)]


_LAYERS = ctypes.POINTER(DeployedLayer)
SIGNATURES = {
    "bl_pack5_ldp": (_I64, [_I64]),
    "bl_quantize_weights_workspace_size": (_SZ, [_I64, _I64]),
    "bl_absmean": (_I, [_P, _I64, _I64, _F, _P, _P, _SZ, _P]),
    "bl_ternarize": (_I, [_P, _I64, _I64, _P, _P, _P]),
    "bl_ternarize_pack5": (_I, [_P, _I64, _I64, _P, _P, _I64, _P]),
    "bl_quantize_weights": (_I, [_P, _I64, _I64, _F, _P, _P, _P, _SZ, _P]),
    "bl_quantize_weights_pack5": (_I, [_P, _I64, _I64, _F, _P, _I64, _P, _P, _SZ, _P]),
    "bl_pack": (_I, [_P, _I64, _I64, _P, _I64, _P]),
    "bl_unpack": (_I, [_P, _I64, _I64, _I64, _P, _P]),
    "bl_quantize_act": (_I, [_P, _I64, _I64, _F, _P, _P, _P]),
    "bl_rmsnorm_quantize_act": (_I, [_P, _I64, _I64, _P, _F, _F, _P, _P, _P]),
    "bl_linear_workspace_size": (_SZ, [_I64, _I64, _I64, _I]),
    "bl_linear_ex_workspace_size": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "bl_linear": (_I, [_P, _I64, _I64, _P, _I, _I64, _I64, _P, _P, _F, _P, _P, _SZ, _P]),
    "bl_linear_ex": (_I, [_P, _I64, _I64, _P, _I, _I64, _I64, _P, _P, _F, _P, _P, _SZ, _I, _P]),
    "bl_linear_group_workspace_size": (_SZ, [_CALLS, _I]),
    "bl_linear_group": (_I, [_CALLS, _I, _I, _P, _SZ, _P]),
    "bl_linear_group_host": (_I, [_CALLS, _IOS, _I, _I, _P, _SZ, _P]),
    "bl_linear_noalloc": (_I, [_P, _I64, _I64, _P, _I, _I64, _I64, _P, _P, _F, _P, _P]),
    "bl_bitlinear_forward_workspace_size": (_SZ, [_I64, _I64, _I64, _I]),
    "bl_bitlinear_forward": (_I, [_P, _I64, _I64, _P, _I, _I64, _F, _P, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bl_linear_plan": (_I, [_I64, _I64, _I64, _I, _I, ctypes.POINTER(ctypes.c_int)]),
    "bl_linear_acc": (_I, [_P, _I64, _I64, _P, _I, _I64, _I64, _P, _P]),
    "bl_linear_acc_workspace_size": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "bl_linear_acc_ex": (_I, [_P, _I64, _I64, _P, _I, _I64, _I64, _P, _P, _SZ, _I, _P]),
    "bl_linear_backward_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "bl_linear_backward": (_I, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P]),
    "bl_save_deployed": (_I, [ctypes.c_char_p, _LAYERS, _I, _P]),
    "bl_deployed_count": (_I, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_int)]),
    "bl_deployed_layer_info": (_I, [ctypes.c_char_p, _I, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                    ctypes.POINTER(ctypes.c_int), ctypes.c_char_p, _SZ]),
    "bl_load_deployed_layer": (_I, [ctypes.c_char_p, _I, _P, _I64, _P, _P, _P]),
    "bl_selftest_wait_timeout": (_I, [_I64, _P]),
    "bl_sync_status": (_I, [_P]),
    "bl_status_string": (ctypes.c_char_p, [_I]),
}

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code
        self.status = STATUS.get(code, str(code))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with python -m int8_row_absmax_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _torch():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("BitLinear runs on the GPU only: no CUDA device is visible")
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(torch, t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise BitLinearError(fn, code)


def _dev(t, dtype=None):
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"expected {dtype}, got {t.dtype}")
    return t


def pack5_ldp(K: int) -> int:
    return int(load().bl_pack5_ldp(K))


def workspace(nbytes: int, device):
    """A zero-filled, 256-byte aligned device byte buffer (torch allocations are
    512-byte aligned).  The weight-quantization calls need it zero on first use
    and leave it zero, so one workspace can be reused across calls."""
    torch = _torch()
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def quantize_weights(W, eps: float = 1e-5, ws=None, out=None, beta=None):
    """W [N,K] float32 -> (Wq int8 [N,K], beta float32 [1] on the device)."""
    torch, lib = _torch(), load()
    _dev(W, torch.float32)
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if out is None else out
    beta = torch.empty(1, dtype=torch.float32, device=W.device) if beta is None else beta
    need = lib.bl_quantize_weights_workspace_size(N, K)
    ws = workspace(need, W.device) if ws is None else ws
    _check("bl_quantize_weights", lib.bl_quantize_weights(
        _ptr(W), N, K, eps, _ptr(Wq), _ptr(beta), _ptr(ws), ws.numel(), _stream(torch, W)))
    return Wq, beta


def quantize_weights_pack5(W, eps: float = 1e-5, ws=None, out=None, beta=None):
    """W [N,K] float32 -> (Wp uint8 [N, ldp], beta float32 [1] on the device)."""
    torch, lib = _torch(), load()
    _dev(W, torch.float32)
    N, K = W.shape
    ldp = pack5_ldp(K)
    Wp = torch.empty((N, ldp), dtype=torch.uint8, device=W.device) if out is None else out
    beta = torch.empty(1, dtype=torch.float32, device=W.device) if beta is None else beta
    need = lib.bl_quantize_weights_workspace_size(N, K)
    ws = workspace(need, W.device) if ws is None else ws
    _check("bl_quantize_weights_pack5", lib.bl_quantize_weights_pack5(
        _ptr(W), N, K, eps, _ptr(Wp), Wp.shape[1], _ptr(beta), _ptr(ws), ws.numel(),
        _stream(torch, W)))
    return Wp, beta


def absmean(W, eps: float = 1e-5, ws=None, beta=None):
    """beta = mean|W| + eps as a float32 [1] device tensor."""
    torch, lib = _torch(), load()
    _dev(W, torch.float32)
    N, K = W.shape
    beta = torch.empty(1, dtype=torch.float32, device=W.device) if beta is None else beta
    ws = workspace(lib.bl_quantize_weights_workspace_size(N, K), W.device) if ws is None else ws
    _check("bl_absmean", lib.bl_absmean(_ptr(W), N, K, eps, _ptr(beta), _ptr(ws), ws.numel(),
                                        _stream(torch, W)))
    return beta


def ternarize(W, beta, out=None):
    torch, lib = _torch(), load()
    _dev(W, torch.float32)
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if out is None else out
    _check("bl_ternarize", lib.bl_ternarize(_ptr(W), N, K, _ptr(beta), _ptr(Wq), _stream(torch, W)))
    return Wq


def ternarize_pack5(W, beta, out=None):
    torch, lib = _torch(), load()
    _dev(W, torch.float32)
    N, K = W.shape
    Wp = torch.empty((N, pack5_ldp(K)), dtype=torch.uint8, device=W.device) if out is None else out
    _check("bl_ternarize_pack5", lib.bl_ternarize_pack5(_ptr(W), N, K, _ptr(beta), _ptr(Wp),
                                                        Wp.shape[1], _stream(torch, W)))
    return Wp


def pack(Wq, ldp: Optional[int] = None):
    torch, lib = _torch(), load()
    _dev(Wq, torch.int8)
    N, K = Wq.shape
    ldp = pack5_ldp(K) if ldp is None else ldp
    Wp = torch.empty((N, ldp), dtype=torch.uint8, device=Wq.device)
    _check("bl_pack", lib.bl_pack(_ptr(Wq), N, K, _ptr(Wp), ldp, _stream(torch, Wq)))
    return Wp


def unpack(Wp, K: int):
    torch, lib = _torch(), load()
    _dev(Wp, torch.uint8)
    N, ldp = Wp.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=Wp.device)
    _check("bl_unpack", lib.bl_unpack(_ptr(Wp), N, K, ldp, _ptr(Wq), _stream(torch, Wp)))
    return Wq


def quantize_act(X, eps: float = 1e-5) -> Tuple:
    """X [M,K] float32 -> (Xq int8 [M,K], s float32 [M])."""
    torch, lib = _torch(), load()
    _dev(X, torch.float32)
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check("bl_quantize_act", lib.bl_quantize_act(_ptr(X), M, K, eps, _ptr(Xq), _ptr(s),
                                                  _stream(torch, X)))
    return Xq, s


def rmsnorm_quantize_act(X, g, eps_norm: float = 1e-5, eps: float = 1e-5) -> Tuple:
    """RMSNorm with gain g, then per-row int8 quantization: (Xq int8 [M,K], s float32 [M])."""
    torch, lib = _torch(), load()
    _dev(X, torch.float32)
    _dev(g, torch.float32)
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s = torch.empty((M,), dtype=torch.float32, device=X.device)
    _check("bl_rmsnorm_quantize_act", lib.bl_rmsnorm_quantize_act(
        _ptr(X), M, K, _ptr(g), eps_norm, eps, _ptr(Xq), _ptr(s), _stream(torch, X)))
    return Xq, s


def linear_plan(M: int, N: int, K: int, fmt: int, path: int = PATH_AUTO):
    """(resolved path, kernel launches) that bl_linear_ex would use; path -1 = unsupported."""
    n = ctypes.c_int(0)
    p = load().bl_linear_plan(M, N, K, fmt, path, ctypes.byref(n))
    return int(p), int(n.value)


def linear_workspace_size(M: int, N: int, K: int, fmt: int) -> int:
    return int(load().bl_linear_workspace_size(M, N, K, fmt))


def linear(X, W, fmt: int, N: int, K: int, beta, bias=None, eps: float = 1e-5,
           path: int = PATH_AUTO, ws=None, out=None, static_weights: bool = False):
    """Y = (X_q W_q^T)(s beta) + bias for X [M,K] float32 and W in format fmt.
    static_weights: W is not written by a kernel still in flight (BL_FLAG_STATIC_WEIGHTS)."""
    torch, lib = _torch(), load()
    path = path | (FLAG_STATIC_WEIGHTS if static_weights else 0)
    _dev(X, torch.float32)
    M = X.shape[0]
    if X.shape[1] != K or W.shape[0] != N:
        raise ValueError("shape mismatch")
    Y = torch.empty((M, N), dtype=torch.float32, device=X.device) if out is None else out
    need = lib.bl_linear_ex_workspace_size(M, N, K, fmt, path)
    if ws is None and need:
        ws = workspace(need, X.device)
    _check("bl_linear_ex", lib.bl_linear_ex(
        _ptr(X), M, K, _ptr(W), fmt, N, W.shape[1], _ptr(beta), _ptr(bias), eps, _ptr(Y),
        _ptr(ws), 0 if ws is None else ws.numel(), path, _stream(torch, X)))
    return Y


def _call_array(calls, outs=None):
    torch = _torch()
    arr = (LinearCall * max(1, len(calls)))()
    Ys = []
    for i, (X, W, fmt, N, K, beta, bias, eps) in enumerate(calls):
        _dev(X, torch.float32)
        M = X.shape[0]
        if X.shape[1] != K or W.shape[0] != N:
            raise ValueError("shape mismatch")
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device) if outs is None else outs[i]
        Ys.append(Y)
        arr[i] = LinearCall(_ptr(X), M, K, _ptr(W), N, W.shape[1], fmt, eps, _ptr(beta), _ptr(bias), _ptr(Y))
    return arr, Ys


def linear_group_workspace_size(calls) -> int:
    arr, _ = _call_array(calls, outs=[None] * len(calls))
    return int(load().bl_linear_group_workspace_size(arr, len(calls)))


def linear_group(calls, static_weights: bool = False, ws=None, outs=None):
    """bl_linear_group: several independent linears, calls = [(X, W, fmt, N, K, beta, bias, eps)];
    returns the list of Y (written into `outs` when given)."""
    torch, lib = _torch(), load()
    arr, Ys = _call_array(calls, outs)
    need = lib.bl_linear_group_workspace_size(arr, len(calls))
    if ws is None and need:
        ws = workspace(need, calls[0][0].device)
    stream = _stream(torch, calls[0][0]) if calls else None
    _check("bl_linear_group", lib.bl_linear_group(
        arr, len(calls), FLAG_STATIC_WEIGHTS if static_weights else 0, _ptr(ws),
        0 if ws is None else ws.numel(), stream))
    return Ys


def _host(t, shape):
    torch = _torch()
    if t.is_cuda:
        raise ValueError("host tensor expected")
    if not t.is_contiguous() or t.dtype != torch.float32 or tuple(t.shape) != tuple(shape):
        raise ValueError(f"expected a contiguous float32 host tensor of shape {tuple(shape)}")
    return t


class LinearGroupHost:
    """bl_linear_group_host with its arguments marshalled once: calling the object
    enqueues, on the stream current at construction, the copies of every host X
    into its device staging tensor, the group, and the copies of every Y back to
    its host tensor (no host synchronization; synchronize the stream before
    reading the host Y).  calls = [(X_dev, W, fmt, N, K, beta, bias, eps)] as for
    linear_group; hX[i] [M_i, K_i] and hY[i] [M_i, N_i] float32 host tensors
    (page-locked for asynchronous copies).  The tensors stay referenced by the
    object."""

    def __init__(self, calls, hX, hY, static_weights: bool = False, ws=None, outs=None):
        torch, self._lib = _torch(), load()
        if not (len(calls) == len(hX) == len(hY)):
            raise ValueError("calls, hX and hY differ in length")
        self._calls, self._ys = _call_array(calls, outs)
        self._io = (HostIO * max(1, len(calls)))()
        for i, (c, x, y) in enumerate(zip(calls, hX, hY)):
            _host(x, c[0].shape)
            _host(y, (c[0].shape[0], c[3]))
            self._io[i] = HostIO(x.data_ptr(), y.data_ptr())
        need = self._lib.bl_linear_group_workspace_size(self._calls, len(calls))
        if ws is None and need:
            ws = workspace(need, calls[0][0].device)
        self._keep = (calls, hX, hY, ws, outs)
        self._args = (self._calls, self._io, len(calls), FLAG_STATIC_WEIGHTS if static_weights else 0,
                      _ptr(ws), 0 if ws is None else ws.numel(),
                      _stream(torch, calls[0][0]) if calls else None)

    @property
    def device_outputs(self):
        return self._ys

    def __call__(self):
        _check("bl_linear_group_host", self._lib.bl_linear_group_host(*self._args))


def linear_group_host(calls, hX, hY, static_weights: bool = False, ws=None, outs=None):
    """bl_linear_group_host once: enqueue host X -> device, the group, Y -> host hY;
    returns the device Y list.  Synchronize the stream before reading hY."""
    g = LinearGroupHost(calls, hX, hY, static_weights, ws, outs)
    g()
    return g.device_outputs


def bitlinear_forward(X, W, fmt: int = PACK5, bias=None, eps: float = 1e-5, ws=None, w_out=None,
                      beta=None, out=None):
    """The BitLinear forward: W [N,K] and X [M,K] float32 -> (Y [M,N], codes, beta).
    Codes: packed [N, ldp] uint8 (PACK5) or int8 [N,K] (I8)."""
    torch, lib = _torch(), load()
    _dev(X, torch.float32)
    _dev(W, torch.float32)
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("shape mismatch")
    if w_out is None:
        w_out = (torch.empty((N, pack5_ldp(K)), dtype=torch.uint8, device=W.device) if fmt == PACK5
                 else torch.empty((N, K), dtype=torch.int8, device=W.device))
    beta = torch.empty(1, dtype=torch.float32, device=W.device) if beta is None else beta
    Y = torch.empty((M, N), dtype=torch.float32, device=X.device) if out is None else out
    ws = workspace(lib.bl_bitlinear_forward_workspace_size(M, N, K, fmt), W.device) if ws is None else ws
    _check("bl_bitlinear_forward", lib.bl_bitlinear_forward(
        _ptr(X), M, K, _ptr(W), fmt, N, eps, _ptr(w_out), w_out.shape[1], _ptr(beta), _ptr(bias),
        _ptr(Y), _ptr(ws), ws.numel(), _stream(torch, X)))
    return Y, w_out, beta


NOALLOC_SCRATCH_BYTES = 16 << 20


def linear_noalloc(X, W, fmt: int, N: int, K: int, beta, out, bias=None, eps: float = 1e-5):
    """bl_linear_noalloc: Y written into the caller's `out`; the library's static
    scratch array replaces the workspace, so no device memory is allocated."""
    torch, lib = _torch(), load()
    _dev(X, torch.float32)
    _dev(out, torch.float32)
    _check("bl_linear_noalloc", lib.bl_linear_noalloc(
        _ptr(X), X.shape[0], K, _ptr(W), fmt, N, W.shape[1], _ptr(beta), _ptr(bias), eps,
        _ptr(out), _stream(torch, X)))
    return out


def linear_acc(Xq, W, fmt: int, N: int, K: int, path: int = PATH_AUTO, ws=None,
               static_weights: bool = False):
    """acc = X_q W_q^T in int32 from pre-quantized Xq [M,K] int8."""
    torch, lib = _torch(), load()
    path = path | (FLAG_STATIC_WEIGHTS if static_weights else 0)
    _dev(Xq, torch.int8)
    M = Xq.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    need = lib.bl_linear_acc_workspace_size(M, N, K, fmt, path)
    if ws is None and need:
        ws = workspace(need, Xq.device)
    _check("bl_linear_acc_ex", lib.bl_linear_acc_ex(
        _ptr(Xq), M, K, _ptr(W), fmt, N, W.shape[1], _ptr(acc), _ptr(ws),
        0 if ws is None else ws.numel(), path, _stream(torch, Xq)))
    return acc


def linear_backward(dY, X, W, want=("dX", "dW", "db"), ws=None):
    """Straight-through backward: (dX [M,K], dW [N,K], db [N]) float32; entries
    not in `want` come back as None."""
    torch, lib = _torch(), load()
    _dev(dY, torch.float32)
    M, N = dY.shape
    K = W.shape[1] if W is not None else X.shape[1]
    dX = torch.empty((M, K), dtype=torch.float32, device=dY.device) if "dX" in want else None
    dW = torch.empty((N, K), dtype=torch.float32, device=dY.device) if "dW" in want else None
    db = torch.empty((N,), dtype=torch.float32, device=dY.device) if "db" in want else None
    need = lib.bl_linear_backward_workspace_size(M, N, K) if (dX is not None or dW is not None) else 0
    if ws is None and need:
        ws = workspace(need, dY.device)
    _check("bl_linear_backward", lib.bl_linear_backward(
        _ptr(dY), _ptr(X), _ptr(W), M, N, K, _ptr(dX), _ptr(dW), _ptr(db), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(torch, dY)))
    return dX, dW, db


def save_deployed(path: str, layers):
    """bl_save_deployed: layers = [dict(name, Wp [N, ldp] uint8, K, beta [1], bias [N] or None)]."""
    torch, lib = _torch(), load()
    arr = (DeployedLayer * max(1, len(layers)))()
    for i, L in enumerate(layers):
        Wp = _dev(L["Wp"], torch.uint8)
        arr[i] = DeployedLayer(L.get("name", "").encode(), Wp.shape[0], L["K"], _ptr(Wp), Wp.shape[1],
                               _ptr(L["beta"]), _ptr(L.get("bias")))
    stream = _stream(torch, layers[0]["Wp"]) if layers else ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    _check("bl_save_deployed", lib.bl_save_deployed(path.encode(), arr, len(layers), stream))


def load_deployed(path: str, device=None):
    """bl_deployed_count / bl_deployed_layer_info / bl_load_deployed_layer: every
    layer into new device tensors: dict(name, N, K, Wp [N, pack5_ldp(K)], beta, bias)."""
    torch, lib = _torch(), load()
    device = torch.device("cuda") if device is None else device
    n = ctypes.c_int(0)
    _check("bl_deployed_count", lib.bl_deployed_count(path.encode(), ctypes.byref(n)))
    out = []
    for i in range(n.value):
        N, K, hb = _I64(0), _I64(0), ctypes.c_int(0)
        name = ctypes.create_string_buffer(256)
        _check("bl_deployed_layer_info", lib.bl_deployed_layer_info(
            path.encode(), i, ctypes.byref(N), ctypes.byref(K), ctypes.byref(hb), name, 256))
        Wp = torch.empty((N.value, pack5_ldp(K.value)), dtype=torch.uint8, device=device)
        beta = torch.empty(1, dtype=torch.float32, device=device)
        bias = torch.empty(N.value, dtype=torch.float32, device=device) if hb.value else None
        _check("bl_load_deployed_layer", lib.bl_load_deployed_layer(
            path.encode(), i, _ptr(Wp), Wp.shape[1], _ptr(beta), _ptr(bias), _stream(torch, Wp)))
        out.append({"name": name.value.decode(), "N": N.value, "K": K.value, "Wp": Wp, "beta": beta, "bias": bias})
    return out


def selftest_wait_timeout(limit_ns: int = 2_000_000):
    """bl_selftest_wait_timeout on the current stream: a bounded wait that runs out
    and records BL_ERR_DEVICE_TIMEOUT for the next sync_status()."""
    torch, lib = _torch(), load()
    _check("bl_selftest_wait_timeout",
           lib.bl_selftest_wait_timeout(int(limit_ns), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def sync_status(device=None) -> str:
    """Synchronize the current stream and return the device status ("BL_OK" ...)."""
    torch, lib = _torch(), load()
    dev = torch.device("cuda") if device is None else device
    code = lib.bl_sync_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    return STATUS.get(code, str(code))
