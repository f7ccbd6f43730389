"""BitNet b1.58 BitLinear on B200 (sm_100a): Python binding of libbitlinear.so.

The functions named ``bitlinear_*`` mirror the C ABI in include/bitlinear.h
one to one and only marshal arguments: torch CUDA tensors in (PyTorch
provides device memory and streams), raw device pointers out to the library.
All arithmetic runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback -- if the library is missing, every call raises.

A few helpers (``pack``, ``quant_act``, ``forward``, ``forward_x``) allocate
the outputs with torch and then call the same entry points.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitlinear.so")

BL_OK, BL_ERR_NULL, BL_ERR_SHAPE, BL_ERR_ALIGN, BL_ERR_DTYPE = 0, 1, 2, 3, 4
BL_ERR_WORKSPACE, BL_ERR_OVERFLOW, BL_ERR_NONFINITE, BL_ERR_CUDA, BL_ERR_ARG, BL_ERR_TIMEOUT = 5, 6, 7, 8, 9, 10
BL_F32, BL_BF16 = 0, 1
BL_DECODE_AUTO, BL_DECODE_TENSOR, BL_DECODE_DP4A, BL_DECODE_TILE, BL_DECODE_LUT = 0, 1, 2, 3, 4

# Every symbol include/bitlinear.h declares, with (restype, argtypes).
_vp, _i64, _i32 = C.c_void_p, C.c_int64, C.c_int
SIGNATURES = {
    "bitlinear_padded_k": (_i64, [_i64]),
    "bitlinear_packed_bytes": (_i64, [_i64, _i64]),
    "bitlinear_pack_workspace_bytes": (_i64, [_i64, _i64]),
    "bitlinear_pack_weights": (_i32, [_vp, _i64, _i64, C.c_double, _vp, _vp, _vp, _vp, C.c_size_t, _vp]),
    "bitlinear_pack_weights_noalloc": (_i32, [_vp, _i64, _i64, C.c_double, _vp, _vp, _vp, _vp]),
    "bitlinear_quant_act": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _vp]),
    "bitlinear_forward": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp]),
    "bitlinear_forward_x": (_i32, [_vp, _i32, _vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp]),
    "bitlinear_forward_x_grouped": (_i32, [_i32, _vp, _i32, _vp, _vp, _i64, _vp, _vp, _vp, _i32, _vp]),
    "bitlinear_forward_x_supported": (_i32, [_i64, _i64]),
    "bitlinear_decode_workspace_bytes": (_i64, [_i32, _i64, _vp]),
    "bitlinear_forward_x_grouped_ws": (_i32, [_i32, _vp, _i32, _vp, _vp, _i64, _vp, _vp, _vp, _i32, _vp, _i64,
                                              _vp]),
    "bitlinear_forward_x_rmsnorm_grouped_ws": (_i32, [_i32, _vp, _i32, _vp, C.c_double, _vp, _vp, _i64, _vp, _vp,
                                                      _vp, _i32, _vp, _i64, _vp]),
    "bitlinear_rmsnorm_quant_act": (_i32, [_vp, _i32, _vp, C.c_double, _i64, _i64, _vp, _vp, _vp]),
    "bitlinear_forward_x_rmsnorm_grouped": (_i32, [_i32, _vp, _i32, _vp, C.c_double, _vp, _vp, _i64, _vp, _vp,
                                                   _vp, _i32, _vp]),
    "bitlinear_get_status": (_i32, [_vp]),
    "bitlinear_set_decode_kernel": (_i32, [_i32]),
    "bitlinear_get_decode_kernel": (_i32, []),
    "bitlinear_status_string": (C.c_char_p, [_i32]),
}

_lib = None


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> C.CDLL:
    """Load libbitlinear.so (build it first with __graft_entry__.build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python __graft_entry__.py build` "
                               "or ternary_weight_linear_absmean_b200/_build.py")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bitlinear_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != BL_OK:
        raise BitLinearError(status, where)


def _torch():
    import torch
    return torch


def _dptr(t, name: str) -> int:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(dt) -> int:
    torch = _torch()
    if dt == torch.float32:
        return BL_F32
    if dt == torch.bfloat16:
        return BL_BF16
    raise ValueError(f"unsupported dtype {dt}; use float32 or bfloat16")


# ------------------------------------------------------- C ABI mirror ----
def bitlinear_padded_k(K: int) -> int:
    return int(lib().bitlinear_padded_k(K))


def bitlinear_forward_x_supported(M: int, K: int) -> bool:
    """Whether the fused decode forms take M tokens of K columns."""
    return bool(lib().bitlinear_forward_x_supported(M, K))


def bitlinear_packed_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_packed_bytes(N, K))


def bitlinear_pack_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_pack_workspace_bytes(N, K))


def bitlinear_pack_weights(W, eps, packed, gamma64, gamma32, workspace, stream=None) -> None:
    N, K = W.shape
    st = lib().bitlinear_pack_weights(_dptr(W, "W"), N, K, float(eps), _dptr(packed, "packed"),
                                      _dptr(gamma64, "gamma64"), _dptr(gamma32, "gamma32"),
                                      _dptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                      _stream(stream))
    _check(st, "bitlinear_pack_weights")


def bitlinear_pack_weights_noalloc(W, eps, packed, gamma64, gamma32, stream=None) -> None:
    """bitlinear_pack_weights with its scratch in the library's own fixed
    device array: for callers that cannot allocate device memory."""
    N, K = W.shape
    st = lib().bitlinear_pack_weights_noalloc(_dptr(W, "W"), N, K, float(eps), _dptr(packed, "packed"),
                                              _dptr(gamma64, "gamma64"), _dptr(gamma32, "gamma32"),
                                              _stream(stream))
    _check(st, "bitlinear_pack_weights_noalloc")


def bitlinear_quant_act(x, q, s, stream=None) -> None:
    M, K = x.shape
    st = lib().bitlinear_quant_act(_dptr(x, "x"), _dtype_code(x.dtype), M, K, _dptr(q, "q"),
                                   _dptr(s, "s"), _stream(stream))
    _check(st, "bitlinear_quant_act")


def bitlinear_forward(q, s, packed, gamma32, M, N, K, y, acc_debug=None, stream=None) -> None:
    st = lib().bitlinear_forward(_dptr(q, "q"), _dptr(s, "s"), _dptr(packed, "packed"),
                                 _dptr(gamma32, "gamma32"), M, N, K, _dptr(y, "y"), _dtype_code(y.dtype),
                                 _dptr(acc_debug, "acc_debug"), _stream(stream))
    _check(st, "bitlinear_forward")


def bitlinear_forward_x(x, packed, gamma32, N, K, y, stream=None) -> None:
    M = x.shape[0]
    st = lib().bitlinear_forward_x(_dptr(x, "x"), _dtype_code(x.dtype), _dptr(packed, "packed"),
                                   _dptr(gamma32, "gamma32"), M, N, K, _dptr(y, "y"), _dtype_code(y.dtype),
                                   _stream(stream))
    _check(st, "bitlinear_forward_x")


def bitlinear_decode_workspace_bytes(M: int, Ks) -> int:
    """Device workspace bytes of the grouped calls' workspace forms."""
    n = len(Ks)
    return int(lib().bitlinear_decode_workspace_bytes(n, M, (C.c_int64 * n)(*Ks)))


def decode_workspace(M: int, Ks, device):
    """A workspace tensor for the grouped calls (uint8, device)."""
    torch = _torch()
    nbytes = bitlinear_decode_workspace_bytes(M, Ks)
    if nbytes <= 0:
        raise ValueError("no workspace size for these shapes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _ws_args(workspace):
    return _dptr(workspace, "workspace"), workspace.numel() * workspace.element_size()


def bitlinear_forward_x_grouped(xs, packeds, gammas, Ns, Ks, ys, stream=None, workspace=None) -> None:
    """One launch over the problems; with a workspace (decode_workspace)
    and M >= 2, a quantiser launch first and the product on the codes."""
    n = len(xs)
    if not (len(packeds) == len(gammas) == len(Ns) == len(Ks) == len(ys) == n):
        raise ValueError("grouped arguments must all have the same length")
    M = xs[0].shape[0]
    arr_p = C.c_void_p * n
    arr_i = C.c_int64 * n
    args = (n, arr_p(*[_dptr(t, "x") for t in xs]), _dtype_code(xs[0].dtype),
            arr_p(*[_dptr(t, "packed") for t in packeds]), arr_p(*[_dptr(t, "gamma32") for t in gammas]), M,
            arr_i(*Ns), arr_i(*Ks), arr_p(*[_dptr(t, "y") for t in ys]), _dtype_code(ys[0].dtype))
    if workspace is None:
        _check(lib().bitlinear_forward_x_grouped(*args, _stream(stream)), "bitlinear_forward_x_grouped")
    else:
        _check(lib().bitlinear_forward_x_grouped_ws(*args, *_ws_args(workspace), _stream(stream)),
               "bitlinear_forward_x_grouped_ws")


def bitlinear_rmsnorm_quant_act(x, gain, eps, q, s, stream=None) -> None:
    M, K = x.shape
    st = lib().bitlinear_rmsnorm_quant_act(_dptr(x, "x"), _dtype_code(x.dtype), _dptr(gain, "gain"), float(eps), M,
                                           K, _dptr(q, "q"), _dptr(s, "s"), _stream(stream))
    _check(st, "bitlinear_rmsnorm_quant_act")


def bitlinear_forward_x_rmsnorm_grouped(xs, gains, eps, packeds, gammas, Ns, Ks, ys, stream=None,
                                        workspace=None) -> None:
    n = len(xs)
    if not (len(gains) == len(packeds) == len(gammas) == len(Ns) == len(Ks) == len(ys) == n):
        raise ValueError("grouped arguments must all have the same length")
    M = xs[0].shape[0]
    arr_p = C.c_void_p * n
    arr_i = C.c_int64 * n
    args = (n, arr_p(*[_dptr(t, "x") for t in xs]), _dtype_code(xs[0].dtype), arr_p(*[_dptr(t, "gain") for t in gains]),
            float(eps), arr_p(*[_dptr(t, "packed") for t in packeds]), arr_p(*[_dptr(t, "gamma32") for t in gammas]),
            M, arr_i(*Ns), arr_i(*Ks), arr_p(*[_dptr(t, "y") for t in ys]), _dtype_code(ys[0].dtype))
    if workspace is None:
        _check(lib().bitlinear_forward_x_rmsnorm_grouped(*args, _stream(stream)),
               "bitlinear_forward_x_rmsnorm_grouped")
    else:
        _check(lib().bitlinear_forward_x_rmsnorm_grouped_ws(*args, *_ws_args(workspace), _stream(stream)),
               "bitlinear_forward_x_rmsnorm_grouped_ws")


class GroupedDecode:
    """A prepared grouped decode call (bitlinear_forward_x_grouped_ws, or
    its SubLN form when gains are given): the pointer and size arrays are
    marshalled and the workspace allocated once, so each call costs one C
    call (for decode loops that run the same layers every token).  The
    tensors must stay alive and in place while the object is used, and one
    object must not run on two streams at once (they share the workspace)."""

    def __init__(self, xs, packeds, gammas, Ns, Ks, ys, gains=None, eps=1e-6):
        n = len(xs)
        if not (len(packeds) == len(gammas) == len(Ns) == len(Ks) == len(ys) == n):
            raise ValueError("grouped arguments must all have the same length")
        if gains is not None and len(gains) != n:
            raise ValueError("grouped arguments must all have the same length")
        arr_p = C.c_void_p * n
        arr_i = C.c_int64 * n
        M = xs[0].shape[0]
        self.workspace = decode_workspace(M, Ks, xs[0].device)
        self._keep = (list(xs), list(packeds), list(gammas), list(ys), list(gains or []))
        head = (n, arr_p(*[_dptr(t, "x") for t in xs]), _dtype_code(xs[0].dtype))
        if gains is not None:
            head += (arr_p(*[_dptr(t, "gain") for t in gains]), float(eps))
        self._args = head + (arr_p(*[_dptr(t, "packed") for t in packeds]),
                             arr_p(*[_dptr(t, "gamma32") for t in gammas]), M, arr_i(*Ns), arr_i(*Ks),
                             arr_p(*[_dptr(t, "y") for t in ys]), _dtype_code(ys[0].dtype),
                             *_ws_args(self.workspace))
        self._name = "bitlinear_forward_x_rmsnorm_grouped_ws" if gains is not None else "bitlinear_forward_x_grouped_ws"
        self._fn = getattr(lib(), self._name)

    def __call__(self, stream=None) -> None:
        _check(self._fn(*self._args, _stream(stream)), self._name)


def bitlinear_get_status(stream=None) -> int:
    return int(lib().bitlinear_get_status(_stream(stream)))


def bitlinear_set_decode_kernel(kind: int) -> None:
    _check(lib().bitlinear_set_decode_kernel(int(kind)), "bitlinear_set_decode_kernel")


def bitlinear_get_decode_kernel() -> int:
    return int(lib().bitlinear_get_decode_kernel())


bitlinear_status_string = status_string


# ------------------------------------------------ allocating helpers ----
def pack(W, eps: float = 1e-5, stream=None):
    """Returns (packed uint8, gamma64 float64[1], gamma32 float32[1])."""
    torch = _torch()
    N, K = W.shape
    dev = W.device
    packed = torch.empty(bitlinear_packed_bytes(N, K), dtype=torch.uint8, device=dev)
    g64 = torch.empty(1, dtype=torch.float64, device=dev)
    g32 = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(bitlinear_pack_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
    bitlinear_pack_weights(W, eps, packed, g64, g32, ws, stream)
    return packed, g64, g32


def quant_act(x, stream=None):
    """Returns (q int8 [M, Kp], s float32 [M])."""
    torch = _torch()
    M, K = x.shape
    q = torch.empty((M, bitlinear_padded_k(K)), dtype=torch.int8, device=x.device)
    s = torch.empty(M, dtype=torch.float32, device=x.device)
    bitlinear_quant_act(x, q, s, stream)
    return q, s


def rmsnorm_quant_act(x, gain, eps: float = 1e-6, stream=None):
    """SubLN (RMS normalisation with gain) then the quantiser.  Returns
    (q int8 [M, Kp], s float32 [M])."""
    torch = _torch()
    M, K = x.shape
    q = torch.empty((M, bitlinear_padded_k(K)), dtype=torch.int8, device=x.device)
    s = torch.empty(M, dtype=torch.float32, device=x.device)
    bitlinear_rmsnorm_quant_act(x, gain, eps, q, s, stream)
    return q, s


def forward(q, s, packed, gamma32, N, K, out_dtype=None, acc_debug=False, stream=None):
    torch = _torch()
    M = q.shape[0]
    y = torch.empty((M, N), dtype=out_dtype or torch.float32, device=q.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=q.device) if acc_debug else None
    bitlinear_forward(q, s, packed, gamma32, M, N, K, y, acc, stream)
    return (y, acc) if acc_debug else y


def forward_x(x, packed, gamma32, N, K, out_dtype=None, stream=None):
    torch = _torch()
    y = torch.empty((x.shape[0], N), dtype=out_dtype or torch.float32, device=x.device)
    bitlinear_forward_x(x, packed, gamma32, N, K, y, stream)
    return y
