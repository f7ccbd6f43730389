"""CPU oracle for the BitNet b1.58 BitLinear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it, and
the two share no code: the oracle is a plain C file (``bitlinear_oracle.c``,
``philox_oracle.c``) compiled with gcc and called here through ctypes over
numpy arrays.  Each C function cites the page section it restates.

Every function is pinned by ``tests/test_oracle_pins.py`` against values the
definition fixes independently (hand-built cases, closed forms, invariants,
exact rational arithmetic, published generator vectors).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SOURCES = [os.path.join(_HERE, f) for f in ("bitlinear_oracle.c", "philox_oracle.c")]
LIB_PATH = os.path.join(_HERE, "liboracle_bitlinear.so")
CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-pthread", "-Wall", "-Wextra", "-Wno-unused-parameter"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (no FMA contraction)."""
    stale = force or not os.path.exists(LIB_PATH) or any(
        os.path.getmtime(s) > os.path.getmtime(LIB_PATH) for s in _SOURCES)
    if stale:
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, *_SOURCES, "-lm"], check=True)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def _i64(*a):
    return [C.c_int64(int(v)) for v in a]


def lib() -> C.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(LIB_PATH)
            vp = C.c_void_p
            i64 = C.c_int64
            L.orc_absmean_gamma.restype = C.c_double
            L.orc_absmean_gamma.argtypes = [vp, i64, i64]
            L.orc_ternary_codes.restype = i64
            L.orc_ternary_codes.argtypes = [vp, i64, i64, C.c_double, C.c_double, vp, vp]
            for f in ("orc_padded_k", "orc_padded_n"):
                getattr(L, f).restype = i64
                getattr(L, f).argtypes = [i64]
            L.orc_packed_bytes.restype = i64
            L.orc_packed_bytes.argtypes = [i64, i64]
            L.orc_pack.restype = None
            L.orc_pack.argtypes = [vp, i64, i64, vp]
            L.orc_unpack.restype = i64
            L.orc_unpack.argtypes = [vp, i64, i64, vp]
            L.orc_quant_act_f32.restype = i64
            L.orc_quant_act_f32.argtypes = [vp, i64, i64, vp, vp]
            L.orc_quant_act_bf16.restype = i64
            L.orc_quant_act_bf16.argtypes = [vp, i64, i64, vp, vp]
            L.orc_rms_factor.restype = C.c_float
            L.orc_rms_factor.argtypes = [vp, i64, C.c_double]
            L.orc_rmsnorm_quant_act.restype = i64
            L.orc_rmsnorm_quant_act.argtypes = [vp, C.c_int, vp, C.c_double, i64, i64, vp, vp, vp]
            L.orc_int_matmul.restype = C.c_int
            L.orc_int_matmul.argtypes = [vp, vp, i64, i64, i64, vp]
            L.orc_int_matmul_sampled.restype = C.c_int
            L.orc_int_matmul_sampled.argtypes = [vp, vp, i64, vp, vp, i64, vp]
            L.orc_rescale_one.restype = C.c_float
            L.orc_rescale_one.argtypes = [C.c_int32, C.c_float, C.c_float]
            L.orc_rescale.restype = None
            L.orc_rescale.argtypes = [vp, vp, C.c_float, i64, i64, vp]
            L.orc_f32_to_bf16.restype = C.c_uint16
            L.orc_f32_to_bf16.argtypes = [C.c_float]
            L.orc_to_bf16.restype = None
            L.orc_to_bf16.argtypes = [vp, i64, vp]
            L.orc_forward_bf16_mt.restype = C.c_int
            L.orc_forward_bf16_mt.argtypes = [vp, vp, C.c_float, i64, i64, i64, vp, C.c_int, vp, vp]
            L.orc_philox4x32_10.restype = None
            L.orc_philox4x32_10.argtypes = [vp, vp, vp]
            L.orc_synth_weights.restype = None
            L.orc_synth_weights.argtypes = [C.c_uint32, C.c_uint32, i64, i64, i64, vp]
            L.orc_synth_weights_mt.restype = None
            L.orc_synth_weights_mt.argtypes = [C.c_uint32, C.c_uint32, i64, i64, i64, vp, C.c_int]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- A1 ----
def absmean_gamma(W: np.ndarray) -> float:
    W = _c(W, np.float32)
    N, K = W.shape
    return float(lib().orc_absmean_gamma(_p(W), N, K))


def ternary_codes(W: np.ndarray, gamma64: float, eps: float = 1e-5):
    """Returns (codes int8 [N, K], boundary uint8 [N, K], boundary count)."""
    W = _c(W, np.float32)
    N, K = W.shape
    code = np.empty((N, K), np.int8)
    bnd = np.empty((N, K), np.uint8)
    nb = lib().orc_ternary_codes(_p(W), N, K, float(gamma64), float(eps), _p(code), _p(bnd))
    return code, bnd, int(nb)


# ---------------------------------------------------------------- A2 ----
def padded_k(K: int) -> int:
    return int(lib().orc_padded_k(K))


def padded_n(N: int) -> int:
    return int(lib().orc_padded_n(N))


def packed_bytes(N: int, K: int) -> int:
    return int(lib().orc_packed_bytes(N, K))


def pack(code: np.ndarray) -> np.ndarray:
    code = _c(code, np.int8)
    N, K = code.shape
    out = np.empty(packed_bytes(N, K), np.uint8)
    lib().orc_pack(_p(code), N, K, _p(out))
    return out


def unpack(packed: np.ndarray, N: int, K: int):
    """Returns (codes int8 [N, K], number of malformed fields)."""
    packed = _c(packed, np.uint8)
    assert packed.size == packed_bytes(N, K)
    code = np.empty((N, K), np.int8)
    bad = lib().orc_unpack(_p(packed), N, K, _p(code))
    return code, int(bad)


# ---------------------------------------------------------------- A3 ----
def quant_act(x: np.ndarray, dtype: str):
    """x: float32 [M, K] (dtype 'f32') or bf16 bit patterns uint16 [M, K]
    (dtype 'bf16').  Returns (q int8 [M, K], s float32 [M], clipped count)."""
    if dtype == "f32":
        x = _c(x, np.float32)
        fn = lib().orc_quant_act_f32
    elif dtype == "bf16":
        x = _c(x, np.uint16)
        fn = lib().orc_quant_act_bf16
    else:
        raise ValueError(dtype)
    M, K = x.shape
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    clipped = fn(_p(x), M, K, _p(q), _p(s))
    if clipped < 0:
        raise MemoryError("oracle quant_act allocation failed")
    return q, s, int(clipped)


def rms_factor(x_row: np.ndarray, eps: float) -> np.float32:
    """r32 = (float)(1 / sqrt(mean(x^2) + eps)), mean square summed in fp64."""
    x_row = _c(x_row, np.float32)
    return np.float32(lib().orc_rms_factor(_p(x_row), x_row.size, float(eps)))


def rmsnorm_quant_act(x: np.ndarray, dtype: str, gain: np.ndarray, eps: float):
    """SubLN (RMS normalisation with per-channel gain) then the per-token
    int8 quantiser.  x as in quant_act.  Returns (xn float32 [M, K], q int8
    [M, K], s float32 [M], clipped count)."""
    if dtype == "f32":
        x = _c(x, np.float32)
        xt = 0
    elif dtype == "bf16":
        x = _c(x, np.uint16)
        xt = 1
    else:
        raise ValueError(dtype)
    M, K = x.shape
    gain = _c(gain, np.float32)
    assert gain.shape == (K,)
    xn = np.empty((M, K), np.float32)
    q = np.empty((M, K), np.int8)
    s = np.empty(M, np.float32)
    clipped = lib().orc_rmsnorm_quant_act(_p(x), xt, _p(gain), float(eps), M, K, _p(xn), _p(q), _p(s))
    if clipped < 0:
        raise MemoryError("oracle rmsnorm_quant_act allocation failed")
    return xn, q, s, int(clipped)


# ---------------------------------------------------------------- A4 ----
def int_matmul(q: np.ndarray, code: np.ndarray) -> np.ndarray:
    q = _c(q, np.int8)
    code = _c(code, np.int8)
    M, K = q.shape
    N, K2 = code.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    if lib().orc_int_matmul(_p(q), _p(code), M, N, K, _p(acc)) != 0:
        raise OverflowError("accumulator exceeds int32")
    return acc


def int_matmul_sampled(q: np.ndarray, code: np.ndarray, ms, ns) -> np.ndarray:
    q = _c(q, np.int8)
    code = _c(code, np.int8)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    K = q.shape[1]
    assert code.shape[1] == K and ms.shape == ns.shape
    acc = np.empty(ms.size, np.int32)
    if lib().orc_int_matmul_sampled(_p(q), _p(code), K, _p(ms), _p(ns), ms.size, _p(acc)) != 0:
        raise OverflowError("accumulator exceeds int32")
    return acc


# ---------------------------------------------------------------- A5 ----
def rescale(acc: np.ndarray, s: np.ndarray, gamma32: float) -> np.ndarray:
    acc = _c(acc, np.int32)
    s = _c(s, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    lib().orc_rescale(_p(acc), _p(s), C.c_float(gamma32), M, N, _p(y))
    return y


def rescale_one(acc: int, gamma32: float, s: float) -> float:
    return float(lib().orc_rescale_one(int(acc), C.c_float(gamma32), C.c_float(s)))


def to_bf16(y: np.ndarray) -> np.ndarray:
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint16)
    lib().orc_to_bf16(_p(y), y.size, _p(out))
    return out


# ------------------------------------------------------- whole layer ----
def bitlinear(W: np.ndarray, x: np.ndarray, xdtype: str, eps: float = 1e-5):
    """The whole layer on the CPU: every intermediate, as a dict."""
    g64 = absmean_gamma(W)
    g32 = float(np.float32(g64))
    code, bnd, nb = ternary_codes(W, g64, eps)
    q, s, clipped = quant_act(x, xdtype)
    acc = int_matmul(q, code)
    y = rescale(acc, s, g32)
    return dict(gamma64=g64, gamma32=g32, code=code, boundary=bnd, n_boundary=nb,
                packed=pack(code), q=q, s=s, clipped=clipped, acc=acc, y=y)


def bitlinear_rmsnorm(W: np.ndarray, x: np.ndarray, xdtype: str, gain: np.ndarray, eps_norm: float,
                      eps: float = 1e-5):
    """SubLN (RMS normalisation, reading R16) then the whole layer."""
    g64 = absmean_gamma(W)
    g32 = float(np.float32(g64))
    code, bnd, nb = ternary_codes(W, g64, eps)
    xn, q, s, clipped = rmsnorm_quant_act(x, xdtype, gain, eps_norm)
    acc = int_matmul(q, code)
    y = rescale(acc, s, g32)
    return dict(gamma64=g64, gamma32=g32, code=code, boundary=bnd, n_boundary=nb,
                packed=pack(code), xn=xn, q=q, s=s, clipped=clipped, acc=acc, y=y)


def forward_bf16_mt(x_bf16: np.ndarray, code: np.ndarray, gamma32: float, threads: int) -> np.ndarray:
    """quantise + multiply + rescale with output rows split over threads."""
    x_bf16 = _c(x_bf16, np.uint16)
    code = _c(code, np.int8)
    M, K = x_bf16.shape
    N = code.shape[0]
    y = np.empty((M, N), np.float32)
    qs = np.empty((M, K), np.int8)
    ss = np.empty(M, np.float32)
    rc = lib().orc_forward_bf16_mt(_p(x_bf16), _p(code), C.c_float(gamma32), M, N, K, _p(y),
                                   int(threads), _p(qs), _p(ss))
    if rc != 0:
        raise RuntimeError(f"oracle forward failed ({rc})")
    return y


# --------------------------------------------- counter-based generator ----
def philox4x32_10(ctr, key) -> np.ndarray:
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    out = np.empty(4, np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def synth_weights(seed: int, g: int, row0: int, rows: int, K: int, threads: int = 1) -> np.ndarray:
    W = np.empty((rows, K), np.float32)
    if threads > 1:
        lib().orc_synth_weights_mt(seed, g, row0, rows, K, _p(W), int(threads))
    else:
        lib().orc_synth_weights(seed, g, row0, rows, K, _p(W))
    return W
