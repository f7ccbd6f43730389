"""GPU side of the counter-based weight generator (synth/csrc/synth_philox.cu).

Used only where inputs are too large to draw on the host (the 100B-class
decode sweep).  The CPU oracle regenerates the same weights with its own
implementation of the same published generator.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "synth_philox.cu")
LIB_PATH = os.path.join(HERE, "libbitlinear_synth.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(SRC) > os.path.getmtime(LIB_PATH):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run([os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-fmad=false",
                        "-o", tmp, SRC], check=True)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB_PATH)
        L.synth_weights_device.restype = C.c_int
        L.synth_weights_device.argtypes = [C.c_void_p, C.c_uint32, C.c_uint32, C.c_int64, C.c_int64, C.c_int64,
                                           C.c_void_p]
        L.synth_philox_device.restype = C.c_int
        L.synth_philox_device.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p]
        _lib = L
    return _lib


def weights(out, seed: int, g: int, row0: int = 0, stream=None) -> None:
    """Fill the fp32 CUDA tensor `out` [rows, K] with rows row0.. of matrix g."""
    import torch
    rows, K = out.shape
    st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = lib().synth_weights_device(out.data_ptr(), seed, g, row0, rows, K, st)
    if rc != 0:
        raise RuntimeError(f"synth_weights_device failed ({rc})")


def philox(vectors):
    """vectors: list of (c0, c1, c2, c3, k0, k1) -> list of 4-tuples, on the GPU."""
    import numpy as np
    import torch
    a = torch.from_numpy(np.asarray(vectors, dtype=np.uint32).view(np.int32).ravel()).cuda()
    out = torch.empty(4 * len(vectors), dtype=torch.int32, device="cuda")
    rc = lib().synth_philox_device(a.data_ptr(), out.data_ptr(), len(vectors),
                                   torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"synth_philox_device failed ({rc})")
    return out.cpu().numpy().view(np.uint32).reshape(-1, 4)
