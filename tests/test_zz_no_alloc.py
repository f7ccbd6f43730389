"""GPU test of bitlinear_pack_weights_noalloc, the packer entry point for
callers that cannot allocate device memory (a framework hook with no
allocator, a fixed memory plan that forbids cudaMalloc after start-up).

It calls the entry point through the C ABI twice in a row, on two weight
tensors of different sizes, and checks each result against the regular
bitlinear_pack_weights (which takes a caller-provided workspace): the same
packed bytes, and gamma within the parity tolerance (in fact identical,
since both run the same kernels in the same order).  The file is named so
that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest

import synth
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bl():
    import torch  # noqa: F401
    import ternary_weight_linear_absmean_b200 as m
    from ternary_weight_linear_absmean_b200 import _build
    _build.build()
    return m


def test_noalloc_pack_matches_workspace_pack_on_two_calls(bl):
    import torch
    lib = bl.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # first call: 200 reduction blocks; second: 3 -- the second must not see
    # anything the first left in the shared scratch array
    for N, K, seed in [(640, 2560, 5), (97, 200, 6)]:
        W = torch.from_numpy(synth.weights(N, K, seed)).cuda()
        ref_packed, ref_g64, ref_g32 = bl.pack(W)

        packed = torch.full((bl.bitlinear_packed_bytes(N, K),), 0x5A, dtype=torch.uint8, device="cuda")
        g64 = torch.zeros(1, dtype=torch.float64, device="cuda")
        g32 = torch.zeros(1, dtype=torch.float32, device="cuda")
        st = lib.bitlinear_pack_weights_noalloc(C.c_void_p(W.data_ptr()), N, K, C.c_double(1e-5),
                                                C.c_void_p(packed.data_ptr()), C.c_void_p(g64.data_ptr()),
                                                C.c_void_p(g32.data_ptr()), C.c_void_p(stream))
        assert st == bl.BL_OK, bl.status_string(st)
        torch.cuda.synchronize()
        assert bl.bitlinear_get_status() == bl.BL_OK
        ref = {"gamma64": float(ref_g64.item()), "gamma32": float(ref_g32.item())}
        P.check_gamma(float(g64.item()), float(g32.item()), ref, N * K)
        assert np.array_equal(packed.cpu().numpy(), ref_packed.cpu().numpy())


def test_noalloc_rejects_bad_arguments(bl):
    lib = bl.lib()
    assert lib.bitlinear_pack_weights_noalloc(None, 8, 64, 1e-5, 0x10000, 0x10000, 0x10000, None) == bl.BL_ERR_NULL
    assert lib.bitlinear_pack_weights_noalloc(0x10000, 0, 64, 1e-5, 0x10000, 0x10000, 0x10000, None) == \
        bl.BL_ERR_SHAPE
    assert lib.bitlinear_pack_weights_noalloc(0x10004, 8, 64, 1e-5, 0x10000, 0x10000, 0x10000, None) == \
        bl.BL_ERR_ALIGN
    assert lib.bitlinear_pack_weights_noalloc(0x10000, 8, 64, -1.0, 0x10000, 0x10000, 0x10000, None) == \
        bl.BL_ERR_ARG
