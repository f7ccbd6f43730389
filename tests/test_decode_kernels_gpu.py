"""GPU parity of every decode kernel (M <= 16): the tensor-core kernel, the
dp4a streaming kernel and the per-tile kernel, each forced through
bitlinear_set_decode_kernel, against the CPU oracle on the same seeded
inputs.  Decode results are exact: acc bit for bit, fp32 y equal to the
oracle's (float)((double)acc * gamma32 / s)."""
import numpy as np
import pytest

import oracle
import synth
from tests import parity as P

pytestmark = pytest.mark.gpu

KINDS = {"tensor": 1, "dp4a": 2, "tile": 3}


@pytest.fixture(scope="module")
def bl():
    import torch  # noqa: F401
    import ternary_weight_linear_absmean_b200 as m
    from ternary_weight_linear_absmean_b200 import _build
    _build.build()
    return m


@pytest.fixture(params=list(KINDS))
def kind(request, bl):
    bl.bitlinear_set_decode_kernel(KINDS[request.param])
    assert bl.bitlinear_get_decode_kernel() == KINDS[request.param]
    yield request.param
    bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)


def _packed(bl, W):
    return bl.pack(P.to_dev_f32(W))


def _xdev(x, xd):
    return P.to_dev_f32(x) if xd == "f32" else P.to_dev_bf16(x)


# shapes span several 8-row tiles, ragged N and K, several stages per job for
# every token-slot count, and (the last two) several jobs per CTA with a
# ragged last job
CASES = [(1, 13, 200, "bf16"), (2, 40, 320, "f32"), (3, 100, 1000, "bf16"), (4, 33, 4097, "bf16"),
         (5, 64, 64, "f32"), (8, 300, 1000, "bf16"), (9, 96, 2560, "bf16"), (16, 256, 768, "bf16"),
         (1, 2560, 640, "bf16"), (4, 6000, 320, "bf16"), (16, 20000, 256, "f32")]


@pytest.mark.parametrize("M,N,K,xd", CASES)
def test_forward_unfused(bl, kind, M, N, K, xd):
    import torch
    W = synth.weights(N, K, seed=3 * N + K)
    x = synth.activations(M, K, seed=7 * M + K, dtype=xd, outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, xd)
    packed, _, g32 = _packed(bl, W)
    q, s = bl.quant_act(_xdev(x, xd))
    y, acc = bl.forward(q, s, packed, g32, N, K, acc_debug=True)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("M,N,K,xd", CASES)
def test_forward_fused(bl, kind, M, N, K, xd):
    import torch
    W = synth.weights(N, K, seed=5 * N + K)
    x = synth.activations(M, K, seed=11 * M + K, dtype=xd, outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, xd)
    packed, _, g32 = _packed(bl, W)
    y = bl.forward_x(_xdev(x, xd), packed, g32, N, K)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("M", [1, 3, 16])
def test_forward_bf16_out(bl, kind, M):
    import torch
    N, K = 300, 640
    W = synth.weights(N, K, seed=2)
    x = synth.activations(M, K, seed=3, dtype="bf16")
    ref = oracle.bitlinear(W, x, "bf16")
    packed, _, g32 = _packed(bl, W)
    y = bl.forward_x(P.to_dev_bf16(x), packed, g32, N, K, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert np.array_equal(P.bf16_dev_to_bits(y), oracle.to_bf16(ref["y"]))


@pytest.mark.parametrize("M", [1, 2, 7])
def test_grouped(bl, kind, M):
    # one launch over linears of different K and N (as for a transformer
    # block); every output checked against the oracle
    import torch
    shapes = [(640, 2560), (2560, 640), (96, 4097), (8, 64)]
    xs, ps, gs, ys, refs = [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=100 + i)
        x = synth.activations(M, K, seed=200 + i, dtype="bf16", outlier_frac=0.01)
        refs.append(oracle.bitlinear(W, x, "bf16"))
        p, _, g = _packed(bl, W)
        xs.append(P.to_dev_bf16(x))
        ps.append(p)
        gs.append(g)
        ys.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
    bl.bitlinear_forward_x_grouped(xs, ps, gs, [s[0] for s in shapes], [s[1] for s in shapes], ys)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


def test_set_decode_kernel_rejects_unknown(bl):
    assert bl.lib().bitlinear_set_decode_kernel(5) == bl.BL_ERR_ARG
    assert bl.lib().bitlinear_set_decode_kernel(-1) == bl.BL_ERR_ARG
    assert bl.bitlinear_get_decode_kernel() == bl.BL_DECODE_AUTO


@pytest.mark.parametrize("M,K", [(16, 11008), (8, 16384)])
def test_tensor_kernel_large_operand(bl, M, K):
    # M * Kp too large for the deep prefetch rings: the tensor-core kernel
    # keeps the resident operand and runs with shallower rings
    import torch
    N = 200
    W = synth.weights(N, K, seed=K + M)
    x = synth.activations(M, K, seed=M * 3 + K, dtype="bf16", outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, "bf16")
    packed, _, g32 = _packed(bl, W)
    q, s = bl.quant_act(P.to_dev_bf16(x))
    bl.bitlinear_set_decode_kernel(bl.BL_DECODE_TENSOR)
    try:
        y, acc = bl.forward(q, s, packed, g32, N, K, acc_debug=True)
        torch.cuda.synchronize()
    finally:
        bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)
    assert bl.bitlinear_get_status() == bl.BL_OK
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("N,K", [(13, 200), (300, 1000), (33, 4097), (2560, 640), (640, 2560), (6912, 2560),
                                 (2560, 6912), (20000, 64)])
def test_lut_kernel(bl, N, K):
    # table-lookup decode (M = 1, unfused form) against the oracle
    import torch
    W = synth.weights(N, K, seed=N + 7 * K)
    x = synth.activations(1, K, seed=K, dtype="bf16", outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, "bf16")
    packed, _, g32 = _packed(bl, W)
    q, s = bl.quant_act(P.to_dev_bf16(x))
    bl.bitlinear_set_decode_kernel(bl.BL_DECODE_LUT)
    try:
        y, acc = bl.forward(q, s, packed, g32, N, K, acc_debug=True)
        torch.cuda.synchronize()
    finally:
        bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)
    assert bl.bitlinear_get_status() == bl.BL_OK
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


def test_lut_kernel_limits(bl):
    # M > 1, tables beyond shared memory, and the fused calls are refused
    import torch
    W = synth.weights(64, 256, seed=1)
    packed, _, g32 = _packed(bl, W)
    x2 = P.to_dev_bf16(synth.activations(2, 256, seed=2, dtype="bf16"))
    q2, s2 = bl.quant_act(x2)
    big = torch.zeros((1, 28672), dtype=torch.bfloat16, device="cuda")
    Wb = torch.zeros((8, 28672), dtype=torch.float32, device="cuda")
    pb, _, gb = bl.pack(Wb)
    qb, sb = bl.quant_act(big)
    bl.bitlinear_set_decode_kernel(bl.BL_DECODE_LUT)
    try:
        with pytest.raises(bl.BitLinearError):
            bl.forward(q2, s2, packed, g32, 64, 256)
        with pytest.raises(bl.BitLinearError):
            bl.forward(qb, sb, pb, gb, 8, 28672)
        with pytest.raises(bl.BitLinearError):
            bl.forward_x(x2[:1], packed, g32, 64, 256)
    finally:
        bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)
    torch.cuda.synchronize()


def test_prepared_grouped_call_matches_direct_call(bl):
    # GroupedDecode marshals once; its results equal the plain grouped call's
    import torch
    shapes = [(640, 2560), (96, 4097), (300, 1000)]
    xs, ps, gs, y1, y2 = [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=400 + i)
        x = synth.activations(1, K, seed=500 + i, dtype="bf16")
        p, _, g = _packed(bl, W)
        xs.append(P.to_dev_bf16(x))
        ps.append(p)
        gs.append(g)
        y1.append(torch.empty((1, N), dtype=torch.float32, device="cuda"))
        y2.append(torch.empty((1, N), dtype=torch.float32, device="cuda"))
    Ns, Ks = [s[0] for s in shapes], [s[1] for s in shapes]
    call = bl.GroupedDecode(xs, ps, gs, Ns, Ks, y1)
    call()
    call()
    bl.bitlinear_forward_x_grouped(xs, ps, gs, Ns, Ks, y2)
    torch.cuda.synchronize()
    for a, b in zip(y1, y2):
        assert np.array_equal(a.cpu().numpy(), b.cpu().numpy())


@pytest.mark.parametrize("M,N,K", [(16, 200, 11008), (12, 96, 11776), (1, 64, 150000)])
def test_fused_beyond_the_streaming_limit(bl, M, N, K):
    # activations above 160 KiB per CTA: only the tensor-core kernel holds
    # them, and AUTO falls through to it for the fused form too
    import torch
    assert bl.bitlinear_forward_x_supported(M, K)
    W = synth.weights(N, K, seed=K + 5 * M)
    x = synth.activations(M, K, seed=M + K, dtype="bf16", outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, "bf16")
    packed, _, g32 = _packed(bl, W)
    y = bl.forward_x(P.to_dev_bf16(x), packed, g32, N, K)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)
    bl.bitlinear_set_decode_kernel(bl.BL_DECODE_DP4A)
    try:
        with pytest.raises(bl.BitLinearError):
            bl.forward_x(P.to_dev_bf16(x), packed, g32, N, K)
    finally:
        bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)


@pytest.mark.parametrize("M", [9, 16])
def test_grouped_mixed_ring_depths(bl, M):
    # one launch over a long-K problem (shallow rings) and short-K problems
    # (their CTAs take deeper rings from the same shared-memory region)
    import torch
    shapes = [(96, 11008), (200, 4096), (64, 1000), (8, 64)]
    xs, ps, gs, ys, refs = [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=700 + i)
        x = synth.activations(M, K, seed=800 + i, dtype="bf16", outlier_frac=0.01)
        refs.append(oracle.bitlinear(W, x, "bf16"))
        p, _, g = _packed(bl, W)
        xs.append(P.to_dev_bf16(x))
        ps.append(p)
        gs.append(g)
        ys.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
    bl.bitlinear_forward_x_grouped(xs, ps, gs, [s[0] for s in shapes], [s[1] for s in shapes], ys)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)



@pytest.mark.parametrize("M", [1, 2, 3, 8, 16])
def test_workspace_form(bl, kind, M):
    # quantise-once launch + product on the codes (M >= 2): the same y, bit
    # for bit, as the single-launch form and the oracle; the workspace is
    # reused by a second call
    import torch
    shapes = [(640, 2560), (96, 4097), (300, 1000), (8, 64)]
    xs, ps, gs, y1, y2, refs = [], [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=1100 + i)
        x = synth.activations(M, K, seed=1200 + i + M, dtype="bf16", outlier_frac=0.01)
        refs.append(oracle.bitlinear(W, x, "bf16"))
        p, _, g = _packed(bl, W)
        xs.append(P.to_dev_bf16(x))
        ps.append(p)
        gs.append(g)
        y1.append(torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda"))
        y2.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
    Ns, Ks = [s[0] for s in shapes], [s[1] for s in shapes]
    ws = bl.decode_workspace(M, Ks, "cuda")
    bl.bitlinear_forward_x_grouped(xs, ps, gs, Ns, Ks, y1, workspace=ws)
    bl.bitlinear_forward_x_grouped(xs, ps, gs, Ns, Ks, y1, workspace=ws)
    bl.bitlinear_forward_x_grouped(xs, ps, gs, Ns, Ks, y2)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for a, b, ref in zip(y1, y2, refs):
        assert np.array_equal(a.cpu().numpy(), b.cpu().numpy())
        P.check_y_f32(a.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("M", [4, 16])
def test_workspace_form_beyond_the_streaming_limit(bl, M):
    import torch
    shapes = [(200, 11008), (128, 4096)]
    xs, ps, gs, ys, refs = [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=1300 + i)
        x = synth.activations(M, K, seed=1400 + i, dtype="f32", outlier_frac=0.01)
        refs.append(oracle.bitlinear(W, x, "f32"))
        p, _, g = _packed(bl, W)
        xs.append(P.to_dev_f32(x))
        ps.append(p)
        gs.append(g)
        ys.append(torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
    Ns, Ks = [s[0] for s in shapes], [s[1] for s in shapes]
    bl.bitlinear_forward_x_grouped(xs, ps, gs, Ns, Ks, ys, workspace=bl.decode_workspace(M, Ks, "cuda"))
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for y, ref in zip(ys, refs):
        assert np.array_equal(P.bf16_dev_to_bits(y), oracle.to_bf16(ref["y"]))


def test_prepared_grouped_call_with_gains(bl):
    # GroupedDecode with gains: the SubLN workspace form, equal to the plain
    # SubLN grouped call
    import torch
    M, eps, shapes = 5, 1e-6, [(640, 2560), (96, 4097)]
    xs, gains, ps, gs, y1, y2 = [], [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=1500 + i)
        xs.append(P.to_dev_bf16(synth.activations(M, K, seed=1600 + i, dtype="bf16")))
        gains.append(P.to_dev_f32((1.0 + 0.25 * np.random.default_rng(K).standard_normal(K)).astype(np.float32)))
        p, _, g = _packed(bl, W)
        ps.append(p)
        gs.append(g)
        y1.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
        y2.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
    Ns, Ks = [s[0] for s in shapes], [s[1] for s in shapes]
    bl.GroupedDecode(xs, ps, gs, Ns, Ks, y1, gains=gains, eps=eps)()
    bl.bitlinear_forward_x_rmsnorm_grouped(xs, gains, eps, ps, gs, Ns, Ks, y2)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for a, b in zip(y1, y2):
        assert np.array_equal(a.cpu().numpy(), b.cpu().numpy())
