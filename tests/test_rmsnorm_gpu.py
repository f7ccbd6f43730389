"""GPU parity of the SubLN (RMS normalisation) paths against the oracle:
the standalone normalise-and-quantise kernel, and the fused decode forms of
every streaming decode kernel.  Bit-exact, except that rows whose fp64
normalisation factor lies within 1e-13 of an fp32 rounding midpoint may
round either way (different fp64 summation orders); such rows are counted
and skipped (none is expected)."""
import numpy as np
import pytest

import oracle
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


def _x_f32(x, xd):
    return synth.bf16_bits_to_f32(x) if xd == "bf16" else np.asarray(x, np.float32)


def straddle_rows(x, xd, eps):
    """Rows whose factor 1/sqrt(ms + eps) sits within 1e-13 of an fp32 midpoint."""
    xf = _x_f32(x, xd).astype(np.float64)
    r = 1.0 / np.sqrt((xf * xf).sum(axis=1) / xf.shape[1] + eps)
    r32 = r.astype(np.float32)
    other = np.where(r32.astype(np.float64) < r, np.nextafter(r32, np.float32(np.inf)),
                     np.nextafter(r32, np.float32(0)))
    mid = (r32.astype(np.float64) + other.astype(np.float64)) / 2
    return np.abs(r - mid) <= 1e-13 * r


def _gain(K, seed):
    rng = np.random.default_rng(seed)
    return (1.0 + 0.25 * rng.standard_normal(K)).astype(np.float32)


@pytest.mark.parametrize("xd", ["f32", "bf16"])
@pytest.mark.parametrize("M,K,eps", [(1, 7, 1e-6), (3, 64, 1e-6), (2, 2560, 1e-5), (17, 6912, 1e-6),
                                     (2, 9000, 1e-6), (1, 28672, 1e-6), (4, 1000, 1e-2)])
def test_rmsnorm_quant_act(bl, xd, M, K, eps):
    import torch
    x = synth.activations(M, K, seed=M * 31 + K, dtype=xd, outlier_frac=0.01)
    g = _gain(K, K)
    _, qr, sr, clipped = oracle.rmsnorm_quant_act(x, xd, g, eps)
    xdev = P.to_dev_f32(x) if xd == "f32" else P.to_dev_bf16(x)
    q, s = bl.rmsnorm_quant_act(xdev, P.to_dev_f32(g), eps)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    q, s = q.cpu().numpy(), s.cpu().numpy()
    skip = straddle_rows(x, xd, eps)
    assert clipped == 0 and skip.sum() == 0
    assert np.array_equal(q[:, :K], qr)
    assert np.all(q[:, K:] == 0)
    assert np.array_equal(s.view(np.uint32), sr.view(np.uint32))


KINDS = {"auto": 0, "tensor": 1, "dp4a": 2}


@pytest.mark.parametrize("kind", list(KINDS))
@pytest.mark.parametrize("M", [1, 3, 8])
def test_fused_rmsnorm_grouped(bl, kind, M):
    # q/k/v-like group sharing one normalised input, plus a linear with its
    # own input and gain; every output against the oracle
    import torch
    eps = 1e-6
    K1, K2 = 2560, 1000
    x1 = synth.activations(M, K1, seed=71, dtype="bf16", outlier_frac=0.01)
    x2 = synth.activations(M, K2, seed=72, dtype="bf16", outlier_frac=0.01)
    g1, g2 = _gain(K1, 1), _gain(K2, 2)
    shapes = [(640, x1, g1), (2560, x1, g1), (96, x1, g1), (300, x2, g2)]
    xs_dev = {id(x1): P.to_dev_bf16(x1), id(x2): P.to_dev_bf16(x2)}
    gs_dev = {id(g1): P.to_dev_f32(g1), id(g2): P.to_dev_f32(g2)}
    xs, gains, ps, gms, ys, refs, Ns, Ks = [], [], [], [], [], [], [], []
    for i, (N, x, g) in enumerate(shapes):
        K = x.shape[1]
        W = synth.weights(N, K, seed=300 + i)
        refs.append(oracle.bitlinear_rmsnorm(W, x, "bf16", g, eps))
        p, _, gm = bl.pack(P.to_dev_f32(W))
        xs.append(xs_dev[id(x)])
        gains.append(gs_dev[id(g)])
        ps.append(p)
        gms.append(gm)
        ys.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
        Ns.append(N)
        Ks.append(K)
    bl.bitlinear_set_decode_kernel(KINDS[kind])
    try:
        bl.bitlinear_forward_x_rmsnorm_grouped(xs, gains, eps, ps, gms, Ns, Ks, ys)
        torch.cuda.synchronize()
    finally:
        bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)
    assert bl.bitlinear_get_status() == bl.BL_OK
    assert straddle_rows(x1, "bf16", eps).sum() == 0 and straddle_rows(x2, "bf16", eps).sum() == 0
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


def test_fused_rmsnorm_equals_separate(bl):
    # fused prologue == standalone normalise-and-quantise kernel + product
    import torch
    M, N, K, eps = 2, 700, 2560, 1e-6
    x = synth.activations(M, K, seed=5, dtype="bf16")
    g = _gain(K, 9)
    W = synth.weights(N, K, seed=6)
    p, _, gm = bl.pack(P.to_dev_f32(W))
    y1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    bl.bitlinear_forward_x_rmsnorm_grouped([P.to_dev_bf16(x)], [P.to_dev_f32(g)], eps, [p], [gm], [N], [K], [y1])
    q, s = bl.rmsnorm_quant_act(P.to_dev_bf16(x), P.to_dev_f32(g), eps)
    y2 = bl.forward(q, s, p, gm, N, K)
    torch.cuda.synchronize()
    assert np.array_equal(y1.cpu().numpy(), y2.cpu().numpy())


def test_rmsnorm_then_prefill_gemm(bl):
    # the prefill path: normalise-and-quantise then the tensor-core GEMM
    import torch
    M, N, K, eps = 96, 384, 1024, 1e-6
    x = synth.activations(M, K, seed=8, dtype="bf16")
    g = _gain(K, 4)
    W = synth.weights(N, K, seed=7)
    ref = oracle.bitlinear_rmsnorm(W, x, "bf16", g, eps)
    p, _, gm = bl.pack(P.to_dev_f32(W))
    q, s = bl.rmsnorm_quant_act(P.to_dev_bf16(x), P.to_dev_f32(g), eps)
    y, acc = bl.forward(q, s, p, gm, N, K, acc_debug=True)
    torch.cuda.synchronize()
    assert straddle_rows(x, "bf16", eps).sum() == 0
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    P.check_y_f32(y.cpu().numpy(), ref["y"])


def test_rmsnorm_grouped_beyond_the_streaming_limit(bl):
    # M = 16 at K = 11008: the activations fit only the tensor-core kernel
    import torch
    M, eps, shapes = 16, 1e-6, [(64, 11008), (128, 4096)]
    xs, gains, ps, gs, ys, refs, xs_host = [], [], [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=900 + i)
        x = synth.activations(M, K, seed=910 + i, dtype="bf16", outlier_frac=0.01)
        g = _gain(K, 920 + i)
        refs.append(oracle.bitlinear_rmsnorm(W, x, "bf16", g, eps))
        p, _, g32 = bl.pack(P.to_dev_f32(W))
        xs.append(P.to_dev_bf16(x))
        xs_host.append(x)
        gains.append(P.to_dev_f32(g))
        ps.append(p)
        gs.append(g32)
        ys.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
    bl.bitlinear_forward_x_rmsnorm_grouped(xs, gains, eps, ps, gs, [s[0] for s in shapes],
                                           [s[1] for s in shapes], ys)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    assert all(straddle_rows(x, "bf16", eps).sum() == 0 for x in xs_host)
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("kind", ["auto", "tensor", "dp4a", "tile"])
@pytest.mark.parametrize("M", [2, 16])
def test_rmsnorm_workspace_form(bl, kind, M):
    # SubLN quantised once per row (grouped quantiser launch), then the
    # product on the codes: against the oracle, every decode kernel
    import torch
    eps = 1e-6
    shapes = [(640, 2560), (96, 4097), (8, 64)]
    xs, gains, ps, gs, ys, refs, xs_host = [], [], [], [], [], [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, seed=1700 + i)
        x = synth.activations(M, K, seed=1800 + i, dtype="bf16", outlier_frac=0.01)
        g = _gain(K, 1900 + i)
        refs.append(oracle.bitlinear_rmsnorm(W, x, "bf16", g, eps))
        p, _, g32 = bl.pack(P.to_dev_f32(W))
        xs.append(P.to_dev_bf16(x))
        xs_host.append(x)
        gains.append(P.to_dev_f32(g))
        ps.append(p)
        gs.append(g32)
        ys.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
    Ns, Ks = [s[0] for s in shapes], [s[1] for s in shapes]
    bl.bitlinear_set_decode_kernel({"tile": bl.BL_DECODE_TILE}.get(kind, KINDS.get(kind)))
    try:
        bl.bitlinear_forward_x_rmsnorm_grouped(xs, gains, eps, ps, gs, Ns, Ks, ys,
                                               workspace=bl.decode_workspace(M, Ks, "cuda"))
        torch.cuda.synchronize()
    finally:
        bl.bitlinear_set_decode_kernel(bl.BL_DECODE_AUTO)
    assert bl.bitlinear_get_status() == bl.BL_OK
    assert all(straddle_rows(x, "bf16", eps).sum() == 0 for x in xs_host)
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)
