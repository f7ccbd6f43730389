"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
the same seeded inputs, element by element.  See tests/parity.py for the
tolerances."""
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


def gpu_pack(bl, W, eps=1e-5):
    import torch
    packed, g64, g32 = bl.pack(P.to_dev_f32(W), eps)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), float(g64.item()), float(g32.item())


def x_dev(x, dtype):
    return P.to_dev_f32(x) if dtype == "f32" else P.to_dev_bf16(x)


# ------------------------------------------------------------------ A1+A2
@pytest.mark.parametrize("N,K", [(1, 1), (3, 64), (8, 65), (13, 200), (9, 70), (64, 512), (512, 512),
                                 (100, 1000), (7, 4097)])
def test_pack_small_and_ragged(bl, N, K):
    W = synth.weights(N, K, seed=N * 7 + K)
    ref = oracle.bitlinear(W, np.zeros((1, K), np.float32), "f32")
    packed, g64, g32 = gpu_pack(bl, W)
    P.check_gamma(g64, g32, ref, N * K)
    assert P.compare_packed(packed, ref, N, K) <= max(1, ref["n_boundary"])


def test_pack_exact_ties_hand_built(bl):
    # gamma = 1 exactly, eps = 0: |W| = 0.5 sits on the tie (code 0 either
    # way), 1.5 clips to 1, values just off the tie decide by side.
    W = np.array([[0.5, -0.5, 1.5, -1.5, 0.25, -1.75, 2.0, 0.0]], np.float32)
    packed, g64, g32 = gpu_pack(bl, W, eps=0.0)
    assert g64 == 1.0 and g32 == 1.0
    code, bad = oracle.unpack(packed, 1, 8)
    assert bad == 0 and code.tolist() == [[0, 0, 1, -1, 0, -1, 1, 0]]


@pytest.mark.parametrize("N,K", [(6912, 2560), (2560, 6912), (2560, 2560), (640, 2560),
                                 (11008, 4096), (4096, 11008), (4096, 4096)])
def test_pack_full_sizes(bl, N, K):
    W = synth.weights(N, K, seed=1)
    g64 = oracle.absmean_gamma(W)
    code, bnd, nb = oracle.ternary_codes(W, g64, 1e-5)
    ref = dict(gamma64=g64, gamma32=float(np.float32(g64)), code=code, boundary=bnd, packed=oracle.pack(code))
    packed, gg64, gg32 = gpu_pack(bl, W)
    P.check_gamma(gg64, gg32, ref, N * K)
    assert P.compare_packed(packed, ref, N, K) <= max(1, nb)


def test_pack_deterministic(bl):
    W = synth.weights(4096, 4096, seed=3)
    a = gpu_pack(bl, W)
    b = gpu_pack(bl, W)
    assert np.array_equal(a[0], b[0]) and a[1] == b[1]


# --------------------------------------------------------------------- A3
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(1, 1), (1, 7), (3, 64), (2, 100), (8, 512), (1, 2560), (4, 6912),
                                 (2048, 2560), (1, 28672)])
def test_quant_act(bl, dtype, M, K):
    import torch
    x = synth.activations(M, K, seed=M + K, dtype=dtype, outlier_frac=0.01)
    if M > 1:
        x[M // 2] = 0   # an all-zero token
    q, s = bl.quant_act(x_dev(x, dtype))
    torch.cuda.synchronize()
    q, s = q.cpu().numpy(), s.cpu().numpy()
    qr, sr, clipped = oracle.quant_act(x, dtype)
    assert clipped == 0
    assert np.array_equal(q[:, :K], qr)
    assert np.all(q[:, K:] == 0)
    assert np.array_equal(s.view(np.uint32), sr.view(np.uint32))


# ----------------------------------------------------------------- A4+A5
def run_layer(bl, W, x, xdtype, out_dtype="f32", fused=False):
    import torch
    N, K = W.shape
    packed, g64, g32 = bl.pack(P.to_dev_f32(W))
    xd = x_dev(x, xdtype)
    odt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    if fused:
        y = bl.forward_x(xd, packed, g32, N, K, odt)
        acc = None
    else:
        q, s = bl.quant_act(xd)
        y, acc = bl.forward(q, s, packed, g32, N, K, odt, acc_debug=True)
    torch.cuda.synchronize()
    yv = y.cpu().numpy() if out_dtype == "f32" else P.bf16_dev_to_bits(y)
    return yv, (acc.cpu().numpy() if acc is not None else None)


@pytest.mark.parametrize("M,N,K,xd", [(8, 512, 512, "f32"), (1, 13, 200, "bf16"), (3, 9, 70, "f32"),
                                      (2, 64, 64, "bf16"), (5, 100, 1000, "bf16"), (16, 256, 768, "bf16"),
                                      (1, 1, 1, "f32"), (7, 33, 4097, "bf16"), (24, 40, 320, "bf16")])
def test_forward_small_and_ragged(bl, M, N, K, xd):
    W = synth.weights(N, K, seed=M + N + K)
    x = synth.activations(M, K, seed=5 * M + K, dtype=xd, outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, xd)
    y, acc = run_layer(bl, W, x, xd)
    assert np.array_equal(acc, ref["acc"])
    P.check_y_f32(y, ref["y"], exact=(M <= 16))


@pytest.mark.parametrize("M,N,K", [(1, 640, 2560), (4, 300, 1000), (16, 96, 2560)])
def test_forward_x_matches_oracle_and_unfused(bl, M, N, K):
    W = synth.weights(N, K, seed=11)
    x = synth.activations(M, K, seed=12, dtype="bf16", outlier_frac=0.01)
    ref = oracle.bitlinear(W, x, "bf16")
    yf, _ = run_layer(bl, W, x, "bf16", fused=True)
    yu, _ = run_layer(bl, W, x, "bf16", fused=False)
    assert np.array_equal(yf, yu)
    P.check_y_f32(yf, ref["y"], exact=True)


def test_forward_bf16_output(bl):
    W = synth.weights(300, 640, seed=2)
    x = synth.activations(4, 640, seed=3, dtype="bf16")
    ref = oracle.bitlinear(W, x, "bf16")
    y, acc = run_layer(bl, W, x, "bf16", out_dtype="bf16")
    assert np.array_equal(acc, ref["acc"])
    P.check_y_bf16(y, ref["y"])


def test_block2b_grouped_single_launch(bl):
    import torch
    lin = synth.block2b_inputs(0, M=1)
    xs, ps, gs, ys, refs = [], [], [], [], []
    for L in lin:
        packed, _, g32 = bl.pack(P.to_dev_f32(L["W"]))
        xs.append(P.to_dev_bf16(L["x"]))
        ps.append(packed)
        gs.append(g32)
        ys.append(torch.empty((1, L["N"]), dtype=torch.float32, device="cuda"))
        refs.append(oracle.bitlinear(L["W"], L["x"], "bf16"))
    bl.bitlinear_forward_x_grouped(xs, ps, gs, [L["N"] for L in lin], [L["K"] for L in lin], ys)
    torch.cuda.synchronize()
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("M", synth.M_7B)
def test_7b_group_as_benched(bl, M):
    # the 7B-class decode step exactly as bench.py times it: the three
    # linears' inputs from the same seeds, one prepared grouped call
    # (workspace form: for M >= 2 a quantiser launch, then the product on the
    # codes), every output element against the oracle
    import torch
    xs, ps, gs, ys, refs, Ns, Ks = [], [], [], [], [], [], []
    for i, (K, N, _) in enumerate(synth.SHAPES_7B):
        W = synth.weights(N, K, 10 + i)
        x = synth.activations(M, K, 2000 + i, "bf16")
        refs.append(oracle.bitlinear(W, x, "bf16"))
        packed, _, g32 = bl.pack(P.to_dev_f32(W))
        xs.append(P.to_dev_bf16(x))
        ps.append(packed)
        gs.append(g32)
        ys.append(torch.empty((M, N), dtype=torch.float32, device="cuda"))
        Ns.append(N)
        Ks.append(K)
    step = bl.GroupedDecode(xs, ps, gs, Ns, Ks, ys)
    step()
    step()
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for y, ref in zip(ys, refs):
        P.check_y_f32(y.cpu().numpy(), ref["y"], exact=True)


@pytest.mark.parametrize("K,N", [(K, N) for K, N, _ in synth.SHAPES_7B])
@pytest.mark.parametrize("M", synth.M_7B)
def test_7b_shapes_full(bl, M, K, N):
    W = synth.weights(N, K, seed=K + N)
    x = synth.activations(M, K, seed=M, dtype="bf16")
    ref = oracle.bitlinear(W, x, "bf16")
    y, acc = run_layer(bl, W, x, "bf16")
    assert np.array_equal(acc, ref["acc"])
    P.check_y_f32(y, ref["y"], exact=True)


@pytest.mark.parametrize("K,N", [(K, N) for K, N, _ in synth.PREFILL])
def test_prefill_sampled(bl, K, N):
    # M = 2048 tokens, bf16 in, bf16 out.  The oracle computes codes and q in
    # full and acc/y at 4096 sampled outputs plus two full token rows.
    import torch
    M = synth.M_PREFILL
    W = synth.weights(N, K, seed=21)
    x = synth.activations(M, K, seed=22, dtype="bf16")
    g64 = oracle.absmean_gamma(W)
    code, _, _ = oracle.ternary_codes(W, g64, 1e-5)
    qr, sr, _ = oracle.quant_act(x, "bf16")
    g32 = float(np.float32(g64))
    y, acc = run_layer(bl, W, x, "bf16", out_dtype="bf16")
    rng = np.random.default_rng(0)
    ms = np.concatenate([rng.integers(0, M, 4096), np.full(N, 0), np.full(N, M - 1)])
    ns = np.concatenate([rng.integers(0, N, 4096), np.arange(N), np.arange(N)])
    acc_ref = oracle.int_matmul_sampled(qr, code, ms, ns)
    assert np.array_equal(acc[ms, ns], acc_ref)
    y_ref = np.array([oracle.rescale_one(a, g32, sr[m]) for a, m in zip(acc_ref, ms)], np.float32)
    P.check_y_bf16(y[ms, ns], y_ref)


# ------------------------------------------------------------ status word
def test_nonfinite_inputs_set_status(bl):
    import torch
    assert bl.bitlinear_get_status() == bl.BL_OK
    W = synth.weights(16, 64, seed=1)
    W[3, 5] = np.nan
    bl.pack(P.to_dev_f32(W))
    assert bl.bitlinear_get_status() == bl.BL_ERR_NONFINITE
    assert bl.bitlinear_get_status() == bl.BL_OK          # cleared by the read
    x = synth.activations(2, 64, seed=1, dtype="f32")
    x[1, 0] = np.inf
    bl.quant_act(P.to_dev_f32(x))
    assert bl.bitlinear_get_status() == bl.BL_ERR_NONFINITE
    torch.cuda.synchronize()


def test_api_errors_raise(bl):
    import torch
    x = torch.zeros((17, 64), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros(bl.bitlinear_packed_bytes(8, 64), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    with pytest.raises(bl.BitLinearError) as e:
        bl.forward_x(x, packed, g, 8, 64)
    assert e.value.status == bl.BL_ERR_SHAPE
