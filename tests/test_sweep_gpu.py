"""100B-class decode sweep (80 layers x 7 linears, M = 1): weights are drawn
on each side by the counter-based generator (GPU: synth/csrc, oracle: its own
C implementation), so the GPU parity checks here cover sampled layers, each
in full, plus the generator itself against its published vectors."""
import os

import numpy as np
import pytest

import oracle
import synth
from tests import parity as P

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SEED = 1234


@pytest.fixture(scope="module")
def dev():
    import torch  # noqa: F401
    import synth.device as sd
    import ternary_weight_linear_absmean_b200 as bl
    from ternary_weight_linear_absmean_b200 import _build
    _build.build()
    sd.build()
    return sd, bl


def test_device_philox_known_answers(dev):
    sd, _ = dev
    vecs, want = [], []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                v = [int(t, 16) for t in line.split()]
                vecs.append(v[:6])
                want.append(v[6:10])
    assert sd.philox(vecs).tolist() == want


@pytest.mark.parametrize("row0,rows,K", [(0, 3, 8192), (1000, 5, 28672), (7, 4, 1023), (3, 1, 1)])
def test_device_weights_equal_oracle_generator(dev, row0, rows, K):
    import torch
    sd, _ = dev
    W = torch.empty((rows, K), dtype=torch.float32, device="cuda")
    sd.weights(W, SEED, 11, row0)
    torch.cuda.synchronize()
    ref = oracle.synth_weights(SEED, 11, row0, rows, K)
    assert np.array_equal(W.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("layer", [0, 79])
def test_sweep_layer_parity(dev, layer):
    # one full layer of the sweep: 7 matrices generated on the GPU, packed by
    # the library, and run through the grouped fused decode launch; the
    # oracle regenerates every weight on the host and checks codes and y.
    import torch
    sd, bl = dev
    threads = os.cpu_count() or 1
    xs, ps, gs, ys, refs = [], [], [], [], []
    for j, (K, N, name) in enumerate(synth.LAYER100B):
        g = layer * 7 + j
        W = torch.empty((N, K), dtype=torch.float32, device="cuda")
        sd.weights(W, SEED, g)
        packed, g64, g32 = bl.pack(W)
        del W
        x = synth.activations(1, K, 50_000 + g, "bf16")
        xs.append(P.to_dev_bf16(x))
        ps.append(packed)
        gs.append(g32)
        ys.append(torch.empty((1, N), dtype=torch.float32, device="cuda"))
        refs.append((K, N, g, x, g64))
    bl.bitlinear_forward_x_grouped(xs, ps, gs, [r[1] for r in refs], [r[0] for r in refs], ys)
    torch.cuda.synchronize()
    assert bl.bitlinear_get_status() == bl.BL_OK
    for (K, N, g, x, g64), packed, g32, y in zip(refs, ps, gs, ys):
        Wh = oracle.synth_weights(SEED, g, 0, N, K, threads=threads)
        gr = oracle.absmean_gamma(Wh)
        code, bnd, nb = oracle.ternary_codes(Wh, gr, 1e-5)
        del Wh
        ref = dict(gamma64=gr, gamma32=float(np.float32(gr)), code=code, boundary=bnd, packed=oracle.pack(code))
        P.check_gamma(float(g64.item()), float(g32.item()), ref, N * K)
        assert P.compare_packed(packed.cpu().numpy(), ref, N, K) <= max(1, nb)
        q, s, _ = oracle.quant_act(x, "bf16")
        yr = oracle.rescale(oracle.int_matmul(q, code), s, ref["gamma32"])
        P.check_y_f32(y.cpu().numpy(), yr, exact=True)
