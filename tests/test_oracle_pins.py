"""Pins of the CPU oracle against facts fixed independently of it.

Each check comes from the definition on the BitNet b1.58 pages or from
mathematics, not from re-running the oracle's own formula: hand-derived
cases, closed forms, invariants, exact rational arithmetic, library routines
for the special cases that reduce to them, and published generator vectors.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------ gamma (A1)
def test_gamma_constant_magnitude_closed_form():
    # |W| = c everywhere -> mean|W| = c exactly (c and the count are exact).
    g = np.random.default_rng(1)
    W = np.where(g.random((37, 53)) < 0.5, 0.75, -0.75).astype(np.float32)
    assert oracle.absmean_gamma(W) == 0.75


def test_gamma_counts_every_element():
    # One zero row among N: mean = c * (N - 1) / N; catches a wrong divisor
    # (N or K instead of N*K) or a skipped row.
    W = np.full((8, 16), -0.5, np.float32)
    W[3] = 0.0
    assert oracle.absmean_gamma(W) == 0.5 * 7 / 8


def test_gamma_matches_exact_rational_mean():
    # Exact mean as a Fraction vs the fp64 running sum: the running sum of n
    # non-negative terms is within (n-1)*u*sum of the exact sum (Higham,
    # "Accuracy and Stability of Numerical Algorithms", sec. 4.2), plus one
    # rounding for the division.
    W = synth.weights(64, 96, seed=7)
    exact = sum(Fraction(float(abs(v))) for v in W.ravel()) / W.size
    g = Fraction(oracle.absmean_gamma(W))
    u = Fraction(1, 2 ** 53)
    bound = (W.size + 1) * u * exact
    assert abs(g - exact) <= bound


def test_gamma_gaussian_expectation():
    # E|W| = sigma * sqrt(2/pi) for W ~ N(0, sigma^2); std of the mean of
    # |W| is sigma * sqrt(1 - 2/pi) / sqrt(n).
    sigma, n_rows, n_cols = 0.02, 512, 1024
    W = synth.weights(n_rows, n_cols, seed=3, sigma=sigma)
    g = oracle.absmean_gamma(W)
    mu = sigma * math.sqrt(2 / math.pi)
    se = sigma * math.sqrt(1 - 2 / math.pi) / math.sqrt(W.size)
    assert abs(g - mu) < 6 * se


# ------------------------------------------------------------ codes (A1)
def test_codes_hand_built_ties_and_clip():
    # mean|W| = 8/8 = 1 exactly.  With eps = 0, r = W:
    #   0.5 -> rint 0 (tie to even), -0.5 -> 0, 1.5 -> 2 -> clip 1,
    #   -1.5 -> -1, 0.25 -> 0, -1.75 -> -2 -> clip -1, 2.0 -> 1, 0 -> 0.
    W = np.array([[0.5, -0.5, 1.5, -1.5, 0.25, -1.75, 2.0, 0.0]], np.float32)
    g = oracle.absmean_gamma(W)
    assert g == 1.0
    code, bnd, nb = oracle.ternary_codes(W, g, eps=0.0)
    assert code.tolist() == [[0, 0, 1, -1, 0, -1, 1, 0]]
    assert bnd.tolist() == [[1, 1, 0, 0, 0, 0, 0, 0]] and nb == 2


def test_codes_eps_enters_the_threshold():
    # gamma = 1 (values sum to 4 over 4 elements).  0.5000038 is above the
    # threshold 0.5*gamma but below 0.5*(gamma + 1e-5) = 0.500005.
    v = np.float32(0.5000038)
    W = np.array([[v, np.float32(4.0) - v - np.float32(1.0) - np.float32(1.0), 1.0, -1.0]], np.float32)
    g = oracle.absmean_gamma(W)
    assert g == 1.0
    assert oracle.ternary_codes(W, g, eps=0.0)[0][0, 0] == 1
    assert oracle.ternary_codes(W, g, eps=1e-5)[0][0, 0] == 0


def test_codes_exact_rational_classification():
    # Brute force over random W: code = sign(W) * [|W|/(g+eps) > 1/2], decided
    # in exact rational arithmetic.  Values within 1e-9 of the boundary are
    # skipped (ties are the documented exception).
    W = synth.weights(24, 40, seed=11)
    eps = 1e-5
    g = oracle.absmean_gamma(W)
    code, _, _ = oracle.ternary_codes(W, g, eps)
    d = Fraction(g) + Fraction(eps)
    checked = 0
    for (n, k), w in np.ndenumerate(W):
        r = Fraction(float(w)) / d
        if abs(abs(r) - Fraction(1, 2)) < Fraction(1, 10 ** 9):
            continue
        want = 0 if abs(r) < Fraction(1, 2) else (1 if r > 0 else -1)
        assert code[n, k] == want, (n, k, float(r))
        checked += 1
    assert checked > 900


def test_codes_zero_fraction_closed_form():
    # For Gaussian W, gamma -> sigma*sqrt(2/pi) and a code is 0 iff
    # |W| <= (gamma + eps)/2, so P(0) = 2*Phi(t) - 1 with t = (gamma+eps)/(2 sigma)
    # (about 0.310 at eps = 0).  Binomial +-5 sigma window.
    sigma = 0.02
    W = synth.weights(1024, 1024, seed=5, sigma=sigma)
    g = oracle.absmean_gamma(W)
    code, _, _ = oracle.ternary_codes(W, g, 1e-5)
    t = (sigma * math.sqrt(2 / math.pi) + 1e-5) / (2 * sigma)
    p = math.erf(t / math.sqrt(2))
    n = W.size
    frac = float(np.mean(code == 0))
    assert abs(frac - p) < 5 * math.sqrt(p * (1 - p) / n)
    assert abs(p - 0.3101) < 0.001


def test_codes_values_sign_symmetry_and_power_of_two_scaling():
    W = synth.weights(64, 128, seed=9)
    g = oracle.absmean_gamma(W)
    code, _, _ = oracle.ternary_codes(W, g, 0.0)
    assert set(np.unique(code).tolist()) <= {-1, 0, 1}
    neg, _, _ = oracle.ternary_codes(-W, oracle.absmean_gamma(-W), 0.0)
    assert np.array_equal(neg, -code)
    for e in (-3, 5):
        Ws = (W * np.float32(2.0 ** e)).astype(np.float32)
        cs, _, _ = oracle.ternary_codes(Ws, oracle.absmean_gamma(Ws), 0.0)
        assert np.array_equal(cs, code)


@pytest.mark.parametrize("c", [3.0, 0.7])
def test_codes_scaling_flips_only_near_boundary(c):
    # Scaling W by c > 0 scales gamma by c; with eps > 0 the threshold moves
    # by eps/(c*gamma) relative, so a flip may only happen where
    # |r - 1/2| < eps/gamma + 1e-6.
    eps = 1e-5
    W = synth.weights(128, 256, seed=13)
    g = oracle.absmean_gamma(W)
    code, _, _ = oracle.ternary_codes(W, g, eps)
    Ws = (W.astype(np.float64) * c).astype(np.float32)
    gs = oracle.absmean_gamma(Ws)
    cs, _, _ = oracle.ternary_codes(Ws, gs, eps)
    r = np.abs(W.astype(np.float64) / (g + eps))
    flips = cs != code
    assert np.all(np.abs(r[flips] - 0.5) < eps / g + 1e-6)


# -------------------------------------------------------------- pack (A2)
def _hexbytes(s):
    return np.frombuffer(bytes.fromhex(s), np.uint8)


def test_pack_all_plus_one_and_all_minus_one():
    # The layout stores u = code + 1 (include/bitlinear.h): +1 -> 10, 0 -> 01,
    # -1 -> 00, padding 01.  N=1, K=64 -> 8 padded rows x 1 chunk = 128 bytes.
    # Row 0 is bytes 0..15: all +1 -> 0b10101010 = 0xAA; all -1 -> 0x00.
    # Padded rows 1..7 are all 01 -> 0x55.
    plus = oracle.pack(np.ones((1, 64), np.int8))
    minus = oracle.pack(-np.ones((1, 64), np.int8))
    assert np.array_equal(plus, _hexbytes("aa" * 16 + "55" * 112))
    assert np.array_equal(minus, _hexbytes("00" * 16 + "55" * 112))


def test_pack_single_code_position():
    # Zero codes are 01 -> bytes 0x55.  k = 45 = 16*2 + 4*3 + 1 -> word 2,
    # field 3, byte 1 -> byte offset 2*4 + 1 = 9, bits 6..7:
    #   +1 (10): 0b10_01_01_01 = 0x95;  -1 (00): 0b00_01_01_01 = 0x15.
    code = np.zeros((1, 64), np.int8)
    code[0, 45] = 1
    assert np.array_equal(oracle.pack(code), _hexbytes("55" * 9 + "95" + "55" * 6 + "55" * 112))
    code[0, 45] = -1
    assert np.array_equal(oracle.pack(code), _hexbytes("55" * 9 + "15" + "55" * 6 + "55" * 112))


def test_pack_ragged_tile_and_chunk():
    # N=9, K=70 -> Np=16, Kp=128, C=2, 512 bytes.  Row 8 is row 0 of tile 1
    # (tile stride 8*2*16 = 256).  k = 69: chunk 1, word 0, field 1, byte 1
    # -> offset 256 + (1*8 + 0)*16 + 1 = 385.  That byte's fields cover
    # k = 65 (code 0 -> 01), 69 (+1 -> 10), 73 and 77 (padding -> 01):
    # 0b01_01_10_01 = 0x59.
    code = np.zeros((9, 70), np.int8)
    code[8, 69] = 1
    p = oracle.pack(code)
    assert p.size == 512
    assert p[385] == 0x59
    # Row 9 (tile 1, r = 1) is padding: offsets 256 + (c*8 + 1)*16 .. +16.
    for c in range(2):
        assert np.all(p[256 + (c * 8 + 1) * 16: 256 + (c * 8 + 2) * 16] == 0x55)
    # Row 0, chunk 0 (offset 0..15) is a full chunk of zero codes.
    assert np.all(p[0:16] == 0x55)


@pytest.mark.parametrize("N,K", [(1, 1), (3, 64), (8, 65), (13, 200), (64, 256)])
def test_pack_roundtrip_and_size(N, K):
    g = np.random.default_rng(N * 1000 + K)
    code = g.integers(-1, 2, size=(N, K)).astype(np.int8)
    p = oracle.pack(code)
    assert p.size == ((N + 7) // 8 * 8) * ((K + 63) // 64 * 64) // 4
    back, bad = oracle.unpack(p, N, K)
    assert bad == 0 and np.array_equal(back, code)


# ----------------------------------------------------------- quant (A3)
def test_quant_hand_built_row():
    # amax = 2 -> s = 127/2 = 63.5; x*s = 63.5, -31.75, 15.875, 127
    # -> rint: 64 (tie to even), -32, 16, 127.
    x = np.array([[1.0, -0.5, 0.25, 2.0]], np.float32)
    q, s, clipped = oracle.quant_act(x, "f32")
    assert q.tolist() == [[64, -32, 16, 127]] and s[0] == 63.5 and clipped == 0


def test_quant_extremes_range_and_scaling():
    x = synth.activations(16, 300, seed=2, dtype="f32", outlier_frac=0.01)
    q, s, clipped = oracle.quant_act(x, "f32")
    assert clipped == 0 and q.min() >= -127 and q.max() <= 127
    am = np.argmax(np.abs(x), axis=1)
    for m in range(16):
        assert abs(int(q[m, am[m]])) == 127
        assert np.sign(q[m, am[m]]) == np.sign(x[m, am[m]])
    for e in (-4, 6):
        q2, s2, _ = oracle.quant_act((x * np.float32(2.0 ** e)).astype(np.float32), "f32")
        assert np.array_equal(q2, q) and np.array_equal(s2, (s * np.float32(2.0 ** -e)))


def test_quant_zero_row_and_bf16_widening():
    x = np.zeros((2, 64), np.float32)
    x[1, 5] = -3.0
    q, s, _ = oracle.quant_act(x, "f32")
    assert np.all(q[0] == 0) and s[0] == np.float32(127.0) / np.float32(1e-5)
    assert q[1, 5] == -127 and np.count_nonzero(q[1]) == 1
    xb = synth.activations(5, 130, seed=4, dtype="bf16", outlier_frac=0.01)
    qa, sa, _ = oracle.quant_act(xb, "bf16")
    qb, sb, _ = oracle.quant_act(synth.bf16_bits_to_f32(xb), "f32")
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb)


# ------------------------------------------------------------ matmul (A4)
def test_int_matmul_against_numpy_and_closed_form():
    g = np.random.default_rng(21)
    q = g.integers(-127, 128, size=(5, 333)).astype(np.int8)
    code = g.integers(-1, 2, size=(7, 333)).astype(np.int8)
    acc = oracle.int_matmul(q, code)
    assert np.array_equal(acc, q.astype(np.int64) @ code.astype(np.int64).T)
    K = 28672
    acc = oracle.int_matmul(np.full((1, K), 127, np.int8), np.ones((2, K), np.int8))
    assert acc.tolist() == [[127 * K, 127 * K]]
    ms, ns = np.array([4, 0, 2]), np.array([6, 1, 1])
    full = oracle.int_matmul(q, code)
    assert np.array_equal(oracle.int_matmul_sampled(q, code, ms, ns), full[ms, ns])


# ----------------------------------------------------------- rescale (A5)
def test_rescale_exact_values():
    assert oracle.rescale_one(127, 0.5, 127.0) == 0.5
    assert oracle.rescale_one(-254, 0.25, 63.5) == -1.0
    assert oracle.rescale_one(0, 0.3, 7.0) == 0.0


def test_layer_matches_fp64_matmul_of_dequantised_operands():
    # y = (code * gamma32) @ (q / s)^T evaluated as an fp64 matmul; the
    # oracle's y must agree to 1e-6 relative (it is a different evaluation
    # order of the same exact quantity).
    W = synth.weights(96, 512, seed=0)
    x = synth.activations(8, 512, seed=1, dtype="f32")
    r = oracle.bitlinear(W, x, "f32")
    deq_w = r["code"].astype(np.float64) * r["gamma32"]
    deq_x = r["q"].astype(np.float64) / r["s"].astype(np.float64)[:, None]
    ref = deq_x @ deq_w.T
    nz = ref != 0
    assert np.all(r["y"][~nz] == 0)
    assert np.max(np.abs(r["y"][nz] - ref[nz]) / np.abs(ref[nz])) <= 1e-6
    # Closed form: for Gaussian W and threshold t = (gamma+eps)/(2 sigma),
    # corr(W, code) = E|W|1[|W|>t sigma] / sqrt(E W^2 P(code != 0))
    #               = 2 phi(t) / sqrt(2 (1 - Phi(t)))  (about 0.887),
    # and y inherits it against the unquantised x @ W^T.
    full = x.astype(np.float64) @ W.astype(np.float64).T
    corr = np.corrcoef(full.ravel(), r["y"].ravel())[0, 1]
    t = (r["gamma64"] + 1e-5) / (2 * float(W.std()))
    phi = math.exp(-t * t / 2) / math.sqrt(2 * math.pi)
    tail = 0.5 * math.erfc(t / math.sqrt(2))
    want = 2 * phi / math.sqrt(2 * tail)
    assert abs(corr - want) < 0.03 and abs(want - 0.887) < 0.01


def test_bf16_round_to_nearest_even():
    # 1.0 = 0x3F800000 -> 0x3F80.  0x3F808000 is halfway between 0x3F80 and
    # 0x3F81 -> even 0x3F80; 0x3F818000 -> even 0x3F82; 0x3F808001 -> 0x3F81.
    vals = np.array([0x3F800000, 0x3F808000, 0x3F818000, 0x3F808001, 0xBF808000], np.uint32)
    out = oracle.to_bf16(vals.view(np.float32))
    assert out.tolist() == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xBF80]


def test_threaded_forward_equals_single_thread_pipeline():
    W = synth.weights(50, 320, seed=4)
    x = synth.activations(3, 320, seed=8, dtype="bf16", outlier_frac=0.01)
    r = oracle.bitlinear(W, x, "bf16")
    y = oracle.forward_bf16_mt(x, r["code"], r["gamma32"], threads=4)
    assert np.array_equal(y, r["y"])


# ------------------------------------------- counter-based generator ----
def _kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                v = [int(t, 16) for t in line.split()]
                rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


def test_philox_known_answers():
    for ctr, key, want in _kat():
        assert oracle.philox4x32_10(ctr, key).tolist() == want


def test_synth_weights_recipe_and_distribution():
    # Element (n, k) draws Philox at counter (e//2, 0, g, 0), key (seed, 0),
    # e = n*K + k, using words 2*(e%2) and 2*(e%2)+1.  The Irwin-Hall sum is
    # exact in fp32, so z*65536 + 131072 - 2 is the integer sum of the four
    # 16-bit halves; only the final scale rounds.
    seed, g, K = 7, 3, 100
    W = oracle.synth_weights(seed, g, 5, 2, K)
    scale = np.array([0x3D0DE3BD], np.uint32).view(np.float32)[0]
    for (r, k) in [(0, 0), (0, 1), (1, 99), (1, 42)]:
        e = (5 + r) * K + k
        out = oracle.philox4x32_10([e // 2, 0, g, 0], [seed, 0])
        a, b = int(out[2 * (e % 2)]), int(out[2 * (e % 2) + 1])
        hsum = (a & 0xFFFF) + (a >> 16) + (b & 0xFFFF) + (b >> 16)
        z = np.float32((hsum + 2) / 65536.0 - 2.0)   # exact: fits 19 bits
        assert W[r, k] == np.float32(z * scale)
    big = oracle.synth_weights(1, 0, 0, 256, 1024, threads=4)
    assert np.array_equal(big[:3], oracle.synth_weights(1, 0, 0, 3, 1024))
    assert abs(float(big.mean())) < 1e-4
    assert abs(float(big.std()) - 0.02) < 2e-4


# ------------------------------------------------------------ SubLN (R16)
# RMS normalisation before the quantiser, pinned against torch's own
# rms_norm (a library routine, run in fp64), closed forms and invariants.

def _torch_rms_norm_f64(x, g, eps):
    import torch
    t = torch.from_numpy(np.asarray(x, np.float64))
    return torch.nn.functional.rms_norm(t, (t.shape[-1],), torch.from_numpy(np.asarray(g, np.float64)),
                                        eps).numpy()


@pytest.mark.parametrize("K,eps", [(1, 1e-6), (7, 1e-6), (512, 1e-6), (2560, 1e-5), (64, 1e-2)])
def test_rmsnorm_matches_library_rms_norm(K, eps):
    rng = np.random.default_rng(K)
    x = (rng.standard_normal((3, K)) * np.array([[1.0], [0.05], [3.0]])).astype(np.float32)
    g = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    xn, q, s, clipped = oracle.rmsnorm_quant_act(x, "f32", g, eps)
    ref = _torch_rms_norm_f64(x, g, eps)
    # three fp32 roundings (the factor, x*r, *g): within 2^-22 relative
    assert np.all(np.abs(xn - ref) <= 2.0 ** -22 * np.abs(ref) + 1e-30)
    # the quantiser then runs on xn exactly as on any input
    q2, s2, _ = oracle.quant_act(xn, "f32")
    assert np.array_equal(q, q2) and np.array_equal(s, s2) and clipped == 0


def test_rmsnorm_eps_inside_the_root():
    # small-magnitude row where eps dominates: sqrt(ms + eps), not sqrt(ms) + eps
    x = np.full((1, 16), 1e-3, np.float32)
    g = np.ones(16, np.float32)
    xn, _, _, _ = oracle.rmsnorm_quant_act(x, "f32", g, 1e-2)
    want = 1e-3 / np.sqrt(1e-6 + 1e-2)
    assert abs(float(xn[0, 0]) - want) <= 2.0 ** -22 * want


def test_rmsnorm_constant_row_and_unit_rms():
    g = np.ones(300, np.float32)
    for c in (0.75, -3.0, 1e-4, 123.0):
        x = np.full((1, 300), c, np.float32)
        xn, _, _, _ = oracle.rmsnorm_quant_act(x, "f32", g, 0.0)
        assert np.all(np.abs(np.abs(xn) - 1.0) <= 2.0 ** -22)
        assert np.all(np.sign(xn) == np.sign(c))
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 1000)).astype(np.float32)
    xn, _, _, _ = oracle.rmsnorm_quant_act(x, "f32", np.ones(1000, np.float32), 0.0)
    ms = (xn.astype(np.float64) ** 2).mean(axis=1)
    assert np.all(np.abs(ms - 1.0) < 1e-6)


def test_rmsnorm_power_of_two_scaling_is_exact():
    # eps = 0: scaling x by 2^j scales the mean square by 4^j exactly, so the
    # factor by 2^-j and every normalised value is bit-identical; a gain of
    # 2^i scales the output exactly
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 777)).astype(np.float32)
    g = (1 + 0.2 * rng.standard_normal(777)).astype(np.float32)
    a, qa, sa, _ = oracle.rmsnorm_quant_act(x, "f32", g, 0.0)
    b, qb, sb, _ = oracle.rmsnorm_quant_act(x * np.float32(8.0), "f32", g, 0.0)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb)
    c, _, _, _ = oracle.rmsnorm_quant_act(x, "f32", g * np.float32(0.25), 0.0)
    assert np.array_equal((a * np.float32(0.25)).view(np.uint32), c.view(np.uint32))


def test_rmsnorm_permutation_equivariant_on_exact_sums():
    # small integers: every fp64 partial sum is exact, so the order of the
    # sum cannot matter and a permuted row gives the permuted result
    rng = np.random.default_rng(9)
    x = rng.integers(-20, 21, size=(1, 256)).astype(np.float32)
    g = (1 + 0.3 * rng.standard_normal(256)).astype(np.float32)
    perm = rng.permutation(256)
    a, _, _, _ = oracle.rmsnorm_quant_act(x, "f32", g, 1e-6)
    b, _, _, _ = oracle.rmsnorm_quant_act(x[:, perm], "f32", g[perm], 1e-6)
    assert np.array_equal(a[:, perm].view(np.uint32), b.view(np.uint32))


def test_rmsnorm_bf16_input_is_widened_exactly():
    rng = np.random.default_rng(11)
    xf = rng.standard_normal((2, 300)).astype(np.float32)
    bits = synth.f32_to_bf16_bits(xf)
    g = np.ones(300, np.float32)
    a, qa, sa, _ = oracle.rmsnorm_quant_act(bits, "bf16", g, 1e-6)
    b, qb, sb, _ = oracle.rmsnorm_quant_act(synth.bf16_bits_to_f32(bits), "f32", g, 1e-6)
    assert np.array_equal(a, b) and np.array_equal(qa, qb) and np.array_equal(sa, sb)
