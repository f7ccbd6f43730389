"""Comparison helpers shared by the GPU parity tests (test code only).

Tolerances, from the layer's definition (include/bitlinear.h):
  * ternary codes, packed bytes, int8 q and int32 acc: bit-exact; the only
    allowed code differences are at weights whose |W/(gamma+eps)| lies within
    1e-6 of 1/2 (the oracle's boundary mask), and they are counted;
  * gamma64: different fp64 summation orders agree to within the running-sum
    bound (n+1)*2^-53 relative; gamma32 = (float)gamma64 must be equal;
  * fp32 y: relative error <= 1e-6 (the decode kernel is in fact bit-exact);
  * bf16 y: equal after rounding, or 1 bf16 ulp apart where the oracle's fp32
    value lies within 1e-6 relative of the midpoint between the two
    candidates (a rounding straddle).
"""
from __future__ import annotations

import numpy as np

import oracle
import synth

REL_TOL_F32 = 1e-6


def torch_mod():
    import torch
    return torch


def to_dev_f32(a: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def to_dev_bf16(bits: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_dev_to_bits(t) -> np.ndarray:
    torch = torch_mod()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compare_packed(gpu_packed: np.ndarray, ref: dict, N: int, K: int) -> int:
    """Packed bytes equal except at boundary codes; returns #code mismatches."""
    exp = ref["packed"]
    assert gpu_packed.shape == exp.shape
    if np.array_equal(gpu_packed, exp):
        return 0
    got, bad = oracle.unpack(gpu_packed, N, K)
    assert bad == 0, "GPU packed buffer has malformed fields or padding"
    diff = got != ref["code"]
    assert np.all(ref["boundary"][diff] == 1), "code mismatch outside the 1e-6 boundary band"
    return int(diff.sum())


def check_gamma(g64_gpu: float, g32_gpu: float, ref: dict, count: int) -> None:
    bound = (count + 1) * 2.0 ** -53
    assert abs(g64_gpu - ref["gamma64"]) <= bound * abs(ref["gamma64"]), (g64_gpu, ref["gamma64"])
    assert np.float32(g32_gpu) == np.float32(ref["gamma32"])


def check_y_f32(y_gpu: np.ndarray, y_ref: np.ndarray, exact: bool = False) -> float:
    y_gpu = np.asarray(y_gpu, np.float32)
    y_ref = np.asarray(y_ref, np.float32)
    assert y_gpu.shape == y_ref.shape
    zero = y_ref == 0
    assert np.all(y_gpu[zero] == 0)
    rel = np.abs(y_gpu[~zero].astype(np.float64) - y_ref[~zero]) / np.abs(y_ref[~zero].astype(np.float64))
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= REL_TOL_F32, worst
    if exact:
        assert np.array_equal(y_gpu, y_ref)
    return worst


def check_y_bf16(y_gpu_bits: np.ndarray, y_ref_f32: np.ndarray) -> int:
    """Returns the number of allowed 1-ulp rounding straddles."""
    ref_bits = oracle.to_bf16(y_ref_f32)
    diff = y_gpu_bits != ref_bits
    if not diff.any():
        return 0
    g = y_gpu_bits[diff].astype(np.int64)
    r = ref_bits[diff].astype(np.int64)
    assert np.all(np.abs(g - r) == 1), "bf16 outputs differ by more than one ulp"
    lo = np.minimum(g, r).astype(np.uint16)
    hi = np.maximum(g, r).astype(np.uint16)
    mid = (synth.bf16_bits_to_f32(lo).astype(np.float64) + synth.bf16_bits_to_f32(hi)) / 2
    yv = y_ref_f32[diff].astype(np.float64)
    assert np.all(np.abs(yv - mid) <= 1e-6 * np.abs(yv)), "bf16 difference is not a rounding straddle"
    return int(diff.sum())
