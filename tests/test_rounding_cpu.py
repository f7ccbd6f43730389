"""The activation codes' rounding by addition, checked on the CPU.

The kernels round x*s to an int8 code by adding 1.5 * 2^23 in fp32 and
keeping the low byte of the sum's bit pattern (rint_low_byte in
csrc/bl_internal.cuh).  In [2^23, 2^24) the fp32 spacing is 1, so the IEEE
round-to-nearest-even addition rounds to an integer with ties to even.  This
test replays that arithmetic in numpy fp32 (IEEE, round to nearest even) on
every tie, the floats around every tie and the range ends, and 4 million
random values, against np.rint.  The GPU parity tests check the kernels'
codes against the oracle; this checks the reasoning."""
import numpy as np

MAGIC = np.float32(12582912.0)   # 1.5 * 2^23


def low_byte_code(v: np.ndarray) -> np.ndarray:
    s = (v.astype(np.float32) + MAGIC).astype(np.float32)
    return (s.view(np.uint32) & np.uint32(0xFF)).astype(np.uint8).view(np.int8)


def test_ties_and_neighbours():
    ties = np.arange(-255, 256, dtype=np.float32) / np.float32(2)       # -127.5 .. 127.5 step 0.5
    vals = [ties]
    for direction in (np.float32(np.inf), np.float32(-np.inf)):
        nb = ties.copy()
        for _ in range(3):
            nb = np.nextafter(nb, direction)
            vals.append(nb)
    v = np.concatenate(vals)
    v = v[np.abs(v) <= 127.5]
    assert np.array_equal(low_byte_code(v), np.rint(v).astype(np.int8))


def test_random_values():
    rng = np.random.default_rng(0)
    v = rng.uniform(-127.5, 127.5, 4_000_000).astype(np.float32)
    assert np.array_equal(low_byte_code(v), np.rint(v).astype(np.int8))


def test_signed_zero_and_ends():
    v = np.array([0.0, -0.0, 0.49999997, -0.49999997, 0.5, -0.5, 1.5, -1.5, 126.5, -126.5, 127.0, -127.0],
                 dtype=np.float32)
    assert low_byte_code(v).tolist() == [0, 0, 0, 0, 0, 0, 2, -2, 126, -126, 127, -127]
