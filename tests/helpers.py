"""Small numpy helpers shared by the tests (bit patterns, ulp distance)."""
import numpy as np


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 (exact)."""
    return (np.asarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits_rne(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (test-side helper, float inputs only)."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    out = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(a, dtype=np.float32))
    out[nan] = (np.asarray(a, dtype=np.float32).view(np.uint32)[nan] >> 16).astype(np.uint16) | 0x40
    return out


def ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance between bf16 bit patterns in units in the last place.

    Maps each pattern to an order-preserving integer (+0 and -0 both to 0) and
    subtracts. NaN patterns are not expected in these tests.
    """
    def key(x):
        x = np.asarray(x, dtype=np.uint16).astype(np.int32)
        mag = x & 0x7FFF
        return np.where(x & 0x8000, -mag, mag)
    return np.abs(key(a) - key(b))
