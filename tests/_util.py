"""Helpers shared by the tests (comparison only; no method arithmetic)."""
import numpy as np


def fp16_ordered(x: np.ndarray) -> np.ndarray:
    """Map fp16 bit patterns to integers whose order is the numeric order
    (+0 and -0 both map to 0), so |a - b| counts ulps between fp16 values."""
    bits = np.asarray(x, dtype=np.float16).view(np.uint16).astype(np.int32)
    mag = bits & 0x7FFF
    return np.where(bits & 0x8000, -mag, mag)


def max_ulp_fp16(a: np.ndarray, b: np.ndarray) -> int:
    a = np.asarray(a, dtype=np.float16)
    b = np.asarray(b, dtype=np.float16)
    assert a.shape == b.shape
    if a.size == 0:
        return 0
    assert not np.isnan(a).any() and not np.isnan(b).any()
    return int(np.max(np.abs(fp16_ordered(a) - fp16_ordered(b))))
