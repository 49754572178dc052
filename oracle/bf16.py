"""bfloat16 bit patterns to float64 (exact).

A bfloat16 value is the upper 16 bits of an IEEE float32; widening it to
float32 and then float64 is exact, so the oracle sees precisely the values
the GPU reads.
"""

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    f32 = (b.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return f32.astype(np.float64)
