"""Constructed momentum inputs (float32 / bf16 values) on which rounding the
float64 sum mu m + g to the storage type rounds twice and differs from
rounding the exact value once.  Shared by the oracle pins and the GPU parity
tests; no arithmetic of the method lives here."""
import numpy as np

import oracle as orc


def crafted_fp32_tie():
    """mu, m, g (float32 values, 0.5 <= mu < 1) with mu m = 2^-24 (1 - d 2^-47),
    0 < d < 2^18, and g = 1 + 2^-23: the float64 sum is exactly the float32
    midpoint 1 + 2^-23 + 2^-24 (its ties-to-even neighbour is 1 + 2^-22),
    while the exact value lies just below it (nearest: 1 + 2^-23)."""
    for a in range(2 ** 24 - 1, 2 ** 23, -1):
        b = 2 ** 47 // a
        d = 2 ** 47 - a * b
        if 0 < d < 2 ** 18 and 2 ** 23 <= b < 2 ** 24:
            return a / 2.0 ** 24, b / 2.0 ** 47, 1.0 + 2.0 ** -23
    raise AssertionError("no crafted case")


def crafted_bf16_tie():
    """mu = 0.75 and the bf16 m = 129/128, so mu m = 387/512 lies exactly
    halfway between two bf16 values, and a gradient of +-2^-80 that moves the
    exact value off the midpoint towards the odd neighbour: the float64 sum
    rounds back onto the midpoint."""
    m = 1.0 + 1.0 / 128
    p = 0.75 * m                        # 387/512: a tie at bf16 precision
    lo = float(orc.round_bf16(np.float64(p) - 2.0 ** -12))
    down_is_even = orc.round_bf16(np.float64(p)) == lo
    g = (2.0 ** -80) * (1.0 if down_is_even else -1.0)
    return 0.75, m, g
