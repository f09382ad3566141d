"""Readers for the text fixtures in tests/golden and an exact float32
rounding helper used to re-derive expected values with rational arithmetic."""
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def value_table(name):
    out = {}
    for line in _lines(name):
        code, val = line.split()
        out[int(code, 16)] = float(val)
    return out


def cases(name):
    cur = None
    out = []
    for line in _lines(name):
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
            out.append(cur)
        else:
            cur[key] = rest.split()
    return out


def f32_round(r: Fraction) -> np.float32:
    """Round a rational to the nearest float32, ties to even, exactly
    (including subnormals; no overflow handling needed here)."""
    if r == 0:
        return np.float32(0.0)
    x = np.float32(float(r))
    cands = {x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(-np.inf))}

    def key(c):
        return (abs(Fraction(float(c)) - r), int(np.array(c, dtype=np.float32).view(np.uint32)) & 1)

    return min(cands, key=key)


def rne_int(r: Fraction) -> int:
    fl = r.numerator // r.denominator
    frac = r - fl
    if frac > Fraction(1, 2):
        return fl + 1
    if frac < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1
