"""Writes tests/golden/rmsnorm_pins.txt: rows for which each reading of the
RMSNorm steps that the pages leave open, and its alternative, round one
output element to different bf16 values.  Everything is derived with the
exact rational model in tests/exact_binary32.py (no oracle, no GPU): a seeded
random row of bf16 activations with bf16 gains near 1, searched for an
element whose bf16 output differs between the two readings.

    python tests/golden/make_rmsnorm_pins.py
"""
import os
import struct
import sys
from fractions import Fraction

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
import exact_binary32 as xb  # noqa: E402

K = 192
EPS = Fraction(float(np.float32(1e-6)))
ALT = {"summation": dict(summation="sequential"), "mean": dict(mean="reciprocal"),
       "rsqrt": dict(rsqrt="rsqrt"), "order": dict(order="r_gamma_first")}


def bf16_bits(v: Fraction) -> int:
    return struct.unpack("<I", struct.pack("<f", float(v)))[0] >> 16


def from_bf16(b: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", b << 16))[0])


def row(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(K) * np.exp2(rng.integers(-3, 4, K))).astype(np.float32)
    g = (1.0 + 0.25 * rng.standard_normal(K)).astype(np.float32)
    xbits = [bf16_bits(xb.bf16_rne(Fraction(float(v)))) for v in x]
    gbits = [bf16_bits(xb.bf16_rne(Fraction(float(v)))) for v in g]
    return xbits, gbits


def find(reading):
    """The first seeded row whose factor r differs between the two readings
    (for the product order: any row) and one of whose elements rounds to a
    different bf16 under the two; returns the row, the gains, the element's
    index and its two bf16 values."""
    alt = ALT[reading]
    order = {k: v for k, v in alt.items() if k == "order"}
    for seed in range(5000):
        xbits, gbits = row(1000 * len(reading) + seed)
        x = [from_bf16(b) for b in xbits]
        g = [from_bf16(b) for b in gbits]
        r0 = xb.rms_scale(x, EPS)
        r1 = xb.rms_scale(x, EPS, **{k: v for k, v in alt.items() if k != "order"})
        if r0 == r1 and not order:
            continue
        for i in range(K):
            y0, y1 = xb.rms_out(x[i], r0, g[i]), xb.rms_out(x[i], r1, g[i], **order)
            if y0 != y1:
                return xbits, gbits, i, bf16_bits(y0), bf16_bits(y1)
    raise SystemExit(f"no separating row found for {reading}")


def main():
    lines = ["# RMSNorm reading pins: name | reading | K | eps (binary32 hex) | x (bf16 hex) | gamma (bf16 hex) |",
             "#   i | y[i] under this library's reading | y[i] under the alternative  (bf16 hex; derived by",
             "#   make_rmsnorm_pins.py in exact arithmetic)"]
    for reading in ALT:
        xbits, gbits, i, y0, y1 = find(reading)
        lines.append(" | ".join([f"rms_{reading}", reading, str(K), float(EPS).hex(),
                                 " ".join(f"{b:04x}" for b in xbits), " ".join(f"{b:04x}" for b in gbits),
                                 str(i), f"{y0:04x}", f"{y1:04x}"]))
        print(reading, i, hex(y0), hex(y1), flush=True)
    with open(os.path.join(HERE, "rmsnorm_pins.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
