"""Independent reference constructions used to pin the oracle.

Nothing here imports the oracle.  The E4M3FN grid is built from a different
description of the format than the oracle's encoder uses: the set of finite
magnitudes {0} + {j * 2^-9, j = 1..7} + {(1 + f/8) * 2^p, p = -6..8, f = 0..7},
capped at 448, listed in increasing order.  E4M3FN codes 0x00..0x7E are
monotone in magnitude, so a magnitude's code is its index in that list.
Rounding is brute force: the nearest grid point, ties to the even code.
"""
from __future__ import annotations

import numpy as np
import torch


def e4m3_grid() -> np.ndarray:
    mags = [0.0] + [j / 512.0 for j in range(1, 8)]
    for p in range(-6, 9):
        for f in range(8):
            v = (1.0 + f / 8.0) * 2.0 ** p
            if v <= 448.0:
                mags.append(v)
    g = np.array(sorted(mags), dtype=np.float64)
    assert g.size == 127
    return g


GRID = e4m3_grid()


def bruteforce_e4m3(values) -> np.ndarray:
    """Nearest E4M3FN code (ties to even code), saturating at +-448, sign kept."""
    v = np.asarray(values, dtype=np.float64).reshape(-1)
    neg = np.signbit(v)
    a = np.minimum(np.abs(v), 448.0)
    hi = np.searchsorted(GRID, a, side="left")          # GRID[hi] >= a
    hi = np.clip(hi, 0, GRID.size - 1)
    lo = np.clip(hi - 1, 0, GRID.size - 1)
    dlo = a - GRID[lo]
    dhi = GRID[hi] - a
    code = np.where(dlo < dhi, lo, hi)
    tie = dlo == dhi
    code = np.where(tie, np.where(lo % 2 == 0, lo, hi), code)
    code = np.where(a == GRID[hi], hi, code)
    out = code.astype(np.uint8) | np.where(neg, 0x80, 0).astype(np.uint8)
    return out.reshape(np.shape(values))


def e4m3_spacing(mag) -> np.ndarray:
    """Distance between adjacent E4M3 values around magnitude mag (<= 448)."""
    a = np.asarray(mag, dtype=np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 2.0 ** (e - 3)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its uint16 bit patterns as a numpy array."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def load_hand_rows(path):
    rows = []
    with open(path, encoding="utf-8") as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, xs, codes = [p.strip() for p in line.split("|")]
            kind, qmax = head.split()
            x = [float(v) for v in xs.split()]
            if kind == "fp8":
                c = [int(v, 16) for v in codes.split()]
            else:
                c = [int(v) for v in codes.split()]
            rows.append((kind, float(qmax), x, c))
    return rows
