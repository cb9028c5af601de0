"""Test-side statements of the number formats and storage layouts.

These are written independently of the oracle's vectorised rounding so that the
tests can pin the oracle to the format definitions:

* e2m1 and e4m3 (OCP FP4 E2M1 / FP8 E4M3FN) are enumerated as value tables from their
  bit fields; nearest-even rounding is a search over the table where a tie goes to the
  neighbour with the even code (the code's lowest bit is the mantissa's lowest bit).
* The block-scale storage layout used by the tensor-core GEMM: the scales of a
  128-row x 4-group block (128 rows x 64 elements) are 512 contiguous bytes, the byte of
  (row m, group g) at (m % 32) * 16 + (m // 32) * 4 + g; blocks run along K first, then
  along the rows.
"""
from __future__ import annotations

import numpy as np


def e2m1_table():
    """Non-negative e2m1 values indexed by the 3-bit magnitude code (exponent bias 1)."""
    vals = []
    for code in range(8):
        e, m = code >> 1, code & 1
        vals.append(m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1))
    return np.array(vals)


def e4m3_table():
    """Non-negative finite E4M3FN values indexed by code 0x00..0x7E (bias 7)."""
    vals = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        vals.append(m / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


def brute_round_code(x: float, table) -> int:
    """Code of the nearest table value to |x|, ties to the even code, saturating."""
    a = abs(float(x))
    if a >= table[-1]:
        return len(table) - 1
    best = None
    for i, t in enumerate(table):
        d = abs(a - t)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def brute_e2m1(x: float) -> float:
    t = e2m1_table()
    v = t[brute_round_code(x, t)]
    return -v if (x < 0 and v != 0) else v


def brute_e4m3(x: float) -> float:
    t = e4m3_table()
    v = t[brute_round_code(x, t)]
    return -v if (x < 0 and v != 0) else v


def brute_e2m1_code(x: float) -> int:
    c = brute_round_code(x, e2m1_table())
    return c | (8 if (x < 0 and c != 0) else 0)


def scale_offset(m, g, n_groups):
    """Byte offset of (row m, group g) in the block-scale layout (n_groups = K / 16)."""
    m = np.asarray(m)
    g = np.asarray(g)
    blocks_k = n_groups // 4
    return ((m // 128) * blocks_k + g // 4) * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + g % 4


def scales_to_blocked(sc, rows_padded: int):
    sc = np.asarray(sc, dtype=np.uint8)
    rows, ng = sc.shape
    out = np.zeros(rows_padded * ng, dtype=np.uint8)
    m = np.arange(rows)[:, None]
    g = np.arange(ng)[None, :]
    out[scale_offset(m, g, ng)] = sc
    return out


def blocked_to_scales(buf, rows: int, n_groups: int):
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    m = np.arange(rows)[:, None]
    g = np.arange(n_groups)[None, :]
    return buf[scale_offset(m, g, n_groups)]
