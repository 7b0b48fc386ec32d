"""Low-precision router keys: summary keys stored as FP8 E4M3 with one fp32
scale per key row, float64 elsewhere.

TEST INFRASTRUCTURE (see the package docstring): imported only by the tests,
the smoke check and the CPU legs of the benchmark.

"Subquadratic Attention with a Hierarchical Tree-Structured Indexer" (ZHA),
Figure 16 caption: the router can run in low precision -- its operands, its
reference-key cache and its scoring -- while the backbone, the KV cache and
the sparse attention stay in BF16.  The issue digest on the same pages notes
FP8 index keys with per-token scales as the deployed form of such an indexer.

Readings (the pages name the formats, not the encoding details):
  * format: FP8 E4M3 as defined by the OCP 8-bit floating point
    specification (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
    no infinities, largest finite value 448, subnormals down to 2^-9);
  * one fp32 scale per key row: scale = max|x| / 448 (0 for an all-zero row),
    code_j = E4M3 of x_j / scale rounded to nearest, ties to even, saturated
    at +-448; the stored key is code_j * scale;
  * the tree keeps only the quantized keys, so a parent key pools its
    children's stored (dequantized) keys and is then quantized itself;
    values stay in float (they are not router operands);
  * the query and the scoring stay in float: score = q . (code * scale).

Pins (tests/test_oracle_pins.py): decoding every one of the 256 codes matches
the format's closed form; rounding maps every representable value to itself,
midpoints to the even neighbour and overflow to 448, and agrees with torch's
float8_e4m3fn conversion inside the finite range; a quantized tree's keys lie
within half a quantum of the float keys pooled from the same quantized
children.
"""

from __future__ import annotations

from typing import List, Tuple

import numpy as np

from .recsa import level_counts, pool_keys

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of one E4M3 code (0..255); NaN for the two NaN codes."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 value (ties to even), saturated to +-448, elementwise."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                      # a = f * 2^e, f in [0.5, 1): leading bit 2^(e-1)
    lead = np.maximum(e - 1, -6)            # normals; below 2^-6 the subnormal quantum
    quantum = np.ldexp(1.0, lead - 3)       # 3 mantissa bits
    r = np.round(a / quantum) * quantum     # exact in float64; np.round ties to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def quantize_row(x: np.ndarray) -> Tuple[np.ndarray, float]:
    """(E4M3 values of x / scale, scale) of one key row."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.max(np.abs(x)))
    if amax == 0.0:
        return np.zeros_like(x), 0.0
    scale = amax / E4M3_MAX
    return e4m3_round(x / scale), scale


def dequantize_row(x: np.ndarray) -> np.ndarray:
    q, scale = quantize_row(x)
    return q * scale


def build_tree_fp8(K: np.ndarray, V: np.ndarray, r: np.ndarray, B: int, b: int
                   ) -> List[Tuple[np.ndarray, np.ndarray]]:
    """Tree whose keys are stored in E4M3 with a scale per row; returns the
    stored (dequantized) keys and the float values, per level, like
    build_tree: [(keys_l [n_l, d], vals_l [n_l, d])]."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    levels: List[Tuple[np.ndarray, np.ndarray]] = []
    for lev, n in enumerate(level_counts(K.shape[0], B, b)):
        fan = B if lev == 0 else b
        src_k = K if lev == 0 else levels[-1][0]
        src_v = V if lev == 0 else levels[-1][1]
        keys = np.empty((n, K.shape[1]))
        vals = np.empty((n, K.shape[1]))
        for j in range(n):
            keys[j] = dequantize_row(pool_keys(src_k[j * fan:(j + 1) * fan], r))
            vals[j] = src_v[j * fan:(j + 1) * fan].mean(axis=0)
        levels.append((keys, vals))
    return levels


def build_tree_fp8_multi(K, V, Rq, B: int, b: int):
    """build_tree_fp8 for each reference query, keys stacked [n_l, R, d]."""
    Rq = np.atleast_2d(np.asarray(Rq, dtype=np.float64))
    per = [build_tree_fp8(K, V, Rq[j], B, b) for j in range(Rq.shape[0])]
    return [(np.stack([per[j][lev][0] for j in range(Rq.shape[0])], axis=1), per[0][lev][1])
            for lev in range(len(per[0]))]


def near_rounding_boundary(x: np.ndarray, tol: float) -> np.ndarray:
    """Elements of x (already divided by the row scale, so the row's largest
    magnitude is 448) within tol of a midpoint between two E4M3 values, where
    a float32 computation of x -- whose error scales with the row's largest
    element, not with the element itself -- may round to the other neighbour."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    frac = a / quantum - np.floor(a / quantum)
    return np.abs(frac - 0.5) * quantum < tol


__all__ = ["E4M3_MAX", "e4m3_decode", "e4m3_round", "quantize_row", "dequantize_row",
           "build_tree_fp8", "build_tree_fp8_multi", "near_rounding_boundary"]
