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

NVFP4 (the format the caption names) is below, with its own readings.

Pins (tests/test_oracle_pins.py): decoding every one of the 256 E4M3 codes
matches the format's closed form; rounding maps every representable value to
itself, midpoints to the even neighbour and overflow to 448, and agrees with
torch's float8_e4m3fn conversion inside the finite range; a quantized tree's
keys lie within half a quantum of the float keys pooled from the same
quantized children.  E2M1: the 16 codes, fixed points, ties to even,
saturation; an NVFP4 row: every element an E2M1 value times its block's scale,
within half a step of the input, block scales E4M3 values.
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


# ---------------------------------------------------------------------------
# NVFP4: E2M1 elements in blocks of 16 with an E4M3 block scale
# ---------------------------------------------------------------------------
#
# Readings: E2M1 as the OCP microscaling specification defines it (1 sign
# bit, 2 exponent bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1,
# 1.5, 2, 3, 4, 6), nearest with ties to even, saturated at +-6; blocks of 16
# consecutive elements share an E4M3 scale; the second-level fp32 scale that
# NVFP4 keeps per tensor is kept here per key row (a growing cache has no
# fixed tensor): row scale = max|x| / (6 * 448), block scale = E4M3(block
# max / (6 * row scale)), code = E2M1(x / (block scale * row scale)).

E2M1_MAX = 6.0
NVFP4_BLOCK = 16


def e2m1_decode(code: int) -> float:
    """Value of one E2M1 code (0..15)."""
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * 0.5 * m
    return s * (1.0 + 0.5 * m) * 2.0 ** (e - 1)


def e2m1_round(x: np.ndarray) -> np.ndarray:
    """Nearest E2M1 value (ties to even), saturated to +-6, elementwise."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                      # leading bit 2^(e-1)
    lead = np.maximum(e - 1, 0)             # below 1 the subnormal quantum 0.5
    quantum = np.ldexp(1.0, lead - 1)       # 1 mantissa bit
    r = np.minimum(np.round(a / quantum) * quantum, E2M1_MAX)
    return np.copysign(r, x)


def quantize_row_nvfp4(x: np.ndarray) -> np.ndarray:
    """Stored (decoded) value of one key row under the NVFP4 readings above."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.max(np.abs(x)))
    out = np.zeros_like(x)
    if amax == 0.0:
        return out
    g = amax / (E2M1_MAX * E4M3_MAX)
    for b0 in range(0, x.shape[0], NVFP4_BLOCK):
        blk = x[b0:b0 + NVFP4_BLOCK]
        sb = float(e4m3_round(np.max(np.abs(blk)) / (E2M1_MAX * g)))
        if sb == 0.0:
            continue
        out[b0:b0 + NVFP4_BLOCK] = e2m1_round(blk / (sb * g)) * (sb * g)
    return out


def build_tree_nvfp4_multi(K, V, Rq, B: int, b: int):
    """Tree with NVFP4 key rows for each reference query, keys [n_l, R, d];
    a parent pools its children's stored keys (as with FP8)."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    Rq = np.atleast_2d(np.asarray(Rq, dtype=np.float64))
    per = []
    for j in range(Rq.shape[0]):
        levels = []
        for lev, n in enumerate(level_counts(K.shape[0], B, b)):
            fan = B if lev == 0 else b
            src_k = K if lev == 0 else levels[-1][0]
            src_v = V if lev == 0 else levels[-1][1]
            keys = np.empty((n, K.shape[1]))
            vals = np.empty((n, K.shape[1]))
            for i in range(n):
                keys[i] = quantize_row_nvfp4(pool_keys(src_k[i * fan:(i + 1) * fan], Rq[j]))
                vals[i] = src_v[i * fan:(i + 1) * fan].mean(axis=0)
            levels.append((keys, vals))
        per.append(levels)
    return [(np.stack([per[j][lev][0] for j in range(Rq.shape[0])], axis=1), per[0][lev][1])
            for lev in range(len(per[0]))]


__all__ = ["E4M3_MAX", "e4m3_decode", "e4m3_round", "quantize_row", "dequantize_row",
           "build_tree_fp8", "build_tree_fp8_multi", "near_rounding_boundary",
           "E2M1_MAX", "NVFP4_BLOCK", "e2m1_decode", "e2m1_round", "quantize_row_nvfp4",
           "build_tree_nvfp4_multi"]
