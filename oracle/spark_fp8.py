"""Double-precision CPU oracle of the FP8 (e4m3) variant of the two-branch attention.

TEST INFRASTRUCTURE, like ``spark_oracle``: only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; it shares no code with
``block_sparse_attention_gather_b200`` and never imports it.  Everything is float64 numpy.

Source: the Spark-H3 blog, section "Benchmark Results", reports Spark-H3's attention latency
with FP8 as well as with BF16, without describing the FP8 scheme.  Readings taken here (each
is also listed in the design notes):

F1  Only the logits' product is taken in FP8: the queries Qp, the exact keys Kp, the summary
    keys k~ and the context keys Kc are quantised to e4m3 right before the attention; the
    routing, the anchor, the summaries themselves (k~, v~, c) and the value side (Vp, v~, Vc,
    the probabilities) stay as in the BF16 path.
F2  e4m3 is the OCP "E4M3FN" format: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
    no infinities, largest finite value 448, subnormals down to 2^-9.  Values are rounded to
    nearest, ties to even, and saturated to +-448.
F3  Scales are powers of two, one per group of rows: each query block, each key block, each
    128-row tile of the summary rows and each 128-row tile of the context rows.  A group's
    exponent e is the smallest integer with amax <= 448 * 2^e (amax = the group's largest
    |value|; e = 0 for an all-zero group), so x * 2^-e is exact and its e4m3 code decides
    the value code * 2^e.
F4  The summary keys are quantised from their bf16 values (the precision in which the path
    stores them), so that both sides take each code from the same number.
"""

from __future__ import annotations

import math

import numpy as np

from oracle import spark_oracle as O

__all__ = [
    "E4M3_MAX",
    "TILE_ROWS",
    "bf16_round",
    "e4m3_round",
    "group_exponent",
    "quantize_groups",
    "fixed_groups",
    "offset_groups",
    "forward_head_fp8",
]

E4M3_MAX = 448.0
TILE_ROWS = 128


def _round_to_bits(x: np.ndarray, mant_bits: int, min_exp: int) -> np.ndarray:
    """x rounded to nearest, ties to even, on the grid of a binary format with `mant_bits`
    stored mantissa bits and smallest normal exponent `min_exp` (subnormals below it), with
    unbounded range.  The quantum of a value with exponent E is 2^(max(E, min_exp) -
    mant_bits); dividing by a power of two is exact in float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    safe = np.where(a > 0, a, 1.0)
    E = np.floor(np.log2(safe))
    E = np.where(2.0 ** E > safe, E - 1, E)          # guard log2 rounding at powers of two
    E = np.where(2.0 ** (E + 1) <= safe, E + 1, E)
    q = 2.0 ** (np.maximum(E, min_exp) - mant_bits)
    m = a / q
    r = np.floor(m)
    frac = m - r
    r = r + ((frac > 0.5) | ((frac == 0.5) & (np.mod(r, 2) == 1)))
    return np.where(a > 0, np.copysign(r * q, x), 0.0 * x)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """F4: the nearest bf16 value (7 stored mantissa bits, smallest normal 2^-126), ties to
    even."""
    return _round_to_bits(x, 7, -126)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """F2: the nearest e4m3 value (3 stored mantissa bits, smallest normal 2^-6), ties to
    even, saturated to +-448."""
    r = _round_to_bits(x, 3, -6)
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def group_exponent(X: np.ndarray) -> int:
    """F3: the smallest integer e with max|X| <= 448 * 2^e, at least -126 (so 2^e is a normal
    float32); 0 for an all-zero group."""
    amax = float(np.max(np.abs(X))) if np.size(X) else 0.0
    if amax == 0.0:
        return 0
    e = math.ceil(math.log2(amax / E4M3_MAX))
    while amax > E4M3_MAX * 2.0 ** e:
        e += 1
    while amax <= E4M3_MAX * 2.0 ** (e - 1):
        e -= 1
    return max(e, -126)


def fixed_groups(rows: int, size: int = TILE_ROWS):
    """Row ranges [g*size, min((g+1)*size, rows)) covering `rows` rows."""
    return [(g, min(g + size, rows)) for g in range(0, rows, size)]


def offset_groups(offsets):
    """Row ranges of the blocks given by offsets."""
    offsets = np.asarray(offsets, dtype=np.int64)
    return [(int(offsets[i]), int(offsets[i + 1])) for i in range(len(offsets) - 1)]


def quantize_groups(X: np.ndarray, groups):
    """F2, F3: (dequantised values, exponents) of the rows of X, one power-of-two scale per
    group of rows.  Dequantised = e4m3(X * 2^-e) * 2^e."""
    X = np.asarray(X, dtype=np.float64)
    out = np.zeros_like(X)
    exps = []
    for lo, hi in groups:
        e = group_exponent(X[lo:hi])
        out[lo:hi] = e4m3_round(X[lo:hi] * 2.0 ** (-e)) * 2.0 ** e
        exps.append(e)
    return out, np.array(exps, dtype=np.int64)


def forward_head_fp8(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, ratio, *, sel=None,
                     blocks=None, Kc=None, Vc=None) -> O.HeadResult:
    """One head of the FP8 variant (F1-F4): the BF16 path's steps (``spark_oracle``) for the
    layout, anchor, summaries and routing, then the attention with the logits taken from the
    dequantised e4m3 queries and keys."""
    Q = np.asarray(Q, dtype=np.float64)
    base = O.forward_head(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, ratio, sel=sel,
                          blocks=[], Kc=Kc, Vc=Vc)
    N, d = Q.shape
    scale = 1.0 / math.sqrt(d)
    q_perm = np.asarray(q_perm, dtype=np.int64)
    k_perm = np.asarray(k_perm, dtype=np.int64)
    q_offsets = np.asarray(q_offsets, dtype=np.int64)
    k_offsets = np.asarray(k_offsets, dtype=np.int64)
    Qp = O.gather_rows(Q, q_perm)
    Kp = O.gather_rows(np.asarray(K, dtype=np.float64), k_perm)
    Vp = O.gather_rows(np.asarray(V, dtype=np.float64), k_perm)
    Qq, _ = quantize_groups(Qp, offset_groups(q_offsets))
    Kq, _ = quantize_groups(Kp, offset_groups(k_offsets))
    ktq, _ = quantize_groups(bf16_round(base.k_tilde), fixed_groups(len(base.k_tilde)))
    Kcq = None
    if Kc is not None:
        Kc = np.asarray(Kc, dtype=np.float64).reshape(-1, d)
        Kcq, _ = quantize_groups(Kc, fixed_groups(len(Kc)))
    sel_use = base.sel if sel is None else np.asarray(sel, dtype=np.int64)
    out = np.full((N, d), np.nan)
    todo = range(len(q_offsets) - 1) if blocks is None else blocks
    for A in todo:
        lo, hi = q_offsets[A], q_offsets[A + 1]
        o = O.attend_block(Qq[lo:hi], Kq, Vp, k_offsets, sel_use[A], ktq, base.v_tilde,
                           base.c, scale, Kc=Kcq, Vc=Vc)
        out[q_perm[lo:hi]] = o
    return O.HeadResult(out, base.qbar, base.qbar_blocks, base.kbar, base.k_tilde,
                        base.v_tilde, base.c, sel_use, base.scores)
