"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle on the same
seeded inputs, and compare with the tolerances of the method's parity contract.

Tolerances (bf16 tensor-core operands, fp32 accumulation):
  * out: relative L2 error <= 1e-2 and max abs error <= 2e-2 against the float64 oracle;
  * sel: identical, except where the oracle's scores of the differing blocks lie within
    1e-5 * max|S| of the k-th largest score (then both selections are correct; the oracle
    is re-run with the GPU's selection before the outputs are compared);
  * reblocked Q/K/V: bit-exact (pure data movement of bf16 values);
  * fp32 block means / anchor: relative 1e-5 of the row norm;
  * bf16 summaries k~, v~: within 2 bf16 ulps of the oracle value (+1e-3 absolute);
  * summary offsets c_B: 1e-2 absolute (the GPU's c_B is taken against its bf16 k~).
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import spark_oracle as O

OUT_REL_L2 = 1e-2
OUT_MAX_ABS = 2e-2
NEAR_TIE_REL = 1e-5


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_64(t: torch.Tensor) -> np.ndarray:
    """The bf16 value the kernels compute on (fp32 inputs are rounded to nearest-even bf16
    on entry), as float64."""
    return t.detach().to(torch.bfloat16).to("cpu", torch.float64).numpy()


def head_inputs(x: dict, h: int) -> dict:
    """CPU float64 copies of one head's inputs (and context rows, if any), rounded to bf16 as
    the library does."""
    hi = dict(Q=bf16_64(x["Q"][h]), K=bf16_64(x["K"][h]), V=bf16_64(x["V"][h]),
              q_perm=x["q_perm"][h].cpu().numpy().astype(np.int64),
              k_perm=x["k_perm"][h].cpu().numpy().astype(np.int64),
              q_offsets=x["q_offsets"].cpu().numpy().astype(np.int64),
              k_offsets=x["k_offsets"].cpu().numpy().astype(np.int64),
              Kc=None, Vc=None)
    if x.get("Kc") is not None:
        hi["Kc"], hi["Vc"] = bf16_64(x["Kc"][h]), bf16_64(x["Vc"][h])
    return hi


def oracle_head(x: dict, h: int, ratio: float, blocks=None, sel=None, hi=None):
    hi = head_inputs(x, h) if hi is None else hi
    return O.forward_head(hi["Q"], hi["K"], hi["V"], hi["q_perm"], hi["k_perm"],
                          hi["q_offsets"], hi["k_offsets"], ratio, blocks=blocks, sel=sel,
                          Kc=hi["Kc"], Vc=hi["Vc"])


def compare_sel(gpu_sel: np.ndarray, ref_sel: np.ndarray, scores: np.ndarray, k: int):
    """Checks the GPU selection row by row; returns the number of rows that differ (all of
    them near-ties).  Raises AssertionError on any difference outside the near-tie rule or
    on an invalid selection (not ascending, duplicates, out of range)."""
    nqb, nkb = scores.shape
    assert gpu_sel.shape == (nqb, k)
    assert (gpu_sel >= 0).all() and (gpu_sel < nkb).all(), "selected id out of range"
    assert (np.diff(gpu_sel, axis=1) > 0).all(), "selection not strictly ascending"
    diff_rows = 0
    for A in range(nqb):
        if np.array_equal(gpu_sel[A], ref_sel[A]):
            continue
        diff_rows += 1
        S = scores[A]
        tol = NEAR_TIE_REL * float(np.abs(S).max())
        kth = float(np.sort(S)[::-1][k - 1])
        g, r = set(gpu_sel[A].tolist()), set(ref_sel[A].tolist())
        for B in g ^ r:
            assert abs(float(S[B]) - kth) <= tol, (
                f"row {A}: block {B} differs with score {S[B]} vs k-th {kth} (tol {tol})")
        # the GPU's set must be a valid top-k under the slack
        sel_min = min(float(S[B]) for B in g)
        rest = [float(S[B]) for B in range(nkb) if B not in g]
        if rest:
            assert max(rest) <= sel_min + 2 * tol
    return diff_rows


def compare_out(got: np.ndarray, ref: np.ndarray, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.abs(got - ref).max()) if got.size else 0.0
    assert rel <= OUT_REL_L2, f"{what}: rel-L2 {rel:.3e} > {OUT_REL_L2}"
    assert mx <= OUT_MAX_ABS, f"{what}: max-abs {mx:.3e} > {OUT_MAX_ABS}"
    return rel, mx


def rows_of_blocks(q_perm: np.ndarray, q_offsets: np.ndarray, blocks) -> np.ndarray:
    """Original-order token ids of the given query blocks."""
    return np.concatenate([q_perm[q_offsets[A]:q_offsets[A + 1]] for A in blocks])
