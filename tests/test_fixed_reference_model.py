"""A float32 model of the attention kernel's softmax scheme, checked against float64 softmax on
the CPU (no GPU).

The kernel does not keep an online maximum. Its scheme is:
- exponentiate every tile against a fixed reference per row, the larger of the first two
  tiles' row maxima;
- round P to bf16, sum p in fp32 and accumulate P V in fp32;
- a row whose sum leaves [2^-60, 2^60] repeats the pass with a maximum recorded only from
  64-column chunks whose own sum left [2^-40, 2^40].

This file models that arithmetic (not the kernel's code) and pins the argument the design rests
on:
- in-window rows lose nothing to the missing rescale;
- a row out of window is always detected;
- the recorded maximum is close enough for the second pass, whatever the logits.
"""

import numpy as np
import pytest
import torch

CHUNK = 64
TILE = 128


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(
        torch.float32).numpy()


def one_pass(tiles, values, m_ref):
    """tiles: list of [rows, 128] logits in log2 units (-inf = masked); values: [128, d]."""
    rows = tiles[0].shape[0]
    d = values[0].shape[1]
    l = np.zeros(rows, dtype=np.float32)
    O = np.zeros((rows, d), dtype=np.float32)
    m_seen = np.full(rows, -np.inf, dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        for x, v in zip(tiles, values):
            x = x.astype(np.float32)
            p = np.exp2(x - m_ref[:, None]).astype(np.float32)      # ex2: inf on overflow
            for c0 in range(0, TILE, CHUNK):
                cs = p[:, c0:c0 + CHUNK].sum(axis=1, dtype=np.float32)
                bad = ~((cs >= 2.0 ** -40) & (cs <= 2.0 ** 40))
                m_seen = np.where(bad, np.maximum(m_seen, x[:, c0:c0 + CHUNK].max(axis=1)),
                                  m_seen)
            l += p.sum(axis=1, dtype=np.float32)
            O += bf16(p) @ v.astype(np.float32)
    return O, l, m_seen


def fixed_reference_attention(tiles, values):
    m_ref = np.maximum(tiles[0].max(axis=1), tiles[1].max(axis=1) if len(tiles) > 1
                       else -np.inf).astype(np.float32)
    m_ref = np.where(np.isfinite(m_ref), m_ref, 0.0).astype(np.float32)
    O, l, m_seen = one_pass(tiles, values, m_ref)
    out_of_window = ~((l >= 2.0 ** -60) & (l <= 2.0 ** 60))
    reran = bool(out_of_window.any())
    if reran:                                       # the whole CTA repeats with m_seen
        m2 = np.where(out_of_window, m_seen, m_ref).astype(np.float32)
        m2 = np.where(np.isfinite(m2), m2, 0.0).astype(np.float32)
        O, l, _ = one_pass(tiles, values, m2)
    return O / l[:, None], reran


def softmax64(tiles, values):
    X = np.concatenate(tiles, axis=1).astype(np.float64) * np.log(2.0)
    V = np.concatenate(values, axis=0).astype(np.float64)
    X = X - X.max(axis=1, keepdims=True)
    P = np.exp(X)
    return (P / P.sum(axis=1, keepdims=True)) @ V


def make(rng, n_tiles, rows=32, d=16, spread=6.0):
    tiles = [rng.standard_normal((rows, TILE)) * spread for _ in range(n_tiles)]
    values = [rng.standard_normal((TILE, d)) for _ in range(n_tiles)]
    return tiles, values


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_ordinary_logits_need_no_second_pass():
    rng = np.random.default_rng(0)
    tiles, values = make(rng, 40)
    out, reran = fixed_reference_attention(tiles, values)
    assert not reran
    assert rel(out, softmax64(tiles, values)) < 1e-2


@pytest.mark.parametrize("lift", [70.0, 150.0, 400.0])
def test_a_late_key_far_above_the_reference_forces_the_second_pass(lift):
    rng = np.random.default_rng(1)
    tiles, values = make(rng, 30)
    tiles[25][:, 17] += lift                        # log2 units above everything else
    out, reran = fixed_reference_attention(tiles, values)
    assert reran
    assert rel(out, softmax64(tiles, values)) < 1e-2


def test_masked_first_tiles_and_very_negative_logits():
    """The first two tiles fully masked (reference 0) and every logit near -300: the sums
    underflow, the chunks record their maxima, and the second pass recovers the softmax."""
    rng = np.random.default_rng(2)
    tiles, values = make(rng, 12)
    tiles[0][:] = -np.inf
    tiles[1][:] = -np.inf
    for t in tiles[2:]:
        t -= 300.0
    out, reran = fixed_reference_attention(tiles, values)
    assert reran
    assert rel(out, softmax64(tiles, values)) < 1e-2


def test_many_moderate_chunks_cannot_leave_the_window_unrecorded():
    """Each chunk's sum up to 2^40 with fewer than 2^16 chunks keeps the row sum below 2^56,
    inside the window: rows with every chunk in range never need the recorded maximum."""
    n_chunks = 2 ** 15
    assert n_chunks * 2.0 ** 40 < 2.0 ** 60
    rng = np.random.default_rng(3)
    tiles, values = make(rng, 20, spread=2.0)
    for t in tiles:
        t += 30.0                               # every p near 2^30 against a reference at 30
    tiles[0] -= 30.0
    tiles[1] -= 30.0                            # reference from the first tiles: ~0
    out, reran = fixed_reference_attention(tiles, values)
    # p ~ 2^30 per column, 2^36 per chunk: in range, no chunk records; the row sum ~2^41 is
    # in the window, so no repeat either, and the result is still exact up to rounding
    assert not reran
    assert rel(out, softmax64(tiles, values)) < 1e-2
