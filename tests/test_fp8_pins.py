"""Pins of the FP8 oracle (``oracle/spark_fp8.py``) against what the format and the
mathematics fix, independent of the oracle's own code (no GPU).

* e4m3 rounding against PyTorch's float8_e4m3fn cast (an independent implementation of the
  OCP format) on every representable value, on every midpoint between neighbours (ties to
  even) and on random values; saturation and the subnormal range by hand.
* bf16 rounding against PyTorch's bfloat16 cast on float32 inputs (exact in float32, so the
  cast rounds once).
* The group exponent at the edges of its rule, and the per-group structure of the scales.
* The forward pass: with inputs on a grid that e4m3 represents exactly under the exponent
  every group gets, the FP8 forward equals the BF16 oracle's (dense limit, sparse ratios with
  blocks of identical keys, context rows); with ordinary inputs it stays within the error the
  format implies.
"""

import math

import numpy as np
import pytest
import torch

from oracle import spark_fp8 as F
from oracle import spark_oracle as O


def e4m3_all_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    v = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return np.unique(v[np.isfinite(v)])


def torch_e4m3(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_representable_values_are_fixed_points():
    v = e4m3_all_values()
    assert v.max() == 448.0 and v.min() == -448.0
    assert np.array_equal(F.e4m3_round(v), v)


def test_e4m3_midpoints_round_to_even():
    v = e4m3_all_values()
    v = v[v >= 0]
    mids = (v[:-1] + v[1:]) / 2
    got = F.e4m3_round(mids)
    assert np.array_equal(got, torch_e4m3(mids))
    assert np.array_equal(F.e4m3_round(-mids), -got)


def test_e4m3_random_values_match_the_format():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(50000) * 30, rng.uniform(-448, 448, 50000),
                        rng.standard_normal(20000) * 1e-2])
    x = x[np.abs(x) <= 448]
    assert np.array_equal(F.e4m3_round(x), torch_e4m3(x))


def test_e4m3_saturation_and_subnormals_by_hand():
    assert F.e4m3_round(np.array([449.0, 464.0, 1e6, -1e6])).tolist() == [448, 448, 448, -448]
    s = 2.0 ** -9                                  # smallest subnormal
    got = F.e4m3_round(np.array([s, s / 2, 3 * s / 2, s / 4, 2.0 ** -6, 7 * s, 7.5 * s]))
    # s/2 ties to 0 (even), 3s/2 ties to 2s (even), 7.5s ties to 8s = 2^-6
    assert got.tolist() == [s, 0.0, 2 * s, 0.0, 2.0 ** -6, 7 * s, 8 * s]


def test_bf16_round_matches_the_format():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(100000) * 10).astype(np.float32).astype(np.float64)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(F.bf16_round(x), ref)


def test_group_exponent_edges():
    cases = {448.0: 0, 448.5: 1, 224.0: -1, 224.5: 0, 1.0: -8, 1.75: -8, 1.76: -7, 0.0: 0,
             1e-40: -126, 3.5: -7, 3e30: 93}
    for amax, e in cases.items():
        assert F.group_exponent(np.array([amax, -amax / 3])) == e, amax
        if amax:
            assert amax <= 448 * 2.0 ** e
            assert e == -126 or amax > 448 * 2.0 ** (e - 1)


def test_quantize_groups_scales_each_group_on_its_own():
    # group 0 has amax 3.5 (e = -7), group 1 has amax 448 (e = 0); 2^-14 survives only under
    # group 0's exponent (it is 2^-7 there, a subnormal code), and 0.3 is off-grid in both
    X = np.array([[3.5, 2.0 ** -14, 0.3], [448.0, 2.0 ** -14, 0.3]])
    q, e = F.quantize_groups(X, [(0, 1), (1, 2)])
    assert e.tolist() == [-7, 0]
    assert q[0, 1] == 2.0 ** -14 and q[1, 1] == 0.0
    assert q[0, 2] == F.e4m3_round(np.array([0.3 * 2 ** 7]))[0] * 2.0 ** -7
    assert q[1, 2] == F.e4m3_round(np.array([0.3]))[0]
    qm, em = F.quantize_groups(X, [(0, 2)])           # one group: the tiny value is lost
    assert em.tolist() == [0] and qm[0, 1] == 0.0


def test_quantize_error_bound():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((300, 64)) * np.exp(rng.uniform(-3, 3, (300, 1)))
    groups = F.fixed_groups(300, 128)
    q, e = F.quantize_groups(X, groups)
    for (lo, hi), eg in zip(groups, e):
        err = np.abs(q[lo:hi] - X[lo:hi])
        # half a quantum: 2^-4 relative for normal codes, 2^-10 * 2^e below them
        assert (err <= 2.0 ** -4 * np.abs(X[lo:hi]) + 2.0 ** (eg - 10) + 1e-300).all()


def grid_inputs(seed, N, d, nq_rows, identical_keys_per_block=None, k_offsets=None):
    """Values from {0, +-0.25, ..., +-3} with 3.5 in every row: every group gets e = -7 and
    every value times 2^7 is an e4m3 value (32 .. 448)."""
    rng = np.random.default_rng(seed)
    grid = np.array([0, 0.25, 0.5, 0.75, 1, 1.5, 2, 3, -0.25, -0.5, -0.75, -1, -1.5, -2, -3])

    def mat(rows):
        m = rng.choice(grid, size=(rows, d))
        m[:, rng.integers(0, d)] = 3.5
        return m

    Q, K, V = mat(nq_rows), mat(N), rng.standard_normal((N, d))
    if identical_keys_per_block is not None:
        for lo, hi in zip(k_offsets[:-1], k_offsets[1:]):
            K[lo:hi] = K[lo]
    return Q, K, V


def offsets(N, size):
    return np.array(list(range(0, N, size)) + [N])


@pytest.mark.parametrize("with_context", [False, True])
def test_grid_inputs_dense_limit_equals_bf16_oracle(with_context):
    N, d = 300, 32
    Q, K, V = grid_inputs(3, N, d, N)
    rng = np.random.default_rng(4)
    qp, kp = rng.permutation(N), rng.permutation(N)
    qo, ko = offsets(N, 64), offsets(N, 50)
    Kc = Vc = None
    if with_context:
        Kc, _, Vc = grid_inputs(5, 70, d, 70)
        Vc = rng.standard_normal((70, d))
    a = F.forward_head_fp8(Q, K, V, qp, kp, qo, ko, 1.0, Kc=Kc, Vc=Vc)
    b = O.forward_head(Q, K, V, qp, kp, qo, ko, 1.0, Kc=Kc, Vc=Vc)
    assert np.abs(a.out - b.out).max() < 1e-12


@pytest.mark.parametrize("ratio", [0.1, 0.4])
def test_grid_inputs_with_identical_block_keys_equal_bf16_oracle(ratio):
    """k~ of a block of identical keys is that key (P2 of the BF16 oracle), so the summary
    rows are on the grid too and the compressed branch is exact in FP8."""
    N, d = 400, 32
    qo, ko = offsets(N, 40), offsets(N, 40)
    Q, K, V = grid_inputs(6, N, d, N, identical_keys_per_block=True, k_offsets=ko)
    rng = np.random.default_rng(7)
    qp = rng.permutation(N)
    kp = np.arange(N)
    a = F.forward_head_fp8(Q, K, V, qp, kp, qo, ko, ratio)
    b = O.forward_head(Q, K, V, qp, kp, qo, ko, ratio)
    assert np.array_equal(a.sel, b.sel)
    assert np.abs(a.out - b.out).max() < 1e-12


def test_off_grid_inputs_stay_within_the_format_error():
    rng = np.random.default_rng(8)
    N, d = 600, 64
    Q, K, V = (rng.standard_normal((N, d)) * 1.5 for _ in range(3))
    qp, kp = rng.permutation(N), rng.permutation(N)
    qo, ko = offsets(N, 100), offsets(N, 75)
    a = F.forward_head_fp8(Q, K, V, qp, kp, qo, ko, 0.25)
    b = O.forward_head(Q, K, V, qp, kp, qo, ko, 0.25)
    rel = np.linalg.norm(a.out - b.out) / np.linalg.norm(b.out)
    # Each factor of a product q_i k_i carries a rounding error of RMS ~2^-4/sqrt(3) = 3.6%,
    # so a logit sigma q.k moves by ~sigma * sqrt(2 d) * 0.036 * E|q_i k_i| ~ 0.11 nats here
    # (logit spread ~2.25 nats).  That perturbs every probability by ~11% at random, and
    # for random values the output, an average of ~n_eff random rows, moves by about the same
    # fraction of its own size: the FP8 product is this coarse on unstructured data.
    assert 1e-3 < rel < 0.15, rel


def test_groups_follow_blocks_and_tiles():
    """Each query block, key block and 128-row context tile gets its own power-of-two scale
    here; the values stay exact in e4m3 only if every group takes its own exponent, so the FP8
    forward equals the BF16 oracle's only if the groups are the ones F3 names."""
    N, d = 360, 32
    rng = np.random.default_rng(9)
    qo, ko = offsets(N, 45), offsets(N, 60)
    Q, K, V = grid_inputs(10, N, d, N)
    # neighbouring groups 2^18 apart: under a shared exponent the smaller one's values
    # (>= 0.25 * its scale) would fall below e4m3's smallest subnormal
    for A in range(len(qo) - 1):
        Q[qo[A]:qo[A + 1]] *= 2.0 ** (-12 if A % 2 else 6)
    for B in range(len(ko) - 1):
        K[ko[B]:ko[B + 1]] *= 2.0 ** (6 if B % 2 else -12)
    Kc, _, _ = grid_inputs(11, 200, d, 200)
    Kc[:128] *= 2.0 ** -12
    Kc[128:] *= 2.0 ** 6
    Vc = rng.standard_normal((200, d))
    qp, kp = np.arange(N), np.arange(N)          # blocks are runs of original rows
    a = F.forward_head_fp8(Q, K, V, qp, kp, qo, ko, 1.0, Kc=Kc, Vc=Vc)
    b = O.forward_head(Q, K, V, qp, kp, qo, ko, 1.0, Kc=Kc, Vc=Vc)
    assert np.abs(a.out - b.out).max() < 1e-12
    # the same inputs with the context quantised as one group lose its small tile
    Kc_one, _ = F.quantize_groups(Kc, [(0, 200)])
    assert np.abs(Kc_one - Kc).max() > 1e-6


def test_summary_tiles_take_their_own_scale():
    """150 key blocks of identical keys: the summary rows of blocks 0..127 and 128..149 form
    two tiles with different scales; exact only with one exponent per 128-row tile."""
    nb, bs, d = 150, 4, 32
    N = nb * bs
    ko = offsets(N, bs)
    Q, K, V = grid_inputs(12, N, d, N, identical_keys_per_block=True, k_offsets=ko)
    K[: 128 * bs] *= 2.0 ** -12
    K[128 * bs:] *= 2.0 ** 7
    rng = np.random.default_rng(13)
    qo = offsets(N, 100)
    qp, kp = rng.permutation(N), np.arange(N)
    a = F.forward_head_fp8(Q, K, V, qp, kp, qo, ko, 0.2)
    b = O.forward_head(Q, K, V, qp, kp, qo, ko, 0.2)
    assert np.array_equal(a.sel, b.sel)
    assert np.abs(a.out - b.out).max() < 1e-12
