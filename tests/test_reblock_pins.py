"""Pins of the Spark-Reblock oracle against facts fixed by the pages and by mathematics (CPU).

Each pin checks the oracle against something other than itself: another library routine for
the matrix square root (scipy's Schur-based sqrtm), closed forms (the Mahalanobis cosine, the
power-iteration iterate as a matrix power, a diagonal second moment), exhaustive checks of the
block tree, recovery of planted clusters, invariances the distance has by construction, and
the direction of the blog's ablation (reblocking raises attention-mass recall).  Planted
mistakes at the end must each be caught by at least one pin.
"""

import math

import numpy as np
import pytest
import scipy.linalg

from oracle import spark_oracle as SO
from oracle import spark_reblock as R

TOL = 1e-9


def _rng(seed):
    return np.random.default_rng(seed)


def _anisotropic(seed, n, d, scales):
    rng = _rng(seed)
    A = rng.standard_normal((d, d))
    Qo, _ = np.linalg.qr(A)
    return (rng.standard_normal((n, d)) * np.asarray(scales)) @ Qo.T


# ----------------------------------------------------------------------------------- pins

def pin_sqrt_vs_scipy():
    """B1: psd_sqrt agrees with scipy's sqrtm (a Schur method) and squares back to M, also
    for a rank-deficient M."""
    err = 0.0
    for seed, rank in ((1, 6), (2, 3)):
        X = _rng(seed).standard_normal((50, rank)) @ _rng(seed + 9).standard_normal((rank, 6))
        M = R.second_moment(X)
        W = R.psd_sqrt(M)
        err = max(err, float(np.abs(W @ W - M).max()), float(np.abs(W - W.T).max()))
        if rank == 6:
            err = max(err, float(np.abs(W - np.real(scipy.linalg.sqrtm(M))).max()))
    return err


def pin_second_moment_closed_form():
    """B1: rows a*e1 and b*e2 (each half the rows) give M = diag(a^2/2, b^2/2, 0)."""
    X = np.zeros((8, 3))
    X[:4, 0] = 3.0
    X[4:, 1] = -2.0
    return float(np.abs(R.second_moment(X) - np.diag([4.5, 2.0, 0.0])).max())


def pin_mahalanobis_cosine():
    """B2: 1 - x_i.x_j equals the blog's d_Q = 1 - q_i^T M q_j / sqrt(q_i^T M q_i q_j^T M q_j)."""
    rng = _rng(3)
    K = _anisotropic(4, 200, 5, [3, 1, 0.5, 0.2, 0.05])
    Q = rng.standard_normal((30, 5))
    M = R.second_moment(K)
    X = R.whiten_normalize(Q, R.psd_sqrt(M))
    G = Q @ M @ Q.T
    nrm = np.sqrt(np.diag(G))
    ref = 1.0 - G / np.outer(nrm, nrm)
    return float(np.abs((1.0 - X @ X.T) - ref).max())


def pin_tree_levels():
    """B3: for every block count 1..70 the tree's leaves are exactly the single blocks, each
    node gives ceil(m/2) blocks to its left child, and the depth is ceil(log2 nb)."""
    for nb in range(1, 71):
        levels = R.tree_levels(nb)
        if len(levels) != (math.ceil(math.log2(nb)) if nb > 1 else 0):
            return float("inf")
        covered = {(0, nb)}
        for nodes in levels:
            for lo, mid, hi in nodes:
                if (lo, hi) not in covered or mid - lo != (hi - lo + 1) // 2:
                    return float("inf")
                covered |= {(lo, mid), (mid, hi)}
        leaves = sorted((lo, hi) for lo, hi in covered if hi - lo == 1)
        if leaves != [(b, b + 1) for b in range(nb)]:
            return float("inf")
    return 0.0


def pin_power_iteration_closed_form():
    """B4: v = C^T v0 / |C^T v0| (matrix power of the node covariance); with many iterations
    on a clear eigen-gap it is the top eigenvector from eigh (up to sign)."""
    X = _anisotropic(5, 300, 6, [4, 1, 0.8, 0.5, 0.3, 0.1])
    mu, v = R.principal_direction(X, R.POWER_ITERS)
    C = np.cov(X.T, bias=True)
    w = np.linalg.matrix_power(C, R.POWER_ITERS) @ np.full(6, 1 / math.sqrt(6))
    err = float(np.abs(v - w / np.linalg.norm(w)).max())
    err = max(err, float(np.abs(mu - X.mean(0)).max()))
    _, v60 = R.principal_direction(X, 60)
    lam, U = np.linalg.eigh(C)
    err = max(err, 1.0 - abs(float(U[:, -1] @ v60)))
    return err


def pin_split_order_and_ties():
    """B4: the left child holds the `cap` largest projections, ties go to the earlier token,
    both children keep their relative order; on exactly duplicated rows the split falls by
    position."""
    rng = _rng(6)
    X = rng.standard_normal((40, 4))
    X[10] = X[3]
    X[25] = X[3]                                    # three identical rows -> equal projections
    left, right, p = R.split_node(X, 17)
    ok = len(left) == 17 and len(right) == 23 and sorted(np.r_[left, right]) == list(range(40))
    ok &= bool(np.all(np.diff(left) > 0)) and bool(np.all(np.diff(right) > 0))
    ok &= float(p[left].min()) >= float(p[right].max())
    for i in left:                                  # any equal projection on the right comes later
        ok &= all(not (p[j] == p[i] and j < i) for j in right)
    D = np.ones((9, 4))
    l2, r2, _ = R.split_node(D, 4)
    ok &= list(l2) == [0, 1, 2, 3] and list(r2) == [4, 5, 6, 7, 8]
    return 0.0 if ok else float("inf")


def _planted_clusters(seed, n_clusters, b, d, spread=1e-3):
    rng = _rng(seed)
    centers = rng.standard_normal((n_clusters, d)) * 2.0
    lab = np.repeat(np.arange(n_clusters), b)
    order = rng.permutation(len(lab))
    lab = lab[order]
    Q = centers[lab] + spread * rng.standard_normal((len(lab), d))
    K = rng.standard_normal((5 * len(lab), d)) * np.linspace(2.0, 0.5, d)
    return Q, K, lab


def pin_planted_clusters_recovered():
    """Blog "Spark-Reblock": tokens with similar attention preferences share blocks.  Tight
    planted clusters of exactly one block each end up one cluster per leaf, for a power-of-two
    and a ragged block count."""
    for seed, ncl, b in ((7, 8, 16), (8, 5, 12)):
        Q, K, lab = _planted_clusters(seed, ncl, b, 10)
        qp, kp, offs = R.reblock_head(Q, K, b)
        if not np.array_equal(qp, kp) or sorted(qp) != list(range(len(lab))):
            return float("inf")
        for B in range(len(offs) - 1):
            if len(set(lab[qp[offs[B]:offs[B + 1]]])) != 1:
                return float("inf")
    return 0.0


def pin_whitening_side():
    """B1/B2: queries are whitened by the KEYS' second moment.  Keys spread along e1 only, so
    d_Q ignores the large e3 offsets of the queries and the first split separates +e1 from
    -e1 queries; whitening by M_Q, or not at all, would split on e3 instead."""
    rng = _rng(9)
    b = 8
    groups = [(1, 3), (1, -3), (-1, 3), (-1, -3)]
    Q = np.concatenate([np.tile([s1, 0.0, s3, 0.0], (b, 1)) for s1, s3 in groups])
    Q += 1e-3 * rng.standard_normal(Q.shape)
    K = np.zeros((400, 4))
    K[:, 0] = rng.standard_normal(400) * 2.0
    K[:, 1] = rng.standard_normal(400) * 1.0
    K[:, 2] = rng.standard_normal(400) * 1e-3
    K[:, 3] = rng.standard_normal(400) * 1.0
    qp, _, offs = R.reblock_head(Q, K, 2 * b)
    first_half = set((qp[: 2 * b] // b).tolist())
    return 0.0 if first_half in ({0, 1}, {2, 3}) else float("inf")


def pin_invariances():
    """B2: positive rescaling of single queries and a global rescaling of the keys leave
    the partition unchanged; so does relabelling the tokens (as sets per block)."""
    rng = _rng(10)
    w = SO  # noqa: F841  (keeps both oracle modules in one test run)
    Q, K, _ = _planted_clusters(11, 4, 20, 6, spread=0.3)
    qp, _, offs = R.reblock_head(Q, K, 20)
    sets = [frozenset(qp[offs[B]:offs[B + 1]].tolist()) for B in range(len(offs) - 1)]
    s = rng.uniform(0.2, 5.0, size=(len(Q), 1))
    qp2, _, _ = R.reblock_head(Q * s, K * 3.7, 20)
    sets2 = [frozenset(qp2[offs[B]:offs[B + 1]].tolist()) for B in range(len(offs) - 1)]
    relabel = rng.permutation(len(Q))
    qp3, _, _ = R.reblock_head(Q[relabel], K, 20)
    sets3 = [frozenset(relabel[qp3[offs[B]:offs[B + 1]]].tolist()) for B in range(len(offs) - 1)]
    return 0.0 if sets == sets2 and sorted(map(sorted, sets)) == sorted(map(sorted, sets3)) else float("inf")


def pin_separate_mode_swaps_roles():
    """B5: in the separate layout the key partition is the query partition with Q and K
    swapped."""
    Q, K, _ = _planted_clusters(12, 4, 10, 5, spread=0.2)
    K = K[: len(Q)]
    _, kp, _ = R.reblock_head(Q, K, 10, mode="separate")
    qp_sw, _, _ = R.reblock_head(K, Q, 10)
    return 0.0 if np.array_equal(kp, qp_sw) else float("inf")


PINS = [pin_sqrt_vs_scipy, pin_second_moment_closed_form, pin_mahalanobis_cosine,
        pin_tree_levels, pin_power_iteration_closed_form, pin_split_order_and_ties,
        pin_planted_clusters_recovered, pin_whitening_side, pin_invariances,
        pin_separate_mode_swaps_roles]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    assert pin() < TOL


def test_reblock_raises_attention_mass_recall():
    """Blog "Spark-Reblock" table: at a 10% Top-K budget, the reblocked partition has a higher
    attention-mass recall than fixed contiguous blocks (direction only).  Mixture tokens in
    random order stand in for video tokens without a useful spatial order."""
    rng = _rng(13)
    H, N, d, ncomp, b = 1, 1024, 32, 16, 32
    mu = rng.standard_normal((ncomp, d))
    comp = rng.integers(0, ncomp, size=N)
    Q = mu[comp] + 0.6 * rng.standard_normal((N, d))
    K = mu[comp] + 0.6 * rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    ident = np.arange(N)
    offs = R.fixed_block_offsets(N, b)
    qp, kp, _ = R.reblock_head(Q, K, b)
    rec = {}
    for name, pq, pk in (("fixed", ident, ident), ("reblock", qp, kp)):
        r = SO.forward_head(Q, K, V, pq, pk, offs, offs, 0.1, blocks=[])
        Qp, Kp = Q[pq], K[pk]
        rec[name] = np.mean([SO.attention_mass_recall(Qp[offs[A]:offs[A + 1]], Kp, offs, r.sel[A])
                             for A in range(len(offs) - 1)])
    assert rec["reblock"] > rec["fixed"] + 0.05, rec


# ------------------------------------------------------------------- planted mistakes

def _mut_sqrt_is_identity(orig):
    return "psd_sqrt", lambda M: M


def _mut_no_normalisation(orig):
    return "whiten_normalize", lambda X, W: np.asarray(X, dtype=np.float64) @ np.asarray(W).T


def _mut_uncentred(orig):
    def f(Xs, iters=R.POWER_ITERS):
        Xs = np.asarray(Xs, dtype=np.float64)
        n, d = Xs.shape
        v = np.full(d, 1.0 / math.sqrt(d))
        for _ in range(iters):
            w = Xs.T @ (Xs @ v) / n
            v = w / np.linalg.norm(w)
        return Xs.mean(0), v
    return "principal_direction", f


def _mut_smallest_left(orig):
    def f(Xs, cap, iters=R.POWER_ITERS):
        left, right, p = orig(-np.asarray(Xs), cap, iters)
        return left, right, -p
    return "split_node", f


def _mut_floor_left(orig):
    def f(nb):
        levels, frontier = [], [(0, nb)]
        while frontier:
            nodes, nxt = [], []
            for lo, hi in frontier:
                if hi - lo >= 2:
                    mid = lo + (hi - lo) // 2
                    nodes.append((lo, mid, hi))
                    nxt += [(lo, mid), (mid, hi)]
            if nodes:
                levels.append(nodes)
            frontier = nxt
        return levels
    return "tree_levels", f


def _mut_moment_of_queries(orig):
    def f(Q, K, block, mode="q_reuse_k", iters=R.POWER_ITERS):
        return orig(Q, Q, block, mode, iters)
    return "reblock_head", f


def _mut_unstable_children(orig):
    def f(Xs, cap, iters=R.POWER_ITERS):
        mu, v = R.principal_direction(Xs, iters)
        p = (np.asarray(Xs, dtype=np.float64) - mu) @ v
        order = np.lexsort((np.arange(len(p)), -p))
        return order[:cap], order[cap:], p          # children in projection order
    return "split_node", f


MUTATIONS = [_mut_sqrt_is_identity, _mut_no_normalisation, _mut_uncentred, _mut_smallest_left,
             _mut_floor_left, _mut_moment_of_queries, _mut_unstable_children]


@pytest.mark.parametrize("mutation", MUTATIONS, ids=lambda f: f.__name__)
def test_pins_catch_planted_mistake(mutation, monkeypatch):
    name = mutation(lambda *a, **k: None)[0]
    _, bad = mutation(getattr(R, name))
    monkeypatch.setattr(R, name, bad)
    caught = []
    for pin in PINS:
        try:
            e = pin()
        except Exception:
            e = float("inf")
        if not e < TOL:
            caught.append(pin.__name__)
    assert caught, f"no pin caught {mutation.__name__}"
