"""Double-precision CPU oracle of the Spark-Reblock token partitioner.

TEST INFRASTRUCTURE. Like ``spark_oracle``, this module is the independent checker of the
CUDA path: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it, it shares no code with ``block_sparse_attention_gather_b200`` and
never imports it.  Everything is float64 numpy.  Library primitives used as steps:
``ndarray @``, ``np.linalg.eigh`` (the symmetric square root), ``np.lexsort``.

Source: Spark-H3 blog, section "Spark-Reblock".  Queries are grouped under the Mahalanobis
cosine distance d_Q(q_i, q_j) = 1 - cos(M_K^{1/2} q_i, M_K^{1/2} q_j) with M_K = E[k k^T], keys
symmetrically under M_Q = E[q q^T].  Starting from all tokens, a hierarchical partitioner
splits every group level by level into children of assigned capacities, until every leaf
holds exactly one block; the hierarchy costs O(N log N).  The released workflows reuse the
query partition for the keys (``reblock_layout=q_reuse_k``, comfy.icu "Spark-H3" page).

Readings taken where the blog leaves the partitioner open (each is also in the design notes):

B1  M_K is the plain second moment (1/N) sum_j k_j k_j^T over the head's N keys, and M^{1/2}
    its symmetric positive semi-definite square root.
B2  the cosine geometry is realised by the unit vectors x_i = W q_i / |W q_i| (W = M_K^{1/2};
    x_i = 0 when W q_i = 0), so that d_Q(q_i, q_j) = 1 - x_i . x_j.
B3  blocks are fixed-size (the target block size b; the last block takes the remainder) and
    the hierarchy is a binary tree over the block range: a node covering m >= 2 blocks gives
    its left child ceil(m/2) blocks and its right child the rest; a child's capacity is the
    number of tokens in its blocks.  A node of one block is a leaf.
B4  a node is split along the principal direction of its vectors: v = the result of
    ``POWER_ITERS`` power iterations of the node's covariance (1/n) sum (x_i - mu)(x_i - mu)^T
    from v0 = (1, ..., 1)/sqrt(d), each iterate normalised (an iterate of norm 0 keeps the
    previous one).  The left child takes the ``capacity_left`` tokens with the largest
    projections (x_i - mu) . v; equal projections go to the token that comes first in the
    node's current order; both children keep the current relative order of their tokens.
B5  the root's order is the token order 0..N-1; the final permutation lists the leaves in
    block order.  Keys reuse the query partition (q_reuse_k) unless ``mode="separate"``, in
    which case keys are partitioned the same way under d_K (roles of Q and K swapped).
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "POWER_ITERS",
    "second_moment",
    "psd_sqrt",
    "whiten_normalize",
    "fixed_block_offsets",
    "tree_levels",
    "principal_direction",
    "split_node",
    "reblock_level",
    "reblock_perm",
    "reblock_head",
]

POWER_ITERS = 4


def second_moment(X: np.ndarray) -> np.ndarray:
    """B1: M = E[x x^T] = (1/N) X^T X over the rows of X."""
    X = np.asarray(X, dtype=np.float64)
    return (X.T @ X) / X.shape[0]


def psd_sqrt(M: np.ndarray) -> np.ndarray:
    """B1: the symmetric PSD square root U diag(sqrt(max(lambda, 0))) U^T of M."""
    M = np.asarray(M, dtype=np.float64)
    lam, U = np.linalg.eigh(0.5 * (M + M.T))
    return (U * np.sqrt(np.clip(lam, 0.0, None))) @ U.T


def whiten_normalize(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """B2: rows x_i = W x_i / |W x_i| (zero rows stay zero)."""
    Y = np.asarray(X, dtype=np.float64) @ np.asarray(W, dtype=np.float64).T
    n = np.linalg.norm(Y, axis=1, keepdims=True)
    return np.divide(Y, n, out=np.zeros_like(Y), where=n > 0)


def fixed_block_offsets(N: int, b: int) -> np.ndarray:
    """B3: offsets of fixed-size blocks of b tokens; the last block takes the remainder."""
    return np.array(list(range(0, N, b)) + [N], dtype=np.int64)


def tree_levels(nb: int) -> list[list[tuple[int, int, int]]]:
    """B3: the internal nodes (lo, mid, hi) of the block tree, one list per depth; a node
    covers blocks [lo, hi) and its children [lo, mid) and [mid, hi)."""
    levels = []
    frontier = [(0, nb)]
    while frontier:
        nodes, nxt = [], []
        for lo, hi in frontier:
            if hi - lo >= 2:
                mid = lo + (hi - lo + 1) // 2
                nodes.append((lo, mid, hi))
                nxt += [(lo, mid), (mid, hi)]
        if nodes:
            levels.append(nodes)
        frontier = nxt
    return levels


def principal_direction(Xs: np.ndarray, iters: int = POWER_ITERS):
    """B4: (mu, v) of one node: its mean and the power-iteration estimate of the top
    eigenvector of its covariance."""
    Xs = np.asarray(Xs, dtype=np.float64)
    n, d = Xs.shape
    mu = Xs.mean(axis=0)
    Xc = Xs - mu
    v = np.full(d, 1.0 / math.sqrt(d))
    for _ in range(iters):
        w = Xc.T @ (Xc @ v) / n
        nrm = float(np.linalg.norm(w))
        if nrm > 0.0:
            v = w / nrm
    return mu, v


def split_node(Xs: np.ndarray, capacity_left: int, iters: int = POWER_ITERS):
    """B4: positions (0..n-1, in the node's current order) of the left and right children,
    and the projections they were decided on."""
    mu, v = principal_direction(Xs, iters)
    p = (np.asarray(Xs, dtype=np.float64) - mu) @ v
    n = len(p)
    order = np.lexsort((np.arange(n), -p))          # largest projection first, then position
    left = np.sort(order[:capacity_left])
    right = np.sort(order[capacity_left:])
    return left, right, p


def reblock_level(X: np.ndarray, perm: np.ndarray, offsets: np.ndarray, nodes, iters=POWER_ITERS):
    """One level of the hierarchy: every node (lo, mid, hi) of the level splits its token
    range perm[offsets[lo]:offsets[hi]]; everything else is copied."""
    perm = np.asarray(perm, dtype=np.int64)
    out = perm.copy()
    for lo, mid, hi in nodes:
        a, m, e = int(offsets[lo]), int(offsets[mid]), int(offsets[hi])
        toks = perm[a:e]
        left, right, _ = split_node(X[toks], m - a, iters)
        out[a:m] = toks[left]
        out[m:e] = toks[right]
    return out


def reblock_perm(X: np.ndarray, offsets: np.ndarray, iters: int = POWER_ITERS) -> np.ndarray:
    """B3-B5: the partition permutation of the unit vectors X (rows = tokens)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    perm = np.arange(len(X), dtype=np.int64)
    for nodes in tree_levels(len(offsets) - 1):
        perm = reblock_level(X, perm, offsets, nodes, iters)
    return perm


def reblock_head(Q: np.ndarray, K: np.ndarray, block: int, mode: str = "q_reuse_k",
                 iters: int = POWER_ITERS):
    """Spark-Reblock for one head: returns (q_perm, k_perm, offsets).  Query i of block A
    in the reblocked layout is token q_perm[offsets[A] + i]."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    N = Q.shape[0]
    offsets = fixed_block_offsets(N, block)
    Xq = whiten_normalize(Q, psd_sqrt(second_moment(K)))
    q_perm = reblock_perm(Xq, offsets, iters)
    if mode == "q_reuse_k":
        k_perm = q_perm.copy()
    elif mode == "separate":
        Xk = whiten_normalize(K, psd_sqrt(second_moment(Q)))
        k_perm = reblock_perm(Xk, offsets, iters)
    else:
        raise ValueError(mode)
    return q_perm, k_perm, offsets
