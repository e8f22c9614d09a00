"""Double-precision CPU oracle of the Spark-Attn two-branch block-sparse attention forward.

TEST INFRASTRUCTURE. This module is the independent checker of the CUDA path. Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import it.
It shares no code with ``block_sparse_attention_gather_b200`` and never imports it: inputs
arrive as plain arrays from the seeded generators, outputs are compared by the tests.

Everything is float64 numpy. Each step is written the way the method states it, one query
block at a time, with no blocking, fusion or reordering beyond what the definition says.
Library primitives used as steps: ``ndarray @`` (a dot product / matmul), ``np.lexsort``.

Sources (blog "Spark-H3: Adaptive Block Sparse Attention for MiniMax-H3", the project's
extension page "Spark-H3 (comfy.icu)", and the comfyui-wiki news article on Spark-H3):

* Spark-H3 blog, section "Spark-Reblock": tokens are reordered into blocks ("Token IDs track
  membership"), and the BSA equations: per query block A,
  ``BSA(Q_A) = Softmax(Q_A K~_A^T / sqrt(d)) V~_A`` where K~_A, V~_A concatenate, over every
  key block B, the exact rows K_B, V_B when B is in the selected set S_A, and |B| copies of a
  summary row otherwise; one row-wise softmax covers both branches. The selection is a
  fixed Top-K budget ("top 10%" of key blocks).
* Spark-H3 blog, section "Discussion": blocks are scored from block-level means.
* Spark-H3 blog, section "Spark-Reweight": each block is scored once with a representative
  query, the mean of the video queries; the scores give weighted key/value summaries and a
  log-mass bias chosen so that the exponential of the effective logit equals the expected
  exponential E[exp(x)] instead of exp(E[x]); routing is unchanged.
* comfyui-wiki news article, bullet on Spark-Reweight: one anchor (the query mean) per head.
* Spark-H3 blog, section "Spark-Reblock", after the BSA equations: context (sink) tokens are
  always attended exactly and do not count against the Top-K budget of video blocks.

Readings taken where the pages leave a step open (each is also listed in the design notes):

R1  summary weights: the in-block softmax of the anchor logits s_j = q_bar . k_j / sqrt(d).
R2  bias: b_B = log(mean_j exp(s_j)) - q_bar . k~_B / sqrt(d); the |B| copies of the summary
    row become one row whose logit carries + log|B|, so c_B = b_B + log|B|.
R3  anchor: the mean over all N queries of the head.
R4  routing score: S[A,B] = q_bar_A . k_bar_B / sqrt(d) with uniform block means.
R5  k = clamp(ceil(ratio * nKB - 1e-9), 1, nKB).
R6  ties in Top-K: the smaller block index wins; S_A is reported in ascending order.
R7  no causal mask and no forced diagonal block; sink tokens only as the context segment (R15).
R8  each key block is either exact or compressed, never both.
R9  the output row of reblocked position i is written back to original token q_perm[i].
R10 permutations are per head; block offsets are shared by all heads.
R15 context tokens (optional, Kc/Vc [nc, d] per head): every video query attends to all of
    them exactly, inside the same row-wise softmax as both branches.  They form no block, take
    no part in the anchor, the block means, the summaries or the routing, and k is still
    taken over the nKB video blocks.  Context queries are not part of this operation.

Parity: every function here is pinned by the CPU tests (dense attention at ratio 1, blocks of
identical keys, identical queries, an anchor-centred query, the log-mass identity, hand
cases, brute-force Top-K, and permutation invariances).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "topk_count",
    "gather_rows",
    "anchor",
    "block_sizes",
    "block_means",
    "summarize_block",
    "summarize",
    "meanpool_summaries",
    "route_scores",
    "route_block",
    "route",
    "route_threshold_block",
    "attend_block",
    "HeadResult",
    "forward_head",
    "forward",
    "dense_attention",
    "attention_mass_recall",
    "log_mass_error",
]


def topk_count(ratio: float, nkb: int) -> int:
    """Number of exact key blocks per query block (reading R5).

    Spark-H3 blog, "Spark-Reblock": the exact branch covers the top ``ratio`` fraction of the
    key blocks ("top 10%").  The fraction is rounded up, with a 1e-9 guard so that a ratio
    whose product with nKB is an integer in exact arithmetic is not bumped by the binary
    representation of the ratio, and clamped to [1, nKB].
    """
    if not (ratio > 0.0 and ratio <= 1.0):
        raise ValueError(f"topk_ratio must lie in (0, 1], got {ratio}")
    if nkb < 1:
        raise ValueError("need at least one key block")
    k = math.ceil(ratio * nkb - 1e-9)
    return int(min(max(k, 1), nkb))


def gather_rows(X: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Reblocked layout: row i of the result is token ``perm[i]`` of X.

    Spark-H3 blog, "Spark-Reblock": tokens are permuted into blocks and token IDs track their
    membership.
    """
    return np.asarray(X, dtype=np.float64)[np.asarray(perm, dtype=np.int64)]


def anchor(Q: np.ndarray) -> np.ndarray:
    """Representative query of one head: the mean of all N queries (reading R3).

    Spark-H3 blog, "Spark-Reweight" (the mean of the video queries is the representative),
    comfyui-wiki article (one anchor per head).
    """
    Q = np.asarray(Q, dtype=np.float64)
    return Q.sum(axis=0) / Q.shape[0]


def block_sizes(offsets: np.ndarray) -> np.ndarray:
    offsets = np.asarray(offsets, dtype=np.int64)
    return offsets[1:] - offsets[:-1]


def block_means(Xp: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """Uniform mean of each block's rows (Spark-H3 blog, "Discussion": block-level means)."""
    offsets = np.asarray(offsets, dtype=np.int64)
    nb = len(offsets) - 1
    out = np.empty((nb, Xp.shape[1]), dtype=np.float64)
    for b in range(nb):
        rows = Xp[offsets[b]:offsets[b + 1]]
        out[b] = rows.sum(axis=0) / rows.shape[0]
    return out


def _log_mean_exp(s: np.ndarray) -> float:
    m = float(np.max(s))
    return m + math.log(float(np.sum(np.exp(s - m))) / s.shape[0])


def summarize_block(Kp_B: np.ndarray, Vp_B: np.ndarray, qbar: np.ndarray, scale: float):
    """Spark-Reweight summary of one key block (readings R1, R2).

    Spark-H3 blog, "Spark-Reweight": the block is scored once with the representative query;
    the scores weight the key/value summary, and a log-mass bias restores the expected
    exponential.  Returns (k_tilde, v_tilde, b, c) with c = b + log|B| the offset that the
    single summary row carries in place of |B| identical copies.
    """
    s = scale * (Kp_B @ qbar)                       # anchor logits s_j
    w = np.exp(s - np.max(s))
    w = w / np.sum(w)                               # in-block softmax weights
    k_tilde = w @ Kp_B
    v_tilde = w @ Vp_B
    b = _log_mean_exp(s) - scale * float(qbar @ k_tilde)
    c = b + math.log(Kp_B.shape[0])
    return k_tilde, v_tilde, b, c


def summarize(Kp: np.ndarray, Vp: np.ndarray, k_offsets: np.ndarray, qbar: np.ndarray,
              scale: float):
    """All key-block summaries of one head: (k_tilde [nKB,d], v_tilde [nKB,d], c [nKB])."""
    k_offsets = np.asarray(k_offsets, dtype=np.int64)
    nkb = len(k_offsets) - 1
    d = Kp.shape[1]
    kt = np.empty((nkb, d)); vt = np.empty((nkb, d)); c = np.empty(nkb)
    for B in range(nkb):
        lo, hi = k_offsets[B], k_offsets[B + 1]
        kt[B], vt[B], _, c[B] = summarize_block(Kp[lo:hi], Vp[lo:hi], qbar, scale)
    return kt, vt, c


def meanpool_summaries(Kp: np.ndarray, Vp: np.ndarray, k_offsets: np.ndarray):
    """Baseline BSA compressed branch: uniform means repeated |B| times.

    Spark-H3 blog, "Spark-Reblock", BSA equations: the 1_{|B|} k_bar_B^T rows.  As one row the
    repetition is the offset log|B| (no bias).  Diagnostic only.
    """
    kt = block_means(Kp, k_offsets)
    vt = block_means(Vp, k_offsets)
    c = np.log(block_sizes(k_offsets).astype(np.float64))
    return kt, vt, c


def route_scores(qbar_blocks: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Block scores S[A,B] = q_bar_A . k_bar_B / sqrt(d) (reading R4)."""
    return scale * (qbar_blocks @ kbar.T)


def route_block(scores_A: np.ndarray, k: int) -> np.ndarray:
    """Top-k key blocks of one query block, ties to the smaller index, ascending (R6)."""
    nkb = scores_A.shape[0]
    idx = np.arange(nkb)
    order = np.lexsort((idx, -scores_A))            # primary: score desc; secondary: index asc
    return np.sort(order[:k]).astype(np.int64)


def route(qbar_blocks: np.ndarray, kbar: np.ndarray, scale: float, k: int):
    """Selected sets of all query blocks of one head: (sel [nQB,k], S [nQB,nKB])."""
    S = route_scores(qbar_blocks, kbar, scale)
    sel = np.stack([route_block(S[A], k) for A in range(S.shape[0])])
    return sel, S


def route_threshold_block(scores_A: np.ndarray, tau: float, kcap: int) -> np.ndarray:
    """Sol-Attn's content-adaptive routing, as the comparator the Spark-H3 blog's "Discussion"
    describes: the block-level logits of a query block are taken as roughly Gaussian and the
    blocks above mu + tau * sigma get exact attention.  Readings (T1): mu and sigma are the
    mean and the population standard deviation of the query block's nKB scores; "above" is
    strict; at most kcap blocks are kept, the largest (ties to the smaller index), so a caller
    can bound the exact branch; the set is reported ascending and may be empty."""
    S = np.asarray(scores_A, dtype=np.float64)
    thr = S.mean() + tau * S.std()
    above = np.flatnonzero(S > thr)
    if len(above) > kcap:
        return route_block(S, kcap)
    return above.astype(np.int64)


def attend_block(Qp_A: np.ndarray, Kp: np.ndarray, Vp: np.ndarray, k_offsets: np.ndarray,
                 sel_A: np.ndarray, k_tilde: np.ndarray, v_tilde: np.ndarray, c: np.ndarray,
                 scale: float, Kc: np.ndarray | None = None,
                 Vc: np.ndarray | None = None) -> np.ndarray:
    """Two-branch attention of one query block (Spark-H3 blog, BSA equations; R8).

    The exact branch holds every key row of the selected blocks; the compressed branch holds
    one summary row per unselected block whose logit carries the offset c_B.  Context rows
    Kc/Vc, when given, are exact keys outside the Top-K budget (R15).  A single row-wise
    softmax normalises the union.
    """
    k_offsets = np.asarray(k_offsets, dtype=np.int64)
    nkb = len(k_offsets) - 1
    selected = set(int(b) for b in sel_A)
    exact_rows = (np.concatenate([np.arange(k_offsets[B], k_offsets[B + 1])
                                  for B in sorted(selected)])
                  if selected else np.zeros(0, dtype=np.int64))   # threshold routing: may be empty
    comp = np.array([B for B in range(nkb) if B not in selected], dtype=np.int64)

    logits_exact = scale * (Qp_A @ Kp[exact_rows].T)
    values = [Vp[exact_rows]]
    logits = [logits_exact]
    if comp.size:
        logits.append(scale * (Qp_A @ k_tilde[comp].T) + c[comp][None, :])
        values.append(v_tilde[comp])
    if Kc is not None and len(Kc):
        logits.append(scale * (Qp_A @ np.asarray(Kc, dtype=np.float64).T))
        values.append(np.asarray(Vc, dtype=np.float64))
    L = np.concatenate(logits, axis=1)
    Vcat = np.concatenate(values, axis=0)
    L = L - L.max(axis=1, keepdims=True)
    P = np.exp(L)
    P = P / P.sum(axis=1, keepdims=True)
    return P @ Vcat


@dataclass
class HeadResult:
    """Per-head output and intermediates (rows of out in ORIGINAL token order)."""
    out: np.ndarray            # [N, d] (rows not computed are NaN when a subset is requested)
    qbar: np.ndarray           # [d]
    qbar_blocks: np.ndarray    # [nQB, d]
    kbar: np.ndarray           # [nKB, d]
    k_tilde: np.ndarray        # [nKB, d]
    v_tilde: np.ndarray        # [nKB, d]
    c: np.ndarray              # [nKB]
    sel: np.ndarray            # [nQB, k]
    scores: np.ndarray         # [nQB, nKB]


def forward_head(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, ratio, *, mode="reweight",
                 sel=None, blocks=None, Kc=None, Vc=None) -> HeadResult:
    """One head of the forward pass, steps in the pages' order.

    ``sel`` (optional [nQB,k]) replaces the routing result, e.g. with another implementation's
    selection when several selections are correct at a near-tie.  ``blocks`` (optional
    iterable of query-block ids) restricts the attention step to those blocks; summaries and
    routing are always computed for the whole head.  ``Kc``, ``Vc`` (optional [nc, d]) are the
    head's context tokens (R15).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    q_perm = np.asarray(q_perm, dtype=np.int64)
    k_perm = np.asarray(k_perm, dtype=np.int64)
    q_offsets = np.asarray(q_offsets, dtype=np.int64)
    k_offsets = np.asarray(k_offsets, dtype=np.int64)
    N, d = Q.shape
    if (Kc is None) != (Vc is None):
        raise ValueError("Kc and Vc go together")
    if Kc is not None:
        Kc = np.asarray(Kc, dtype=np.float64).reshape(-1, d)
        Vc = np.asarray(Vc, dtype=np.float64).reshape(-1, d)
        if Kc.shape != Vc.shape:
            raise ValueError("Kc and Vc must have the same shape")
    scale = 1.0 / math.sqrt(d)
    nqb = len(q_offsets) - 1
    nkb = len(k_offsets) - 1
    k = topk_count(ratio, nkb)

    # 1. reblocked layout
    Qp = gather_rows(Q, q_perm)
    Kp = gather_rows(K, k_perm)
    Vp = gather_rows(V, k_perm)
    # 2. anchor: mean over all N queries of the head
    qbar = anchor(Q)
    # 3. block means for routing
    qbar_blocks = block_means(Qp, q_offsets)
    kbar = block_means(Kp, k_offsets)
    # 4. compressed-branch summaries
    if mode == "reweight":
        kt, vt, c = summarize(Kp, Vp, k_offsets, qbar, scale)
    elif mode == "meanpool":
        kt, vt, c = meanpool_summaries(Kp, Vp, k_offsets)
    else:
        raise ValueError(mode)
    # 5. routing
    sel_o, S = route(qbar_blocks, kbar, scale, k)
    if sel is None:
        sel = sel_o
    else:
        sel = np.asarray(sel, dtype=np.int64)
        if sel.shape != (nqb, k):
            raise ValueError(f"sel must have shape {(nqb, k)}")
    # 6. attention, written back in original order
    out = np.full((N, d), np.nan)
    todo = range(nqb) if blocks is None else blocks
    for A in todo:
        lo, hi = q_offsets[A], q_offsets[A + 1]
        o = attend_block(Qp[lo:hi], Kp, Vp, k_offsets, sel[A], kt, vt, c, scale, Kc=Kc, Vc=Vc)
        out[q_perm[lo:hi]] = o
    return HeadResult(out, qbar, qbar_blocks, kbar, kt, vt, c, sel, S)


def forward(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, ratio, *, mode="reweight",
            sel=None, blocks=None, Kc=None, Vc=None):
    """All heads: Q,K,V [H,N,d]; perms [H,N]; offsets shared; optional context Kc,Vc
    [H,nc,d].  Returns a list of HeadResult.

    ``blocks`` may be a dict head -> iterable of query blocks (heads absent are skipped for
    the attention step) or None for every block of every head.
    """
    H = np.asarray(Q).shape[0]
    res = []
    for h in range(H):
        if isinstance(blocks, dict):
            bl = blocks.get(h, [])
        else:
            bl = blocks
        res.append(forward_head(Q[h], K[h], V[h], q_perm[h], k_perm[h], q_offsets, k_offsets,
                                ratio, mode=mode, sel=None if sel is None else sel[h],
                                blocks=bl, Kc=None if Kc is None else Kc[h],
                                Vc=None if Vc is None else Vc[h]))
    return res


# ----------------------------------------------------------------------------------------
# Diagnostics (not part of parity): the two quantities the blog's ablation tables report.
# ----------------------------------------------------------------------------------------

def dense_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """softmax(Q K^T / sqrt(d)) V for one head, float64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L = (Q @ K.T) / math.sqrt(Q.shape[1])
    L = L - L.max(axis=1, keepdims=True)
    P = np.exp(L)
    P = P / P.sum(axis=1, keepdims=True)
    return P @ V


def attention_mass_recall(Qp_A, Kp, k_offsets, sel_A) -> float:
    """Mean over the block's queries of the dense attention mass inside the selected blocks.

    Spark-H3 blog, "Spark-Reblock" ablation table ("attention-mass recall").
    """
    k_offsets = np.asarray(k_offsets, dtype=np.int64)
    L = (np.asarray(Qp_A) @ np.asarray(Kp).T) / math.sqrt(Kp.shape[1])
    L = L - L.max(axis=1, keepdims=True)
    P = np.exp(L)
    P = P / P.sum(axis=1, keepdims=True)
    rows = np.concatenate([np.arange(k_offsets[B], k_offsets[B + 1]) for B in sel_A])
    return float(P[:, rows].sum(axis=1).mean())


def log_mass_error(Qp_A, Kp, k_offsets, sel_A, k_tilde, c) -> float:
    """Mean |exact log-mass of the compressed set - its summary approximation| (nats).

    Spark-H3 blog, "Spark-Reweight" ablation table ("absolute log-mass error").
    """
    k_offsets = np.asarray(k_offsets, dtype=np.int64)
    nkb = len(k_offsets) - 1
    scale = 1.0 / math.sqrt(Kp.shape[1])
    selected = set(int(b) for b in sel_A)
    comp = [B for B in range(nkb) if B not in selected]
    if not comp:
        return 0.0
    rows = np.concatenate([np.arange(k_offsets[B], k_offsets[B + 1]) for B in comp])
    Le = scale * (np.asarray(Qp_A) @ np.asarray(Kp)[rows].T)
    La = scale * (np.asarray(Qp_A) @ np.asarray(k_tilde)[comp].T) + np.asarray(c)[comp][None, :]

    def lse(x):
        m = x.max(axis=1, keepdims=True)
        return (m + np.log(np.exp(x - m).sum(axis=1, keepdims=True)))[:, 0]

    return float(np.abs(lse(Le) - lse(La)).mean())
