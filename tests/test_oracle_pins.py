"""Pins of the CPU oracle against facts fixed by the pages and by mathematics (no GPU).

Each pin compares the oracle with something other than itself: a library routine (torch's
scaled-dot-product attention, scipy's logsumexp / entropy), a closed form worked by hand from
the Spark-H3 blog's definitions (tests/golden), exhaustive enumeration, or an invariance.
The mutation test at the end plants plausible mistakes in the oracle and checks that at
least one pin catches each of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

from oracle import spark_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "reweight_hand_cases.json")
TOL = 1e-11


# ------------------------------------------------------------------------ problem builders

def random_offsets(rng, N, lo, hi):
    offs = [0]
    while offs[-1] < N:
        offs.append(min(offs[-1] + int(rng.integers(lo, hi + 1)), N))
    return np.array(offs, dtype=np.int64)


def random_problem(seed, H=2, N=97, d=8, lo=1, hi=17, same_layout=False):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((H, N, d))
    K = rng.standard_normal((H, N, d))
    V = rng.standard_normal((H, N, d))
    q_perm = np.stack([rng.permutation(N) for _ in range(H)])
    k_perm = q_perm.copy() if same_layout else np.stack([rng.permutation(N) for _ in range(H)])
    q_off = random_offsets(rng, N, lo, hi)
    k_off = q_off.copy() if same_layout else random_offsets(rng, N, lo, hi)
    return dict(Q=Q, K=K, V=V, q_perm=q_perm, k_perm=k_perm, q_offsets=q_off, k_offsets=k_off)


def scatter_reblocked(Xp, perm):
    """Original-order array X with X[perm[i]] = Xp[i]."""
    X = np.empty_like(Xp)
    X[perm] = Xp
    return X


def sdpa(Q, K, V):
    """Library dense attention softmax(QK^T/sqrt(d))V, float64 (torch math backend)."""
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()


def run(p, ratio, **kw):
    return O.forward(p["Q"], p["K"], p["V"], p["q_perm"], p["k_perm"], p["q_offsets"],
                     p["k_offsets"], ratio, **kw)


def max_err_vs_dense(p, ratio, heads_rows=None):
    res = run(p, ratio)
    err = 0.0
    for h, r in enumerate(res):
        ref = sdpa(p["Q"][h], p["K"][h], p["V"][h])
        if heads_rows is None:
            err = max(err, float(np.abs(r.out - ref).max()))
        else:
            rows = heads_rows[h]
            err = max(err, float(np.abs(r.out[rows] - ref[rows]).max()))
    return err


# ----------------------------------------------------------------------------------- pins
# Each pin returns its error; the tests assert it is below TOL, and the mutation test
# asserts that a planted mistake pushes at least one pin above it.

def pin_dense_at_ratio_one():
    """P1: topk_ratio = 1 makes every block exact: the result is dense softmax attention."""
    return max(max_err_vs_dense(random_problem(s), 1.0) for s in (1, 2))


def pin_identical_keys_in_blocks():
    """P2: keys identical inside every key block make the compressed row exact, any ratio.

    With k_j = k for j in B the weights are uniform, k~ = k, b = 0 and the single row with
    offset log|B| carries exactly the |B| terms exp(q.k/sqrt d) v_j.
    """
    err = 0.0
    for seed, ratio in ((3, 0.1), (4, 0.3), (5, 0.5)):
        p = random_problem(seed, N=120, lo=3, hi=20)
        rng = np.random.default_rng(seed + 100)
        for h in range(p["Q"].shape[0]):
            Kp = np.empty((p["Q"].shape[1], p["Q"].shape[2]))
            for B in range(len(p["k_offsets"]) - 1):
                Kp[p["k_offsets"][B]:p["k_offsets"][B + 1]] = rng.standard_normal(Kp.shape[1])
            p["K"][h] = scatter_reblocked(Kp, p["k_perm"][h])
        err = max(err, max_err_vs_dense(p, ratio))
    return err


def pin_identical_queries():
    """P4: all queries equal (so each equals the anchor): the result is dense, any ratio."""
    err = 0.0
    for seed, ratio in ((6, 0.1), (7, 0.4)):
        p = random_problem(seed, N=110, lo=2, hi=25)
        for h in range(p["Q"].shape[0]):
            p["Q"][h] = p["Q"][h, :1]
        err = max(err, max_err_vs_dense(p, ratio))
    return err


def pin_anchor_centred_query():
    """P4b: a query equal to the mean of ALL queries of its head gets the dense row.

    Token 0 holds q*, the other tokens come in pairs q* +/- delta placed at random, so the
    head's query mean is q* while no query block is centred on it.  Only the anchor reading
    "mean over all N queries of the head" makes token 0's output exact at any ratio.
    """
    err = 0.0
    for seed, ratio in ((8, 0.1), (9, 0.3)):
        p = random_problem(seed, N=129, lo=4, hi=24)
        rng = np.random.default_rng(seed + 7)
        H, N, d = p["Q"].shape
        rows = {}
        for h in range(H):
            qs = rng.standard_normal(d) * 1.5
            delta = rng.standard_normal(((N - 1) // 2, d))
            others = np.concatenate([qs + delta, qs - delta])
            others = others[rng.permutation(N - 1)]
            p["Q"][h] = np.concatenate([qs[None], others])
            rows[h] = [0]
        err = max(err, max_err_vs_dense(p, ratio, heads_rows=rows))
    return err


def pin_log_mass_identity():
    """P3: q_bar.k~/sqrt d + c = logsumexp_j(q_bar.k_j/sqrt d) and c = entropy(w)."""
    rng = np.random.default_rng(11)
    err = 0.0
    for m in (1, 2, 7, 64, 128):
        d = 16
        Kb = rng.standard_normal((m, d)) * 2.0
        Vb = rng.standard_normal((m, d))
        qbar = rng.standard_normal(d)
        scale = 1.0 / math.sqrt(d)
        kt, vt, b, c = O.summarize_block(Kb, Vb, qbar, scale)
        s = scale * (Kb @ qbar)
        lse = scipy.special.logsumexp(s)
        w = scipy.special.softmax(s)
        err = max(err, abs(scale * float(qbar @ kt) + c - lse))
        err = max(err, abs(c - scipy.stats.entropy(w)))
        err = max(err, abs(b - (c - math.log(m))))
    return err


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _ev(x):
    return float(eval(x, {"__builtins__": {}}, vars(math))) if isinstance(x, str) else float(x)


def pin_golden_single_block():
    """P5: the hand-worked single-block case (tests/golden/reweight_hand_cases.json)."""
    g = _golden()["single_block"]
    K = np.array([[_ev(v) for v in row] for row in g["K"]])
    V = np.array([[_ev(v) for v in row] for row in g["V"]])
    qbar = np.array(g["qbar"], dtype=np.float64)
    kt, vt, b, c = O.summarize_block(K, V, qbar, 1.0)
    e = g["expected"]
    errs = [abs(kt[0] - _ev(e["k_tilde"])), abs(vt[0] - _ev(e["v_tilde"])),
            abs(b - _ev(e["b"])), abs(c - _ev(e["c"])), abs(c - _ev(e["entropy"])),
            abs(float(qbar @ kt) + c - _ev(e["effective_logit"]))]
    return max(errs)


def pin_golden_tiny_forward():
    """P5: hand-worked 4-token forward, in reblocked and in scrambled original order."""
    g = _golden()["tiny_forward"]
    err = 0.0
    for variant in ("identity", "permuted"):
        v = g[variant]
        Q = np.array([[_ev(x)] for x in v["Q"]])[None]
        K = np.array([[_ev(x)] for x in v["K"]])[None]
        V = np.array([[_ev(x)] for x in v["V"]])[None]
        res = O.forward(Q, K, V, np.array([v["q_perm"]]), np.array([v["k_perm"]]),
                        np.array(g["q_offsets"]), np.array(g["k_offsets"]), g["ratio"])[0]
        exp = np.array([_ev(x) for x in v["expected_out"]])
        err = max(err, float(np.abs(res.out[:, 0] - exp).max()))
        if not np.array_equal(res.sel, np.array(g["expected_sel"])):
            err = max(err, 1.0)
        err = max(err, float(np.abs(res.c - np.array([_ev(x) for x in g["expected_c"]])).max()))
    return err


def _brute_topk(S, k):
    """The unique k-subset T with S[b] > S[b'] or (S[b] == S[b'] and b < b') for b in T,
    b' not in T, found by enumerating every k-subset."""
    n = len(S)
    found = []
    for T in itertools.combinations(range(n), k):
        rest = [b for b in range(n) if b not in T]
        if all(S[b] > S[r] or (S[b] == S[r] and b < r) for b in T for r in rest):
            found.append(T)
    assert len(found) == 1
    return np.array(found[0])


def pin_bruteforce_topk():
    """P6: Top-K against exhaustive enumeration, with many exact ties (integer scores)."""
    rng = np.random.default_rng(12)
    bad = 0
    for _ in range(60):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, n + 1))
        S = rng.integers(-2, 3, size=n).astype(np.float64)
        if not np.array_equal(O.route_block(S, k), _brute_topk(S, k)):
            bad += 1
    return float(bad)


def pin_scores_are_block_mass_order():
    """P6b: with identical queries inside each query block, identical keys inside each key
    block and equal block sizes, the block score order is the order of the dense attention
    mass per key block, so the selection is the top-k blocks by dense mass (torch softmax)."""
    rng = np.random.default_rng(13)
    bad = 0
    H, nb, bs, d = 2, 8, 6, 8
    N = nb * bs
    for trial in range(4):
        for ratio in (0.25, 0.5):
            p = random_problem(100 + trial, H=H, N=N, d=d)
            p["q_offsets"] = np.arange(0, N + 1, bs)
            p["k_offsets"] = np.arange(0, N + 1, bs)
            for h in range(H):
                Qp = np.repeat(rng.standard_normal((nb, d)), bs, axis=0)
                Kp = np.repeat(rng.standard_normal((nb, d)), bs, axis=0)
                p["Q"][h] = scatter_reblocked(Qp, p["q_perm"][h])
                p["K"][h] = scatter_reblocked(Kp, p["k_perm"][h])
            res = run(p, ratio)
            k = O.topk_count(ratio, nb)
            for h in range(H):
                Qp = torch.from_numpy(p["Q"][h][p["q_perm"][h]])
                Kp = torch.from_numpy(p["K"][h][p["k_perm"][h]])
                P = torch.softmax(Qp @ Kp.T / math.sqrt(d), dim=-1)
                mass = P.reshape(N, nb, bs).sum(-1).reshape(nb, bs, nb)[:, 0, :].numpy()
                for A in range(nb):
                    want = np.sort(np.argsort(-mass[A], kind="stable")[:k])
                    if not np.array_equal(res[h].sel[A], want):
                        bad += 1
    return float(bad)


def pin_invariances():
    """P7: relabelling tokens inside blocks, or reordering whole blocks consistently, leaves
    the output (in original token order) unchanged."""
    err = 0.0
    for ratio in (0.2, 0.5):
        p = random_problem(21, N=100, lo=3, hi=15)
        ref = [r.out for r in run(p, ratio)]
        rng = np.random.default_rng(22)
        # (a) shuffle tokens inside each block
        q = dict(p)
        q["q_perm"] = p["q_perm"].copy()
        q["k_perm"] = p["k_perm"].copy()
        for h in range(p["Q"].shape[0]):
            for offs, key in ((p["q_offsets"], "q_perm"), (p["k_offsets"], "k_perm")):
                for B in range(len(offs) - 1):
                    seg = q[key][h, offs[B]:offs[B + 1]]
                    q[key][h, offs[B]:offs[B + 1]] = seg[rng.permutation(len(seg))]
        out_a = [r.out for r in run(q, ratio)]
        # (b) reorder whole blocks (queries and keys independently)
        r = dict(p)
        for offs_key, perm_key in (("q_offsets", "q_perm"), ("k_offsets", "k_perm")):
            offs = p[offs_key]
            nb = len(offs) - 1
            new_order = rng.permutation(nb)
            sizes = offs[1:] - offs[:-1]
            r[offs_key] = np.concatenate([[0], np.cumsum(sizes[new_order])])
            r[perm_key] = np.stack([np.concatenate([p[perm_key][h, offs[B]:offs[B + 1]]
                                                    for B in new_order])
                                    for h in range(p["Q"].shape[0])])
        out_b = [x.out for x in run(r, ratio)]
        for h in range(len(ref)):
            err = max(err, float(np.abs(out_a[h] - ref[h]).max()),
                      float(np.abs(out_b[h] - ref[h]).max()))
    return err


def pin_literal_copies():
    """The single summary row with offset log|B| equals the BSA equations' literal form:
    |B| copies of the summary row (logit q.k~/sqrt d + b) concatenated with the exact rows,
    one softmax over all of them; likewise |B| copies of the uniform mean row (mean pooling)."""
    p = random_problem(31, H=1, N=90, d=8, lo=2, hi=16)
    err = 0.0
    for mode in ("reweight", "meanpool"):
        res = run(p, 0.3, mode=mode)[0]
        Qp = p["Q"][0][p["q_perm"][0]]
        Kp = p["K"][0][p["k_perm"][0]]
        Vp = p["V"][0][p["k_perm"][0]]
        offs = p["k_offsets"]
        scale = 1 / math.sqrt(8)
        qoffs = p["q_offsets"]
        for A in range(len(qoffs) - 1):
            rowsK, rowsV, bias = [], [], []
            for B in range(len(offs) - 1):
                m = offs[B + 1] - offs[B]
                if B in set(res.sel[A].tolist()):
                    rowsK.append(Kp[offs[B]:offs[B + 1]]); rowsV.append(Vp[offs[B]:offs[B + 1]])
                    bias.append(np.zeros(m))
                else:
                    rowsK.append(np.repeat(res.k_tilde[B][None], m, 0))
                    rowsV.append(np.repeat(res.v_tilde[B][None], m, 0))
                    b = res.c[B] - math.log(m)          # per-copy bias (0 for mean pooling)
                    bias.append(np.full(m, b))
            Kt = torch.from_numpy(np.concatenate(rowsK))
            Vt = torch.from_numpy(np.concatenate(rowsV))
            bt = torch.from_numpy(np.concatenate(bias))
            q = torch.from_numpy(Qp[qoffs[A]:qoffs[A + 1]])
            lit = torch.softmax(q @ Kt.T * scale + bt, dim=-1) @ Vt
            got = res.out[p["q_perm"][0][qoffs[A]:qoffs[A + 1]]]
            err = max(err, float(np.abs(lit.numpy() - got).max()))
        if mode == "meanpool":
            err = max(err, float(np.abs(res.c - np.log(offs[1:] - offs[:-1])).max()))
    return err


def pin_block_means():
    """Block means: |B|-weighted means add up to the column sums of all rows, each mean lies
    between the block's column minimum and maximum, and a constant block gives the constant."""
    rng = np.random.default_rng(51)
    X = rng.standard_normal((300, 6))
    offs = random_offsets(rng, 300, 1, 40)
    m = O.block_means(X, offs)
    sizes = (offs[1:] - offs[:-1]).astype(np.float64)
    err = float(np.abs((sizes[:, None] * m).sum(0) - X.sum(0)).max())
    for B in range(len(offs) - 1):
        blk = X[offs[B]:offs[B + 1]]
        if not ((m[B] >= blk.min(0) - 1e-12).all() and (m[B] <= blk.max(0) + 1e-12).all()):
            err = max(err, 1.0)
    Xc = np.repeat(rng.standard_normal((len(offs) - 1, 6)), offs[1:] - offs[:-1], axis=0)
    err = max(err, float(np.abs(O.block_means(Xc, offs) - Xc[offs[:-1]]).max()))
    return err


def pin_dense_reference():
    """The oracle's dense attention (used by the GPU tests at ratio 1) against torch's
    scaled-dot-product attention."""
    rng = np.random.default_rng(52)
    Q, K, V = (rng.standard_normal((70, 16)) for _ in range(3))
    return float(np.abs(O.dense_attention(Q, K, V) - sdpa(Q, K, V)).max())


def pin_diagnostics():
    """Attention-mass recall is 1 when every block is selected; the log-mass error is 0 when
    every key block holds identical keys (the summary row is then exact)."""
    p = random_problem(53, H=1, N=90, d=8, lo=3, hi=12)
    Qp = p["Q"][0][p["q_perm"][0]]
    Kp = p["K"][0][p["k_perm"][0]]
    offs = p["k_offsets"]
    nkb = len(offs) - 1
    err = abs(O.attention_mass_recall(Qp[:10], Kp, offs, np.arange(nkb)) - 1.0)
    rng = np.random.default_rng(54)
    for B in range(nkb):
        Kp[offs[B]:offs[B + 1]] = rng.standard_normal(8)
    kt, vt, c = O.summarize(Kp, Kp, offs, rng.standard_normal(8), 1 / math.sqrt(8))
    err = max(err, O.log_mass_error(Qp[:10], Kp, offs, [0, 1], kt, c))
    return err


def _with_context(p, seed, nc):
    rng = np.random.default_rng(seed)
    H, _, d = p["Q"].shape
    p["Kc"] = rng.standard_normal((H, nc, d)) * 1.5
    p["Vc"] = rng.standard_normal((H, nc, d))
    return p


def pin_context_dense_at_ratio_one():
    """Context tokens (Spark-H3 blog, "Spark-Reblock": context/sink tokens stay exact, outside
    the Top-K budget): at topk_ratio = 1 the result is dense attention over the video keys
    followed by the context keys, in one softmax."""
    err = 0.0
    for seed, nc in ((81, 1), (82, 13), (83, 40)):
        p = _with_context(random_problem(seed), seed + 1, nc)
        res = run(p, 1.0, Kc=p["Kc"], Vc=p["Vc"])
        for h, r in enumerate(res):
            ref = sdpa(p["Q"][h], np.concatenate([p["K"][h], p["Kc"][h]]),
                       np.concatenate([p["V"][h], p["Vc"][h]]))
            err = max(err, float(np.abs(r.out - ref).max()))
    return err


def pin_context_identical_keys():
    """Context tokens with exact summaries (keys constant inside every video block, as in P2):
    the result is dense over video + context keys at any ratio."""
    err = 0.0
    for seed, ratio, nc in ((84, 0.1, 7), (85, 0.3, 21)):
        p = _with_context(random_problem(seed, N=120, lo=3, hi=20), seed + 1, nc)
        rng = np.random.default_rng(seed + 100)
        for h in range(p["Q"].shape[0]):
            Kp = np.empty((p["Q"].shape[1], p["Q"].shape[2]))
            for B in range(len(p["k_offsets"]) - 1):
                Kp[p["k_offsets"][B]:p["k_offsets"][B + 1]] = rng.standard_normal(Kp.shape[1])
            p["K"][h] = scatter_reblocked(Kp, p["k_perm"][h])
        res = run(p, ratio, Kc=p["Kc"], Vc=p["Vc"])
        for h, r in enumerate(res):
            ref = sdpa(p["Q"][h], np.concatenate([p["K"][h], p["Kc"][h]]),
                       np.concatenate([p["V"][h], p["Vc"][h]]))
            err = max(err, float(np.abs(r.out - ref).max()))
    return err


def pin_context_outside_budget():
    """Context tokens change neither the routing nor the summaries (outside the Top-K budget,
    no part in the anchor), and an empty context is no context."""
    p = random_problem(86, N=150, lo=4, hi=24)
    base = run(p, 0.2)
    q = _with_context(dict(p), 87, 9)
    withc = run(q, 0.2, Kc=q["Kc"], Vc=q["Vc"])
    empty = run(p, 0.2, Kc=np.zeros((2, 0, 8)), Vc=np.zeros((2, 0, 8)))
    err = 0.0
    for a, b, e in zip(base, withc, empty):
        if not np.array_equal(a.sel, b.sel):
            return float("inf")
        err = max(err, float(np.abs(a.k_tilde - b.k_tilde).max()),
                  float(np.abs(a.c - b.c).max()), float(np.abs(a.qbar - b.qbar).max()),
                  float(np.abs(a.out - e.out).max()))
    return err


PINS = [pin_dense_at_ratio_one, pin_identical_keys_in_blocks, pin_identical_queries,
        pin_anchor_centred_query, pin_log_mass_identity, pin_golden_single_block,
        pin_golden_tiny_forward, pin_bruteforce_topk, pin_scores_are_block_mass_order,
        pin_invariances, pin_literal_copies, pin_block_means, pin_dense_reference,
        pin_diagnostics, pin_context_dense_at_ratio_one, pin_context_identical_keys,
        pin_context_outside_budget]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    assert pin() < TOL


def test_topk_count_rounding():
    # "top 10%" of nKB blocks at the workloads' sizes, and the small cases
    assert O.topk_count(0.125, 16) == 2
    assert O.topk_count(0.1, 256) == 26
    assert O.topk_count(0.1, 473) == 48
    assert O.topk_count(0.1, 1890) == 189
    assert O.topk_count(0.2, 1890) == 378
    assert O.topk_count(0.3, 1890) == 567
    assert O.topk_count(1.0, 1890) == 1890
    assert O.topk_count(1e-9, 50) == 1
    for bad in (0.0, -0.1, 1.5, float("nan")):
        with pytest.raises(ValueError):
            O.topk_count(bad, 10)


# ------------------------------------------------------------- qualitative claims (pages)

def _mixture(seed, H, N, d, ncomp, spread, sorted_layout):
    rng = np.random.default_rng(seed)
    mu = rng.standard_normal((H, ncomp, d))
    comp = rng.integers(0, ncomp, size=(H, N))
    Q = np.stack([mu[h, comp[h]] for h in range(H)]) + spread * rng.standard_normal((H, N, d))
    K = np.stack([mu[h, comp[h]] for h in range(H)]) + spread * rng.standard_normal((H, N, d))
    V = rng.standard_normal((H, N, d))
    if sorted_layout:
        perm = np.stack([np.argsort(comp[h] + 0.5 * rng.random(N), kind="stable")
                         for h in range(H)])
    else:
        perm = np.stack([rng.permutation(N) for _ in range(H)])
    return Q, K, V, perm


def test_reweight_lowers_log_mass_error():
    """Spark-H3 blog, "Spark-Reweight" table: weighted summaries with the log-mass bias have a
    smaller absolute log-mass error than mean pooling at 10% density (direction only)."""
    Q, K, V, perm = _mixture(41, 1, 1024, 32, 8, 0.6, sorted_layout=False)
    offs = np.arange(0, 1025, 32)
    errs = {}
    for mode in ("reweight", "meanpool"):
        r = O.forward_head(Q[0], K[0], V[0], perm[0], perm[0], offs, offs, 0.1, mode=mode,
                           blocks=[])
        Qp, Kp = Q[0][perm[0]], K[0][perm[0]]
        errs[mode] = np.mean([O.log_mass_error(Qp[offs[A]:offs[A + 1]], Kp, offs, r.sel[A],
                                               r.k_tilde, r.c) for A in range(len(offs) - 1)])
    assert errs["reweight"] < errs["meanpool"]


def test_reblock_layout_raises_recall():
    """Spark-H3 blog, "Spark-Reblock" table: grouping similar tokens raises attention-mass
    recall at the same Top-K budget (direction only)."""
    rec = {}
    for sorted_layout in (False, True):
        Q, K, V, perm = _mixture(42, 1, 1024, 32, 8, 0.6, sorted_layout)
        offs = np.arange(0, 1025, 32)
        r = O.forward_head(Q[0], K[0], V[0], perm[0], perm[0], offs, offs, 0.1, blocks=[])
        Qp, Kp = Q[0][perm[0]], K[0][perm[0]]
        rec[sorted_layout] = np.mean([O.attention_mass_recall(Qp[offs[A]:offs[A + 1]], Kp,
                                                              offs, r.sel[A])
                                      for A in range(len(offs) - 1)])
    assert rec[True] > rec[False]


# ------------------------------------------------------------------- planted mistakes

def _mut_drop_log_size(orig):
    def f(Kp_B, Vp_B, qbar, scale):
        kt, vt, b, c = orig(Kp_B, Vp_B, qbar, scale)
        return kt, vt, b, b
    return "summarize_block", f


def _mut_uniform_weights(orig):
    def f(Kp_B, Vp_B, qbar, scale):
        kt = Kp_B.mean(0); vt = Vp_B.mean(0)
        s = scale * (Kp_B @ qbar)
        b = math.log(np.mean(np.exp(s))) - scale * float(qbar @ kt)
        return kt, vt, b, b + math.log(Kp_B.shape[0])
    return "summarize_block", f


def _mut_value_from_keys(orig):
    def f(Kp_B, Vp_B, qbar, scale):
        return orig(Kp_B, Kp_B, qbar, scale)
    return "summarize_block", f


def _mut_sign_bias(orig):
    def f(Kp_B, Vp_B, qbar, scale):
        kt, vt, b, c = orig(Kp_B, Vp_B, qbar, scale)
        return kt, vt, -b, -b + math.log(Kp_B.shape[0])
    return "summarize_block", f


def _mut_anchor_half(orig):
    return "anchor", lambda Q: np.asarray(Q)[: len(Q) // 2].mean(0)


def _mut_no_scale(orig):
    def f(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale, **kw):
        return orig(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, 1.0, **kw)
    return "attend_block", f


def _mut_context_own_softmax(orig):
    # context normalised by a softmax of its own and averaged in, instead of sharing the row
    def f(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale, Kc=None, Vc=None):
        o = orig(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale)
        if Kc is None or not len(Kc):
            return o
        L = scale * (Qp_A @ Kc.T)
        P = np.exp(L - L.max(1, keepdims=True))
        return 0.5 * o + 0.5 * (P / P.sum(1, keepdims=True)) @ Vc
    return "attend_block", f


def _mut_context_unscaled(orig):
    def f(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale, Kc=None, Vc=None):
        return orig(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale,
                    Kc=None if Kc is None else Kc / scale, Vc=Vc)
    return "attend_block", f


def _mut_context_values_from_keys(orig):
    def f(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale, Kc=None, Vc=None):
        return orig(Qp_A, Kp, Vp, k_offsets, sel_A, kt, vt, c, scale, Kc=Kc, Vc=Kc)
    return "attend_block", f


def _mut_ties_to_larger(orig):
    def f(scores_A, k):
        idx = np.arange(len(scores_A))
        return np.sort(np.lexsort((-idx, -scores_A))[:k])
    return "route_block", f


def _mut_ignore_perm(orig):
    return "gather_rows", lambda X, perm: np.asarray(X, dtype=np.float64)


def _mut_transposed_scores(orig):
    return "route_scores", lambda qb, kb, scale: scale * (kb @ qb.T)


def _mut_block_mean_off_by_one(orig):
    def f(Xp, offsets):
        offsets = np.asarray(offsets)
        return np.stack([Xp[offsets[b]:max(offsets[b + 1] - 1, offsets[b] + 1)].mean(0)
                         for b in range(len(offsets) - 1)])
    return "block_means", f


def _mut_lowest_scores(orig):
    def f(scores_A, k):
        return orig(-scores_A, k)
    return "route_block", f


MUTATIONS = [_mut_drop_log_size, _mut_uniform_weights, _mut_value_from_keys, _mut_sign_bias,
             _mut_anchor_half, _mut_no_scale, _mut_ties_to_larger, _mut_ignore_perm,
             _mut_transposed_scores, _mut_lowest_scores, _mut_block_mean_off_by_one,
             _mut_context_own_softmax, _mut_context_unscaled, _mut_context_values_from_keys]


@pytest.mark.parametrize("mutation", MUTATIONS, ids=lambda f: f.__name__)
def test_pins_catch_planted_mistake(mutation, monkeypatch):
    name, bad = mutation(getattr(O, name_of(mutation)))
    monkeypatch.setattr(O, name, bad)
    caught = []
    for pin in PINS:
        try:
            e = pin()
        except Exception:                                   # a crash also counts as caught
            e = float("inf")
        if not e < TOL:
            caught.append(pin.__name__)
    assert caught, f"no pin caught {mutation.__name__}"


def name_of(mutation):
    return mutation(lambda *a, **k: None)[0]


# ---------------------------------------------------------------- threshold routing (T1)

def test_threshold_routing_is_affine_invariant_and_monotone():
    """mu + tau*sigma moves with any positive affine change of the scores, so the selection
    does not (a variance in place of sigma, or a dropped mu, breaks this); a larger tau never
    selects more."""
    rng = np.random.default_rng(40)
    for _ in range(50):
        S = rng.standard_normal(300) * rng.uniform(0.1, 5) + rng.uniform(-3, 3)
        tau = rng.uniform(-1, 2.5)
        a = O.route_threshold_block(S, tau, 300)
        for scale, shift in ((3.7, 0.0), (0.21, 5.0), (1.0, -11.0)):
            b = O.route_threshold_block(S * scale + shift, tau, 300)
            assert np.array_equal(a, b)
        c = O.route_threshold_block(S, tau + 0.3, 300)
        assert set(c.tolist()) <= set(a.tolist())


def test_threshold_routing_gaussian_fraction_and_limits():
    """For Gaussian scores the selected fraction is the normal tail 1 - Phi(tau); a very
    negative tau keeps every block, a very large one none; ties at the threshold stay out."""
    from scipy.stats import norm
    rng = np.random.default_rng(41)
    S = rng.standard_normal(200000)
    for tau in (-0.5, 0.0, 1.0, 2.0):
        frac = len(O.route_threshold_block(S, tau, len(S))) / len(S)
        assert abs(frac - (1 - norm.cdf(tau))) < 5e-3
    small = rng.standard_normal(40)
    assert len(O.route_threshold_block(small, -50.0, 40)) == 40
    assert len(O.route_threshold_block(small, 50.0, 40)) == 0
    assert len(O.route_threshold_block(np.full(10, 2.0), 0.0, 10)) == 0     # sigma = 0


def test_threshold_routing_cap_keeps_the_top_blocks():
    """With more blocks above the threshold than the cap, the cap's top blocks by score (ties to
    the smaller index) are kept, i.e. the Top-K router's choice."""
    rng = np.random.default_rng(42)
    S = np.round(rng.standard_normal(500), 1)          # many exact ties
    sel = O.route_threshold_block(S, -1.0, 37)
    assert len(sel) == 37
    assert np.array_equal(sel, O.route_block(S, 37))
    # brute force on a tiny case: the cap's set by enumeration of the order
    S = np.array([0.3, 2.0, 2.0, -1.0, 1.5, 2.0, 0.0])
    assert O.route_threshold_block(S, -0.2, 2).tolist() == [1, 2]


def test_threshold_routing_hand_case():
    """Closed form: S = (0, 0, 0, 0, 10) has mu = 2 and sigma = 4 (population), so tau = -0.4
    puts the threshold at 0.4 (only block 4 is above) and tau = -0.6 at -0.4 (all are)."""
    S = np.array([0.0, 0.0, 0.0, 0.0, 10.0])
    assert O.route_threshold_block(S, -0.4, 5).tolist() == [4]
    assert O.route_threshold_block(S, -0.6, 5).tolist() == [0, 1, 2, 3, 4]
    assert O.route_threshold_block(S, 1.9, 5).tolist() == [4]       # 9.6 < 10
    assert O.route_threshold_block(S, 2.0, 5).tolist() == []        # 10 is not above 10


def test_empty_selection_is_the_compressed_branch_alone():
    """Threshold routing may select no block (T1): the attention is then the compressed branch
    alone, which for blocks of identical keys is still dense attention (pin P2's identity)."""
    rng = np.random.default_rng(43)
    d, nb, bs = 16, 6, 5
    N = nb * bs
    ko = np.arange(0, N + 1, bs)
    K = np.repeat(rng.standard_normal((nb, d)), bs, axis=0)
    V = rng.standard_normal((N, d))
    Q = rng.standard_normal((7, d))
    qbar = rng.standard_normal(d)
    kt, vt, c = O.summarize(K, V, ko, qbar, 1.0 / math.sqrt(d))
    got = O.attend_block(Q, K, V, ko, np.zeros(0, dtype=np.int64), kt, vt, c, 1.0 / math.sqrt(d))
    assert np.abs(got - O.dense_attention(Q, K, V)).max() < 1e-12
