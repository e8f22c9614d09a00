"""GPU parity of the Spark-Reblock partitioner against the float64 CPU oracle.

The partition is an integer result decided by floating-point projections, so the checks
compare what is unique and validate the rest:
  * whitening: the second moment M (fp32 sums) against the oracle's, W = M^{1/2} (fp32
    Newton-Schulz) against the eigendecomposition square root of the same M, and the bf16
    unit rows against the oracle's rows computed with the GPU's W;
  * every tree level, step by step from the GPU's own previous permutation and unit rows:
    each node keeps its tokens, the left child has exactly its capacity, both children keep
    the node's order, and a token may sit on the other side than in the oracle's split only
    if its projection is within 1e-4 * max|p| of the capacity-th largest projection;
  * planted well-separated clusters: the whole partition equals the oracle's exactly;
  * the separate-keys mode is the role swap of the query partition, bit for bit;
  * the 768p workload in full: valid permutations, the fused call equals the step-by-step
    run, and levels 0, 1 and the last are checked against the oracle on one head.
"""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (spark_reblock, spark_reblock_level,
                                                spark_reblock_levels, spark_reblock_whiten)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs
from oracle import spark_oracle as SO
from oracle import spark_reblock as R

pytestmark = pytest.mark.gpu
DEV = "cuda"
NEAR_TIE_REL = 1e-4


def mixture(seed, H, N, d, ncomp, spread, dtype):
    g = torch.Generator().manual_seed(seed)
    mu = torch.randn(H, ncomp, d, generator=g) * torch.linspace(1.5, 0.3, d)
    comp = torch.randint(0, ncomp, (H, N), generator=g)
    hidx = torch.arange(H)[:, None]
    Q = mu[hidx, comp] + spread * torch.randn(H, N, d, generator=g)
    K = mu[hidx, comp] + spread * torch.randn(H, N, d, generator=g)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    return Q.to(tdt).to(DEV).contiguous(), K.to(tdt).to(DEV).contiguous()


def check_level(X64, perm_in, perm_out, offsets, nodes):
    """One level of one head against the oracle's split of the same nodes."""
    inv = np.empty(len(perm_in), dtype=np.int64)
    inv[perm_in] = np.arange(len(perm_in))
    moved = 0
    for lo, mid, hi in nodes:
        a, m, e = int(offsets[lo]), int(offsets[mid]), int(offsets[hi])
        toks = perm_in[a:e]
        gl, gr = perm_out[a:m], perm_out[m:e]
        assert np.array_equal(np.sort(np.r_[gl, gr]), np.sort(toks)), "node lost tokens"
        gl_pos, gr_pos = inv[gl] - a, inv[gr] - a
        assert (np.diff(gl_pos) > 0).all() and (np.diff(gr_pos) > 0).all(), "child not stable"
        left_ref, _, p = R.split_node(X64[toks], m - a)
        diff = np.setxor1d(gl_pos, left_ref)
        if diff.size:
            thr = float(np.sort(p)[::-1][m - a - 1])
            tol = NEAR_TIE_REL * float(np.abs(p).max())
            assert np.all(np.abs(p[diff] - thr) <= tol), (
                f"node {lo}-{hi}: {diff.size} tokens on the wrong side beyond the near-tie rule")
            moved += diff.size
    return moved


@pytest.mark.parametrize("d,dtype", [(64, "fp32"), (128, "bf16"), (128, "fp32")])
def test_whiten_matches_oracle(d, dtype):
    Q, K = mixture(71 + d, H=2, N=3001, d=d, ncomp=8, spread=0.4, dtype=dtype)
    ws, lay, v = spark_reblock_whiten(Q, K, 64)
    torch.cuda.synchronize()
    for h in range(2):
        K64 = P.bf16_64(K[h]) if dtype == "bf16" else P.to64(K[h])
        Q64 = P.bf16_64(Q[h]) if dtype == "bf16" else P.to64(Q[h])
        Mref = R.second_moment(K64)
        Mg = P.to64(v["M"][h])
        assert np.abs(Mg - Mref).max() <= 1e-5 * np.abs(Mref).max()
        Wref = R.psd_sqrt(Mg)
        Wg = P.to64(v["W"][h])
        assert np.abs(Wg - Wref).max() <= 2e-3 * np.abs(Wref).max()
        Xref = R.whiten_normalize(Q64, Wg)
        assert np.abs(P.to64(v["X"][h]) - Xref).max() <= 5e-3


@pytest.mark.parametrize("d,N,block", [(128, 5000, 64), (64, 2049, 128)])
def test_levels_match_oracle(d, N, block):
    H = 2
    Q, K = mixture(81 + d, H=H, N=N, d=d, ncomp=12, spread=0.5, dtype="bf16")
    ws, lay, v = spark_reblock_whiten(Q, K, block)
    offsets = R.fixed_block_offsets(N, block)
    levels = R.tree_levels(len(offsets) - 1)
    assert spark_reblock_levels(N, block) == len(levels) == lay.levels
    X64 = [P.to64(v["X"][h]) for h in range(H)]
    perm = torch.arange(N, dtype=torch.int32, device=DEV).repeat(H, 1).contiguous()
    for lv, nodes in enumerate(levels):
        out = spark_reblock_level(H, N, d, block, lv, perm, ws)
        torch.cuda.synchronize()
        for h in range(H):
            check_level(X64[h], perm[h].cpu().numpy().astype(np.int64),
                        out[h].cpu().numpy().astype(np.int64), offsets, nodes)
        perm = out
    # the fused call reproduces the step-by-step run
    qp, kp, offs = spark_reblock(Q, K, block)
    torch.cuda.synchronize()
    assert torch.equal(qp, perm) and torch.equal(kp, perm)
    assert np.array_equal(offs.cpu().numpy(), offsets)


@pytest.mark.parametrize("d,dtype,block,nclusters", [(64, "fp32", 64, 16), (128, "bf16", 32, 13)])
def test_planted_clusters_exact(d, dtype, block, nclusters):
    g = np.random.default_rng(90 + d)
    H = 2
    Qs, Ks, labs = [], [], []
    for h in range(H):
        centers = g.standard_normal((nclusters, d)) * 2.0
        lab = g.permutation(np.repeat(np.arange(nclusters), block))
        Qs.append(centers[lab] + 1e-3 * g.standard_normal((len(lab), d)))
        Ks.append(g.standard_normal((len(lab), d)) * np.linspace(2.0, 0.5, d))
        labs.append(lab)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    Q = torch.tensor(np.stack(Qs)).to(tdt).to(DEV).contiguous()
    K = torch.tensor(np.stack(Ks)).to(tdt).to(DEV).contiguous()
    qp, kp, offs = spark_reblock(Q, K, block)
    torch.cuda.synchronize()
    for h in range(H):
        q64 = P.bf16_64(Q[h]) if dtype == "bf16" else P.to64(Q[h])
        k64 = P.bf16_64(K[h]) if dtype == "bf16" else P.to64(K[h])
        rq, rk, roffs = R.reblock_head(q64, k64, block)
        assert np.array_equal(qp[h].cpu().numpy(), rq)
        assert np.array_equal(offs.cpu().numpy(), roffs)
        for B in range(nclusters):
            assert len(set(labs[h][rq[roffs[B]:roffs[B + 1]]])) == 1


def test_separate_mode_is_role_swap():
    Q, K = mixture(95, H=2, N=4000, d=128, ncomp=10, spread=0.5, dtype="bf16")
    qp, kp, _ = spark_reblock(Q, K, 128, mode="separate")
    qs, ks, _ = spark_reblock(K, Q, 128)
    qr, kr, _ = spark_reblock(Q, K, 128)
    torch.cuda.synchronize()
    assert torch.equal(kp, qs) and torch.equal(qp, qr) and torch.equal(kr, qr)
    assert torch.equal(ks, qs)


def test_reblocked_partition_raises_recall():
    """Blog "Spark-Reblock" ablation direction on the GPU partition: mixture tokens in random
    order; the reblocked layout has a higher attention-mass recall at 10% than fixed blocks
    over the token order."""
    H, N, d, b = 1, 4096, 64, 64
    g = torch.Generator().manual_seed(97)
    mu = torch.randn(16, d, generator=g)
    comp = torch.randint(0, 16, (N,), generator=g)
    Q = (mu[comp] + 0.6 * torch.randn(N, d, generator=g))[None].float().to(DEV).contiguous()
    K = (mu[comp] + 0.6 * torch.randn(N, d, generator=g))[None].float().to(DEV).contiguous()
    qp, kp, offs = spark_reblock(Q, K, b)
    torch.cuda.synchronize()
    q64, k64 = P.to64(Q[0]), P.to64(K[0])
    V = np.zeros_like(q64)
    o = offs.cpu().numpy().astype(np.int64)
    rec = {}
    for name, pq, pk in (("fixed", np.arange(N), np.arange(N)),
                         ("reblock", qp[0].cpu().numpy().astype(np.int64),
                          kp[0].cpu().numpy().astype(np.int64))):
        r = SO.forward_head(q64, k64, V, pq, pk, o, o, 0.1, blocks=[])
        Qp, Kp = q64[pq], k64[pk]
        rec[name] = np.mean([SO.attention_mass_recall(Qp[o[A]:o[A + 1]], Kp, o, r.sel[A])
                             for A in range(0, len(o) - 1, 4)])
    assert rec["reblock"] > rec["fixed"] + 0.05, rec


def test_full_size_768p_reblock():
    w = WORKLOADS["768p-24x241920-d128"]
    x = make_inputs(w, device=DEV)
    Q, K = x["Q"], x["K"]
    del x
    H, N, d = Q.shape
    block = 128
    qp, kp, offs = spark_reblock(Q, K, block)
    torch.cuda.synchronize()
    assert torch.equal(qp, kp)
    ref_order = torch.arange(N, dtype=torch.int32, device=DEV)
    for h in range(H):
        assert torch.equal(torch.sort(qp[h]).values, ref_order)
    offsets = R.fixed_block_offsets(N, block)
    assert np.array_equal(offs.cpu().numpy(), offsets)
    # step by step: levels 0, 1 and the last against the oracle on head 0
    ws, lay, v = spark_reblock_whiten(Q, K, block)
    levels = R.tree_levels(len(offsets) - 1)
    X64 = P.to64(v["X"][0])
    perm = torch.arange(N, dtype=torch.int32, device=DEV).repeat(H, 1).contiguous()
    for lv, nodes in enumerate(levels):
        out = spark_reblock_level(H, N, d, block, lv, perm, ws)
        if lv in (0, 1, len(levels) - 1):
            torch.cuda.synchronize()
            check_level(X64, perm[0].cpu().numpy().astype(np.int64),
                        out[0].cpu().numpy().astype(np.int64), offsets, nodes)
        perm = out
    torch.cuda.synchronize()
    assert torch.equal(perm, qp)
    del ws, v, Q, K
    torch.cuda.empty_cache()


def test_reblock_then_forward():
    """The partitioner's output drives the attention path: spark_reblock's permutation and
    offsets go straight into spark_bsa_forward, and the result matches the oracle run on the
    same layout; the reblocked layout also recalls more attention mass than a random one."""
    from block_sparse_attention_gather_b200 import spark_bsa_forward
    w = WORKLOADS["small-8x16384-d128-randperm"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    qp, kp, offs = spark_reblock(x["Q"], x["K"], 64)
    out, _, layout = spark_bsa_forward(x["Q"], x["K"], x["V"], qp, kp, offs, offs, w.ratio)
    torch.cuda.synchronize()
    y = dict(x, q_perm=qp, k_perm=kp, q_offsets=offs, k_offsets=offs)
    rng = np.random.default_rng(5)
    rec = {"reblock": [], "random": []}
    for h in (0, 5):
        hi = P.head_inputs(y, h)
        blocks = sorted(rng.choice(len(offs) - 1, size=6, replace=False).tolist())
        ref = P.oracle_head(y, h, w.ratio, blocks=blocks, hi=hi)
        rows = P.rows_of_blocks(hi["q_perm"], hi["q_offsets"], blocks)
        P.compare_out(P.to64(out[h])[rows], ref.out[rows], f"head {h}")
        for name, src in (("reblock", y), ("random", x)):
            hh = P.head_inputs(src, h)
            r = P.oracle_head(src, h, w.ratio, blocks=[], hi=hh)
            Qp, Kp = hh["Q"][hh["q_perm"]], hh["K"][hh["k_perm"]]
            o = hh["q_offsets"]
            rec[name].append(np.mean([SO.attention_mass_recall(Qp[o[A]:o[A + 1]], Kp,
                                                                hh["k_offsets"], r.sel[A])
                                      for A in range(0, len(o) - 1, 16)]))
    assert np.mean(rec["reblock"]) > np.mean(rec["random"]), rec
