"""GPU parity of the threshold-routing comparator (Sol-Attn's mu + tau*sigma cutoff, as the
Spark-H3 blog's "Discussion" describes it) and of the attention with a per-query-block number
of selected blocks, against the oracle's ``route_threshold_block`` and ``attend_block``.

The GPU takes mu, sigma and the threshold in fp32, the oracle in float64: a block may land on
different sides only if its score lies within 1e-5 of the score scale from the threshold (or,
for a capped row, from the cap's last score).  The attention is compared with the oracle run on
the GPU's selection."""

import math

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (
    spark_bsa_anchor, spark_bsa_attend_var, spark_bsa_gather_kv_summarize, spark_bsa_gather_q,
    spark_bsa_read_error, spark_bsa_route_threshold)
from oracle import spark_oracle as O
from test_gpu_parity import custom_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check_row(g, S, tau, kcap):
    """g: the GPU's selection of one row; S: the oracle's scores of that row."""
    ref = O.route_threshold_block(S, tau, kcap)
    eps = 1e-5 * max(float(np.abs(S).max()), 1e-30)
    assert (np.diff(g) > 0).all() and len(g) <= kcap
    if set(g.tolist()) == set(ref.tolist()):
        return 0
    thr = S.mean() + tau * S.std()
    above = np.flatnonzero(S > thr)
    if len(above) > kcap:                      # capped: the Top-K rule at the cap's last score
        kth = np.sort(S)[::-1][kcap - 1]
        diff = set(g.tolist()) ^ set(ref.tolist())
        assert all(abs(S[b] - kth) <= eps for b in diff), "capped row differs beyond ties"
    else:
        diff = set(g.tolist()) ^ set(ref.tolist())
        assert all(abs(S[b] - thr) <= eps for b in diff), "row differs beyond the threshold"
    return 1


@pytest.mark.parametrize("tau,cap_frac,d,dtype", [(1.0, 1.0, 128, "bf16"), (0.5, 0.1, 128, "bf16"),
                                                  (2.0, 1.0, 64, "fp32"), (-0.3, 0.5, 128, "fp32")])
def test_threshold_routing_and_variable_attention(tau, cap_frac, d, dtype):
    x = custom_inputs(110 + d, H=2, N=3300, d=d, dtype=dtype, lo=30, hi=128, lo_k=1, hi_k=128)
    H, N, _ = x["Q"].shape
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    Qp, qbar_blocks = spark_bsa_gather_q(x["Q"], x["q_perm"], x["q_offsets"], err=err)
    qbar = spark_bsa_anchor(qbar_blocks, x["q_offsets"], N)
    Kp, Vp, kbar, kt, vt, cb = spark_bsa_gather_kv_summarize(x["K"], x["V"], x["k_perm"],
                                                             x["k_offsets"], qbar, err=err)
    nkb = x["k_offsets"].numel() - 1
    kcap = max(1, int(nkb * cap_frac))
    sel, count = spark_bsa_route_threshold(qbar_blocks, kbar, tau, kcap, err=err)
    out = spark_bsa_attend_var(Qp, Kp, Vp, kt, vt, cb, sel, count, x["q_perm"], x["q_offsets"],
                               x["k_offsets"], out_dtype=torch.float32, err=err)
    assert spark_bsa_read_error(err) == 0
    scale = 1.0 / math.sqrt(d)
    for h in range(H):
        hi = P.head_inputs(x, h)
        ref = P.oracle_head(x, h, 1.0, blocks=[], hi=hi)        # summaries, anchor, scores
        cnt = count[h].cpu().numpy()
        sh = sel[h].cpu().numpy().astype(np.int64)
        qo = hi["q_offsets"]
        Qp64 = hi["Q"][hi["q_perm"]]
        Kp64, Vp64 = hi["K"][hi["k_perm"]], hi["V"][hi["k_perm"]]
        got = P.to64(out[h])
        for A in range(len(qo) - 1):
            g = sh[A, :cnt[A]]
            check_row(g, ref.scores[A], tau, kcap)
            o = O.attend_block(Qp64[qo[A]:qo[A + 1]], Kp64, Vp64, hi["k_offsets"], g,
                               ref.k_tilde, ref.v_tilde, ref.c, scale)
            rows = hi["q_perm"][qo[A]:qo[A + 1]]
            P.compare_out(got[rows], o, f"head {h} block {A}")
        assert cnt.min() >= 0 and cnt.max() <= kcap
