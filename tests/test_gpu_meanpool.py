"""GPU parity of the baseline BSA compressed branch (the blog's ablation comparator, section
"Spark-Reblock", BSA equations: unselected blocks as their uniform mean key and value repeated
|B| times) against the oracle's ``mode="meanpool"``.  Routing and attention are the same
kernels as in the Spark-Reweight path; only the summaries and their offsets differ."""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (
    spark_bsa_attend, spark_bsa_gather_kv_meanpool, spark_bsa_gather_q, spark_bsa_read_error,
    spark_bsa_route, spark_bsa_topk_count)
from oracle import spark_oracle as O
from test_gpu_parity import custom_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("d,dtype,ratio", [(128, "bf16", 0.1), (64, "fp32", 0.3),
                                           (128, "fp32", 1.0)])
def test_meanpool_branch_matches_oracle(d, dtype, ratio):
    x = custom_inputs(100 + d, H=2, N=2700, d=d, dtype=dtype, lo=20, hi=128, lo_k=1, hi_k=128)
    H, N, _ = x["Q"].shape
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    Qp, qbar_blocks = spark_bsa_gather_q(x["Q"], x["q_perm"], x["q_offsets"], err=err)
    Kp, Vp, kbar, kt, vt, cb = spark_bsa_gather_kv_meanpool(x["K"], x["V"], x["k_perm"],
                                                            x["k_offsets"], err=err)
    nkb = x["k_offsets"].numel() - 1
    k = spark_bsa_topk_count(nkb, ratio)
    sel = spark_bsa_route(qbar_blocks, kbar, k, err=err)
    out = spark_bsa_attend(Qp, Kp, Vp, kt, vt, cb, sel, x["q_perm"], x["q_offsets"],
                           x["k_offsets"], out_dtype=torch.float32, err=err)
    assert spark_bsa_read_error(err) == 0
    sizes = np.diff(x["k_offsets"].cpu().numpy()).astype(np.float64)
    for h in range(H):
        hi = P.head_inputs(x, h)
        ref = O.forward_head(hi["Q"], hi["K"], hi["V"], hi["q_perm"], hi["k_perm"],
                             hi["q_offsets"], hi["k_offsets"], ratio, mode="meanpool",
                             blocks=[])
        gsel = sel[h].cpu().numpy().astype(np.int64)
        P.compare_sel(gsel, ref.sel, ref.scores, k)
        # mean key and value within 2 bf16 ulps, offsets log|B|
        for got, refv in ((kt[h], ref.k_tilde), (vt[h], ref.v_tilde)):
            g = P.to64(got)
            assert (np.abs(g - refv) <= 2 * 2.0 ** -8 * np.abs(refv) + 1e-3).all()
        assert np.abs(P.to64(cb[h]) - np.log(sizes)).max() < 1e-5
        full = O.forward_head(hi["Q"], hi["K"], hi["V"], hi["q_perm"], hi["k_perm"],
                              hi["q_offsets"], hi["k_offsets"], ratio, mode="meanpool",
                              sel=gsel)
        P.compare_out(P.to64(out[h]), full.out, f"meanpool head {h}")
