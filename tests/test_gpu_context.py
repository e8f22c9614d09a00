"""GPU parity of the context (sink) token path against the float64 CPU oracle.

Context tokens (Spark-H3 blog, section "Spark-Reblock": context/sink tokens stay exact and
sit outside the video-block Top-K budget) enter the attention as extra exact key tiles after
the selected video blocks.  The cases cover ragged context lengths around the 128-row tile,
both head sizes and input dtypes, the dense limit at ratio 1, the step entry points with the
oracle's selection injected, an empty context (bit-identical to the call without context)
and the 768p workload with 512 context tokens in bench.py's launch configuration.
"""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (
    spark_bsa_anchor, spark_bsa_attend_ctx, spark_bsa_context_bf16, spark_bsa_forward,
    spark_bsa_forward_ctx, spark_bsa_gather_kv_summarize, spark_bsa_gather_q,
    spark_bsa_read_error, spark_bsa_route, spark_bsa_topk_count, workspace_views)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs, sample_units
from oracle import spark_oracle as O
from test_gpu_parity import custom_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def with_context(x, seed, nc):
    g = torch.Generator().manual_seed(seed)
    H, _, d = x["Q"].shape
    x = dict(x)
    x["Kc"] = (torch.randn(H, nc, d, generator=g) * 1.5).to(x["Q"].dtype).to(DEV)
    x["Vc"] = torch.randn(H, nc, d, generator=g).to(x["Q"].dtype).to(DEV)
    return x


def check_forward_ctx(x, ratio, heads=None, blocks_per_head=None, seed=0):
    out, ws, layout = spark_bsa_forward_ctx(x["Q"], x["K"], x["V"], x["Kc"], x["Vc"],
                                            x["q_perm"], x["k_perm"], x["q_offsets"],
                                            x["k_offsets"], ratio)
    H, N, d = x["Q"].shape
    nqb, nkb = x["q_offsets"].numel() - 1, x["k_offsets"].numel() - 1
    views = workspace_views(ws, layout, H, N, d, nqb, nkb)
    assert spark_bsa_read_error(views["err"]) == 0
    k = layout.k
    heads = range(H) if heads is None else heads
    rng = np.random.default_rng(seed)
    for h in heads:
        hi = P.head_inputs(x, h)
        ref = P.oracle_head(x, h, ratio, blocks=[], hi=hi)
        gsel = views["sel"][h].cpu().numpy().astype(np.int64)
        P.compare_sel(gsel, ref.sel, ref.scores, k)
        if blocks_per_head is None:
            blocks = list(range(nqb))
        else:
            blocks = sorted(rng.choice(nqb, size=min(blocks_per_head, nqb),
                                       replace=False).tolist())
            if nqb - 1 not in blocks:
                blocks.append(nqb - 1)
        ref2 = P.oracle_head(x, h, ratio, blocks=blocks, sel=gsel, hi=hi)
        rows = P.rows_of_blocks(hi["q_perm"], hi["q_offsets"], blocks)
        P.compare_out(P.to64(out[h])[rows], ref2.out[rows], f"head {h}")
    return out


def test_tiny_context_workload_full():
    w = WORKLOADS["tiny-ctx77-1x1024-d64-fp32"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    out = check_forward_ctx(x, w.ratio)
    assert out.dtype == torch.float32


def test_small_context_workload_full():
    w = WORKLOADS["small-ctx300-8x16384-d128-randperm"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    check_forward_ctx(x, w.ratio)


@pytest.mark.parametrize("nc", [1, 127, 128, 129, 300])
@pytest.mark.parametrize("d,dtype", [(64, "fp32"), (128, "bf16")])
def test_ragged_context(nc, d, dtype):
    x = custom_inputs(61 + nc + d, H=2, N=2101, d=d, dtype=dtype, lo=1, hi=128, lo_k=30,
                      hi_k=128)
    check_forward_ctx(with_context(x, 62 + nc, nc), 0.1)


def test_context_ratio_one_is_dense_attention():
    x = with_context(custom_inputs(63, H=2, N=1500, d=128, dtype="bf16", lo=40, hi=128), 64, 200)
    out = check_forward_ctx(x, 1.0)
    for h in range(2):
        q = P.bf16_64(x["Q"][h])
        k = np.concatenate([P.bf16_64(x["K"][h]), P.bf16_64(x["Kc"][h])])
        v = np.concatenate([P.bf16_64(x["V"][h]), P.bf16_64(x["Vc"][h])])
        P.compare_out(P.to64(out[h]), O.dense_attention(q, k, v), "dense with context")


def test_sink_logit_far_above_the_video_rows():
    """A context (sink) key ~100 nats above every video logit of every query: the context
    tiles come after the video tiles, so the reference taken from the first two tiles is far
    below the row maxima and the attention repeats those query blocks with the true maxima."""
    x = custom_inputs(75, H=2, N=2000, d=128, dtype="bf16", lo=40, hi=128)
    H, N, d = x["Q"].shape
    g = torch.Generator().manual_seed(76)
    u = torch.randn(d, generator=g, dtype=torch.float64)
    u /= u.norm()
    x["Q"] = (x["Q"].cpu().double() + 6.0 * u).to(x["Q"].dtype).to(DEV)
    x = with_context(x, 77, 40)
    Kc = x["Kc"].cpu().clone()
    Kc[:, 17] = (300.0 * u).to(Kc.dtype)
    x["Kc"] = Kc.to(DEV)
    check_forward_ctx(x, 0.2)


def test_empty_context_is_the_plain_call():
    x = custom_inputs(65, H=2, N=3000, d=128, dtype="bf16", lo=50, hi=128)
    a, _, _ = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                x["q_offsets"], x["k_offsets"], 0.2)
    b, _, _ = spark_bsa_forward_ctx(x["Q"], x["K"], x["V"], None, None, x["q_perm"],
                                    x["k_perm"], x["q_offsets"], x["k_offsets"], 0.2)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_context_step_entry_points():
    """Context conversion + attention step with the oracle's selection injected."""
    x = with_context(custom_inputs(66, H=2, N=2500, d=128, dtype="fp32", lo=40, hi=128), 67, 150)
    H, N, _ = x["Q"].shape
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    Qp, qbar_blocks = spark_bsa_gather_q(x["Q"], x["q_perm"], x["q_offsets"], err=err)
    qbar = spark_bsa_anchor(qbar_blocks, x["q_offsets"], N)
    Kp, Vp, kbar, kt, vt, cb = spark_bsa_gather_kv_summarize(x["K"], x["V"], x["k_perm"],
                                                             x["k_offsets"], qbar, err=err)
    Kcb, Vcb = spark_bsa_context_bf16(x["Kc"], x["Vc"])
    torch.cuda.synchronize()
    assert torch.equal(Kcb, x["Kc"].to(torch.bfloat16))
    assert torch.equal(Vcb, x["Vc"].to(torch.bfloat16))
    ratio = 0.15
    nkb = x["k_offsets"].numel() - 1
    k = spark_bsa_topk_count(nkb, ratio)
    refs = [P.oracle_head(x, h, ratio, blocks=[]) for h in range(H)]
    inj = torch.from_numpy(np.stack([r.sel for r in refs]).astype(np.int32)).to(DEV)
    out = spark_bsa_attend_ctx(Qp, Kp, Vp, kt, vt, cb, inj, Kcb, Vcb, x["q_perm"],
                               x["q_offsets"], x["k_offsets"], out_dtype=torch.float32, err=err)
    assert spark_bsa_read_error(err) == 0
    for h in range(H):
        full = P.oracle_head(x, h, ratio)
        P.compare_out(P.to64(out[h]), full.out, f"attend_ctx head {h}")


def test_full_size_context_workload():
    w = WORKLOADS["768p-ctx512-24x241920-d128"]
    x = make_inputs(w, device=DEV)
    nqb = x["q_offsets"].numel() - 1
    heads = sorted(sample_units(w, 2, nqb))
    check_forward_ctx(x, w.ratio, heads=heads, blocks_per_head=6, seed=w.seed)
    del x
    torch.cuda.empty_cache()
