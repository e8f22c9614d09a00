"""Routing inside the attention kernel (spark_bsa_forward_fused, spark_bsa_attend_fused) against
the path with the routing kernel: the in-kernel routing does the routing kernel's arithmetic
(sequential fp32 FMA scores, exact radix select, ties to the smaller block), so selections and
outputs must be equal bit for bit; the float64 oracle checks them as well."""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (SparkError, spark_bsa_attend,
                                                spark_bsa_attend_fused, spark_bsa_forward,
                                                spark_bsa_forward_fused,
                                                spark_bsa_fused_supported, spark_bsa_read_error,
                                                workspace_views)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs
from test_gpu_parity import custom_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _both(x, ratio):
    H, N, d = x["Q"].shape
    nqb, nkb = x["q_offsets"].numel() - 1, x["k_offsets"].numel() - 1
    ref, wr, lay = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                     x["q_offsets"], x["k_offsets"], ratio)
    out, wf, _ = spark_bsa_forward_fused(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                         x["q_offsets"], x["k_offsets"], ratio)
    vr = workspace_views(wr, lay, H, N, d, nqb, nkb)
    vf = workspace_views(wf, lay, H, N, d, nqb, nkb)
    assert spark_bsa_read_error(vr["err"]) == 0
    assert spark_bsa_read_error(vf["err"]) == 0
    torch.cuda.synchronize()
    return ref, out, vr, vf


def _dev(x):
    return {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in x.items()}


@pytest.mark.parametrize("name", ["small-8x16384-d128-randperm", "384p-24x60480-d128"])
def test_fused_equals_routing_kernel_path(name):
    w = WORKLOADS[name]
    x = _dev(make_inputs(w))
    nkb = x["k_offsets"].numel() - 1
    assert spark_bsa_fused_supported(w.d, nkb, w.ratio)
    ref, out, vr, vf = _both(x, w.ratio)
    assert torch.equal(vf["sel"], vr["sel"]), "selections differ"
    assert torch.equal(out, ref), "outputs differ"


@pytest.mark.parametrize("lo,hi,ratio", [(20, 128, 0.1), (1, 128, 0.3), (100, 128, 0.05)])
def test_fused_ragged_blocks_against_oracle(lo, hi, ratio):
    x = custom_inputs(211, H=3, N=5000, d=128, dtype="bf16", lo=lo, hi=hi)
    ref, out, vr, vf = _both(x, ratio)
    assert torch.equal(vf["sel"], vr["sel"])
    assert torch.equal(out, ref)
    nkb = x["k_offsets"].numel() - 1
    k = vf["sel"].shape[-1]
    for h in range(3):
        o = P.oracle_head(x, h, ratio)
        P.compare_sel(vf["sel"][h].cpu().numpy().astype(np.int64), o.sel, o.scores, k)
        sel = vf["sel"][h].cpu().numpy().astype(np.int64)
        o2 = P.oracle_head(x, h, ratio, sel=sel)
        P.compare_out(P.to64(out[h]), o2.out, f"fused head {h}")


def test_fused_fewer_query_blocks_than_sms_and_fp32_inputs():
    x = custom_inputs(212, H=1, N=1500, d=128, dtype="fp32", lo=60, hi=128)
    ref, out, vr, vf = _both(x, 0.25)
    assert torch.equal(vf["sel"], vr["sel"])
    assert torch.equal(out, ref)


def test_fused_attend_step_equals_attend_with_routing_kernel_selection():
    w = WORKLOADS["small-8x16384-d128-randperm"]
    x = _dev(make_inputs(w))
    H, N, d = x["Q"].shape
    nqb, nkb = x["q_offsets"].numel() - 1, x["k_offsets"].numel() - 1
    _, ws, lay = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                   x["q_offsets"], x["k_offsets"], w.ratio)
    v = workspace_views(ws, lay, H, N, d, nqb, nkb)
    ref = spark_bsa_attend(v["Qp"], v["Kp"], v["Vp"], v["k_tilde"], v["v_tilde"], v["cbias"],
                           v["sel"], x["q_perm"], x["q_offsets"], x["k_offsets"])
    sel_out = torch.full_like(v["sel"], -1)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = spark_bsa_attend_fused(v["Qp"], v["Kp"], v["Vp"], v["k_tilde"], v["v_tilde"],
                                 v["cbias"], v["qbar_blocks"], v["kbar"], lay.k, x["q_perm"],
                                 x["q_offsets"], x["k_offsets"], sel_out=sel_out, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(sel_out, v["sel"])
    assert torch.equal(out, ref)


def test_fused_unsupported_shapes_are_refused():
    assert not spark_bsa_fused_supported(64, 100, 0.1)          # d = 64
    assert not spark_bsa_fused_supported(128, 100, 1.0)         # k = nkb: no compressed branch
    assert not spark_bsa_fused_supported(128, 12000, 0.1)       # routing state too large
    w = WORKLOADS["tiny-1x1024-d64-fp32"]
    x = _dev(make_inputs(w))
    with pytest.raises(SparkError) as e:
        spark_bsa_forward_fused(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                x["q_offsets"], x["k_offsets"], w.ratio)
    assert e.value.status == 2                                   # SPARK_ERR_UNSUPPORTED
