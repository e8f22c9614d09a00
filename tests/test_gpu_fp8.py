"""GPU parity of the FP8-logit path against the float64 FP8 oracle (``oracle/spark_fp8.py``).

The quantisation is compared bit for bit (codes and power-of-two scales, the decision taken
from the same bf16 numbers on both sides); the attention with FP8 logits is compared with the
oracle's FP8 forward at the bf16 path's tolerance, the remaining differences being fp32
accumulation and the bf16 probabilities.  Its distance to the BF16 oracle is the FP8 format's
own error and is bounded separately.
"""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (
    SparkError, spark_bsa_anchor, spark_bsa_attend_fp8, spark_bsa_forward_fp8,
    spark_bsa_gather_kv_summarize, spark_bsa_gather_q, spark_bsa_quantize_fp8,
    spark_bsa_read_error, spark_bsa_topk_count, workspace_views)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs, sample_units
from oracle import spark_fp8 as F
from test_gpu_parity import custom_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def decode(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


@pytest.mark.parametrize("grouping", ["offsets", "tiles"])
@pytest.mark.parametrize("d", [64, 128])
def test_quantize_matches_oracle_bit_for_bit(grouping, d):
    g = torch.Generator().manual_seed(80 + d)
    H, R = 3, 1000
    x = torch.randn(H, R, d, generator=g) * torch.exp(torch.randn(H, R, 1, generator=g) * 2)
    x[1, 300:420] = 0.0                              # an all-zero group
    x[2, 5, 7] = 1e30                                # one huge value
    x = x.to(torch.bfloat16).to(DEV)
    if grouping == "offsets":
        sizes = torch.randint(1, 129, (R,), generator=g)
        offs = [0]
        for s in sizes.tolist():
            if offs[-1] >= R:
                break
            offs.append(min(R, offs[-1] + s))
        offsets = torch.tensor(offs, dtype=torch.int32, device=DEV)
        groups = F.offset_groups(offs)
    else:
        offsets = None
        groups = F.fixed_groups(R)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    codes, scales = spark_bsa_quantize_fp8(x, offsets, err=err)
    assert spark_bsa_read_error(err) == 0
    for h in range(H):
        ref, e = F.quantize_groups(P.bf16_64(x[h]), groups)
        assert np.array_equal(scales[h].cpu().double().numpy(), 2.0 ** e)
        sc = np.repeat(2.0 ** e, [hi - lo for lo, hi in groups])[:, None]
        got = decode(codes[h]) * sc
        assert np.array_equal(got, ref)


def oracle_fp8_head(x, h, ratio, blocks=None, sel=None, hi=None):
    hi = P.head_inputs(x, h) if hi is None else hi
    return F.forward_head_fp8(hi["Q"], hi["K"], hi["V"], hi["q_perm"], hi["k_perm"],
                              hi["q_offsets"], hi["k_offsets"], ratio, blocks=blocks, sel=sel,
                              Kc=hi["Kc"], Vc=hi["Vc"])


def check_forward_fp8(x, ratio, heads=None, blocks_per_head=None, seed=0):
    Kc, Vc = x.get("Kc"), x.get("Vc")
    out, ws, layout = spark_bsa_forward_fp8(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                            x["q_offsets"], x["k_offsets"], ratio, Kc=Kc, Vc=Vc)
    H, N, d = x["Q"].shape
    nqb, nkb = x["q_offsets"].numel() - 1, x["k_offsets"].numel() - 1
    views = workspace_views(ws, layout, H, N, d, nqb, nkb)
    assert spark_bsa_read_error(views["err"]) == 0
    k = layout.k
    heads = range(H) if heads is None else heads
    rng = np.random.default_rng(seed)
    worst = 0.0
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
        ref8 = oracle_fp8_head(x, h, ratio, blocks=blocks, sel=gsel, hi=hi)
        rows = P.rows_of_blocks(hi["q_perm"], hi["q_offsets"], blocks)
        got = P.to64(out[h])[rows]
        P.compare_out(got, ref8.out[rows], f"fp8 head {h}")
        ref16 = P.oracle_head(x, h, ratio, blocks=blocks, sel=gsel, hi=hi)
        rel16 = np.linalg.norm(got - ref16.out[rows]) / np.linalg.norm(ref16.out[rows])
        worst = max(worst, rel16)
    # distance to the bf16 oracle: the format's own error (oracle pin: <= 0.15 on random data)
    assert worst < 0.15, worst
    return out, worst


def test_tiny_fp8_is_unsupported_for_d64():
    w = WORKLOADS["tiny-1x1024-d64-fp32"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    with pytest.raises(SparkError):
        spark_bsa_forward_fp8(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"], x["q_offsets"],
                              x["k_offsets"], w.ratio)


def test_small_workload_fp8():
    w = WORKLOADS["small-8x16384-d128-randperm"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    check_forward_fp8(x, w.ratio, heads=[0, 5], blocks_per_head=40, seed=w.seed)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("ratio", [0.05, 0.3, 1.0])
def test_ragged_blocks_fp8(dtype, ratio):
    x = custom_inputs(90, H=2, N=3001, d=128, dtype=dtype, lo=1, hi=128, lo_k=20, hi_k=128)
    check_forward_fp8(x, ratio)


def test_context_fp8():
    x = custom_inputs(91, H=2, N=2200, d=128, dtype="bf16", lo=40, hi=128)
    g = torch.Generator().manual_seed(92)
    x["Kc"] = (torch.randn(2, 300, 128, generator=g) * 1.5).to(torch.bfloat16).to(DEV)
    x["Vc"] = torch.randn(2, 300, 128, generator=g).to(torch.bfloat16).to(DEV)
    check_forward_fp8(x, 0.15)


def test_fp8_far_key_forces_the_second_pass():
    from test_gpu_parity import plant_far_key
    x = custom_inputs(93, H=2, N=1800, d=128, dtype="bf16", lo=60, hi=128)
    x, _ = plant_far_key(x, 6.0, 300.0, 94)
    out, _, layout = spark_bsa_forward_fp8(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                           x["q_offsets"], x["k_offsets"], 1.0)
    for h in range(2):
        ref8 = oracle_fp8_head(x, h, 1.0)
        P.compare_out(P.to64(out[h]), ref8.out, f"fp8 far key head {h}")


def test_attend_fp8_step_entry_points():
    """Quantisation and attention steps on caller buffers, the oracle's selection injected."""
    x = custom_inputs(95, H=2, N=2500, d=128, dtype="fp32", lo=40, hi=128)
    H, N, _ = x["Q"].shape
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    Qp, qbar_blocks = spark_bsa_gather_q(x["Q"], x["q_perm"], x["q_offsets"], err=err)
    qbar = spark_bsa_anchor(qbar_blocks, x["q_offsets"], N)
    Kp, Vp, kbar, kt, vt, cb = spark_bsa_gather_kv_summarize(x["K"], x["V"], x["k_perm"],
                                                             x["k_offsets"], qbar, err=err)
    Qp8, qs = spark_bsa_quantize_fp8(Qp, x["q_offsets"], err=err)
    Kp8, ks = spark_bsa_quantize_fp8(Kp, x["k_offsets"], err=err)
    kt8, kts = spark_bsa_quantize_fp8(kt, None, err=err)
    ratio = 0.2
    nkb = x["k_offsets"].numel() - 1
    k = spark_bsa_topk_count(nkb, ratio)
    refs = [oracle_fp8_head(x, h, ratio, blocks=[]) for h in range(H)]
    inj = torch.from_numpy(np.stack([r.sel for r in refs]).astype(np.int32)).to(DEV)
    assert inj.shape[-1] == k
    out = spark_bsa_attend_fp8(Qp8, qs, Kp8, ks, Vp, kt8, kts, vt, cb, inj, x["q_perm"],
                               x["q_offsets"], x["k_offsets"], out_dtype=torch.float32, err=err)
    assert spark_bsa_read_error(err) == 0
    for h in range(H):
        full = oracle_fp8_head(x, h, ratio)
        P.compare_out(P.to64(out[h]), full.out, f"attend_fp8 head {h}")


def test_full_size_fp8_workload():
    w = WORKLOADS["768p-24x241920-d128"]
    x = make_inputs(w, device=DEV)
    nqb = x["q_offsets"].numel() - 1
    heads = sorted(sample_units(w, 2, nqb))
    check_forward_fp8(x, w.ratio, heads=heads, blocks_per_head=4, seed=w.seed)
    del x
    torch.cuda.empty_cache()
