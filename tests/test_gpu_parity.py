"""GPU parity of the CUDA path (through the C ABI) against the float64 CPU oracle.

Every case feeds the same seeded tensors to both sides.  Small cases compare every output
element and every intermediate; the full-size workloads run in the same launch
configuration as bench.py and are compared on whole heads for the routing and on sampled
query blocks for the attention output.
"""

import math

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (
    spark_bsa_anchor, spark_bsa_attend, spark_bsa_forward, spark_bsa_gather_kv_summarize,
    spark_bsa_gather_q, spark_bsa_read_error, spark_bsa_route, spark_bsa_topk_count,
    workspace_views)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs, sample_units
from oracle import spark_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


def custom_inputs(seed, H, N, d, dtype, lo, hi, same_layout=False, lo_k=None, hi_k=None):
    g = torch.Generator().manual_seed(seed)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    x = {}
    for n in ("Q", "K", "V"):
        x[n] = (torch.randn(H, N, d, generator=g) * (1.5 if n != "V" else 1.0)).to(tdt)
    x["q_perm"] = torch.stack([torch.randperm(N, generator=g) for _ in range(H)]).int()
    x["k_perm"] = (x["q_perm"].clone() if same_layout else
                   torch.stack([torch.randperm(N, generator=g) for _ in range(H)]).int())

    def offs(a, b):
        o = [0]
        while o[-1] < N:
            o.append(min(o[-1] + int(torch.randint(a, b + 1, (1,), generator=g)), N))
        return torch.tensor(o, dtype=torch.int32)

    x["q_offsets"] = offs(lo, hi)
    x["k_offsets"] = x["q_offsets"].clone() if same_layout else offs(lo_k or lo, hi_k or hi)
    return {k: v.to(DEV) for k, v in x.items()}


def check_forward(x, ratio, heads=None, blocks_per_head=None, seed=0, check_inter=True):
    """Runs the fused forward on the GPU and compares with the oracle."""
    out, ws, layout = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                        x["q_offsets"], x["k_offsets"], ratio)
    H, N, d = x["Q"].shape
    nqb, nkb = x["q_offsets"].numel() - 1, x["k_offsets"].numel() - 1
    views = workspace_views(ws, layout, H, N, d, nqb, nkb)
    assert spark_bsa_read_error(views["err"]) == 0
    torch.cuda.synchronize()
    k = layout.k
    assert k == O.topk_count(ratio, nkb)
    heads = range(H) if heads is None else heads
    rng = np.random.default_rng(seed)
    worst = (0.0, 0.0)
    for h in heads:
        hi = P.head_inputs(x, h)
        ref = P.oracle_head(x, h, ratio, blocks=[], hi=hi)
        gsel = views["sel"][h].cpu().numpy().astype(np.int64)
        P.compare_sel(gsel, ref.sel, ref.scores, k)
        if check_inter:
            assert np.array_equal(P.to64(views["Qp"][h]), hi["Q"][hi["q_perm"]])
            assert np.array_equal(P.to64(views["Kp"][h]), hi["K"][hi["k_perm"]])
            assert np.array_equal(P.to64(views["Vp"][h]), hi["V"][hi["k_perm"]])
            for name, refv in (("qbar_blocks", ref.qbar_blocks), ("kbar", ref.kbar)):
                got = P.to64(views[name][h])
                if name == "kbar":
                    got = got.T                          # stored d-major [d, nkb]
                err = np.abs(got - refv).max(axis=1) / np.maximum(np.linalg.norm(refv, axis=1), 1e-6)
                assert err.max() < 1e-5, name
            gq = P.to64(views["qbar"][h])
            assert np.abs(gq - ref.qbar).max() <= 1e-5 * max(np.linalg.norm(ref.qbar), 1e-3)
            for name, refv in (("k_tilde", ref.k_tilde), ("v_tilde", ref.v_tilde)):
                got = P.to64(views[name][h])
                assert (np.abs(got - refv) <= 2 * 2.0 ** -8 * np.abs(refv) + 1e-3).all(), name
            assert np.abs(P.to64(views["cbias"][h]) - ref.c).max() < 1e-2
        if blocks_per_head is None:
            blocks = list(range(nqb))
        else:
            blocks = sorted(rng.choice(nqb, size=min(blocks_per_head, nqb), replace=False).tolist())
            if nqb - 1 not in blocks:
                blocks.append(nqb - 1)                   # the ragged last block
        ref2 = P.oracle_head(x, h, ratio, blocks=blocks, sel=gsel, hi=hi)
        rows = P.rows_of_blocks(hi["q_perm"], hi["q_offsets"], blocks)
        got = P.to64(out[h])[rows]
        r = P.compare_out(got, ref2.out[rows], f"head {h}")
        worst = (max(worst[0], r[0]), max(worst[1], r[1]))
    return out, worst


# --------------------------------------------------------------------- seeded workloads

def test_tiny_workload_full():
    w = WORKLOADS["tiny-1x1024-d64-fp32"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    out, _ = check_forward(x, w.ratio)
    assert out.dtype == torch.float32


def test_small_workload_full():
    w = WORKLOADS["small-8x16384-d128-randperm"]
    x = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(w).items()}
    check_forward(x, w.ratio)


# ---------------------------------------------------------- ragged shapes, both d, dtypes

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("ratio", [0.05, 0.3])
def test_ragged_blocks(d, dtype, ratio):
    x = custom_inputs(7 + d + int(ratio * 100), H=3, N=3001, d=d, dtype=dtype, lo=1, hi=128,
                      lo_k=20, hi_k=128)
    check_forward(x, ratio)


def test_ratio_one_is_dense_attention():
    x = custom_inputs(11, H=2, N=2000, d=128, dtype="bf16", lo=30, hi=128)
    out, _ = check_forward(x, 1.0)
    for h in range(2):
        q, k, v = (P.bf16_64(x[n][h]) for n in ("Q", "K", "V"))
        ref = O.dense_attention(q, k, v)
        P.compare_out(P.to64(out[h]), ref, "dense")


def plant_far_key(x, offset, scale, seed):
    """Queries share a direction u (offset * u added to every row) and the first key of the
    last key block is scale * u in every head, so its logit lies far above the logits of the
    first key tiles of every query block."""
    H, N, d = x["Q"].shape
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(d, generator=g, dtype=torch.float64)
    u /= u.norm()
    Q = (x["Q"].cpu().double() + offset * u).to(x["Q"].dtype)
    K = x["K"].cpu().clone()
    last = int(x["k_offsets"][-2])
    for h in range(H):
        K[h, int(x["k_perm"][h, last])] = (scale * u).to(K.dtype)
    x = dict(x)
    x["Q"], x["K"] = Q.to(DEV), K.to(DEV)
    return x, last


def test_logit_far_above_the_first_tiles():
    """The attention exponentiates against a reference taken from the first two key tiles of
    each query block and repeats a query block whose row sums leave [2^-60, 2^60] with the
    true row maxima.  Here a key in the last block sits ~100 nats above every logit of the
    first two blocks, which forces the repeat; dense attention (ratio 1) in float64 is the
    reference."""
    x = custom_inputs(71, H=2, N=1800, d=128, dtype="fp32", lo=60, hi=128)
    x, last = plant_far_key(x, 6.0, 300.0, 72)
    H, N, d = x["Q"].shape
    second = int(x["k_offsets"][2])
    for h in range(H):
        hi = P.head_inputs(x, h)
        s = hi["Q"] @ hi["K"][hi["k_perm"]].T / math.sqrt(d)
        gap = s[:, last] - s[:, :second].max(axis=1)
        assert np.mean(gap > 60 * math.log(2)) > 0.9    # beyond the window for most rows
    # (the summaries' bias is checked elsewhere: at ~150-nat logits its bf16 rounding of k~
    # exceeds that check's absolute bound, while the output is insensitive to it)
    out, _ = check_forward(x, 1.0, check_inter=False)
    for h in range(H):
        q, k, v = P.bf16_64(x["Q"][h]), P.bf16_64(x["K"][h]), P.bf16_64(x["V"][h])
        P.compare_out(P.to64(out[h]), O.dense_attention(q, k, v), "dense, far key")


def test_rerun_keeps_the_reference_of_rows_in_window():
    """One query block holds a row that leaves the window (a key ~100 nats above its first
    tiles) and a row whose logits all sit near +100 nats, in window against its own first
    tiles.  The repeat must give the first row its recorded maximum and leave the second row
    its own reference (a reference of 0 there would overflow)."""
    x = custom_inputs(76, H=1, N=1000, d=128, dtype="fp32", lo=100, hi=100)
    g = torch.Generator().manual_seed(77)
    u = torch.randn(128, generator=g, dtype=torch.float64)
    u /= u.norm()
    v = torch.randn(128, generator=g, dtype=torch.float64)
    v -= (v @ u) * u
    v /= v.norm()
    Q = x["Q"].cpu().double()
    K = x["K"].cpu().double()
    K += 40.0 * u                                 # every key shares a large u component
    r0, r1 = int(x["q_perm"][0, 0]), int(x["q_perm"][0, 1])   # rows of query block 0
    Q[0, r0] = 6.0 * v + 0.1 * Q[0, r0]
    Q[0, r1] = 30.0 * u + 0.1 * Q[0, r1]          # ~106 nats against every key
    far = int(x["k_perm"][0, int(x["k_offsets"][-2])])
    K[0, far] += 300.0 * v                        # ~160 nats for row r0 only
    x = dict(x)
    x["Q"], x["K"] = Q.float().to(DEV), K.float().to(DEV)
    out, _ = check_forward(x, 1.0, check_inter=False)
    q, k, vv = P.bf16_64(x["Q"][0]), P.bf16_64(x["K"][0]), P.bf16_64(x["V"][0])
    ref = O.dense_attention(q, k, vv)
    got = P.to64(out[0])
    assert np.isfinite(got).all()
    P.compare_out(got, ref, "rerun with rows in window")


def test_logit_far_above_at_a_sparse_ratio():
    """The same planted key at ratio 0.1: it sits in the exact branch of the query blocks that
    select the last block and in the compressed branch (through k~, c) of the others."""
    x = custom_inputs(73, H=2, N=2600, d=128, dtype="bf16", lo=40, hi=128)
    x, _ = plant_far_key(x, 6.0, 300.0, 74)
    check_forward(x, 0.1, check_inter=False)


@pytest.mark.parametrize("case", ["single_token", "one_block", "unit_blocks", "two_summary_tiles",
                                  "q_reuse_k", "k_equals_nkb_minus_1"])
def test_edge_cases(case):
    if case == "single_token":
        x = custom_inputs(21, H=2, N=1, d=64, dtype="bf16", lo=1, hi=1)
        check_forward(x, 0.5)
    elif case == "one_block":
        x = custom_inputs(22, H=2, N=100, d=128, dtype="bf16", lo=128, hi=128)
        check_forward(x, 0.1)
    elif case == "unit_blocks":
        x = custom_inputs(23, H=1, N=300, d=64, dtype="bf16", lo=1, hi=1)
        check_forward(x, 0.1)
    elif case == "two_summary_tiles":
        x = custom_inputs(24, H=2, N=129 * 20, d=128, dtype="bf16", lo=20, hi=20)
        assert x["k_offsets"].numel() - 1 == 129
        check_forward(x, 0.02)
    elif case == "q_reuse_k":
        x = custom_inputs(25, H=2, N=4000, d=128, dtype="bf16", lo=60, hi=128, same_layout=True)
        check_forward(x, 0.2)
    else:
        x = custom_inputs(26, H=1, N=1280, d=128, dtype="bf16", lo=128, hi=128)
        assert spark_bsa_topk_count(10, 0.9) == 9
        check_forward(x, 0.9)


@pytest.mark.parametrize("nkb", [7000, 12800])
def test_many_key_blocks(nkb):
    """Unit-size blocks: 7000 key blocks take the routing kernel's 4-row variant and the
    attention kernel's path that reads summary offsets from global memory (they no longer fit
    its shared-memory row); 12800 is the largest block count the library accepts."""
    x = custom_inputs(27 + nkb, H=1, N=nkb, d=128, dtype="bf16", lo=1, hi=1)
    assert x["k_offsets"].numel() - 1 == nkb
    check_forward(x, 0.01, blocks_per_head=6, seed=nkb, check_inter=False)


# ------------------------------------------------------------------- step entry points

@pytest.mark.parametrize("d", [64, 128])
def test_step_entry_points(d):
    """Each step's kernel against the oracle, with the oracle's selection injected into the
    attention step so that it is checked independently of the routing kernel."""
    x = custom_inputs(31 + d, H=2, N=2500, d=d, dtype="bf16", lo=40, hi=128)
    H, N, _ = x["Q"].shape
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    Qp, qbar_blocks = spark_bsa_gather_q(x["Q"], x["q_perm"], x["q_offsets"], err=err)
    qbar = spark_bsa_anchor(qbar_blocks, x["q_offsets"], N)
    Kp, Vp, kbar, kt, vt, cb = spark_bsa_gather_kv_summarize(x["K"], x["V"], x["k_perm"],
                                                             x["k_offsets"], qbar, err=err)
    nkb = x["k_offsets"].numel() - 1
    ratio = 0.15
    k = spark_bsa_topk_count(nkb, ratio)
    sel = spark_bsa_route(qbar_blocks, kbar, k, err=err)
    refs = [P.oracle_head(x, h, ratio, blocks=[]) for h in range(H)]
    inj = torch.from_numpy(np.stack([r.sel for r in refs]).astype(np.int32)).to(DEV)
    out = spark_bsa_attend(Qp, Kp, Vp, kt, vt, cb, inj, x["q_perm"], x["q_offsets"],
                           x["k_offsets"], out_dtype=torch.bfloat16, err=err)
    assert spark_bsa_read_error(err) == 0
    for h in range(H):
        r = refs[h]
        P.compare_sel(sel[h].cpu().numpy().astype(np.int64), r.sel, r.scores, k)
        assert np.abs(P.to64(qbar[h]) - r.qbar).max() < 1e-4
        assert np.abs(P.to64(cb[h]) - r.c).max() < 1e-2
        full = P.oracle_head(x, h, ratio)
        P.compare_out(P.to64(out[h]), full.out, f"attend head {h}")


def test_device_checks_flag_bad_inputs():
    """Out-of-range permutation entries and selected ids are skipped and reported in the
    error word; the kernels never touch memory outside the buffers."""
    x = custom_inputs(41, H=1, N=1000, d=128, dtype="bf16", lo=50, hi=128)
    bad = x["q_perm"].clone()
    bad[0, 5] = 10 ** 6
    bad[0, 7] = -3
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    spark_bsa_gather_q(x["Q"], bad, x["q_offsets"], err=err)
    assert spark_bsa_read_error(err) & 0x1
    err.zero_()
    Qp, qb = spark_bsa_gather_q(x["Q"], x["q_perm"], x["q_offsets"], err=err)
    qbar = spark_bsa_anchor(qb, x["q_offsets"], 1000)
    Kp, Vp, kbar, kt, vt, cb = spark_bsa_gather_kv_summarize(x["K"], x["V"], x["k_perm"],
                                                             x["k_offsets"], qbar, err=err)
    assert spark_bsa_read_error(err) == 0
    nkb = x["k_offsets"].numel() - 1
    sel = torch.zeros(1, x["q_offsets"].numel() - 1, 2, dtype=torch.int32, device=DEV)
    sel[..., 1] = nkb + 5                                   # out of range
    spark_bsa_attend(Qp, Kp, Vp, kt, vt, cb, sel, x["q_perm"], x["q_offsets"], x["k_offsets"],
                     err=err)
    assert spark_bsa_read_error(err) & 0x4


# ------------------------------------------------------------- full-size workloads

FULL = ["384p-24x60480-d128", "768p-24x241920-d128", "768p-24x241920-d128-randperm",
        "768p-varblock-24x241920-d128-r0.1", "768p-varblock-24x241920-d128-r0.2",
        "768p-varblock-24x241920-d128-r0.3", "768p-varblock-24x241920-d128-r1"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads(name):
    w = WORKLOADS[name]
    x = make_inputs(w, device=DEV)
    nqb = x["q_offsets"].numel() - 1
    units = sample_units(w, 2, nqb)                        # two heads at random
    heads = sorted(units)
    _, worst = check_forward(x, w.ratio, heads=heads, blocks_per_head=6, seed=w.seed,
                             check_inter=True)
    del x
    torch.cuda.empty_cache()
