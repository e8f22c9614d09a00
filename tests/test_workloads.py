"""Seeded input generators: shapes, index validity and reproducibility (no GPU)."""

import torch

from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs, make_offsets


def test_offsets_cover_every_token():
    for w in WORKLOADS.values():
        offs = make_offsets(w)
        sizes = offs[1:] - offs[:-1]
        assert offs[0] == 0 and offs[-1] == w.N
        assert int(sizes.min()) >= 1 and int(sizes.max()) <= 128
        if w.var_block is None:
            assert int((sizes == w.block).sum()) == len(sizes) - (0 if w.N % w.block == 0 else 1)
        else:
            lo, hi = w.var_block
            assert int(sizes[:-1].min()) >= lo and int(sizes[:-1].max()) <= hi


def test_block_counts_at_the_workload_sizes():
    nb = {name: len(make_offsets(w)) - 1 for name, w in WORKLOADS.items()}
    assert nb["tiny-1x1024-d64-fp32"] == 16
    assert nb["small-8x16384-d128-randperm"] == 256
    assert nb["384p-24x60480-d128"] == 473      # last block holds 64 tokens
    assert nb["768p-24x241920-d128"] == 1890


def test_small_inputs_valid_and_reproducible():
    for name in ("tiny-1x1024-d64-fp32", "small-8x16384-d128-randperm"):
        w = WORKLOADS[name]
        a = make_inputs(w)
        b = make_inputs(w)
        for key in ("Q", "K", "V", "q_perm", "k_perm", "q_offsets"):
            assert torch.equal(a[key], b[key])
        assert a["Q"].shape == (w.H, w.N, w.d)
        assert a["Q"].dtype == (torch.float32 if w.dtype == "fp32" else torch.bfloat16)
        for h in range(w.H):
            for key in ("q_perm", "k_perm"):
                assert torch.equal(torch.sort(a[key][h].long()).values, torch.arange(w.N))


def test_reblock_layout_groups_components():
    from dataclasses import replace
    w = replace(WORKLOADS["384p-24x60480-d128"], H=2, N=4096)
    x = make_inputs(w)
    assert torch.equal(x["q_perm"], x["k_perm"])
    for h in range(2):
        assert torch.equal(torch.sort(x["k_perm"][h].long()).values, torch.arange(w.N))
