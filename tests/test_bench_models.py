"""The byte and FLOP models behind bench.py's numbers (no GPU): the algorithmic attention
FLOPs count valid rows only, the dense-equivalent FLOPs are 4 H N (N + nc) d, the HBM byte
models of the bandwidth-bound kernels match their closed forms, and the DRAM traffic of the
committed ncu summary is reported only for the attention source it was taken on."""

import json
import types

import torch

import bench


def fake_hotpath(q_sizes, k_sizes, sel, H=1, d=128, nc=0, dtype=torch.bfloat16):
    qo = torch.tensor([0] + list(torch.tensor(q_sizes).cumsum(0).tolist()), dtype=torch.int32)
    ko = torch.tensor([0] + list(torch.tensor(k_sizes).cumsum(0).tolist()), dtype=torch.int32)
    N = int(qo[-1])
    x = {"q_offsets": qo, "k_offsets": ko, "Q": torch.empty(H, N, d, dtype=dtype)}
    hp = types.SimpleNamespace(x=x, v={"sel": torch.tensor(sel, dtype=torch.int32)}, H=H, N=N,
                               d=d, nqb=len(q_sizes), nkb=len(k_sizes), k=len(sel[0][0]), nc=nc)
    return hp


def test_attention_flops_counts_valid_rows_only():
    # 2 query blocks (3 and 5 rows), 3 key blocks (4, 2, 6 rows), k = 1, 7 context rows:
    # A0 selects B2 -> 6 exact + 7 context + 2 summary rows; A1 selects B0 -> 4 + 7 + 2
    hp = fake_hotpath([3, 5], [4, 2, 6], [[[2], [0]]], d=64, nc=7)
    expect = 4 * 64 * (3 * (6 + 7 + 2) + 5 * (4 + 7 + 2))
    assert bench.attention_flops(hp) == expect


def test_dense_flops_closed_form():
    w = types.SimpleNamespace(H=3, N=1000, nc=24, d=128)
    assert bench.dense_flops(w) == 4.0 * 3 * 1000 * 1024 * 128


def test_kernel_byte_models():
    hp = fake_hotpath([64] * 4, [64] * 4, [[[0], [1], [2], [3]]], H=2, d=128, nc=10)
    H, N, d, nqb, nkb, k = 2, 256, 128, 4, 4, 1
    kb = bench.kernel_bytes(hp)
    assert kb["gather_q"] == H * N * d * (2 + 2) + H * N * 4 + H * nqb * d * 4
    assert kb["route"] == H * (nqb + nkb) * d * 4 + H * nqb * k * 4
    assert kb["quantize"] == (2 * H * N * d + H * nkb * d + H * 10 * d) * 3


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    hp = fake_hotpath([64] * 4, [64] * 4, [[[0], [1], [2], [3]]], H=2)
    prof = tmp_path / "dram.json"
    prof.write_text(json.dumps({"attention_sources_sha256_16": bench.attention_sources_hash(),
                                "dram_bytes_per_query_block": 1000.0}))
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(prof))
    assert bench.profiled_traffic(hp) == 1000.0 * 2 * 4
    prof.write_text(json.dumps({"attention_sources_sha256_16": "0" * 16,
                                "dram_bytes_per_query_block": 1000.0}))
    assert bench.profiled_traffic(hp) is None
    # a change to any source the kernel is compiled from invalidates the capture
    monkeypatch.setattr(bench, "ATTENTION_SOURCES", bench.ATTENTION_SOURCES[:1])
    prof.write_text(json.dumps({"attention_sources_sha256_16": bench.attention_sources_hash(),
                                "dram_bytes_per_query_block": 1000.0}))
    monkeypatch.undo()
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(prof))
    assert bench.profiled_traffic(hp) is None


def test_attention_flops_with_threshold_counts():
    # kcap = 2; A0 keeps one block (B2: 6 rows), A1 none: the other blocks are summary rows
    hp = fake_hotpath([3, 5], [4, 2, 6], [[[2, -1], [-1, -1]]], d=32)
    hp.routing = "threshold"
    hp.count = torch.tensor([[1, 0]], dtype=torch.int32)
    expect = 4 * 32 * (3 * (6 + 2) + 5 * (0 + 3))
    assert bench.attention_flops(hp) == expect


def test_issued_flops_follow_the_kernels_tiles():
    # short key blocks (variable tiles): an exact tile covers its rows rounded up to 16; the one
    # summary tile covers 128 keys; 7 context rows make one tile of 16; M is always 128
    hp = fake_hotpath([3, 5], [4, 2, 6], [[[2], [0]]], d=64, nc=7)
    expect = 4 * 128 * 64 * ((16 + 16 + 128) + (16 + 16 + 128))
    assert bench.attention_issued_flops(hp) == expect
    # every key block full (128 rows): every exact tile covers 128 keys, context too
    hp = fake_hotpath([128, 128, 128], [128, 128, 128], [[[2], [0], [1]]], d=64, nc=7)
    expect = 4 * 128 * 64 * 3 * (128 + 128 + 128)
    assert bench.attention_issued_flops(hp) == expect
    # k = nkb: no summary tile
    hp = fake_hotpath([40], [40, 70], [[[0, 1]]], d=32)
    assert bench.attention_issued_flops(hp) == 4 * 128 * 32 * (48 + 80)
