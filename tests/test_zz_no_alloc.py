"""The forward pass for callers that cannot allocate device memory while they run
(spark_bsa_forward_noalloc): its workspace is the library's own static device array, so a
caller whose device memory is owned by someone else, or who is recording a stream capture,
can still run the whole path.  Checked through the C ABI against the ordinary entry point,
whose workspace the caller allocates, on two calls in a row with different problems: both run
the same kernels on the same workspace layout, so the outputs must be equal bit for bit.  The
first problem is also compared with the float64 oracle.

Kept in a file of its own that pytest collects after every other test file."""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (SparkError, spark_bsa_forward,
                                                spark_bsa_forward_noalloc,
                                                spark_bsa_workspace_size)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCRATCH_BYTES = 16 * 1024 * 1024


def ragged_inputs(seed, H, N, d):
    g = torch.Generator().manual_seed(seed)
    x = {n: torch.randn(H, N, d, generator=g).to(torch.bfloat16) for n in ("Q", "K", "V")}
    x["q_perm"] = torch.stack([torch.randperm(N, generator=g) for _ in range(H)]).int()
    x["k_perm"] = torch.stack([torch.randperm(N, generator=g) for _ in range(H)]).int()
    for key in ("q_offsets", "k_offsets"):
        o = [0]
        while o[-1] < N:
            o.append(min(o[-1] + int(torch.randint(10, 129, (1,), generator=g)), N))
        x[key] = torch.tensor(o, dtype=torch.int32)
    return {k: v.to(DEV) for k, v in x.items()}


def run_both(x, ratio):
    ref, _, _ = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                  x["q_offsets"], x["k_offsets"], ratio)
    out = torch.empty_like(x["Q"])
    spark_bsa_forward_noalloc(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"], x["q_offsets"],
                              x["k_offsets"], ratio, out)
    torch.cuda.synchronize()
    return ref, out


def test_noalloc_matches_the_allocating_entry_point_on_two_calls():
    tiny = WORKLOADS["tiny-1x1024-d64-fp32"]
    a = {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in make_inputs(tiny).items()}
    b = ragged_inputs(77, H=2, N=3000, d=128)
    for x, ratio in ((a, tiny.ratio), (b, 0.2)):
        H, N, d = x["Q"].shape
        need = spark_bsa_workspace_size(H, N, d, x["q_offsets"].numel() - 1,
                                        x["k_offsets"].numel() - 1, ratio)
        assert need <= SCRATCH_BYTES
        ref, out = run_both(x, ratio)
        assert torch.equal(out, ref), "noalloc differs from spark_bsa_forward"
        if x is a:
            want = P.oracle_head(x, 0, ratio).out
            P.compare_out(P.to64(out[0]), want, "noalloc vs oracle")


def test_noalloc_rejects_problems_larger_than_its_array():
    x = ragged_inputs(78, H=4, N=20000, d=128)   # ~61 MB of workspace
    out = torch.empty_like(x["Q"])
    with pytest.raises(SparkError) as e:
        spark_bsa_forward_noalloc(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                  x["q_offsets"], x["k_offsets"], 0.1, out)
    assert e.value.status == 3                   # SPARK_ERR_WORKSPACE
