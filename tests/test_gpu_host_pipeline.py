"""The host-buffer entry point (pipelined by head chunks over three streams) against the
device-buffer forward pass: heads are independent, so the results must be identical."""

import pytest
import torch

from block_sparse_attention_gather_b200 import (spark_bsa_forward, spark_bsa_forward_ctx,
                                                spark_bsa_forward_fp8, spark_bsa_forward_host)
from test_gpu_parity import custom_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,hpc", [("bf16", 2), ("fp32", 1), ("bf16", 5), ("bf16", 9)])
def test_host_pipeline_equals_device_forward(dtype, hpc):
    x = custom_inputs(101, H=5, N=2500, d=128 if dtype == "bf16" else 64, dtype=dtype, lo=20,
                      hi=128)
    ref, _, _ = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                  x["q_offsets"], x["k_offsets"], 0.15)
    host = {n: x[n].cpu().pin_memory() for n in x}
    out = spark_bsa_forward_host(host["Q"], host["K"], host["V"], host["q_perm"],
                                 host["k_perm"], host["q_offsets"], host["k_offsets"], 0.15,
                                 heads_per_chunk=hpc)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.cpu())


def _context(seed, H, nc, d, dtype):
    g = torch.Generator().manual_seed(seed)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    return (torch.randn(H, nc, d, generator=g).to(tdt).cuda(),
            torch.randn(H, nc, d, generator=g).to(tdt).cuda())


@pytest.mark.parametrize("dtype,hpc,nc", [("bf16", 2, 77), ("fp32", 3, 130), ("bf16", 5, 1)])
def test_host_pipeline_with_context_equals_device_forward(dtype, hpc, nc):
    d = 128 if dtype == "bf16" else 64
    x = custom_inputs(102, H=5, N=2300, d=d, dtype=dtype, lo=20, hi=128)
    Kc, Vc = _context(103, 5, nc, d, dtype)
    ref, _, _ = spark_bsa_forward_ctx(x["Q"], x["K"], x["V"], Kc, Vc, x["q_perm"], x["k_perm"],
                                      x["q_offsets"], x["k_offsets"], 0.2)
    host = {n: x[n].cpu().pin_memory() for n in x}
    out = spark_bsa_forward_host(host["Q"], host["K"], host["V"], host["q_perm"],
                                 host["k_perm"], host["q_offsets"], host["k_offsets"], 0.2,
                                 heads_per_chunk=hpc, Kc=Kc.cpu().pin_memory(),
                                 Vc=Vc.cpu().pin_memory())
    torch.cuda.synchronize()
    assert torch.equal(out, ref.cpu())


@pytest.mark.parametrize("hpc,nc", [(2, 0), (3, 200)])
def test_host_pipeline_fp8_equals_device_forward(hpc, nc):
    x = custom_inputs(104, H=5, N=2600, d=128, dtype="bf16", lo=20, hi=128)
    Kc, Vc = _context(105, 5, nc, 128, "bf16") if nc else (None, None)
    ref, _, _ = spark_bsa_forward_fp8(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                      x["q_offsets"], x["k_offsets"], 0.15, Kc=Kc, Vc=Vc)
    host = {n: x[n].cpu().pin_memory() for n in x}
    out = spark_bsa_forward_host(host["Q"], host["K"], host["V"], host["q_perm"],
                                 host["k_perm"], host["q_offsets"], host["k_offsets"], 0.15,
                                 heads_per_chunk=hpc, fp8=True,
                                 Kc=Kc.cpu().pin_memory() if nc else None,
                                 Vc=Vc.cpu().pin_memory() if nc else None)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.cpu())
