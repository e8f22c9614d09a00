"""The host-buffer entry point (pipelined by head chunks over three streams) against the
device-buffer forward pass: heads are independent, so the results must be identical."""

import pytest
import torch

from block_sparse_attention_gather_b200 import spark_bsa_forward, spark_bsa_forward_host
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
