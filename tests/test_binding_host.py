"""The Python binding's own argument checks (no GPU): every wrapper refuses host tensors,
wrong dtypes and mismatched shapes with a Python exception before anything reaches the
library, so a misuse never becomes a device fault."""

import pytest
import torch

from block_sparse_attention_gather_b200 import (
    spark_bsa_attend_fp8, spark_bsa_attend_var, spark_bsa_forward, spark_bsa_forward_ctx,
    spark_bsa_forward_fp8, spark_bsa_gather_kv_meanpool, spark_bsa_quantize_fp8,
    spark_bsa_route_threshold)


def cpu_inputs(H=1, N=256, d=128, dtype=torch.bfloat16):
    Q = torch.zeros(H, N, d, dtype=dtype)
    perm = torch.arange(N, dtype=torch.int32).repeat(H, 1)
    offs = torch.arange(0, N + 1, 128, dtype=torch.int32)
    return Q, perm, offs


def test_forward_refuses_host_tensors():
    Q, perm, offs = cpu_inputs()
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_forward(Q, Q, Q, perm, perm, offs, offs, 0.5)
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_forward_ctx(Q, Q, Q, None, None, perm, perm, offs, offs, 0.5)
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_forward_fp8(Q, Q, Q, perm, perm, offs, offs, 0.5)


def test_wrong_dtypes_are_refused():
    Q, perm, offs = cpu_inputs(dtype=torch.float16)
    with pytest.raises((TypeError, ValueError)):
        spark_bsa_forward(Q, Q, Q, perm, perm, offs, offs, 0.5)
    with pytest.raises((TypeError, ValueError)):
        spark_bsa_quantize_fp8(torch.zeros(1, 128, 128, dtype=torch.float32))


def test_step_wrappers_refuse_host_tensors():
    Q, perm, offs = cpu_inputs()
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_gather_kv_meanpool(Q, Q, perm, offs)
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_route_threshold(torch.zeros(1, 2, 128), torch.zeros(1, 128, 2), 1.0, 1)
    u8 = torch.zeros(1, 256, 128, dtype=torch.uint8)
    f = torch.zeros(1, 2)
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_attend_fp8(u8, f, u8, f, Q, u8, f, Q, f, perm, perm, offs, offs)
    sel = torch.zeros(1, 2, 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        spark_bsa_attend_var(Q, Q, Q, Q, Q, f, sel, sel[..., 0], perm, offs, offs)
