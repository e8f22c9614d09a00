"""The bounded waits of the attention kernel, made to run out on purpose (a limit of 0 ns makes
every barrier wait that is not complete at its first test expire).  The kernel must report
SPARK_DEVERR_TIMEOUT in the device error word, stop, release what it holds and return, and
the context must stay usable: the next call, with the default limit back, must be correct.

No fault is involved: the expiry is the kernels' own bounded-wait logic, and every copy or
MMA the kernel issued is waited for (with the default limit) before it exits."""

import numpy as np
import pytest
import torch

import _parity as P
from block_sparse_attention_gather_b200 import (DEVERR, spark_bsa_forward,
                                                spark_bsa_get_wait_limit_ns,
                                                spark_bsa_read_error,
                                                spark_bsa_set_wait_limit_ns, workspace_views)
from block_sparse_attention_gather_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
DEFAULT_NS = 4_000_000_000


def _inputs(name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    return w, {k: v.to(DEV) if torch.is_tensor(v) else v for k, v in x.items()}


def _run(x, ratio):
    out, ws, lay = spark_bsa_forward(x["Q"], x["K"], x["V"], x["q_perm"], x["k_perm"],
                                     x["q_offsets"], x["k_offsets"], ratio)
    H, N, d = x["Q"].shape
    views = workspace_views(ws, lay, H, N, d, x["q_offsets"].numel() - 1,
                            x["k_offsets"].numel() - 1)
    return out, spark_bsa_read_error(views["err"])


@pytest.mark.parametrize("name", ["tiny-1x1024-d64-fp32", "small-8x16384-d128-randperm"])
def test_expired_wait_reports_timeout_and_leaves_the_context_usable(name):
    w, x = _inputs(name)
    assert spark_bsa_get_wait_limit_ns() == DEFAULT_NS
    try:
        spark_bsa_set_wait_limit_ns(0)
        _, flags = _run(x, w.ratio)
    finally:
        spark_bsa_set_wait_limit_ns(DEFAULT_NS)
    torch.cuda.synchronize()
    assert flags & DEVERR["timeout"], f"no timeout reported (error word {flags:#x})"
    assert flags & ~DEVERR["timeout"] == 0, f"unexpected error bits {flags:#x}"
    # the same call with the default limit completes and is correct
    out, flags = _run(x, w.ratio)
    assert flags == 0
    ref = P.oracle_head(x, 0, w.ratio, blocks=None if w.H == 1 else list(range(8)))
    got = P.to64(out[0])
    rows = ~np.isnan(ref.out[:, 0])
    P.compare_out(got[rows], ref.out[rows], f"{name} after a timeout")


def test_a_one_second_limit_changes_nothing():
    w, x = _inputs("small-8x16384-d128-randperm")
    ref, flags = _run(x, w.ratio)
    assert flags == 0
    try:
        spark_bsa_set_wait_limit_ns(1_000_000_000)
        out, flags = _run(x, w.ratio)
    finally:
        spark_bsa_set_wait_limit_ns(DEFAULT_NS)
    assert flags == 0
    assert torch.equal(out, ref)
