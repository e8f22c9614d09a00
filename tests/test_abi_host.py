"""The C ABI without a GPU: the library loads, exports every function the header declares,
and rejects bad arguments on the host before anything touches a device."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spark_bsa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module")
def L():
    from block_sparse_attention_gather_b200.build import build_library, is_stale
    if is_stale():
        build_library()
    from block_sparse_attention_gather_b200 import lib
    return lib()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"SPARK_API\s+[\w\s\*]+?\b(spark_\w+)\s*\(", src)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), f"{n} declared in spark_bsa.h but not exported"
    from block_sparse_attention_gather_b200 import EXPORTED
    assert set(EXPORTED) == set(names)


def test_status_strings(L):
    from block_sparse_attention_gather_b200 import spark_status_string
    for code, name in [(0, "SPARK_OK"), (1, "SPARK_ERR_INVALID_ARG"), (2, "SPARK_ERR_UNSUPPORTED"),
                       (3, "SPARK_ERR_WORKSPACE"), (4, "SPARK_ERR_CUDA"),
                       (5, "SPARK_ERR_DEVICE_CHECK")]:
        assert spark_status_string(code) == name
    assert spark_status_string(99) == "SPARK_UNKNOWN_STATUS"


def test_topk_count_matches_the_oracle(L):
    from block_sparse_attention_gather_b200 import spark_bsa_topk_count
    from oracle import spark_oracle as O
    for nkb in (1, 2, 7, 16, 256, 473, 1890, 2520, 12800):
        for ratio in (1e-6, 0.01, 0.05, 0.1, 0.125, 0.2, 0.3, 1 / 3, 0.5, 0.95, 1.0):
            assert spark_bsa_topk_count(nkb, ratio) == O.topk_count(ratio, nkb)
    assert spark_bsa_topk_count(10, 0.0) == -1
    assert spark_bsa_topk_count(10, 1.5) == -1
    assert spark_bsa_topk_count(0, 0.5) == -1


def test_workspace_layout(L):
    from block_sparse_attention_gather_b200 import (spark_bsa_workspace_layout,
                                                    spark_bsa_workspace_size)
    H, N, d, nqb, nkb = 24, 241920, 128, 1890, 1890
    lay = spark_bsa_workspace_layout(H, N, d, nqb, nkb, 0.1)
    assert lay.k == 189
    offs = [lay.Qp, lay.Kp, lay.Vp, lay.qbar_blocks, lay.qbar, lay.kbar, lay.k_tilde,
            lay.v_tilde, lay.cbias, lay.sel, lay.err, lay.total]
    assert all(o % 256 == 0 for o in offs)
    assert offs == sorted(offs)
    sizes = [H * N * d * 2] * 3 + [H * nqb * d * 4, H * d * 4, H * nkb * d * 4,
                                   H * nkb * d * 2, H * nkb * d * 2, H * nkb * 4,
                                   H * nqb * 189 * 4, 4]
    for a, b, sz in zip(offs, offs[1:], sizes):
        assert b - a >= sz
    assert spark_bsa_workspace_size(H, N, d, nqb, nkb, 0.1) == lay.total
    assert spark_bsa_workspace_size(H, N, 96, nqb, nkb, 0.1) == 0


def _fwd(L, **kw):
    """spark_bsa_forward with fake but aligned pointers: only host checks may run."""
    p = ctypes.c_void_p(0x100000)
    a = dict(Q=p, K=p, V=p, dtype=0, H=2, N=1000, d=128, q_perm=p, k_perm=p, qo=p, nqb=10,
             ko=p, nkb=10, ratio=0.2, out=p, ws=p, ws_bytes=0, stream=None)
    a.update(kw)
    return L.spark_bsa_forward(a["Q"], a["K"], a["V"], a["dtype"], a["H"], a["N"], a["d"],
                               a["q_perm"], a["k_perm"], a["qo"], a["nqb"], a["ko"], a["nkb"],
                               a["ratio"], a["out"], a["ws"], a["ws_bytes"], a["stream"])


def test_forward_rejects_bad_arguments_on_the_host(L):
    assert _fwd(L, Q=None) == INVALID
    assert _fwd(L, out=None) == INVALID
    assert _fwd(L, dtype=7) == INVALID
    assert _fwd(L, d=96) == UNSUPPORTED
    assert _fwd(L, H=0) == INVALID
    assert _fwd(L, nqb=0) == INVALID
    assert _fwd(L, nkb=2000) == INVALID            # more blocks than tokens
    assert _fwd(L, N=20000, nkb=12801) == UNSUPPORTED
    assert _fwd(L, ratio=0.0) == INVALID
    assert _fwd(L, ratio=1.01) == INVALID
    assert _fwd(L, ratio=float("nan")) == INVALID
    assert _fwd(L, Q=ctypes.c_void_p(0x100004)) == INVALID      # not 16-byte aligned
    assert _fwd(L, ws=None) == WORKSPACE
    assert _fwd(L, ws_bytes=1024) == WORKSPACE                  # too small
    assert _fwd(L, ws=ctypes.c_void_p(0x100010), ws_bytes=1 << 40) == WORKSPACE   # misaligned


def test_step_entry_points_reject_bad_arguments(L):
    p = ctypes.c_void_p(0x100000)
    assert L.spark_bsa_gather_q(None, 0, 1, 10, 128, p, p, 1, p, p, None, None) == INVALID
    assert L.spark_bsa_gather_q(p, 0, 1, 10, 80, p, p, 1, p, p, None, None) == UNSUPPORTED
    assert L.spark_bsa_anchor(p, p, 1, 10, 128, 0, p, None) == INVALID
    assert L.spark_bsa_route(p, p, 1, 4, 4, 128, 5, p, None, None) == INVALID     # k > nkb
    assert L.spark_bsa_route(p, p, 1, 4, 4, 128, 0, p, None, None) == INVALID
    assert L.spark_bsa_route(p, p, 1, 4, 13000, 128, 5, p, None, None) == UNSUPPORTED
    assert L.spark_bsa_attend(p, p, p, p, p, p, p, 0, p, p, 1, p, 1, 1, 10, 128, p, 0, None,
                              None) == INVALID                                   # k = 0
    assert L.spark_bsa_attend(p, p, p, p, p, p, p, 1, p, p, 1, p, 1, 1, 10, 128, p, 3, None,
                              None) == INVALID                                   # out dtype
    assert L.spark_bsa_gather_kv_summarize(p, p, 0, 1, 10, 128, p, p, 1, p, p, p, p, p, p,
                                           None, None, None) == INVALID          # cbias NULL
    flags = ctypes.c_uint32(0)
    assert L.spark_bsa_read_error(None, None, ctypes.byref(flags)) == INVALID


def test_threshold_entry_points_reject_bad_arguments(L):
    p = ctypes.c_void_p(0x100000)
    assert L.spark_bsa_route_threshold(p, p, 1, 4, 4, 128, 1.0, 5, p, p, None, None) == INVALID
    assert L.spark_bsa_route_threshold(p, p, 1, 4, 4, 128, 1.0, 0, p, p, None, None) == INVALID
    assert L.spark_bsa_route_threshold(p, p, 1, 4, 4, 128, float("nan"), 2, p, p, None,
                                       None) == INVALID
    assert L.spark_bsa_route_threshold(p, p, 1, 4, 4, 128, 1.0, 2, p, None, None,
                                       None) == INVALID                          # count NULL
    assert L.spark_bsa_route_threshold(p, p, 1, 4, 4, 96, 1.0, 2, p, p, None,
                                       None) == UNSUPPORTED
    assert L.spark_bsa_attend_var(p, p, p, p, p, p, p, 1, None, p, p, 1, p, 1, 1, 10, 128, p, 0,
                                  None, None) == INVALID                         # count NULL
    assert L.spark_bsa_attend_var(p, p, p, p, p, p, p, 2, p, p, p, 1, p, 1, 1, 10, 128, p, 0,
                                  None, None) == INVALID                         # kcap > nkb


def test_meanpool_entry_point_rejects_bad_arguments(L):
    p = ctypes.c_void_p(0x100000)
    assert L.spark_bsa_gather_kv_meanpool(p, p, 0, 1, 10, 128, p, p, 1, p, p, p, p, p, None,
                                          None, None) == INVALID                 # cbias NULL
    assert L.spark_bsa_gather_kv_meanpool(p, p, 2, 1, 10, 128, p, p, 1, p, p, p, p, p, p,
                                          None, None) == INVALID                 # dtype
    assert L.spark_bsa_gather_kv_meanpool(p, p, 0, 1, 10, 96, p, p, 1, p, p, p, p, p, p,
                                          None, None) == UNSUPPORTED             # d


def test_fp8_entry_points_reject_bad_arguments(L):
    p = ctypes.c_void_p(0x100000)
    # quantise: null operands, d not 64/128, tiles with the wrong group count
    assert L.spark_bsa_quantize_fp8(None, 1, 10, 128, None, 1, p, p, None, None) == INVALID
    assert L.spark_bsa_quantize_fp8(p, 1, 10, 96, None, 1, p, p, None, None) == UNSUPPORTED
    assert L.spark_bsa_quantize_fp8(p, 1, 300, 128, None, 2, p, p, None, None) == INVALID
    # FP8 attention: d must be 128; k in [1, nkb]; out dtype
    args = [p] * 10 + [1, p, p, p, 0, p, p, 1, p, 1, 1, 10, 128, p, 0, None, None]
    bad_d = list(args)
    bad_d[22] = 64
    assert L.spark_bsa_attend_fp8(*bad_d) == UNSUPPORTED
    bad_k = list(args)
    bad_k[10] = 2
    assert L.spark_bsa_attend_fp8(*bad_k) == INVALID
    bad_out = list(args)
    bad_out[24] = 3
    assert L.spark_bsa_attend_fp8(*bad_out) == INVALID
    assert L.spark_bsa_workspace_size_fp8(1, 1024, 64, 16, 16, 0.125, 0) == 0
    assert L.spark_bsa_workspace_size_fp8(1, 1024, 128, 16, 16, 0.125, 0) > \
        L.spark_bsa_workspace_size_ctx(1, 1024, 128, 16, 16, 0.125, 0)


def test_context_entry_points_reject_bad_arguments(L):
    from block_sparse_attention_gather_b200 import (spark_bsa_workspace_layout,
                                                    spark_bsa_workspace_size_ctx)
    H, N, d, nqb, nkb = 24, 241920, 128, 1890, 1890
    lay = spark_bsa_workspace_layout(H, N, d, nqb, nkb, 0.1)
    cbytes = (H * 512 * d * 2 + 255) // 256 * 256
    assert spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, 0.1, 0) == lay.total
    assert spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, 0.1, 512) == lay.total + 2 * cbytes
    assert spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, 0.1, -1) == 0
    assert spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, 0.1, (1 << 20) + 1) == 0

    p = ctypes.c_void_p(0x100000)
    def fwd(Kc=p, Vc=p, nc=16, ws_bytes=1 << 40):
        return L.spark_bsa_forward_ctx(p, p, p, Kc, Vc, nc, 0, 2, 1000, 128, p, p, p, 10, p, 10,
                                       0.2, p, p, ws_bytes, None)
    assert fwd(nc=-1) == INVALID
    assert fwd(nc=(1 << 20) + 1) == INVALID
    assert fwd(Kc=None) == INVALID
    assert fwd(Vc=ctypes.c_void_p(0x100008)) == INVALID          # not 16-byte aligned
    small = L.spark_bsa_workspace_size(2, 1000, 128, 10, 10, ctypes.c_double(0.2))
    assert fwd(ws_bytes=small) == WORKSPACE                       # no room for the context rows
    assert L.spark_bsa_context_bf16(p, p, 3, 2, 16, 128, p, p, None) == INVALID    # dtype
    assert L.spark_bsa_context_bf16(p, p, 0, 2, 16, 96, p, p, None) == UNSUPPORTED
    assert L.spark_bsa_context_bf16(p, None, 0, 2, 16, 128, p, p, None) == INVALID
    assert L.spark_bsa_context_bf16(None, None, 0, 2, 0, 128, None, None, None) == 0  # no rows
    assert L.spark_bsa_attend_ctx(p, p, p, p, p, p, p, 1, None, p, 5, p, p, 1, p, 1, 1, 10, 128,
                                  p, 0, None, None) == INVALID   # Kc NULL with nc > 0
    assert L.spark_bsa_attend_ctx(p, p, p, p, p, p, p, 1, p, p, -3, p, p, 1, p, 1, 1, 10, 128,
                                  p, 0, None, None) == INVALID   # nc < 0


def test_reblock_entry_points_reject_bad_arguments(L):
    from block_sparse_attention_gather_b200 import (spark_reblock_levels,
                                                    spark_reblock_workspace_layout,
                                                    spark_reblock_workspace_size)
    lay = spark_reblock_workspace_layout(24, 241920, 128, 128)
    assert lay.nb == 1890 and lay.levels == 11
    assert lay.X % 256 == 0 and lay.total >= lay.X + 24 * 241920 * 128 * 2
    assert spark_reblock_levels(241920, 128) == 11
    assert spark_reblock_levels(1, 64) == 0
    assert spark_reblock_levels(0, 64) == -1
    assert spark_reblock_workspace_size(2, 1000, 96, 64) == 0         # d unsupported
    assert spark_reblock_workspace_size(2, 1000, 128, 129) == 0       # block > 128
    p = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)
    assert L.spark_reblock(p, p, 0, 2, 1000, 128, 64, 2, p, p, p, p, big, None) == INVALID   # mode
    assert L.spark_reblock(p, p, 5, 2, 1000, 128, 64, 0, p, p, p, p, big, None) == INVALID   # dtype
    assert L.spark_reblock(None, p, 0, 2, 1000, 128, 64, 0, p, p, p, p, big, None) == INVALID
    assert L.spark_reblock(p, p, 0, 2, 1000, 128, 64, 0, p, p, p, p, 1024, None) == WORKSPACE
    assert L.spark_reblock_level(2, 1000, 128, 64, 4, p, p, p, big, None) == INVALID    # in == out
    q = ctypes.c_void_p(0x200000)
    assert L.spark_reblock_level(2, 1000, 128, 64, 99, p, q, p, big, None) == INVALID   # level
    assert L.spark_reblock_whiten(p, p, 0, 2, 1000, 64, 64, p, 16, None) == WORKSPACE


def test_host_pipeline_rejects_bad_arguments(L):
    from block_sparse_attention_gather_b200 import spark_bsa_host_staging_size
    import torch
    assert spark_bsa_host_staging_size(24, 241920, 128, torch.bfloat16, 1890, 1890, 4) > 0
    assert spark_bsa_host_staging_size(24, 241920, 128, torch.bfloat16, 1890, 1890, 0) == 0
    four = spark_bsa_host_staging_size(24, 241920, 128, torch.bfloat16, 1890, 1890, 4)
    eight = spark_bsa_host_staging_size(24, 241920, 128, torch.bfloat16, 1890, 1890, 8)
    assert eight > four                                  # two slots of the chunk size
    p = ctypes.c_void_p(0x100000)
    big = ctypes.c_size_t(1 << 40)

    def call(hpc=2, staging_bytes=big, ws_bytes=big, out=p):
        return L.spark_bsa_forward_host(p, p, p, 0, 4, 1000, 128, p, p, p, 10, p, 10,
                                        ctypes.c_double(0.2), out, hpc, p, staging_bytes, p,
                                        ws_bytes, None, None, None)
    assert call(hpc=0) == INVALID
    assert call(out=None) == INVALID
    assert call(staging_bytes=16) == WORKSPACE
    assert call(ws_bytes=16) == WORKSPACE


def test_missing_library_fails_loudly(tmp_path):
    code = ("import block_sparse_attention_gather_b200._native as n;"
            f"n.LIB_PATH = {str(tmp_path / 'nope.so')!r};"
            "n._LIB = None\n"
            "try:\n    n.lib()\nexcept RuntimeError as e:\n    print('RAISED', 'no fallback' in str(e))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True)
    assert "RAISED True" in r.stdout, r.stderr


def test_wait_limit_is_a_process_wide_setting(L):
    from block_sparse_attention_gather_b200 import (spark_bsa_get_wait_limit_ns,
                                                    spark_bsa_set_wait_limit_ns)
    assert spark_bsa_get_wait_limit_ns() == 4_000_000_000         # 4 s by default
    try:
        spark_bsa_set_wait_limit_ns(123)
        assert spark_bsa_get_wait_limit_ns() == 123
        spark_bsa_set_wait_limit_ns(0)
        assert spark_bsa_get_wait_limit_ns() == 0
    finally:
        spark_bsa_set_wait_limit_ns(4_000_000_000)


def test_fused_routing_support_follows_shared_memory(L):
    from block_sparse_attention_gather_b200 import spark_bsa_fused_supported
    assert spark_bsa_fused_supported(128, 1890, 0.1)              # 768p
    assert spark_bsa_fused_supported(128, 473, 0.1)               # 384p
    assert not spark_bsa_fused_supported(64, 1890, 0.1)           # d = 64
    assert not spark_bsa_fused_supported(128, 1890, 1.0)          # no compressed branch
    assert not spark_bsa_fused_supported(128, 2540, 0.1)          # routing state too large
    p = ctypes.c_void_p(0x100000)
    # d = 64: refused before anything is launched
    assert L.spark_bsa_forward_fused(p, p, p, 0, 1, 1024, 64, p, p, p, 16, p, 16,
                                     ctypes.c_double(0.125), p, p, ctypes.c_size_t(1 << 40),
                                     None) == 2


def test_host_pipeline_staging_grows_with_context_rows(L):
    from block_sparse_attention_gather_b200 import spark_bsa_host_staging_size_ex
    import torch
    base = spark_bsa_host_staging_size_ex(24, 241920, 128, torch.bfloat16, 1890, 1890, 1, 0)
    ctx = spark_bsa_host_staging_size_ex(24, 241920, 128, torch.bfloat16, 1890, 1890, 1, 512)
    assert base > 0 and ctx >= base + 2 * 2 * 512 * 128 * 2      # Kc, Vc in both slots
    assert spark_bsa_host_staging_size_ex(24, 241920, 128, torch.bfloat16, 1890, 1890, 1, -1) == 0
