"""ctypes binding of ``libspark_bsa.so`` (include/spark_bsa.h).

Argument marshalling only: every step of the forward pass runs in the library's sm_100a
kernels.  PyTorch provides device memory, the current CUDA stream and dtype/shape checks.
There is no fallback: if the library is missing or was built for another GPU the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB_PATH

__all__ = [
    "SparkError", "SPARK_BF16", "SPARK_F32", "DEVERR", "Layout", "lib",
    "spark_status_string", "spark_bsa_topk_count", "spark_bsa_workspace_layout",
    "spark_bsa_workspace_size", "spark_bsa_forward", "spark_bsa_read_error",
    "spark_bsa_gather_q", "spark_bsa_anchor", "spark_bsa_gather_kv_summarize",
    "spark_bsa_route", "spark_bsa_attend", "workspace_views", "spark_bsa_forward_noalloc",
    "spark_bsa_workspace_size_ctx", "spark_bsa_forward_ctx", "spark_bsa_context_bf16",
    "spark_bsa_attend_ctx", "ReblockLayout", "spark_reblock_workspace_layout",
    "spark_reblock_workspace_size", "spark_reblock_levels", "spark_reblock",
    "spark_reblock_whiten", "spark_reblock_level", "reblock_views",
    "spark_bsa_host_staging_size", "spark_bsa_forward_host", "spark_bsa_quantize_fp8",
    "spark_bsa_attend_fp8", "spark_bsa_workspace_size_fp8", "spark_bsa_forward_fp8",
    "spark_bsa_gather_kv_meanpool", "spark_bsa_route_threshold", "spark_bsa_attend_var",
    "spark_bsa_set_wait_limit_ns", "spark_bsa_get_wait_limit_ns",
    "spark_bsa_host_staging_size_ex", "spark_bsa_fused_supported", "spark_bsa_forward_fused",
    "spark_bsa_attend_fused",
]

SPARK_BF16, SPARK_F32 = 0, 1
DEVERR = {"perm": 0x1, "offsets": 0x2, "sel": 0x4, "timeout": 0x8}
EXPORTED = [
    "spark_status_string", "spark_bsa_topk_count", "spark_bsa_workspace_layout",
    "spark_bsa_workspace_size", "spark_bsa_forward", "spark_bsa_read_error",
    "spark_bsa_gather_q", "spark_bsa_anchor", "spark_bsa_gather_kv_summarize",
    "spark_bsa_route", "spark_bsa_attend", "spark_bsa_forward_noalloc",
    "spark_bsa_workspace_size_ctx", "spark_bsa_forward_ctx", "spark_bsa_context_bf16",
    "spark_bsa_attend_ctx", "spark_reblock_workspace_layout", "spark_reblock_workspace_size",
    "spark_reblock_levels", "spark_reblock", "spark_reblock_whiten", "spark_reblock_level",
    "spark_bsa_host_staging_size", "spark_bsa_forward_host", "spark_bsa_quantize_fp8",
    "spark_bsa_attend_fp8", "spark_bsa_workspace_size_fp8", "spark_bsa_forward_fp8",
    "spark_bsa_gather_kv_meanpool", "spark_bsa_route_threshold", "spark_bsa_attend_var",
    "spark_bsa_set_wait_limit_ns", "spark_bsa_get_wait_limit_ns",
    "spark_bsa_host_staging_size_ex", "spark_bsa_forward_host_ex", "spark_bsa_fused_supported",
    "spark_bsa_forward_fused", "spark_bsa_attend_fused",
]
REBLOCK_MODES = {"q_reuse_k": 0, "separate": 1}


class SparkError(RuntimeError):
    def __init__(self, fn, status, msg=""):
        super().__init__(f"{fn} failed: {spark_status_string(status)} ({status}) {msg}".strip())
        self.status = status


class Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "Qp", "Kp", "Vp", "qbar_blocks", "qbar", "kbar", "k_tilde", "v_tilde", "cbias", "sel",
        "err", "total")] + [("k", ctypes.c_int)]


class ReblockLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("M", "W", "X", "total")] + \
        [("levels", ctypes.c_int), ("nb", ctypes.c_int)]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double
_SZ = ctypes.c_size_t


def lib():
    """Loads the library once; raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_gather_b200.build`"
            " (nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "spark_status_string": (ctypes.c_char_p, [_I]),
        "spark_bsa_topk_count": (_I, [_I, _D]),
        "spark_bsa_set_wait_limit_ns": (None, [ctypes.c_uint64]),
        "spark_bsa_get_wait_limit_ns": (ctypes.c_uint64, []),
        "spark_bsa_workspace_layout": (_I, [_I, _I, _I, _I, _I, _D, ctypes.POINTER(Layout)]),
        "spark_bsa_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _D]),
        "spark_bsa_forward": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _I, _D, _P,
                                   _P, _SZ, _P]),
        "spark_bsa_read_error": (_I, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
        "spark_bsa_gather_q": (_I, [_P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P]),
        "spark_bsa_anchor": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
        "spark_bsa_gather_kv_summarize": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P,
                                               _P, _P, _P, _P, _P, _P]),
        "spark_bsa_route": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
        "spark_bsa_attend": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _P, _I, _I, _I,
                                  _I, _P, _I, _P, _P]),
        "spark_bsa_forward_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _I,
                                           _D, _P, _P]),
        "spark_bsa_workspace_size_ctx": (_SZ, [_I, _I, _I, _I, _I, _D, _I]),
        "spark_bsa_forward_ctx": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _I,
                                       _P, _I, _D, _P, _P, _SZ, _P]),
        "spark_bsa_context_bf16": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
        "spark_bsa_attend_ctx": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _I,
                                      _P, _I, _I, _I, _I, _P, _I, _P, _P]),
        "spark_reblock_workspace_layout": (_I, [_I, _I, _I, _I, ctypes.POINTER(ReblockLayout)]),
        "spark_reblock_workspace_size": (_SZ, [_I, _I, _I, _I]),
        "spark_reblock_levels": (_I, [_I, _I]),
        "spark_reblock": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
        "spark_reblock_whiten": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _SZ, _P]),
        "spark_reblock_level": (_I, [_I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
        "spark_bsa_host_staging_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
        "spark_bsa_host_staging_size_ex": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
        "spark_bsa_fused_supported": (_I, [_I, _I, _D]),
        "spark_bsa_forward_fused": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _I, _D,
                                         _P, _P, _SZ, _P]),
        "spark_bsa_attend_fused": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _P, _I,
                                        _I, _I, _I, _P, _I, _P, _P, _P]),
        "spark_bsa_forward_host_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P,
                                           _P, _I, _P, _I, _D, _P, _I, _P, _SZ, _P, _SZ, _P,
                                           _P, _P]),
        "spark_bsa_forward_host": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _I, _D,
                                        _P, _I, _P, _SZ, _P, _SZ, _P, _P, _P]),
        "spark_bsa_quantize_fp8": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P]),
        "spark_bsa_route_threshold": (_I, [_P, _P, _I, _I, _I, _I, _D, _I, _P, _P, _P, _P]),
        "spark_bsa_attend_var": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _P, _I,
                                      _I, _I, _I, _P, _I, _P, _P]),
        "spark_bsa_gather_kv_meanpool": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P, _P,
                                              _P, _P, _P, _P, _P]),
        "spark_bsa_attend_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I,
                                      _P, _P, _I, _P, _I, _I, _I, _I, _P, _I, _P, _P]),
        "spark_bsa_workspace_size_fp8": (_SZ, [_I, _I, _I, _I, _I, _D, _I]),
        "spark_bsa_forward_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _I,
                                       _P, _I, _D, _P, _P, _SZ, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L


# ---------------------------------------------------------------------------- helpers

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _code(dtype):
    if dtype == torch.bfloat16:
        return SPARK_BF16
    if dtype == torch.float32:
        return SPARK_F32
    raise TypeError(f"unsupported dtype {dtype}")


def _check(fn, status):
    if status != 0:
        raise SparkError(fn, status)


# ------------------------------------------------------------------------- host calls

def spark_status_string(status: int) -> str:
    return lib().spark_status_string(int(status)).decode()


def spark_bsa_topk_count(nkb: int, topk_ratio: float) -> int:
    return int(lib().spark_bsa_topk_count(int(nkb), float(topk_ratio)))


def spark_bsa_set_wait_limit_ns(limit_ns: int) -> None:
    """Process-wide limit of the kernels' bounded waits (nanoseconds; default 4e9)."""
    lib().spark_bsa_set_wait_limit_ns(int(limit_ns))


def spark_bsa_get_wait_limit_ns() -> int:
    return int(lib().spark_bsa_get_wait_limit_ns())


def spark_bsa_workspace_layout(H, N, d, nqb, nkb, topk_ratio) -> Layout:
    L = Layout()
    _check("spark_bsa_workspace_layout",
           lib().spark_bsa_workspace_layout(H, N, d, nqb, nkb, float(topk_ratio), ctypes.byref(L)))
    return L


def spark_bsa_workspace_size(H, N, d, nqb, nkb, topk_ratio) -> int:
    return int(lib().spark_bsa_workspace_size(H, N, d, nqb, nkb, float(topk_ratio)))


def workspace_views(workspace: torch.Tensor, layout: Layout, H, N, d, nqb, nkb) -> dict:
    """Typed views of the intermediates a spark_bsa_forward call left in `workspace`."""
    def view(off, count, dt):
        nbytes = count * torch.empty(0, dtype=dt).element_size()
        return workspace[off:off + nbytes].view(dt)
    k = layout.k
    return {
        "Qp": view(layout.Qp, H * N * d, torch.bfloat16).view(H, N, d),
        "Kp": view(layout.Kp, H * N * d, torch.bfloat16).view(H, N, d),
        "Vp": view(layout.Vp, H * N * d, torch.bfloat16).view(H, N, d),
        "qbar_blocks": view(layout.qbar_blocks, H * nqb * d, torch.float32).view(H, nqb, d),
        "qbar": view(layout.qbar, H * d, torch.float32).view(H, d),
        "kbar": view(layout.kbar, H * nkb * d, torch.float32).view(H, d, nkb),   # d-major
        "k_tilde": view(layout.k_tilde, H * nkb * d, torch.bfloat16).view(H, nkb, d),
        "v_tilde": view(layout.v_tilde, H * nkb * d, torch.bfloat16).view(H, nkb, d),
        "cbias": view(layout.cbias, H * nkb, torch.float32).view(H, nkb),
        "sel": view(layout.sel, H * nqb * k, torch.int32).view(H, nqb, k),
        "err": view(layout.err, 1, torch.int32),
    }


# --------------------------------------------------------------------------- device calls

def spark_bsa_forward(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, topk_ratio, out=None,
                      workspace=None, stream=None):
    """The whole forward pass on the current CUDA stream; returns (out, workspace, layout)."""
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    dev = Q.device
    for n, t in (("K", K), ("V", V)):
        _need(t, n, Q.dtype, dev)
    H, N, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V must share the shape [H, N, d]")
    for n, t in (("q_perm", q_perm), ("k_perm", k_perm)):
        _need(t, n, torch.int32, dev)
        if t.shape != (H, N):
            raise ValueError(f"{n} must have shape [H, N]")
    for n, t in (("q_offsets", q_offsets), ("k_offsets", k_offsets)):
        _need(t, n, torch.int32, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    layout = spark_bsa_workspace_layout(H, N, d, nqb, nkb, topk_ratio)
    if out is None:
        out = torch.empty_like(Q)
    _need(out, "out", Q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(layout.total, dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    st = lib().spark_bsa_forward(_ptr(Q), _ptr(K), _ptr(V), _code(Q.dtype), H, N, d,
                                 _ptr(q_perm), _ptr(k_perm), _ptr(q_offsets), nqb,
                                 _ptr(k_offsets), nkb, float(topk_ratio), _ptr(out),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check("spark_bsa_forward", st)
    return out, workspace, layout


def spark_bsa_fused_supported(d: int, nkb: int, topk_ratio: float) -> bool:
    return bool(lib().spark_bsa_fused_supported(int(d), int(nkb), float(topk_ratio)))


def spark_bsa_forward_fused(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, topk_ratio, out=None,
                            workspace=None, stream=None):
    """spark_bsa_forward with the routing inside the attention kernel; returns (out, workspace,
    layout) with the selections copied to the workspace's sel region."""
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    dev = Q.device
    for n, t in (("K", K), ("V", V)):
        _need(t, n, Q.dtype, dev)
    H, N, d = Q.shape
    for n, t in (("q_perm", q_perm), ("k_perm", k_perm), ("q_offsets", q_offsets),
                 ("k_offsets", k_offsets)):
        _need(t, n, torch.int32, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    layout = spark_bsa_workspace_layout(H, N, d, nqb, nkb, topk_ratio)
    if out is None:
        out = torch.empty_like(Q)
    _need(out, "out", Q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(layout.total, dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    st = lib().spark_bsa_forward_fused(_ptr(Q), _ptr(K), _ptr(V), _code(Q.dtype), H, N, d,
                                       _ptr(q_perm), _ptr(k_perm), _ptr(q_offsets), nqb,
                                       _ptr(k_offsets), nkb, float(topk_ratio), _ptr(out),
                                       _ptr(workspace), workspace.numel(), _stream(stream))
    _check("spark_bsa_forward_fused", st)
    return out, workspace, layout


def spark_bsa_attend_fused(Qp, Kp, Vp, k_tilde, v_tilde, cbias, qbar_blocks, kbar, k, q_perm,
                           q_offsets, k_offsets, out_dtype=torch.bfloat16, out=None, sel_out=None,
                           err=None, stream=None):
    _need(Qp, "Qp", torch.bfloat16)
    dev = Qp.device
    H, N, d = Qp.shape
    for n, t, dt in (("Kp", Kp, torch.bfloat16), ("Vp", Vp, torch.bfloat16),
                     ("k_tilde", k_tilde, torch.bfloat16), ("v_tilde", v_tilde, torch.bfloat16),
                     ("cbias", cbias, torch.float32), ("qbar_blocks", qbar_blocks, torch.float32),
                     ("kbar", kbar, torch.float32), ("q_perm", q_perm, torch.int32),
                     ("q_offsets", q_offsets, torch.int32), ("k_offsets", k_offsets, torch.int32)):
        _need(t, n, dt, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    if out is None:
        out = torch.empty(H, N, d, dtype=out_dtype, device=dev)
    st = lib().spark_bsa_attend_fused(_ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(k_tilde), _ptr(v_tilde),
                                      _ptr(cbias), _ptr(qbar_blocks), _ptr(kbar), int(k),
                                      _ptr(q_perm), _ptr(q_offsets), nqb, _ptr(k_offsets), nkb,
                                      H, N, d, _ptr(out), _code(out.dtype), _ptr(sel_out),
                                      _ptr(err), _stream(stream))
    _check("spark_bsa_attend_fused", st)
    return out


def spark_bsa_read_error(err_word: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device error word (0 = no error)."""
    _need(err_word, "err_word")
    flags = ctypes.c_uint32(0)
    st = lib().spark_bsa_read_error(_ptr(err_word), _stream(stream), ctypes.byref(flags))
    if st not in (0, 5):
        raise SparkError("spark_bsa_read_error", st)
    return int(flags.value)


def spark_bsa_gather_q(Q, q_perm, q_offsets, Qp=None, qbar_blocks=None, err=None, stream=None):
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    H, N, d = Q.shape
    nqb = q_offsets.numel() - 1
    Qp = torch.empty(H, N, d, dtype=torch.bfloat16, device=Q.device) if Qp is None else Qp
    qbar_blocks = (torch.empty(H, nqb, d, dtype=torch.float32, device=Q.device)
                   if qbar_blocks is None else qbar_blocks)
    for n, t, dt in (("q_perm", q_perm, torch.int32), ("q_offsets", q_offsets, torch.int32),
                     ("Qp", Qp, torch.bfloat16), ("qbar_blocks", qbar_blocks, torch.float32)):
        _need(t, n, dt, Q.device)
    st = lib().spark_bsa_gather_q(_ptr(Q), _code(Q.dtype), H, N, d, _ptr(q_perm),
                                  _ptr(q_offsets), nqb, _ptr(Qp), _ptr(qbar_blocks), _ptr(err),
                                  _stream(stream))
    _check("spark_bsa_gather_q", st)
    return Qp, qbar_blocks


def spark_bsa_anchor(qbar_blocks, q_offsets, N, qbar=None, stream=None):
    _need(qbar_blocks, "qbar_blocks", torch.float32)
    H, nqb, d = qbar_blocks.shape
    qbar = torch.empty(H, d, dtype=torch.float32, device=qbar_blocks.device) if qbar is None else qbar
    _need(q_offsets, "q_offsets", torch.int32, qbar_blocks.device)
    _need(qbar, "qbar", torch.float32, qbar_blocks.device)
    st = lib().spark_bsa_anchor(_ptr(qbar_blocks), _ptr(q_offsets), H, N, d, nqb, _ptr(qbar),
                                _stream(stream))
    _check("spark_bsa_anchor", st)
    return qbar


def spark_bsa_gather_kv_summarize(K, V, k_perm, k_offsets, qbar, err=None, stream=None):
    _need(K, "K", (torch.bfloat16, torch.float32))
    _need(V, "V", K.dtype, K.device)
    H, N, d = K.shape
    nkb = k_offsets.numel() - 1
    dev = K.device
    _need(k_perm, "k_perm", torch.int32, dev)
    _need(k_offsets, "k_offsets", torch.int32, dev)
    _need(qbar, "qbar", torch.float32, dev)
    Kp = torch.empty(H, N, d, dtype=torch.bfloat16, device=dev)
    Vp = torch.empty_like(Kp)
    kbar = torch.empty(H, d, nkb, dtype=torch.float32, device=dev)          # d-major
    k_tilde = torch.empty(H, nkb, d, dtype=torch.bfloat16, device=dev)
    v_tilde = torch.empty_like(k_tilde)
    cbias = torch.empty(H, nkb, dtype=torch.float32, device=dev)
    st = lib().spark_bsa_gather_kv_summarize(
        _ptr(K), _ptr(V), _code(K.dtype), H, N, d, _ptr(k_perm), _ptr(k_offsets), nkb,
        _ptr(qbar), _ptr(Kp), _ptr(Vp), _ptr(kbar), _ptr(k_tilde), _ptr(v_tilde), _ptr(cbias),
        _ptr(err), _stream(stream))
    _check("spark_bsa_gather_kv_summarize", st)
    return Kp, Vp, kbar, k_tilde, v_tilde, cbias


def spark_bsa_route_threshold(qbar_blocks, kbar, tau, kcap, err=None, stream=None):
    """Threshold routing (mu + tau*sigma per query block, at most kcap blocks); returns
    (sel [H, nqb, kcap] with the first count entries of each row valid, count [H, nqb])."""
    _need(qbar_blocks, "qbar_blocks", torch.float32)
    _need(kbar, "kbar", torch.float32, qbar_blocks.device)
    H, nqb, d = qbar_blocks.shape
    nkb = kbar.shape[2]                                                     # kbar is [H, d, nkb]
    sel = torch.full((H, nqb, kcap), -1, dtype=torch.int32, device=qbar_blocks.device)
    count = torch.empty(H, nqb, dtype=torch.int32, device=qbar_blocks.device)
    st = lib().spark_bsa_route_threshold(_ptr(qbar_blocks), _ptr(kbar), H, nqb, nkb, d,
                                         float(tau), int(kcap), _ptr(sel), _ptr(count),
                                         _ptr(err), _stream(stream))
    _check("spark_bsa_route_threshold", st)
    return sel, count


def spark_bsa_attend_var(Qp, Kp, Vp, k_tilde, v_tilde, cbias, sel, count, q_perm, q_offsets,
                         k_offsets, out_dtype=torch.bfloat16, out=None, err=None, stream=None):
    """spark_bsa_attend with a per-query-block count of selected blocks (sel [H, nqb, kcap])."""
    _need(Qp, "Qp", torch.bfloat16)
    dev = Qp.device
    H, N, d = Qp.shape
    for n, t, dt in (("Kp", Kp, torch.bfloat16), ("Vp", Vp, torch.bfloat16),
                     ("k_tilde", k_tilde, torch.bfloat16), ("v_tilde", v_tilde, torch.bfloat16),
                     ("cbias", cbias, torch.float32), ("sel", sel, torch.int32),
                     ("count", count, torch.int32), ("q_perm", q_perm, torch.int32),
                     ("q_offsets", q_offsets, torch.int32), ("k_offsets", k_offsets, torch.int32)):
        _need(t, n, dt, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    kcap = sel.shape[-1]
    if out is None:
        out = torch.empty(H, N, d, dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, dev)
    st = lib().spark_bsa_attend_var(_ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(k_tilde), _ptr(v_tilde),
                                    _ptr(cbias), _ptr(sel), kcap, _ptr(count), _ptr(q_perm),
                                    _ptr(q_offsets), nqb, _ptr(k_offsets), nkb, H, N, d,
                                    _ptr(out), _code(out_dtype), _ptr(err), _stream(stream))
    _check("spark_bsa_attend_var", st)
    return out


def spark_bsa_gather_kv_meanpool(K, V, k_perm, k_offsets, err=None, stream=None):
    """The baseline BSA compressed branch (mean key, mean value, offset log|B|) with the same
    gathered Kp, Vp and key-block means as spark_bsa_gather_kv_summarize; returns
    (Kp, Vp, kbar, k_tilde, v_tilde, cbias)."""
    _need(K, "K", (torch.bfloat16, torch.float32))
    dev = K.device
    H, N, d = K.shape
    _need(V, "V", K.dtype, dev)
    _need(k_perm, "k_perm", torch.int32, dev)
    _need(k_offsets, "k_offsets", torch.int32, dev)
    nkb = k_offsets.numel() - 1
    Kp = torch.empty(H, N, d, dtype=torch.bfloat16, device=dev)
    Vp = torch.empty_like(Kp)
    kbar = torch.empty(H, d, nkb, dtype=torch.float32, device=dev)          # d-major
    k_tilde = torch.empty(H, nkb, d, dtype=torch.bfloat16, device=dev)
    v_tilde = torch.empty_like(k_tilde)
    cbias = torch.empty(H, nkb, dtype=torch.float32, device=dev)
    st = lib().spark_bsa_gather_kv_meanpool(
        _ptr(K), _ptr(V), _code(K.dtype), H, N, d, _ptr(k_perm), _ptr(k_offsets), nkb, _ptr(Kp),
        _ptr(Vp), _ptr(kbar), _ptr(k_tilde), _ptr(v_tilde), _ptr(cbias), _ptr(err),
        _stream(stream))
    _check("spark_bsa_gather_kv_meanpool", st)
    return Kp, Vp, kbar, k_tilde, v_tilde, cbias


def spark_bsa_route(qbar_blocks, kbar, k, err=None, stream=None):
    _need(qbar_blocks, "qbar_blocks", torch.float32)
    _need(kbar, "kbar", torch.float32, qbar_blocks.device)
    H, nqb, d = qbar_blocks.shape
    nkb = kbar.shape[2]                                                     # kbar is [H, d, nkb]
    sel = torch.empty(H, nqb, k, dtype=torch.int32, device=qbar_blocks.device)
    st = lib().spark_bsa_route(_ptr(qbar_blocks), _ptr(kbar), H, nqb, nkb, d, int(k), _ptr(sel),
                               _ptr(err), _stream(stream))
    _check("spark_bsa_route", st)
    return sel


def spark_bsa_attend(Qp, Kp, Vp, k_tilde, v_tilde, cbias, sel, q_perm, q_offsets, k_offsets,
                     out_dtype=torch.bfloat16, out=None, err=None, stream=None):
    _need(Qp, "Qp", torch.bfloat16)
    dev = Qp.device
    H, N, d = Qp.shape
    for n, t, dt in (("Kp", Kp, torch.bfloat16), ("Vp", Vp, torch.bfloat16),
                     ("k_tilde", k_tilde, torch.bfloat16), ("v_tilde", v_tilde, torch.bfloat16),
                     ("cbias", cbias, torch.float32), ("sel", sel, torch.int32),
                     ("q_perm", q_perm, torch.int32), ("q_offsets", q_offsets, torch.int32),
                     ("k_offsets", k_offsets, torch.int32)):
        _need(t, n, dt, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    k = sel.shape[-1]
    if out is None:
        out = torch.empty(H, N, d, dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, dev)
    st = lib().spark_bsa_attend(_ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(k_tilde), _ptr(v_tilde),
                                _ptr(cbias), _ptr(sel), k, _ptr(q_perm), _ptr(q_offsets), nqb,
                                _ptr(k_offsets), nkb, H, N, d, _ptr(out), _code(out_dtype),
                                _ptr(err), _stream(stream))
    _check("spark_bsa_attend", st)
    return out


def spark_bsa_forward_noalloc(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, topk_ratio,
                              out, stream=None):
    """The forward pass with the library's static scratch array as its workspace (for callers
    that cannot allocate device memory while they run); `out` must be preallocated.  Small
    problems only: the workspace must fit SPARK_NOALLOC_SCRATCH_BYTES (16 MiB)."""
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    dev = Q.device
    H, N, d = Q.shape
    for n, t in (("K", K), ("V", V), ("out", out)):
        _need(t, n, Q.dtype, dev)
    for n, t in (("q_perm", q_perm), ("k_perm", k_perm), ("q_offsets", q_offsets),
                 ("k_offsets", k_offsets)):
        _need(t, n, torch.int32, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    st = lib().spark_bsa_forward_noalloc(_ptr(Q), _ptr(K), _ptr(V), _code(Q.dtype), H, N, d,
                                         _ptr(q_perm), _ptr(k_perm), _ptr(q_offsets), nqb,
                                         _ptr(k_offsets), nkb, float(topk_ratio), _ptr(out),
                                         _stream(stream))
    _check("spark_bsa_forward_noalloc", st)
    return out


# ------------------------------------------------------------------ context (sink) tokens

def spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, topk_ratio, nc) -> int:
    return int(lib().spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, float(topk_ratio), int(nc)))


def _context_args(Kc, Vc, H, d, dtype, dev):
    if Kc is None and Vc is None:
        return None, None, 0
    _need(Kc, "Kc", dtype, dev)
    _need(Vc, "Vc", dtype, dev)
    if Kc.dim() != 3 or Kc.shape[0] != H or Kc.shape[2] != d or Vc.shape != Kc.shape:
        raise ValueError("Kc and Vc must have the shape [H, nc, d]")
    return Kc, Vc, Kc.shape[1]


def spark_bsa_forward_ctx(Q, K, V, Kc, Vc, q_perm, k_perm, q_offsets, k_offsets, topk_ratio,
                          out=None, workspace=None, stream=None):
    """spark_bsa_forward with context (sink) tokens Kc, Vc [H, nc, d] (same dtype as Q);
    returns (out, workspace, layout).  The workspace holds the layout's intermediates followed
    by the bf16 context rows."""
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    dev = Q.device
    H, N, d = Q.shape
    for n, t in (("K", K), ("V", V)):
        _need(t, n, Q.dtype, dev)
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V must share the shape [H, N, d]")
    Kc, Vc, nc = _context_args(Kc, Vc, H, d, Q.dtype, dev)
    for n, t in (("q_perm", q_perm), ("k_perm", k_perm)):
        _need(t, n, torch.int32, dev)
        if t.shape != (H, N):
            raise ValueError(f"{n} must have shape [H, N]")
    for n, t in (("q_offsets", q_offsets), ("k_offsets", k_offsets)):
        _need(t, n, torch.int32, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    layout = spark_bsa_workspace_layout(H, N, d, nqb, nkb, topk_ratio)
    size = spark_bsa_workspace_size_ctx(H, N, d, nqb, nkb, topk_ratio, nc)
    if out is None:
        out = torch.empty_like(Q)
    _need(out, "out", Q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(size, dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    st = lib().spark_bsa_forward_ctx(_ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(Vc), nc,
                                     _code(Q.dtype), H, N, d, _ptr(q_perm), _ptr(k_perm),
                                     _ptr(q_offsets), nqb, _ptr(k_offsets), nkb,
                                     float(topk_ratio), _ptr(out), _ptr(workspace),
                                     workspace.numel(), _stream(stream))
    _check("spark_bsa_forward_ctx", st)
    return out, workspace, layout


def spark_bsa_context_bf16(Kc, Vc, Kc_bf16=None, Vc_bf16=None, stream=None):
    """bf16 copies of the context rows ([H, nc, d]); returns (Kc_bf16, Vc_bf16)."""
    _need(Kc, "Kc", (torch.bfloat16, torch.float32))
    H, nc, d = Kc.shape
    Kc, Vc, nc = _context_args(Kc, Vc, H, d, Kc.dtype, Kc.device)
    if Kc_bf16 is None:
        Kc_bf16 = torch.empty(H, nc, d, dtype=torch.bfloat16, device=Kc.device)
    if Vc_bf16 is None:
        Vc_bf16 = torch.empty(H, nc, d, dtype=torch.bfloat16, device=Kc.device)
    _need(Kc_bf16, "Kc_bf16", torch.bfloat16, Kc.device)
    _need(Vc_bf16, "Vc_bf16", torch.bfloat16, Kc.device)
    st = lib().spark_bsa_context_bf16(_ptr(Kc), _ptr(Vc), _code(Kc.dtype), H, nc, d,
                                      _ptr(Kc_bf16), _ptr(Vc_bf16), _stream(stream))
    _check("spark_bsa_context_bf16", st)
    return Kc_bf16, Vc_bf16


def spark_bsa_attend_ctx(Qp, Kp, Vp, k_tilde, v_tilde, cbias, sel, Kc, Vc, q_perm, q_offsets,
                         k_offsets, out_dtype=torch.bfloat16, out=None, err=None, stream=None):
    """spark_bsa_attend with bf16 context rows Kc, Vc [H, nc, d]."""
    _need(Qp, "Qp", torch.bfloat16)
    dev = Qp.device
    H, N, d = Qp.shape
    for n, t, dt in (("Kp", Kp, torch.bfloat16), ("Vp", Vp, torch.bfloat16),
                     ("k_tilde", k_tilde, torch.bfloat16), ("v_tilde", v_tilde, torch.bfloat16),
                     ("cbias", cbias, torch.float32), ("sel", sel, torch.int32),
                     ("q_perm", q_perm, torch.int32), ("q_offsets", q_offsets, torch.int32),
                     ("k_offsets", k_offsets, torch.int32)):
        _need(t, n, dt, dev)
    Kc, Vc, nc = _context_args(Kc, Vc, H, d, torch.bfloat16, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    k = sel.shape[-1]
    if out is None:
        out = torch.empty(H, N, d, dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, dev)
    st = lib().spark_bsa_attend_ctx(_ptr(Qp), _ptr(Kp), _ptr(Vp), _ptr(k_tilde), _ptr(v_tilde),
                                    _ptr(cbias), _ptr(sel), k, _ptr(Kc), _ptr(Vc), nc,
                                    _ptr(q_perm), _ptr(q_offsets), nqb, _ptr(k_offsets), nkb,
                                    H, N, d, _ptr(out), _code(out_dtype), _ptr(err),
                                    _stream(stream))
    _check("spark_bsa_attend_ctx", st)
    return out


# ------------------------------------------------------------------------- FP8 logits

def spark_bsa_quantize_fp8(src, group_offsets=None, dst=None, scales=None, err=None,
                           stream=None):
    """e4m3 codes (torch.uint8 [H, R, d]) and power-of-two group scales (fp32 [H, ngroups]) of
    bf16 rows src [H, R, d]; groups are the blocks of group_offsets (int32 [ngroups+1]) or,
    when it is None, 128-row tiles.  Returns (dst, scales)."""
    _need(src, "src", torch.bfloat16)
    dev = src.device
    H, R, d = src.shape
    if group_offsets is None:
        ngroups = (R + 127) // 128
    else:
        _need(group_offsets, "group_offsets", torch.int32, dev)
        ngroups = group_offsets.numel() - 1
    if dst is None:
        dst = torch.empty(H, R, d, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(H, ngroups, dtype=torch.float32, device=dev)
    _need(dst, "dst", torch.uint8, dev)
    _need(scales, "scales", torch.float32, dev)
    st = lib().spark_bsa_quantize_fp8(_ptr(src), H, R, d, _ptr(group_offsets), ngroups,
                                      _ptr(dst), _ptr(scales), _ptr(err), _stream(stream))
    _check("spark_bsa_quantize_fp8", st)
    return dst, scales


def spark_bsa_attend_fp8(Qp8, q_scale, Kp8, k_scale, Vp, kt8, kt_scale, v_tilde, cbias, sel,
                         q_perm, q_offsets, k_offsets, Kc8=None, kc_scale=None, Vc=None,
                         out_dtype=torch.bfloat16, out=None, err=None, stream=None):
    """The attention step with FP8 logits (codes and scales from spark_bsa_quantize_fp8,
    values in bf16; d = 128)."""
    _need(Qp8, "Qp8", torch.uint8)
    dev = Qp8.device
    H, N, d = Qp8.shape
    for n, t, dt in (("q_scale", q_scale, torch.float32), ("Kp8", Kp8, torch.uint8),
                     ("k_scale", k_scale, torch.float32), ("Vp", Vp, torch.bfloat16),
                     ("kt8", kt8, torch.uint8), ("kt_scale", kt_scale, torch.float32),
                     ("v_tilde", v_tilde, torch.bfloat16), ("cbias", cbias, torch.float32),
                     ("sel", sel, torch.int32), ("q_perm", q_perm, torch.int32),
                     ("q_offsets", q_offsets, torch.int32), ("k_offsets", k_offsets, torch.int32)):
        _need(t, n, dt, dev)
    nc = 0
    if Kc8 is not None:
        _need(Kc8, "Kc8", torch.uint8, dev)
        _need(kc_scale, "kc_scale", torch.float32, dev)
        _need(Vc, "Vc", torch.bfloat16, dev)
        nc = Kc8.shape[1]
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    k = sel.shape[-1]
    if out is None:
        out = torch.empty(H, N, d, dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, dev)
    st = lib().spark_bsa_attend_fp8(_ptr(Qp8), _ptr(q_scale), _ptr(Kp8), _ptr(k_scale), _ptr(Vp),
                                    _ptr(kt8), _ptr(kt_scale), _ptr(v_tilde), _ptr(cbias),
                                    _ptr(sel), k, _ptr(Kc8), _ptr(kc_scale), _ptr(Vc), nc,
                                    _ptr(q_perm), _ptr(q_offsets), nqb, _ptr(k_offsets), nkb,
                                    H, N, d, _ptr(out), _code(out_dtype), _ptr(err),
                                    _stream(stream))
    _check("spark_bsa_attend_fp8", st)
    return out


def spark_bsa_workspace_size_fp8(H, N, d, nqb, nkb, topk_ratio, nc=0) -> int:
    return int(lib().spark_bsa_workspace_size_fp8(H, N, d, nqb, nkb, float(topk_ratio), int(nc)))


def spark_bsa_forward_fp8(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, topk_ratio, Kc=None,
                          Vc=None, out=None, workspace=None, stream=None):
    """spark_bsa_forward_ctx with FP8 logits (d = 128); returns (out, workspace, layout)."""
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    dev = Q.device
    H, N, d = Q.shape
    for n, t in (("K", K), ("V", V)):
        _need(t, n, Q.dtype, dev)
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K, V must share the shape [H, N, d]")
    Kc, Vc, nc = _context_args(Kc, Vc, H, d, Q.dtype, dev)
    for n, t in (("q_perm", q_perm), ("k_perm", k_perm)):
        _need(t, n, torch.int32, dev)
    for n, t in (("q_offsets", q_offsets), ("k_offsets", k_offsets)):
        _need(t, n, torch.int32, dev)
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    layout = spark_bsa_workspace_layout(H, N, d, nqb, nkb, topk_ratio)
    size = spark_bsa_workspace_size_fp8(H, N, d, nqb, nkb, topk_ratio, nc)
    if size == 0:
        raise SparkError("spark_bsa_workspace_size_fp8", 2)
    if out is None:
        out = torch.empty_like(Q)
    _need(out, "out", Q.dtype, dev)
    if workspace is None:
        workspace = torch.empty(size, dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    st = lib().spark_bsa_forward_fp8(_ptr(Q), _ptr(K), _ptr(V), _ptr(Kc), _ptr(Vc), nc,
                                     _code(Q.dtype), H, N, d, _ptr(q_perm), _ptr(k_perm),
                                     _ptr(q_offsets), nqb, _ptr(k_offsets), nkb,
                                     float(topk_ratio), _ptr(out), _ptr(workspace),
                                     workspace.numel(), _stream(stream))
    _check("spark_bsa_forward_fp8", st)
    return out, workspace, layout


# ------------------------------------------------------------ Spark-Reblock partitioner

def spark_reblock_workspace_layout(H, N, d, block) -> ReblockLayout:
    L = ReblockLayout()
    _check("spark_reblock_workspace_layout",
           lib().spark_reblock_workspace_layout(H, N, d, block, ctypes.byref(L)))
    return L


def spark_reblock_workspace_size(H, N, d, block) -> int:
    return int(lib().spark_reblock_workspace_size(H, N, d, block))


def spark_reblock_levels(N, block) -> int:
    return int(lib().spark_reblock_levels(N, block))


def reblock_views(workspace: torch.Tensor, layout: ReblockLayout, H, N, d) -> dict:
    """Typed views of M, W (fp32 [H,d,d]) and X (bf16 [H,N,d]) in a reblock workspace."""
    def view(off, count, dt):
        nbytes = count * torch.empty(0, dtype=dt).element_size()
        return workspace[off:off + nbytes].view(dt)
    return {"M": view(layout.M, H * d * d, torch.float32).view(H, d, d),
            "W": view(layout.W, H * d * d, torch.float32).view(H, d, d),
            "X": view(layout.X, H * N * d, torch.bfloat16).view(H, N, d)}


def spark_reblock(Q, K, block, mode="q_reuse_k", workspace=None, stream=None):
    """Spark-Reblock partition of Q, K [H, N, d]; returns (q_perm, k_perm, offsets)."""
    _need(Q, "Q", (torch.bfloat16, torch.float32))
    _need(K, "K", Q.dtype, Q.device)
    H, N, d = Q.shape
    if K.shape != Q.shape:
        raise ValueError("Q and K must share the shape [H, N, d]")
    layout = spark_reblock_workspace_layout(H, N, d, block)
    if workspace is None:
        workspace = torch.empty(layout.total, dtype=torch.uint8, device=Q.device)
    _need(workspace, "workspace", torch.uint8, Q.device)
    q_perm = torch.empty(H, N, dtype=torch.int32, device=Q.device)
    k_perm = torch.empty_like(q_perm)
    offsets = torch.empty(layout.nb + 1, dtype=torch.int32, device=Q.device)
    st = lib().spark_reblock(_ptr(Q), _ptr(K), _code(Q.dtype), H, N, d, int(block),
                             REBLOCK_MODES[mode], _ptr(q_perm), _ptr(k_perm), _ptr(offsets),
                             _ptr(workspace), workspace.numel(), _stream(stream))
    _check("spark_reblock", st)
    return q_perm, k_perm, offsets


def spark_reblock_whiten(X, Y, block, workspace=None, stream=None):
    """Step: second moment of Y, its square root W, unit rows of W x into the workspace;
    returns (workspace, layout, views)."""
    _need(X, "X", (torch.bfloat16, torch.float32))
    _need(Y, "Y", X.dtype, X.device)
    H, N, d = X.shape
    layout = spark_reblock_workspace_layout(H, N, d, block)
    if workspace is None:
        workspace = torch.empty(layout.total, dtype=torch.uint8, device=X.device)
    st = lib().spark_reblock_whiten(_ptr(X), _ptr(Y), _code(X.dtype), H, N, d, int(block),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _check("spark_reblock_whiten", st)
    return workspace, layout, reblock_views(workspace, layout, H, N, d)


def spark_reblock_level(H, N, d, block, level, perm_in, workspace, perm_out=None, stream=None):
    """Step: the splits of one tree level over the workspace's X rows; returns perm_out."""
    _need(perm_in, "perm_in", torch.int32)
    if perm_out is None:
        perm_out = torch.empty_like(perm_in)
    st = lib().spark_reblock_level(H, N, d, int(block), int(level), _ptr(perm_in),
                                   _ptr(perm_out), _ptr(workspace), workspace.numel(),
                                   _stream(stream))
    _check("spark_reblock_level", st)
    return perm_out


# ------------------------------------------------ host buffers, pipelined by head chunks

def spark_bsa_host_staging_size(H, N, d, dtype, nqb, nkb, heads_per_chunk) -> int:
    return int(lib().spark_bsa_host_staging_size(H, N, d, _code(dtype), nqb, nkb,
                                                  heads_per_chunk))


def _need_host(t, name, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")


def spark_bsa_host_staging_size_ex(H, N, d, dtype, nqb, nkb, heads_per_chunk, nc) -> int:
    return int(lib().spark_bsa_host_staging_size_ex(H, N, d, _code(dtype), nqb, nkb,
                                                    heads_per_chunk, nc))


def spark_bsa_forward_host(Q, K, V, q_perm, k_perm, q_offsets, k_offsets, topk_ratio, out=None,
                           heads_per_chunk=1, device=None, staging=None, workspace=None,
                           streams=None, Kc=None, Vc=None, fp8=False):
    """The forward pass on HOST tensors (page-locked for overlap), pipelined by head chunks
    over three CUDA streams; returns `out` (host) once the work is enqueued on the compute
    stream (synchronise that stream, or the device, before reading it).  Kc, Vc (host
    [H, nc, d]) add context rows; fp8=True takes the logits in e4m3 (d = 128)."""
    _need_host(Q, "Q", (torch.bfloat16, torch.float32))
    for n, t in (("K", K), ("V", V)):
        _need_host(t, n, Q.dtype)
    for n, t in (("q_perm", q_perm), ("k_perm", k_perm), ("q_offsets", q_offsets),
                 ("k_offsets", k_offsets)):
        _need_host(t, n, torch.int32)
    H, N, d = Q.shape
    nc = 0
    if Kc is not None or Vc is not None:
        for n, t in (("Kc", Kc), ("Vc", Vc)):
            _need_host(t, n, Q.dtype)
        if Kc.shape != Vc.shape or Kc.shape[0] != H or Kc.shape[2] != d:
            raise ValueError("Kc, Vc must have the shape [H, nc, d]")
        nc = Kc.shape[1]
    nqb, nkb = q_offsets.numel() - 1, k_offsets.numel() - 1
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    hpc = max(1, min(int(heads_per_chunk), H))
    if out is None:
        out = torch.empty_like(Q).pin_memory()
    _need_host(out, "out", Q.dtype)
    if staging is None:
        staging = torch.empty(spark_bsa_host_staging_size_ex(H, N, d, Q.dtype, nqb, nkb, hpc, nc),
                              dtype=torch.uint8, device=dev)
    if workspace is None:
        size = (spark_bsa_workspace_size_fp8(hpc, N, d, nqb, nkb, topk_ratio, nc) if fp8 else
                spark_bsa_workspace_size_ctx(hpc, N, d, nqb, nkb, topk_ratio, nc))
        workspace = torch.empty(size, dtype=torch.uint8, device=dev)
    if streams is None:
        streams = (torch.cuda.current_stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    sc, sh, sd = (ctypes.c_void_p(s.cuda_stream) for s in streams)
    st = lib().spark_bsa_forward_host_ex(_ptr(Q), _ptr(K), _ptr(V),
                                         _ptr(Kc) if nc else None, _ptr(Vc) if nc else None, nc,
                                         1 if fp8 else 0, _code(Q.dtype), H, N, d,
                                         _ptr(q_perm), _ptr(k_perm), _ptr(q_offsets), nqb,
                                         _ptr(k_offsets), nkb, float(topk_ratio), _ptr(out), hpc,
                                         _ptr(staging), staging.numel(), _ptr(workspace),
                                         workspace.numel(), sc, sh, sd)
    _check("spark_bsa_forward_host", st)
    return out
