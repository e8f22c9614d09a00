"""B200 (sm_100a) Spark-Attn two-branch block-sparse attention forward.

The compute lives in ``libspark_bsa.so`` (hand-written CUDA for sm_100a, C ABI declared in
``include/spark_bsa.h``); this package is its ctypes binding plus the seeded input
generators.  The library is loaded on first use and its absence is an error: there is no
CPU or PyTorch fallback.

Typical use, with Q, K, V as CUDA tensors [H, N, d] (bf16 or fp32, d = 64 or 128), per-head
token orders q_perm, k_perm [H, N] int32 (block i of the layout holds tokens
perm[offsets[i]:offsets[i+1]]) and block offsets [nb + 1] int32 (1..128 tokens per block):

    out, workspace, layout = spark_bsa_forward(Q, K, V, q_perm, k_perm, q_offsets, k_offsets,
                                               topk_ratio=0.1)

``out`` is in the original token order.  The partition can come from the GPU partitioner:
``spark_reblock(Q, K, block=128)`` returns (q_perm, k_perm, offsets).  Variants:
- ``spark_bsa_forward_ctx`` adds always-exact context (sink) rows;
- ``spark_bsa_forward_fp8`` takes the logit product in e4m3;
- ``spark_bsa_forward_host`` runs from host buffers with the copies overlapped.

The step entry points (``spark_bsa_gather_q``, ``spark_bsa_anchor``,
``spark_bsa_gather_kv_summarize``, ``spark_bsa_route``, ``spark_bsa_attend`` and the comparator
steps) expose each kernel on caller buffers.
"""
from ._native import *  # noqa: F401,F403
from ._native import EXPORTED, lib  # noqa: F401
