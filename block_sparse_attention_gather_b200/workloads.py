"""Seeded synthetic inputs for the two-branch block-sparse attention forward.

This module only draws random numbers and lays out integer index arrays; it holds none of
the method's arithmetic.  Both the CUDA path and the CPU oracle consume its tensors.

The shapes stand in for MiniMax-H3 video-latent attention, whose activations are not
available: 60 latent frames x (24 x 42) tokens for the 384p draft and 60 x (48 x 84) for
768p (1344x768, 240 frames, assuming 16x spatial / 4x temporal compression), d = 128.
Q and K come from a 32-component Gaussian mixture per head (component means N(0, I_d),
shared by Q and K; each token draws one component for both its query and its key; spread
0.3), so attention is peaky the way the Spark-H3 blog's attention maps are; V is N(0, 1).

Layouts (the reblocked partition is an input of the method):

* ``identity``  - q_perm = k_perm = arange(N), contiguous blocks.
* ``random``    - independent seeded random permutations for queries and keys.
* ``reblock``   - a stand-in for the Spark-Reblock partitioner's output: tokens stable-sorted
  by mixture component with a random order inside each component; queries reuse the key
  partition (the pages' ``reblock_layout=q_reuse_k``).

Block offsets are shared by all heads: fixed-size blocks whose last block takes the
remainder, or sizes drawn uniformly in [lo, hi] until they cover N (the last block takes the
remainder).

Context (sink) tokens, when a workload has ``nc > 0``: Kc, Vc [H, nc, d] drawn after
everything else from a generator of their own (so the video tensors do not change), keys
from the same mixture as the video keys, values N(0, 1).  The pages give no context length;
512 stands in for a text prompt's tokens.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "make_offsets", "make_inputs", "sample_units"]


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    N: int
    d: int
    dtype: str                 # "fp32" or "bf16": the type of Q, K, V and out
    ratio: float               # topk_ratio
    layout: str                # "identity" | "random" | "reblock"
    structure: str             # "iid" | "mixture"
    seed: int
    block: int = 128           # fixed block size, when var_block is None
    var_block: tuple | None = None   # (lo, hi) for variable block sizes
    n_components: int = 32
    spread: float = 0.3
    nc: int = 0                # context (sink) tokens per head

    def with_ratio(self, ratio: float) -> "Workload":
        return replace(self, ratio=ratio, name=f"{self.name.rsplit('-r', 1)[0]}-r{ratio:g}")


def _mk_var(ratio: float) -> Workload:
    return Workload(f"768p-varblock-24x241920-d128-r{ratio:g}", 24, 241920, 128, "bf16", ratio,
                    "reblock", "mixture", 1005, var_block=(64, 128))


WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny-1x1024-d64-fp32", 1, 1024, 64, "fp32", 0.125, "identity", "iid", 1001,
             block=64),
    Workload("small-8x16384-d128-randperm", 8, 16384, 128, "bf16", 0.1, "random", "mixture",
             1002, block=64),
    Workload("384p-24x60480-d128", 24, 60480, 128, "bf16", 0.1, "reblock", "mixture", 1003),
    Workload("768p-24x241920-d128", 24, 241920, 128, "bf16", 0.1, "reblock", "mixture", 1004),
    Workload("768p-24x241920-d128-randperm", 24, 241920, 128, "bf16", 0.1, "random",
             "mixture", 1004),
    _mk_var(0.1), _mk_var(0.2), _mk_var(0.3), _mk_var(1.0),
    Workload("tiny-ctx77-1x1024-d64-fp32", 1, 1024, 64, "fp32", 0.125, "identity", "iid",
             1006, block=64, nc=77),
    Workload("small-ctx300-8x16384-d128-randperm", 8, 16384, 128, "bf16", 0.1, "random",
             "mixture", 1007, block=64, nc=300),
    Workload("768p-ctx512-24x241920-d128", 24, 241920, 128, "bf16", 0.1, "reblock", "mixture",
             1008, nc=512),
]}


def make_offsets(w: Workload) -> torch.Tensor:
    """int32 block offsets [nB+1] from 0 to N (CPU; identical for every device)."""
    if w.var_block is None:
        starts = list(range(0, w.N, w.block))
        return torch.tensor(starts + [w.N], dtype=torch.int32)
    lo, hi = w.var_block
    g = torch.Generator(device="cpu").manual_seed(w.seed * 7919 + 17)
    offs = [0]
    while offs[-1] < w.N:
        size = int(torch.randint(lo, hi + 1, (1,), generator=g))
        offs.append(min(offs[-1] + size, w.N))
    return torch.tensor(offs, dtype=torch.int32)


def make_inputs(w: Workload, device="cpu") -> dict:
    """Q, K, V [H,N,d], q_perm, k_perm [H,N] int32, q_offsets, k_offsets int32 (device)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    H, N, d = w.H, w.N, w.d
    tdt = torch.float32 if w.dtype == "fp32" else torch.bfloat16
    comp = None
    if w.structure == "iid":
        Q = torch.randn(H, N, d, generator=g, device=device).to(tdt)
        K = torch.randn(H, N, d, generator=g, device=device).to(tdt)
    elif w.structure == "mixture":
        mu = torch.randn(H, w.n_components, d, generator=g, device=device)
        comp = torch.randint(0, w.n_components, (H, N), generator=g, device=device)
        hidx = torch.arange(H, device=device)[:, None]
        Q = (mu[hidx, comp] + w.spread * torch.randn(H, N, d, generator=g, device=device)).to(tdt)
        K = (mu[hidx, comp] + w.spread * torch.randn(H, N, d, generator=g, device=device)).to(tdt)
    else:
        raise ValueError(w.structure)
    V = torch.randn(H, N, d, generator=g, device=device).to(tdt)

    if w.layout == "identity":
        q_perm = torch.arange(N, device=device, dtype=torch.int32).expand(H, N).contiguous()
        k_perm = q_perm.clone()
    elif w.layout == "random":
        q_perm = torch.stack([torch.randperm(N, generator=g, device=device) for _ in range(H)])
        k_perm = torch.stack([torch.randperm(N, generator=g, device=device) for _ in range(H)])
        q_perm, k_perm = q_perm.to(torch.int32), k_perm.to(torch.int32)
    elif w.layout == "reblock":
        if comp is None:
            raise ValueError("reblock layout needs mixture structure")
        rows = []
        for h in range(H):
            r = torch.randperm(N, generator=g, device=device)
            order = torch.argsort(comp[h, r], stable=True)
            rows.append(r[order])
        k_perm = torch.stack(rows).to(torch.int32)
        q_perm = k_perm.clone()
    else:
        raise ValueError(w.layout)

    offs = make_offsets(w).to(device)
    x = dict(Q=Q.contiguous(), K=K.contiguous(), V=V.contiguous(),
             q_perm=q_perm.contiguous(), k_perm=k_perm.contiguous(),
             q_offsets=offs, k_offsets=offs.clone(), ratio=w.ratio)
    if w.nc > 0:
        gc = torch.Generator(device=device).manual_seed(w.seed * 104729 + 11)
        if w.structure == "mixture":
            cc = torch.randint(0, w.n_components, (H, w.nc), generator=gc, device=device)
            Kc = mu[torch.arange(H, device=device)[:, None], cc] + \
                w.spread * torch.randn(H, w.nc, d, generator=gc, device=device)
        else:
            Kc = torch.randn(H, w.nc, d, generator=gc, device=device)
        Vc = torch.randn(H, w.nc, d, generator=gc, device=device)
        x["Kc"] = Kc.to(tdt).contiguous()
        x["Vc"] = Vc.to(tdt).contiguous()
    return x


def sample_units(w: Workload, n_units: int, nqb: int, seed_offset: int = 0):
    """Seeded sample of (head, query block) pairs, as a dict head -> sorted block list."""
    g = torch.Generator(device="cpu").manual_seed(w.seed * 31 + 5 + seed_offset)
    total = w.H * nqb
    n = min(n_units, total)
    picks = torch.randperm(total, generator=g)[:n].tolist()
    out: dict[int, list[int]] = {}
    for p in picks:
        out.setdefault(p // nqb, []).append(p % nqb)
    return {h: sorted(v) for h, v in sorted(out.items())}
