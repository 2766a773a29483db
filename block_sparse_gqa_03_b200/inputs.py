"""Seeded synthetic inputs for MSA problems.

This module only draws random tensors; it holds none of the method's
arithmetic, and both the CUDA path's tests and the float64 oracle consume the
same tensors it returns.

Recipe (one fixed order per problem, so a seed pins every value):
  1. ``q``      [batch, n_q, H, d]        N(0, 1), fp32 draw rounded to bf16 (RNE)
  2. ``k``      [batch, max_kv, h, d]     same
  3. ``v``      [batch, max_kv, h, d]     same
  4. ``q_idx``  [batch, n_q, h, d_idx]    same
  5. ``k_idx``  [batch, max_kv, d_idx]    same
  6. ``seq_lens`` [batch] int32, only when ``len_range`` is set: integers drawn
     uniformly from [lo, hi]; otherwise every sequence has ``max_kv`` tokens.
  7. planted blocks, only when ``plant_frac`` > 0 (decode workloads): for each
     sequence i, one random permutation of its visible blocks is cut into h
     disjoint runs of round(plant_frac * nblk) blocks, one run per group g; every
     token j of group g's blocks gets ``k_idx[i, j] += plant_scale * q_idx[i, 0, g]``
     (added in fp32, then rounded to bf16).  This shifts those tokens' index
     scores for group g up by about plant_scale * d_idx, far above the spread of
     the block maxima of unshifted blocks, so the true top-k is well separated.
  Optionally ``tail_fill`` writes a constant (e.g. NaN) into k, v and k_idx at
  token positions >= seq_lens[b]; the method never reads those tokens.

Tensors are drawn on ``device`` with a ``torch.Generator`` of that device, in
chunks so that the fp32 staging stays small.  Values drawn on the CPU and on a
GPU differ (different generators); each test draws once and hands host copies
of the same tensors to the oracle.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Problem:
    """Shapes and flags of one MSA problem."""

    name: str
    batch: int
    n_q: int
    max_kv: int
    H: int
    h: int
    d: int
    d_idx: int
    block: int
    topk: int
    causal: bool = True
    force_own: bool = False
    seed: int = 0
    len_range: tuple[int, int] | None = None
    plant_frac: float = 0.0
    plant_scale: float = 0.5

    @property
    def G(self) -> int:
        return self.H // self.h

    @property
    def nblk(self) -> int:
        return (self.max_kv + self.block - 1) // self.block

    @property
    def is_decode(self) -> bool:
        return self.n_q == 1

    def with_(self, **kw) -> "Problem":
        return replace(self, **kw)


# The five workloads named for this method, as concrete problems.
WORKLOADS = {
    # Prefill reference: 6 query heads / 2 index queries as in the pages' figure.
    "prefill_1k": Problem("prefill_1k", batch=1, n_q=1024, max_kv=1024, H=6, h=2, d=64, d_idx=32,
                          block=64, topk=4, causal=True, force_own=True, seed=1001),
    # Decode at 128K context with planted, well-separated blocks (4% per group).
    "decode_128k": Problem("decode_128k", batch=16, n_q=1, max_kv=131072, H=64, h=8, d=128,
                           d_idx=128, block=64, topk=128, causal=True, seed=1002,
                           plant_frac=0.04),
    # Prefill at 32K, own block forced.
    "prefill_32k": Problem("prefill_32k", batch=2, n_q=32768, max_kv=32768, H=32, h=4, d=128,
                           d_idx=64, block=64, topk=32, causal=True, force_own=True, seed=1003),
    # Prefill at 128K, block 128, about 6% of blocks per query.
    "prefill_128k": Problem("prefill_128k", batch=1, n_q=131072, max_kv=131072, H=48, h=8, d=128,
                            d_idx=128, block=128, topk=64, causal=True, seed=1004),
    # Decode at 1M context, variable lengths in [768K, 1M].
    "decode_1m": Problem("decode_1m", batch=4, n_q=1, max_kv=1048576, H=64, h=8, d=128, d_idx=128,
                         block=64, topk=1024, causal=True, seed=1005,
                         len_range=(786432, 1048576)),
}


def _randn_bf16(shape, gen: torch.Generator, device, chunk: int = 1 << 26) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
    return out


def make_inputs(prob: Problem, device="cpu", seed: int | None = None, tail_fill: float | None = None):
    """Draw the tensors of ``prob``; returns a dict of tensors on ``device``."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(prob.seed if seed is None else seed)
    B, n, L = prob.batch, prob.n_q, prob.max_kv
    q = _randn_bf16((B, n, prob.H, prob.d), gen, device)
    k = _randn_bf16((B, L, prob.h, prob.d), gen, device)
    v = _randn_bf16((B, L, prob.h, prob.d), gen, device)
    q_idx = _randn_bf16((B, n, prob.h, prob.d_idx), gen, device)
    k_idx = _randn_bf16((B, L, prob.d_idx), gen, device)
    seq_lens = None
    if prob.len_range is not None:
        lo, hi = prob.len_range
        seq_lens = torch.randint(lo, hi + 1, (B,), generator=gen, device=device,
                                 dtype=torch.int64).to(torch.int32)
    planted = None
    if prob.plant_frac > 0:
        nplant = int(round(prob.plant_frac * prob.nblk))
        planted = torch.full((B, prob.h, nplant), -1, dtype=torch.int32)
        for i in range(B):
            Li = int(seq_lens[i]) if seq_lens is not None else L
            nb = (Li + prob.block - 1) // prob.block
            if nplant * prob.h > nb:
                raise ValueError("not enough blocks to plant disjoint sets")
            perm = torch.randperm(nb, generator=gen, device=device)
            for g in range(prob.h):
                blocks = perm[g * nplant:(g + 1) * nplant]
                planted[i, g] = blocks.to(torch.int32).cpu()
                shift = prob.plant_scale * q_idx[i, 0, g].float()
                for beta in blocks.tolist():
                    j0, j1 = beta * prob.block, min((beta + 1) * prob.block, Li)
                    k_idx[i, j0:j1] = (k_idx[i, j0:j1].float() + shift).to(torch.bfloat16)
    if tail_fill is not None and seq_lens is not None:
        for i in range(B):
            Li = int(seq_lens[i])
            k[i, Li:] = tail_fill
            v[i, Li:] = tail_fill
            k_idx[i, Li:] = tail_fill
    return {"q": q, "k": k, "v": v, "q_idx": q_idx, "k_idx": k_idx, "seq_lens": seq_lens,
            "planted": planted}
