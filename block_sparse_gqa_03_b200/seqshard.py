"""Sequence-sharded MSA decode: one decode step over a KV cache split by token
range across GPUs, one process per GPU, NCCL all-gathers between the phases.

MSA itself ("MiniMax goes sparse" (atlascloud.ai), section 1, steps 1 and 2)
is unchanged by the split; the pages do not shard it.  At 1M-token context the
cache of a batch outgrows one GPU's share of a serving node, and a decode step
is HBM-bound, so splitting every sequence's tokens over N GPUs divides both
the memory and the step's bytes by N.  Shard r holds blocks [r * S, (r + 1) * S)
of every sequence (S = ceil(nblk / N) blocks, the last shard may be shorter).
A step:

  1. local candidates: the index scan over the shard and the shard's own top-k
     of its blocks, with their scores (msa_index_candidates; the shard's token
     counts from msa_shard_lengths);
  2. all-gather of the k (score, id) lists of every row;
  3. global top-k from the gathered lists (msa_select_candidates): a row's
     global top-k blocks are each among the top-k of the shard holding them, so
     this is the single-device selection; each GPU keeps the winners in its
     shard, in its local numbering;
  4. attention over those winners on the shard (msa_sparse_attn): a partial
     output and its log-sum-exp per head (a head with no winner here gives
     lse = -inf);
  5. all-gather of the partials and their merge by log-sum-exp weights
     (msa_merge_partials), identical on every GPU.

Every compute step is a kernel of libmsa.so; this module only sequences the
calls and the collectives (``torch.distributed``: NCCL on GPUs).  The phases
are also exposed one by one (``local_candidates``, ``local_attention``,
``merge``) so that the exchange can be driven by another transport.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import msa


@dataclass(frozen=True)
class ShardLayout:
    """Block ranges of the shards of a cache of ``max_kv`` tokens."""

    max_kv: int
    block: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.block < 1 or self.max_kv < 1:
            raise ValueError("bad shard layout")
        if -(-self.nblk // self.shard_blocks) != self.world:
            raise ValueError("%d blocks cannot give each of %d shards a block"
                             % (self.nblk, self.world))

    @property
    def nblk(self) -> int:
        return -(-self.max_kv // self.block)

    @property
    def shard_blocks(self) -> int:
        return -(-self.nblk // self.world)

    def first_block(self, rank: int) -> int:
        return rank * self.shard_blocks

    def blocks(self, rank: int) -> int:
        return min(self.nblk, (rank + 1) * self.shard_blocks) - self.first_block(rank)

    def first_token(self, rank: int) -> int:
        return self.first_block(rank) * self.block

    def tokens(self, rank: int) -> int:
        return min(self.max_kv, (rank + 1) * self.shard_blocks * self.block) - self.first_token(rank)

    def token_slice(self, rank: int) -> slice:
        t0 = self.first_token(rank)
        return slice(t0, t0 + self.tokens(rank))


class TorchDistComm:
    """All-gather over a ``torch.distributed`` process group (NCCL for GPU tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        out = torch.empty((self.world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        if self.dist.get_backend(self.group) == "nccl":
            self.dist.all_gather_into_tensor(out, t, group=self.group)
        else:
            self.dist.all_gather(list(out.unbind(0)), t, group=self.group)
        return out


class LibraryOps:
    """The library calls of each phase (CUDA tensors)."""

    def __init__(self, workspace: msa.Workspace | None = None):
        self.ws = workspace

    def shard_lengths(self, seq_lens, batch, max_kv, base, count, device):
        return msa.msa_shard_lengths(seq_lens, batch=batch, max_kv=max_kv, token_base=base,
                                     token_count=count, workspace=self.ws, device=device)

    def candidates(self, q_idx, k_idx, lens, block, topk):
        return msa.msa_index_candidates(q_idx, k_idx, block=block, topk=topk, causal=True,
                                        seq_lens=lens, workspace=self.ws)

    def select(self, cand_scores, cand_ids, *, seq_lens, max_kv, block, topk, shard_blocks,
               force_own, block_base, nblk_local):
        ids, local = msa.msa_select_candidates(
            cand_scores, cand_ids, max_kv=max_kv, block=block, topk=topk,
            shard_blocks=shard_blocks, causal=True, force_own_block=force_own,
            seq_lens=seq_lens, block_base=block_base, nblk_local=nblk_local, want_global=True,
            want_local=True, workspace=self.ws)
        return ids, local

    def attend(self, q, k, v, local_ids, lens, block):
        return msa.msa_sparse_attn(q, k, v, local_ids, block=block, causal=True, seq_lens=lens,
                                   return_lse=True, workspace=self.ws)

    def merge(self, part_out, part_lse, out=None):
        return msa.msa_merge_partials(part_out, part_lse, out=out)


class ShardedDecode:
    """One rank's side of sequence-sharded decode.

    ``k``, ``v``, ``k_idx`` given to the phases are this rank's shard of the
    cache: tokens ``layout.token_slice(rank)`` of every sequence, [batch,
    tokens, h, d] and [batch, tokens, d_idx] (views of a larger cache are fine).
    ``seq_lens`` are the global lengths (int32 [batch]; None: all max_kv).
    """

    def __init__(self, layout: ShardLayout, rank: int, comm=None, ops=None):
        if not 0 <= rank < layout.world:
            raise ValueError("rank outside the layout")
        self.layout = layout
        self.rank = rank
        self.comm = comm
        self.ops = ops or LibraryOps()
        self.last_ids = None  # the global selection of the last step

    def _lens(self, seq_lens, batch, device):
        lay, r = self.layout, self.rank
        return self.ops.shard_lengths(seq_lens, batch, lay.max_kv, lay.first_token(r),
                                      lay.tokens(r), device)

    def local_candidates(self, q_idx, k_idx, seq_lens, topk):
        """Phase 1: (ids, scores) [batch, 1, h, topk] of this shard's own top-k
        (ids in the shard's numbering, -1 / -inf padded)."""
        if q_idx.shape[1] != 1:
            raise ValueError("sequence-sharded decode takes one query token per sequence")
        lens = self._lens(seq_lens, q_idx.shape[0], q_idx.device)
        return self.ops.candidates(q_idx, k_idx, lens, self.layout.block, topk)

    def local_attention(self, cand_ids, cand_scores, q, k, v, seq_lens, topk, force_own=False):
        """Phase 2, given every shard's lists ([world, batch, 1, h, topk], shard
        order): the global selection and this shard's partial (out, lse)."""
        lay, r = self.layout, self.rank
        ids, local = self.ops.select(cand_scores, cand_ids, seq_lens=seq_lens, max_kv=lay.max_kv,
                                     block=lay.block, topk=topk, shard_blocks=lay.shard_blocks,
                                     force_own=force_own, block_base=lay.first_block(r),
                                     nblk_local=lay.blocks(r))
        self.last_ids = ids
        lens = self._lens(seq_lens, q.shape[0], q.device)
        return self.ops.attend(q, k, v, local, lens, lay.block)

    def merge(self, part_out, part_lse, out=None):
        """Phase 3: the merged output from every shard's partials ([world, ...])."""
        return self.ops.merge(part_out, part_lse, out=out)

    def step(self, q, q_idx, k, v, k_idx, seq_lens, topk, force_own=False, out=None):
        """One decode step with this rank's shard; collective over ``comm``."""
        if self.comm is None:
            raise ValueError("step() needs a communicator")
        ids, scores = self.local_candidates(q_idx, k_idx, seq_lens, topk)
        g_ids = self.comm.all_gather(ids)
        g_scores = self.comm.all_gather(scores)
        o, lse = self.local_attention(g_ids, g_scores, q, k, v, seq_lens, topk, force_own)
        return self.merge(self.comm.all_gather(o), self.comm.all_gather(lse), out=out)
