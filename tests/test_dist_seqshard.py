"""Sequence-sharded decode on the CPU: the protocol of
``block_sparse_gqa_03_b200.seqshard`` (shard layout, per-shard lengths and
candidate lists, the all-gathers, the global selection from the gathered lists,
per-shard attention over the winners, the log-sum-exp merge) run by two and
three ``gloo`` ranks, with every compute phase done by the float64 oracle, must
reproduce the oracle's single-device decode step: the same block ids and the
same outputs up to float64 rounding.  The CUDA kernels of the phases are
checked on a GPU in ``test_gpu_seqshard.py``.
"""

from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs
from block_sparse_gqa_03_b200.seqshard import ShardedDecode, ShardLayout, TorchDistComm

HERE = os.path.dirname(os.path.abspath(__file__))

PROB = Problem("seqshard_cpu", batch=3, n_q=1, max_kv=1500, H=8, h=4, d=64, d_idx=32, block=16,
               topk=6, causal=True, seed=301, len_range=(1, 1500))


def _cfg(p, max_kv, topk=None, force_own=None):
    return oracle.Config(p.batch, 1, max_kv, p.H, p.h, p.d, p.d_idx, p.block,
                         p.topk if topk is None else topk, causal=True,
                         force_own=p.force_own if force_own is None else force_own)


class OracleOps:
    """The phases of seqshard on the CPU in float64, through the oracle."""

    def __init__(self, prob):
        self.p = prob

    def shard_lengths(self, seq_lens, batch, max_kv, base, count, device):
        L = seq_lens if seq_lens is not None else torch.full((batch,), max_kv, dtype=torch.int32)
        return (L.to(torch.int64) - base).clamp(0, count).to(torch.int32)

    def candidates(self, q_idx, k_idx, lens, block, topk):
        cfg = _cfg(self.p, k_idx.shape[1], topk=topk, force_own=False)
        sc = oracle.block_scores(cfg, q_idx, k_idx, seq_lens=lens)
        ids = oracle.select(cfg, sc, seq_lens=lens)
        kept = np.where(ids >= 0, np.take_along_axis(sc, np.maximum(ids, 0), axis=2), -np.inf)
        b, h = self.p.batch, self.p.h
        return (torch.as_tensor(ids).view(b, 1, h, topk),
                torch.as_tensor(kept).view(b, 1, h, topk))

    def select(self, cand_scores, cand_ids, *, seq_lens, max_kv, block, topk, shard_blocks,
               force_own, block_base, nblk_local):
        # the gathered lists as one dense row of block scores (-inf where no shard
        # listed a block), then the oracle's own selection
        cfg = _cfg(self.p, max_kv, topk=topk, force_own=force_own)
        world = cand_ids.shape[0]
        ci = cand_ids.reshape(world, -1, self.p.h, cand_ids.shape[-1]).numpy()
        cs = cand_scores.reshape(world, -1, self.p.h, cand_ids.shape[-1]).numpy()
        dense = np.full((ci.shape[1], self.p.h, cfg.nblk), -np.inf)
        for r in range(world):
            for i, g, j in zip(*np.nonzero(ci[r] >= 0)):
                dense[i, g, ci[r, i, g, j] + r * shard_blocks] = cs[r, i, g, j]
        ids = oracle.select(cfg, dense, seq_lens=seq_lens)
        local = np.where((ids >= block_base) & (ids < block_base + nblk_local), ids - block_base, -1)
        shape = (self.p.batch, 1, self.p.h, topk)
        return torch.as_tensor(ids).view(shape), torch.as_tensor(local.astype(np.int32)).view(shape)

    def attend(self, q, k, v, local_ids, lens, block):
        cfg = _cfg(self.p, k.shape[1], topk=local_ids.shape[-1])
        o, l = oracle.sparse_attn(cfg, q, k, v, local_ids.reshape(-1, self.p.h, cfg.topk),
                                  seq_lens=lens)
        return (torch.as_tensor(o).view(self.p.batch, 1, self.p.H, self.p.d),
                torch.as_tensor(l).view(self.p.batch, 1, self.p.H))

    def merge(self, part_out, part_lse, out=None):
        lse = part_lse.numpy()
        M = lse.max(axis=0)
        w = np.where(np.isneginf(lse), 0.0, np.exp(lse - np.where(np.isneginf(M), 0.0, M)))
        den = w.sum(axis=0)
        o = (w[..., None] * part_out.numpy()).sum(axis=0)
        return torch.as_tensor(np.where(den[..., None] > 0, o / np.maximum(den, 1e-300)[..., None],
                                        0.0))


def _rank_main(rank, world, port, force_own, queue):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        prob = PROB.with_(force_own=force_own)
        x = make_inputs(prob, device="cpu")
        lay = ShardLayout(prob.max_kv, prob.block, world)
        sl = lay.token_slice(rank)
        sd = ShardedDecode(lay, rank, TorchDistComm(), OracleOps(prob))
        out = sd.step(x["q"], x["q_idx"], x["k"][:, sl], x["v"][:, sl], x["k_idx"][:, sl],
                      x["seq_lens"], prob.topk, force_own=force_own)
        ids = sd.last_ids.numpy().reshape(prob.batch, prob.h, prob.topk)
        ref_ids, ref_out, _ = oracle.forward(_cfg(prob, prob.max_kv), x["q"], x["k"], x["v"],
                                             x["q_idx"], x["k_idx"], seq_lens=x["seq_lens"])
        err = float(np.abs(out.numpy().reshape(ref_out.shape) - ref_out).max())
        queue.put((rank, bool(np.array_equal(ids, ref_ids)), err))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        queue.put((rank, False, repr(e)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,force_own", [(2, False), (3, True)])
def test_sharded_decode_protocol_matches_single_device_oracle(world, force_own):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, force_own, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same_ids, err in sorted(res):
        assert same_ids, (rank, err)
        assert isinstance(err, float) and err < 1e-9, (rank, err)


def test_shard_layout():
    lay = ShardLayout(max_kv=1500, block=16, world=3)  # 94 blocks: 32, 32, 30
    assert (lay.nblk, lay.shard_blocks) == (94, 32)
    assert [lay.blocks(r) for r in range(3)] == [32, 32, 30]
    assert [lay.tokens(r) for r in range(3)] == [512, 512, 476]
    assert lay.token_slice(2) == slice(1024, 1500)
    with pytest.raises(ValueError):
        ShardLayout(max_kv=64, block=16, world=8)  # 4 blocks cannot feed 8 shards
