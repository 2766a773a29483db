"""Sequence-sharded decode with the library's kernels, on one GPU.

The ranks of ``block_sparse_gqa_03_b200.seqshard`` are run one after another on
the same device, each with its own token shard of the cache (views of one
cache), and the all-gathers are replaced by stacking the ranks' tensors in rank
order: nothing waits on anything else, so no rank depends on another's kernels
running at the same time.  The result must be the single-device result: the
global block ids bit for bit (the shards' scans compute the same fp32 block
scores), the outputs within the attention tolerance of the single-device
msa_forward (the shards' partial outputs are rounded to bf16 once more before
the merge) and of the float64 oracle.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import WORKLOADS, Problem, make_inputs
from block_sparse_gqa_03_b200.seqshard import ShardedDecode, ShardLayout
from msa_check import check_attn, oracle_cfg

pytestmark = pytest.mark.gpu


def run_sharded(prob, x, world, force_own):
    lay = ShardLayout(prob.max_kv, prob.block, world)
    ranks = [ShardedDecode(lay, r) for r in range(world)]
    shard = [lay.token_slice(r) for r in range(world)]
    sl = x["seq_lens"]
    cands = [rk.local_candidates(x["q_idx"], x["k_idx"][:, s], sl, prob.topk)
             for rk, s in zip(ranks, shard)]
    g_ids = torch.stack([c[0] for c in cands])
    g_sc = torch.stack([c[1] for c in cands])
    parts = [rk.local_attention(g_ids, g_sc, x["q"], x["k"][:, s], x["v"][:, s], sl, prob.topk,
                                force_own) for rk, s in zip(ranks, shard)]
    p_out = torch.stack([p[0] for p in parts])
    p_lse = torch.stack([p[1] for p in parts])
    outs = [rk.merge(p_out, p_lse) for rk in ranks]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])  # every rank merges the same partials
    for rk in ranks[1:]:
        assert torch.equal(rk.last_ids, ranks[0].last_ids)
    return outs[0], ranks[0].last_ids


CASES = [
    # 1M-context decode workload split over two and four GPUs
    (WORKLOADS["decode_1m"], 2, False),
    (WORKLOADS["decode_1m"], 4, False),
    # short and empty sequences on the trailing shards, forced own block, block 16
    (Problem("seqshard_small", batch=5, n_q=1, max_kv=5000, H=16, h=4, d=64, d_idx=32, block=16,
             topk=8, causal=True, seed=302, len_range=(0, 5000)), 3, True),
    # 128K decode workload over eight shards of 256 blocks (k = 128 per shard)
    (WORKLOADS["decode_128k"].with_(batch=4), 8, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s_w%d" % (c[0].name, c[1]))
def test_sharded_decode_equals_single_device(case):
    prob, world, force_own = case
    x = make_inputs(prob, device="cuda")
    kw = dict(block=prob.block, causal=True, seq_lens=x["seq_lens"])
    out1, ids1, lse1 = msa.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"],
                                       topk=prob.topk, force_own_block=force_own,
                                       return_ids=True, return_lse=True, **kw)
    out, ids = run_sharded(prob, x, world, force_own)
    assert torch.equal(ids, ids1)
    err = (out.float() - out1.float()).abs()
    assert float(err.max()) <= 2e-2 and float(err.mean()) <= 2e-3
    # and against the float64 oracle on the same selection
    cfg = oracle_cfg(prob.with_(force_own=force_own))
    o, l = oracle.sparse_attn(cfg, x["q"].cpu(), x["k"].cpu(), x["v"].cpu(),
                              ids.cpu().reshape(-1, prob.h, prob.topk),
                              seq_lens=None if x["seq_lens"] is None else x["seq_lens"].cpu())
    check_attn(out.float().cpu().numpy().reshape(o.shape), None, o, l)


def test_merge_partials_matches_oracle_lse_weights():
    # partials over disjoint key sets of the same rows (two halves of the selected
    # blocks) merged by the kernel = attention over the union
    prob = Problem("merge", batch=2, n_q=1, max_kv=4096, H=16, h=2, d=128, d_idx=64, block=64,
                   topk=16, causal=True, seed=303)
    x = make_inputs(prob, device="cuda")
    ids = msa.msa_index_select(x["q_idx"], x["k_idx"], block=prob.block, topk=prob.topk)
    a = ids.clone()
    b = ids.clone()
    a[..., 8:] = -1
    b[..., :8] = -1
    oa, la = msa.msa_sparse_attn(x["q"], x["k"], x["v"], a, block=prob.block, return_lse=True)
    ob, lb = msa.msa_sparse_attn(x["q"], x["k"], x["v"], b, block=prob.block, return_lse=True)
    lse = torch.empty_like(la)
    out = msa.msa_merge_partials(torch.stack([oa, ob]), torch.stack([la, lb]), lse=lse)
    o, l = oracle.sparse_attn(oracle_cfg(prob), x["q"].cpu(), x["k"].cpu(), x["v"].cpu(),
                              ids.cpu().reshape(-1, prob.h, prob.topk))
    check_attn(out.float().cpu().numpy().reshape(o.shape), lse.cpu().numpy().reshape(l.shape),
               o, l)
    # a row that no part saw: out 0, lse -inf
    none = torch.full_like(la, float("-inf"))
    out0 = msa.msa_merge_partials(torch.stack([oa, ob]), torch.stack([none, none]), lse=lse)
    assert torch.all(out0 == 0) and torch.all(torch.isneginf(lse))


def test_index_candidates_scores_are_the_block_scores_of_the_ids():
    prob = Problem("cands", batch=3, n_q=1, max_kv=70000, H=8, h=8, d=64, d_idx=128, block=64,
                   topk=100, causal=True, seed=304, len_range=(50, 70000))
    x = make_inputs(prob, device="cuda")
    kw = dict(block=prob.block, topk=prob.topk, seq_lens=x["seq_lens"])
    ids, kept = msa.msa_index_candidates(x["q_idx"], x["k_idx"], **kw)
    ids2, sc = msa.msa_index_select(x["q_idx"], x["k_idx"], return_scores=True, **kw)
    assert torch.equal(ids, ids2)
    want = torch.where(ids >= 0, torch.gather(sc, 3, ids.clamp(min=0).long()),
                       torch.full_like(kept, float("-inf")))
    assert torch.equal(kept, want)
    # the scan alone gives the same block scores
    sc2 = msa.msa_block_scores(x["q_idx"], x["k_idx"], block=prob.block, seq_lens=x["seq_lens"])
    assert torch.equal(torch.nan_to_num(sc2), torch.nan_to_num(sc))
