"""Paged KV cache: the block table maps each (sequence, logical block) to a page of
the K, V and K_idx pools.  The layout is storage only, so on the same inputs the
paged path must give exactly the contiguous path's ids, block scores, outputs
and log-sum-exps (the same kernels run the same arithmetic), and a page id
outside the pool must be recorded, never read.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs
from msa_check import check_attn, oracle_cfg, take_rows

pytestmark = pytest.mark.gpu


def to_pages(x, prob, spare=5, seed=0):
    """Scatters the contiguous k, v and k_idx into shuffled page pools (plus unused
    spare pages filled with noise) and returns the pools and the block table."""
    B, nb = prob.block, (prob.max_kv + prob.block - 1) // prob.block
    n_pages = prob.batch * nb + spare
    g = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[:prob.batch * nb].view(prob.batch, nb)
    table = perm.to(torch.int32).cuda()
    pools = {}
    for name in ("k", "v", "k_idx"):
        t = x[name]
        pool = torch.randn((n_pages, B) + tuple(t.shape[2:]), generator=g).to(torch.bfloat16).cuda()
        padded = torch.zeros((t.shape[0], nb * B) + tuple(t.shape[2:]), dtype=t.dtype, device=t.device)
        padded[:, :t.shape[1]] = t
        blocks = padded.view((t.shape[0], nb, B) + tuple(t.shape[2:]))
        pool[table.long().view(-1)] = blocks.reshape((-1, B) + tuple(t.shape[2:]))
        pools[name] = pool
    return pools, table


CASES = [
    # decode: index scan with direct loads, streaming attention, variable lengths
    Problem("paged_decode", batch=3, n_q=1, max_kv=9000, H=32, h=8, d=128, d_idx=128, block=64,
            topk=16, causal=True, seed=201, len_range=(3000, 9000)),
    # prefill: tcgen05 index GEMM (one page per 128-key tile) and KV-major attention
    Problem("paged_prefill_b128", batch=1, n_q=700, max_kv=2000, H=12, h=2, d=128, d_idx=128,
            block=128, topk=5, causal=True, seed=202),
    # prefill: two pages per index key tile, block-64 KV-major attention
    Problem("paged_prefill_b64", batch=2, n_q=400, max_kv=1100, H=8, h=2, d=64, d_idx=64,
            block=64, topk=6, causal=True, force_own=True, seed=203),
    # prefill: warp-MMA index scan (d_idx 32) and the row-per-CTA attention (block 32)
    Problem("paged_prefill_b32", batch=1, n_q=300, max_kv=300, H=6, h=2, d=128, d_idx=32,
            block=32, topk=3, causal=True, seed=204),
]


@pytest.mark.parametrize("prob", CASES, ids=lambda p: p.name)
def test_paged_equals_contiguous(prob):
    x = make_inputs(prob, device="cuda")
    sl = x["seq_lens"]
    kw = dict(block=prob.block, causal=prob.causal, seq_lens=sl)
    ids, sc = msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk,
                                   force_own_block=prob.force_own, return_scores=True, **kw)
    out, lse = msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, return_lse=True, **kw)
    pools, table = to_pages(x, prob, seed=prob.seed)
    pkw = dict(kw, block_table=table, max_kv=prob.max_kv)
    ids_p, sc_p = msa.msa_index_select(x["q_idx"], pools["k_idx"], topk=prob.topk,
                                       force_own_block=prob.force_own, return_scores=True, **pkw)
    out_p, lse_p = msa.msa_sparse_attn(x["q"], pools["k"], pools["v"], ids_p, return_lse=True, **pkw)
    out_f, ids_f, lse_f = msa.msa_forward(x["q"], pools["k"], pools["v"], x["q_idx"],
                                          pools["k_idx"], topk=prob.topk,
                                          force_own_block=prob.force_own, return_ids=True,
                                          return_lse=True, **pkw)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(msa._workspace(None, x["q"].device)) == msa.MSA_OK
    assert torch.equal(ids_p, ids) and torch.equal(ids_f, ids)
    assert torch.equal(torch.nan_to_num(sc_p), torch.nan_to_num(sc))
    assert torch.equal(out_p, out) and torch.equal(out_f, out)
    assert torch.equal(lse_p, lse) and torch.equal(lse_f, lse)


def test_paged_prefill_against_oracle():
    prob = CASES[1]
    x = make_inputs(prob, device="cuda")
    pools, table = to_pages(x, prob, seed=7)
    kw = dict(block=prob.block, causal=prob.causal, block_table=table, max_kv=prob.max_kv)
    ids = msa.msa_index_select(x["q_idx"], pools["k_idx"], topk=prob.topk, **kw)
    out, lse = msa.msa_sparse_attn(x["q"], pools["k"], pools["v"], ids, return_lse=True, **kw)
    rows = [(0, t) for t in range(0, prob.n_q, 7)]
    ids_h = ids.cpu()
    o, l = oracle.sparse_attn(oracle_cfg(prob), x["q"].cpu(), x["k"].cpu(), x["v"].cpu(),
                              take_rows(ids_h, rows), rows=rows)
    check_attn(take_rows(out.float(), rows), take_rows(lse, rows), o, l)


def test_bad_page_is_flagged_not_read():
    prob = CASES[0]
    x = make_inputs(prob, device="cuda")
    pools, table = to_pages(x, prob, spare=0, seed=9)
    bad = table.clone()
    bad[1, 3] = pools["k"].shape[0] + 1000  # outside the pool
    ws = msa.Workspace("cuda")
    kw = dict(block=prob.block, causal=True, seq_lens=x["seq_lens"], max_kv=prob.max_kv,
              workspace=ws)
    msa.msa_index_select(x["q_idx"], pools["k_idx"], topk=prob.topk, block_table=bad, **kw)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_ASSERT
    ids = torch.zeros((prob.batch, 1, prob.h, prob.topk), dtype=torch.int32, device="cuda")
    ids[..., 0] = 3
    ids[..., 1:] = -1
    msa.msa_sparse_attn(x["q"], pools["k"], pools["v"], ids, block_table=bad, **kw)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_ASSERT
    # a good table on the same workspace runs clean again
    msa.msa_sparse_attn(x["q"], pools["k"], pools["v"], ids, block_table=table, **kw)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
