"""Top-k selection under exact ties, on rows wide enough (more than 1024 blocks)
for the one-CTA-per-row kernel.

K_idx repeats a few block patterns, so many blocks of a row carry bit-identical
block scores (the same inputs through the same arithmetic).  The selection rule
(score descending, the lower block id winning a tie, the own block first when
forced) then fixes the ids exactly, and they are checked bit for bit against a
host selection from the GPU's own exposed scores, and against the oracle's ids
(near-tie rows aside, as everywhere).  The cases cover a threshold value shared
by hundreds of blocks (every bit of T resolved, ties cut by id), a row whose
visible blocks all score the same, rows with fewer visible blocks than k, and
the forced own block.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs
from msa_check import check_ids, check_scores, oracle_cfg, row_geometry

pytestmark = pytest.mark.gpu


def host_select(scores_row, F, k, own):
    """min(k, F) ids: own first when forced, then score descending, lower id first."""
    cands = sorted((c for c in range(F) if c != own), key=lambda c: (-float(scores_row[c]), c))
    m = min(k, F)
    take = ([own] if own is not None else []) + cands[:m - (1 if own is not None else 0)]
    return sorted(take) + [-1] * (k - m)


def periodic_k_idx(x, prob, period):
    """Token j of every sequence gets the K_idx of token (j // block % period) *
    block + j % block: blocks repeat with the given period."""
    k_idx = x["k_idx"]
    L = k_idx.shape[1]
    j = torch.arange(L, device=k_idx.device)
    src = (j // prob.block % period) * prob.block + j % prob.block
    return k_idx[:, src].contiguous()


CASES = [
    # 2500 blocks per row (256 threads x 16 keys); T shared by ~350 blocks
    (Problem("ties_p7", batch=3, n_q=1, max_kv=40000, H=8, h=2, d=64, d_idx=32, block=16,
             topk=128, seed=301), 7, [40000, 23456, 1600]),
    # every full block scores the same; 2048 blocks (512 threads x 4 keys)
    (Problem("ties_all", batch=2, n_q=1, max_kv=32768, H=8, h=2, d=64, d_idx=32, block=16,
             topk=100, seed=302), 1, [32760, 20000]),
    # own block forced, 5000 blocks (512 threads x 16 keys)
    (Problem("ties_own", batch=2, n_q=1, max_kv=80000, H=4, h=1, d=64, d_idx=64, block=16,
             topk=300, force_own=True, seed=303), 13, [80000, 77777]),
    # 16384 blocks (1024 threads x 16 keys), as in long-context decode
    (Problem("ties_16k", batch=1, n_q=1, max_kv=262144, H=4, h=2, d=64, d_idx=32, block=16,
             topk=1024, seed=304), 29, [262144]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_cta_topk_ties(case):
    prob, period, lens = case
    x = make_inputs(prob, device="cuda")
    k_idx = periodic_k_idx(x, prob, period)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ids, sc = msa.msa_index_select(x["q_idx"], k_idx, topk=prob.topk, block=prob.block,
                                   causal=prob.causal, seq_lens=sl,
                                   force_own_block=prob.force_own, return_scores=True)
    torch.cuda.synchronize()
    ids_h, sc_h = ids.cpu().numpy(), sc.cpu().numpy()
    rows = [(b, 0) for b in range(prob.batch)]
    n_tied = 0
    for b in range(prob.batch):
        L, pos, F, own = row_geometry(prob, lens, b, 0)
        for g in range(prob.h):
            want = host_select(sc_h[b, 0, g], F, prob.topk, own)
            assert list(ids_h[b, 0, g]) == want, "b=%d g=%d" % (b, g)
            m = min(prob.topk, F)
            kept = sorted(sc_h[b, 0, g, :F])[::-1]
            if F > m and kept[m - 1] == kept[m]:
                n_tied += 1
    assert n_tied > 0, "the case has no tie at the threshold"
    # the oracle agrees (its double scores repeat with the same period)
    cfg = oracle_cfg(prob)
    sl_h = sl.cpu()
    o_sc = oracle.block_scores(cfg, x["q_idx"].cpu(), k_idx.cpu(), seq_lens=sl_h, rows=rows)
    o_ids = oracle.select(cfg, o_sc, seq_lens=sl_h, rows=rows)
    F_rows = [row_geometry(prob, lens, b, 0)[2] for b, _ in rows]
    check_scores(sc_h[:, 0], o_sc, F_rows)
    check_ids(prob, rows, lens, ids_h[:, 0], o_ids, o_sc, gpu_scores=sc_h[:, 0])
