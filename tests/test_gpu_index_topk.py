"""msa_index_topk: stage 1 for prefill in one kernel, the top-k kept in the index
GEMM's epilogue.  Its ids must be exactly msa_index_select's (same scores, same
order, same tie rule: the lower block id wins), which the float64 oracle in turn
checks; its optional block scores must be the same scores bit for bit.
"""

import pytest
import torch

import oracle
from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import WORKLOADS, Problem, make_inputs
from msa_check import (check_ids, check_scores, oracle_cfg, row_geometry, sample_rows_chunked,
                       take_rows)

pytestmark = pytest.mark.gpu


def both(prob, x, return_scores=True):
    kw = dict(block=prob.block, topk=prob.topk, causal=prob.causal,
              force_own_block=prob.force_own, seq_lens=x["seq_lens"])
    ids, sc = msa.msa_index_select(x["q_idx"], x["k_idx"], return_scores=True, **kw)
    fid, fsc = msa.msa_index_topk(x["q_idx"], x["k_idx"], return_scores=True, **kw)
    fid2 = msa.msa_index_topk(x["q_idx"], x["k_idx"], **kw)  # without the scores
    torch.cuda.synchronize()
    assert torch.equal(fid, ids)
    assert torch.equal(fid2, ids)
    assert torch.equal(torch.nan_to_num(fsc), torch.nan_to_num(sc))
    return ids, sc


CASES = [
    Problem("t_b128_d128", batch=2, n_q=700, max_kv=700, H=16, h=4, d=128, d_idx=128, block=128,
            topk=3, causal=True, seed=401),
    Problem("t_b64_d64_own", batch=1, n_q=900, max_kv=900, H=8, h=2, d=64, d_idx=64, block=64,
            topk=5, causal=True, force_own=True, seed=402),
    # chunked prefill (queries are the last 300 of 1000 positions), variable lengths
    Problem("t_chunked_varlen", batch=3, n_q=300, max_kv=1000, H=12, h=3, d=128, d_idx=128,
            block=64, topk=7, causal=True, seed=403, len_range=(300, 1000)),
    # top-k larger than many rows' frontier (dense rows), 64 kept, odd group count
    Problem("t_dense_rows", batch=1, n_q=1300, max_kv=1300, H=10, h=5, d=64, d_idx=64, block=64,
            topk=64, causal=True, force_own=True, seed=404),
    # non-causal, top-1
    Problem("t_noncausal_k1", batch=2, n_q=260, max_kv=600, H=4, h=2, d=64, d_idx=128, block=128,
            topk=1, causal=False, seed=405),
]


@pytest.mark.parametrize("prob", CASES, ids=lambda p: p.name)
def test_fused_topk_equals_two_kernel_select_and_oracle(prob):
    x = make_inputs(prob, device="cuda")
    ids, sc = both(prob, x)
    rows = [(b, t) for b in range(prob.batch) for t in range(prob.n_q)]
    cfg = oracle_cfg(prob)
    sl = None if x["seq_lens"] is None else x["seq_lens"].cpu()
    ora_sc = oracle.block_scores(cfg, x["q_idx"].cpu(), x["k_idx"].cpu(), seq_lens=sl)
    ora_ids = oracle.select(cfg, ora_sc, seq_lens=sl)
    F_rows = [row_geometry(prob, sl, b, t)[2] for (b, t) in rows]
    gsc = take_rows(sc, rows)
    check_scores(gsc, ora_sc, F_rows)
    check_ids(prob, rows, sl, take_rows(ids, rows), ora_ids, ora_sc, gsc)


def test_fused_topk_exact_ties_take_the_lower_id():
    # blocks 9..20 repeat blocks 0..11 exactly: every query sees pairs of equal
    # block scores, so the tie rule decides which of a pair is kept
    prob = Problem("t_ties", batch=1, n_q=1536, max_kv=1536, H=8, h=2, d=64, d_idx=64, block=64,
                   topk=10, causal=True, seed=406)
    x = make_inputs(prob, device="cuda")
    B = prob.block
    x["k_idx"][:, 9 * B:21 * B] = x["k_idx"][:, 0:12 * B].clone()
    ids, sc = both(prob, x)
    # some rows really hold ties between kept and dropped blocks
    s = sc[0, -1]
    assert any(len(set(s[g, :21].tolist())) < 21 for g in range(prob.h))


@pytest.mark.parametrize("name", ["prefill_32k", "prefill_128k"])
def test_fused_topk_on_prefill_workloads(name):
    prob = WORKLOADS[name]
    x = make_inputs(prob, device="cuda")
    kw = dict(block=prob.block, topk=prob.topk, causal=prob.causal,
              force_own_block=prob.force_own)
    ids = msa.msa_index_select(x["q_idx"], x["k_idx"], **kw)
    fid = msa.msa_index_topk(x["q_idx"], x["k_idx"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(fid, ids)
    # and the oracle on a stratified sample of rows
    rows = sample_rows_chunked(prob, 256, seed=7)
    cfg = oracle_cfg(prob)
    ora_sc = oracle.block_scores(cfg, x["q_idx"].cpu(), x["k_idx"].cpu(), rows=rows)
    ora_ids = oracle.select(cfg, ora_sc, rows=rows)
    _, gsc = msa.msa_index_topk(x["q_idx"], x["k_idx"], return_scores=True, **kw)
    check_ids(prob, rows, None, take_rows(fid, rows), ora_ids, ora_sc, take_rows(gsc, rows))


def test_fused_topk_rejects_unsupported_shapes():
    prob = WORKLOADS["prefill_1k"]  # d_idx 32: the warp-MMA scan path only
    x = make_inputs(prob, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_index_topk(x["q_idx"], x["k_idx"], block=prob.block, topk=prob.topk)
    assert e.value.code == msa.MSA_ERR_UNSUPPORTED
