"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Every test here needs a B200.  Small problems are checked on every row; the
full-size workloads on every row where the oracle finishes in seconds (decode)
and on a sample of query rows otherwise (prefill), in the launch configuration
the benchmark times.
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import WORKLOADS, Problem, make_inputs
from msa_check import (check_attn, check_ids, check_scores, oracle_cfg, page_pools,
                       row_geometry, sample_rows_chunked, take_rows)

pytestmark = pytest.mark.gpu


def host(t):
    return None if t is None else t.cpu()


def run_and_check(prob: Problem, rows=None, tail_fill=None, with_oracle_ids=True, lens=None,
                  paged=False):
    """Runs msa_index_select, msa_sparse_attn and msa_forward on the seeded inputs
    of ``prob`` and checks every stage against the oracle on ``rows`` (default: all).
    With ``paged`` the GPU reads K, V and K_idx from shuffled page pools through a
    block table; the oracle always reads the contiguous tensors."""
    x = make_inputs(prob, device="cuda", tail_fill=tail_fill)
    if lens is not None:
        x["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device="cuda")
    sl = x["seq_lens"]
    kw = dict(block=prob.block, causal=prob.causal, seq_lens=sl)
    # host copies for the oracle before the cache is paged
    q_h, k_h, v_h = host(x["q"]), host(x["k"]), host(x["v"])
    qi_h, ki_h = host(x["q_idx"]), host(x["k_idx"])
    dk, dv, dki = x["k"], x["v"], x["k_idx"]
    if paged:
        pools, table = page_pools(x, prob, seed=prob.seed)
        dk, dv, dki = pools["k"], pools["v"], pools["k_idx"]
        del x["k"], x["v"], x["k_idx"]
        torch.cuda.empty_cache()
        kw.update(block_table=table, max_kv=prob.max_kv)
    ids_g, sc_g = msa.msa_index_select(x["q_idx"], dki, topk=prob.topk,
                                       force_own_block=prob.force_own, return_scores=True, **kw)
    out_g, lse_g = msa.msa_sparse_attn(x["q"], dk, dv, ids_g, return_lse=True, **kw)
    out_f, ids_f, lse_f = msa.msa_forward(x["q"], dk, dv, x["q_idx"], dki,
                                          topk=prob.topk, force_own_block=prob.force_own,
                                          return_ids=True, return_lse=True, **kw)
    torch.cuda.synchronize()
    assert msa.msa_get_device_status(msa._workspace(None, x["q"].device)) == msa.MSA_OK
    # msa_forward runs the same kernels: identical results
    assert torch.equal(ids_f, ids_g)
    assert torch.equal(out_f, out_g) and torch.equal(lse_f, lse_g)

    if rows is None:
        rows = [(b, t) for b in range(prob.batch) for t in range(prob.n_q)]
    cfg = oracle_cfg(prob)
    sl_h = host(sl)
    ora_sc = oracle.block_scores(cfg, qi_h, ki_h, seq_lens=sl_h, rows=rows)
    ora_ids = oracle.select(cfg, ora_sc, seq_lens=sl_h, rows=rows)
    gpu_sc = take_rows(sc_g, rows)
    gpu_ids = take_rows(ids_g, rows)
    F_rows = [row_geometry(prob, sl_h, b, t)[2] for (b, t) in rows]
    check_scores(gpu_sc, ora_sc, F_rows)
    _, near = check_ids(prob, rows, sl_h, gpu_ids, ora_ids, ora_sc, gpu_sc)

    ora_out, ora_lse = oracle.sparse_attn(cfg, q_h, k_h, v_h, gpu_ids, seq_lens=sl_h, rows=rows)
    stats = check_attn(take_rows(out_g.float(), rows), take_rows(lse_g, rows), ora_out, ora_lse)

    if with_oracle_ids and len(rows) == prob.batch * prob.n_q:
        # stage 2 in isolation on the oracle's own selection
        ids_o = torch.as_tensor(ora_ids.reshape(prob.batch, prob.n_q, prob.h, prob.topk),
                                device="cuda")
        out_o, lse_o = msa.msa_sparse_attn(x["q"], dk, dv, ids_o, return_lse=True, **kw)
        o2, l2 = oracle.sparse_attn(cfg, q_h, k_h, v_h, ora_ids, seq_lens=sl_h, rows=rows)
        check_attn(take_rows(out_o.float(), rows), take_rows(lse_o, rows), o2, l2)
    return x, ids_g, near, stats


SMALL_CASES = [
    Problem("ragged_b16", batch=1, n_q=100, max_kv=100, H=6, h=2, d=64, d_idx=32, block=16,
            topk=3, causal=True, force_own=True, seed=101),
    Problem("noncausal_g1", batch=2, n_q=200, max_kv=200, H=8, h=8, d=128, d_idx=64, block=32,
            topk=5, causal=False, seed=102),
    Problem("g16_b64", batch=1, n_q=300, max_kv=300, H=16, h=1, d=128, d_idx=128, block=64,
            topk=2, causal=True, seed=103),
    Problem("dense_b128", batch=2, n_q=257, max_kv=257, H=12, h=4, d=64, d_idx=128, block=128,
            topk=64, causal=True, seed=104),
    Problem("chunked", batch=2, n_q=50, max_kv=333, H=4, h=2, d=128, d_idx=64, block=16, topk=4,
            causal=True, force_own=True, seed=105),
    Problem("blocklocal", batch=1, n_q=160, max_kv=160, H=8, h=2, d=128, d_idx=32, block=32,
            topk=1, causal=True, force_own=True, seed=106),
    Problem("decode_varlen", batch=5, n_q=1, max_kv=5000, H=32, h=8, d=128, d_idx=128, block=64,
            topk=8, causal=True, seed=107, len_range=(1, 5000)),
    Problem("decode_g1_h16", batch=3, n_q=1, max_kv=3000, H=16, h=16, d=64, d_idx=32, block=16,
            topk=1, causal=True, seed=108),
    Problem("prefill_kv_varlen", batch=3, n_q=300, max_kv=700, H=12, h=2, d=128, d_idx=64,
            block=128, topk=3, causal=True, seed=112, len_range=(300, 700)),
    Problem("prefill_kv_d64_b64", batch=1, n_q=1500, max_kv=1500, H=16, h=1, d=64, d_idx=128,
            block=64, topk=5, causal=True, force_own=True, seed=113),
    # groups of 8 heads: the combine takes one warp per (query, group)
    Problem("prefill_kv_g8_d64", batch=2, n_q=600, max_kv=900, H=16, h=2, d=64, d_idx=64,
            block=64, topk=6, causal=True, seed=114),
    Problem("prefill_kv_g8_d128", batch=1, n_q=777, max_kv=777, H=8, h=1, d=128, d_idx=128,
            block=128, topk=3, causal=True, force_own=True, seed=115),
    Problem("decode_many_splits", batch=2, n_q=1, max_kv=65536, H=64, h=8, d=128, d_idx=128,
            block=64, topk=600, causal=True, seed=109, len_range=(40000, 65536)),
    # groups of 7 and 5 heads in the decode attention (swapped MMA operands: heads
    # past G are zero columns of the n8 tile)
    Problem("decode_g7_d64", batch=3, n_q=1, max_kv=6000, H=14, h=2, d=64, d_idx=64, block=64,
            topk=12, causal=True, seed=125, len_range=(1, 6000)),
    Problem("decode_g5_b128", batch=2, n_q=1, max_kv=9000, H=20, h=4, d=128, d_idx=128,
            block=128, topk=10, causal=True, force_own=True, seed=126),
]


@pytest.mark.parametrize("prob", SMALL_CASES, ids=lambda p: p.name)
def test_small_problem_all_rows(prob):
    run_and_check(prob, tail_fill=float("nan") if prob.len_range else None)


# Decode edge cases of the streaming index scan: empty and one-token sequences (no
# items; every block -inf), fewer items than CTAs, 16 groups (two 8-column query
# tiles), d_idx 64 with block 16 (a ring of sixteen 2 KB stages).
DECODE_EDGE_CASES = [
    (Problem("decode_edges_h8", batch=6, n_q=1, max_kv=3000, H=32, h=8, d=128, d_idx=128,
             block=64, topk=8, seed=121), [0, 1, 63, 64, 65, 3000]),
    (Problem("decode_h16_d64_b16", batch=3, n_q=1, max_kv=5000, H=16, h=16, d=64, d_idx=64,
             block=16, topk=40, seed=122), [5000, 17, 2500]),
    (Problem("decode_few_items", batch=1, n_q=1, max_kv=640, H=8, h=2, d=64, d_idx=128,
             block=64, topk=4, seed=123), [640]),
    # forced own block, many rows per attention CTA, a one-token and an empty
    # sequence
    (Problem("decode_own_forced", batch=6, n_q=1, max_kv=4000, H=16, h=4, d=64, d_idx=64,
             block=32, topk=6, force_own=True, seed=124), [4000, 1, 0, 33, 2500, 3999]),
]


@pytest.mark.parametrize("case", DECODE_EDGE_CASES, ids=lambda c: c[0].name)
def test_decode_scan_edges(case):
    prob, lens = case
    run_and_check(prob, lens=lens)


def test_workload_prefill_1k():
    run_and_check(WORKLOADS["prefill_1k"])


def test_workload_decode_128k_planted_blocks_selected():
    prob = WORKLOADS["decode_128k"]
    x, ids_g, _, _ = run_and_check(prob, with_oracle_ids=False)
    ids = ids_g.cpu()
    for b in range(prob.batch):
        for g in range(prob.h):
            planted = set(x["planted"][b, g].tolist())
            assert planted <= set(ids[b, 0, g].tolist())


def test_workload_decode_1m_varlen():
    run_and_check(WORKLOADS["decode_1m"], with_oracle_ids=False)


# Prefill workloads: 2048 sampled query rows each, stratified over the KV-major
# query chunks (3 at 32K, 18 at 128K) so that every chunk, its first and last
# query included, is checked on at least 64 rows.
def test_workload_prefill_32k_sampled():
    prob = WORKLOADS["prefill_32k"]
    run_and_check(prob, rows=sample_rows_chunked(prob, 2048, seed=3))


def test_workload_prefill_128k_sampled():
    prob = WORKLOADS["prefill_128k"]
    run_and_check(prob, rows=sample_rows_chunked(prob, 2048, seed=4))


# Paged KV cache against the oracle: the decode workloads' shapes (shuffled page
# pools; the 1M lengths vary per sequence) and a prefill case on every row.
def test_paged_decode_128k_against_oracle():
    prob = WORKLOADS["decode_128k"].with_(batch=4)
    x, ids_g, _, _ = run_and_check(prob, with_oracle_ids=False, paged=True)
    ids = ids_g.cpu()
    for b in range(prob.batch):
        for g in range(prob.h):
            assert set(x["planted"][b, g].tolist()) <= set(ids[b, 0, g].tolist())


def test_paged_decode_1m_varlen_against_oracle():
    run_and_check(WORKLOADS["decode_1m"], with_oracle_ids=False, paged=True)


PAGED_PREFILL = [
    # tcgen05 index GEMM (one page per 128-key tile), KV-major attention, block 128
    Problem("paged_prefill_b128_oracle", batch=1, n_q=700, max_kv=2000, H=12, h=2, d=128,
            d_idx=128, block=128, topk=5, causal=True, seed=211),
    # two pages per index key tile, block-64 KV-major attention, own block forced,
    # variable lengths
    Problem("paged_prefill_b64_oracle", batch=2, n_q=400, max_kv=1100, H=8, h=2, d=64, d_idx=64,
            block=64, topk=6, causal=True, force_own=True, seed=212, len_range=(600, 1100)),
]


@pytest.mark.parametrize("prob", PAGED_PREFILL, ids=lambda p: p.name)
def test_paged_prefill_all_rows_against_oracle(prob):
    run_and_check(prob, paged=True, tail_fill=float("nan") if prob.len_range else None)


def test_ids_any_order_with_empty_slots():
    prob = Problem("anyorder", batch=2, n_q=64, max_kv=200, H=6, h=3, d=128, d_idx=32, block=16,
                   topk=6, causal=True, seed=110)
    x = make_inputs(prob, device="cuda")
    rng = np.random.default_rng(5)
    ids = np.full((prob.batch, prob.n_q, prob.h, prob.topk), -1, dtype=np.int32)
    for b in range(prob.batch):
        for t in range(prob.n_q):
            F = (prob.max_kv - prob.n_q + t) // prob.block + 1
            for g in range(prob.h):
                pick = rng.choice(F, size=min(4, F), replace=False)
                ids[b, t, g, rng.permutation(prob.topk)[:len(pick)]] = pick
    out, lse = msa.msa_sparse_attn(x["q"], x["k"], x["v"], torch.as_tensor(ids, device="cuda"),
                                   block=prob.block, causal=True, return_lse=True)
    rows = [(b, t) for b in range(prob.batch) for t in range(prob.n_q)]
    o, l = oracle.sparse_attn(oracle_cfg(prob), host(x["q"]), host(x["k"]), host(x["v"]),
                              ids.reshape(-1, prob.h, prob.topk))
    check_attn(take_rows(out.float(), rows), take_rows(lse, rows), o, l)


def test_out_of_range_id_is_flagged_not_read():
    prob = Problem("badid", batch=1, n_q=1, max_kv=1024, H=8, h=2, d=64, d_idx=32, block=64,
                   topk=4, causal=True, seed=111)
    x = make_inputs(prob, device="cuda")
    ws = msa.Workspace("cuda")
    ids = torch.tensor([[[[0, 3, 99, -1], [1, 2, -1, -1]]]], dtype=torch.int32, device="cuda")
    out = msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, block=prob.block, workspace=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_ASSERT
    assert msa.msa_get_device_status(ws) == msa.MSA_OK  # reading clears it
    good = torch.tensor([[[[0, 3, -1, -1], [1, 2, -1, -1]]]], dtype=torch.int32, device="cuda")
    ref = msa.msa_sparse_attn(x["q"], x["k"], x["v"], good, block=prob.block, workspace=ws)
    assert torch.equal(out, ref)


def test_bounded_wait_reports_timeout():
    buf = torch.empty(4096, dtype=torch.uint8, device="cuda")
    assert msa.msa_workspace_init(buf) == msa.MSA_OK
    assert msa.msa_selftest_wait_timeout(buf, 2_000_000) == msa.MSA_OK  # 2 ms bound
    assert msa.msa_get_device_status(buf) == msa.MSA_ERR_TIMEOUT
    # the context is still usable afterwards
    t = torch.ones(16, device="cuda")
    assert float(t.sum()) == 16.0


def test_workspace_too_small_is_rejected():
    prob = WORKLOADS["prefill_1k"]
    x = make_inputs(prob, device="cuda")
    p = msa.make_params(batch=1, n_q=prob.n_q, max_kv=prob.max_kv, H=prob.H, h=prob.h, d=prob.d,
                        d_idx=prob.d_idx, block=prob.block, topk=prob.topk, q=x["q"], k=x["k"],
                        v=x["v"], q_idx=x["q_idx"], k_idx=x["k_idx"], out=x["q"])
    need = msa.msa_workspace_size(p, msa.MSA_OP_FORWARD)
    buf = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    lib = msa.load_library()
    import ctypes
    rc = lib.msa_forward(ctypes.byref(p), x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                         x["q_idx"].data_ptr(), x["k_idx"].data_ptr(), x["q"].data_ptr(), None,
                         None, None, buf.data_ptr(), buf.numel(), None)
    assert rc == msa.MSA_ERR_WORKSPACE
