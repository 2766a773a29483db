"""Pins for the float64 oracle (CPU only, no GPU).

Each test checks the oracle against something other than itself: a torch
library routine (matmul + amax pooling, topk, scaled_dot_product_attention,
logsumexp), brute-force enumeration on tiny inputs, closed forms (full top-k is
dense attention; k = 1 with the own block forced is block-local attention) or
invariants the method fixes (group-shared selection, scale invariance of the
ids, order invariance of the id list).  Sources: "MiniMax goes sparse"
(atlascloud.ai) section 1 steps 1-2; "MiniMax M3 的 MSA 与阶跃 Step 3.7 Flash 的
MFA" (ai.air7.fun) section "MSA：稀疏注意力的一种极简实现".
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def cfg_of(p: Problem, **kw) -> oracle.Config:
    c = oracle.Config(p.batch, p.n_q, p.max_kv, p.H, p.h, p.d, p.d_idx, p.block, p.topk,
                      causal=p.causal, force_own=p.force_own)
    for k_, v_ in kw.items():
        setattr(c, k_, v_)
    return c


def positions(p: Problem, seq_lens):
    """Absolute query positions p[b, t] = L_b - n_q + t."""
    L = (torch.full((p.batch,), p.max_kv) if seq_lens is None else seq_lens.long())
    return L[:, None] - p.n_q + torch.arange(p.n_q)[None, :], L


def torch_block_scores(p: Problem, x, seq_lens=None):
    """Token scores by matmul, causal/length mask, then max over each block (amax)."""
    qi = x["q_idx"].double()  # [b, n, h, di]
    ki = x["k_idx"].double()  # [b, L, di]
    s = torch.einsum("bngd,bld->bngl", qi, ki)
    pos, L = positions(p, seq_lens)
    j = torch.arange(p.max_kv)
    vis = j[None, None, :] < L[:, None, None]
    if p.causal:
        vis = vis & (j[None, None, :] <= pos[:, :, None])
    s = s.masked_fill(~vis[:, :, None, :], -math.inf)
    pad = p.nblk * p.block - p.max_kv
    s = F.pad(s, (0, pad), value=-math.inf)
    return s.view(p.batch, p.n_q, p.h, p.nblk, p.block).amax(-1)


def torch_attn(p: Problem, x, key_mask, scale=None):
    """Softmax attention by torch SDPA (float64) under a boolean key mask
    [b, n, H, L]; also returns the logsumexp of the scaled logits."""
    G = p.H // p.h
    q = x["q"].double().permute(0, 2, 1, 3)  # [b, H, n, d]
    k = x["k"].double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)  # [b, H, L, d]
    v = x["v"].double().repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    m = key_mask.permute(0, 2, 1, 3)  # [b, H, n, L]
    sc = 1.0 / math.sqrt(p.d) if scale is None else scale
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=sc)
    z = (q @ k.transpose(-1, -2)) * sc
    lse = torch.logsumexp(z.masked_fill(~m, -math.inf), dim=-1)
    return o.permute(0, 2, 1, 3), lse.permute(0, 2, 1)


def visible_mask(p: Problem, seq_lens=None):
    pos, L = positions(p, seq_lens)
    j = torch.arange(p.max_kv)
    vis = j[None, None, :] < L[:, None, None]
    if p.causal:
        vis = vis & (j[None, None, :] <= pos[:, :, None])
    return vis  # [b, n, L]


def ids_mask(p: Problem, ids, seq_lens=None):
    """Key mask [b, n, H, L] from block ids [b, n, h, k]; head hq uses group hq // G."""
    G = p.H // p.h
    blk = torch.arange(p.max_kv) // p.block
    sel = torch.zeros(p.batch, p.n_q, p.h, p.max_kv, dtype=torch.bool)
    idt = torch.as_tensor(ids).long()
    for s in range(idt.shape[-1]):
        col = idt[..., s]
        sel |= (blk[None, None, None, :] == col[..., None]) & (col[..., None] >= 0)
    sel = sel & visible_mask(p, seq_lens)[:, :, None, :]
    return sel.repeat_interleave(G, dim=2)


SMALL = Problem("small", batch=2, n_q=100, max_kv=100, H=6, h=2, d=16, d_idx=8, block=16,
                topk=3, causal=True, force_own=False, seed=7)


@pytest.mark.parametrize("prob", [
    SMALL,
    SMALL.with_(causal=False, seed=8),
    SMALL.with_(n_q=1, max_kv=77, seed=9),  # decode: p = L - 1
    SMALL.with_(n_q=5, max_kv=70, block=8, seed=10),  # chunked: p = L - n_q + t
])
def test_block_scores_match_matmul_and_amax(prob):
    x = make_inputs(prob)
    ref = torch_block_scores(prob, x).reshape(-1, prob.h, prob.nblk).numpy()
    got = oracle.block_scores(cfg_of(prob), x["q_idx"], x["k_idx"])
    assert np.array_equal(np.isinf(ref), np.isinf(got))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(got[fin], ref[fin], rtol=0, atol=1e-12)


def test_block_scores_variable_lengths():
    prob = SMALL.with_(n_q=1, max_kv=96, batch=3, seed=11, len_range=(40, 96))
    x = make_inputs(prob)
    sl = x["seq_lens"]
    ref = torch_block_scores(prob, x, sl).reshape(-1, prob.h, prob.nblk).numpy()
    got = oracle.block_scores(cfg_of(prob), x["q_idx"], x["k_idx"], seq_lens=sl)
    assert np.array_equal(np.isinf(ref), np.isinf(got))
    fin = np.isfinite(ref)
    np.testing.assert_allclose(got[fin], ref[fin], rtol=0, atol=1e-12)


def brute_force_ids(scores, F_, k, own=None):
    """The unique subset T (|T| = min(k, F)) such that every member outranks every
    non-member under (score desc, id asc); with ``own`` forced, own is in T and the
    rule holds for the rest."""
    m = min(k, F_)
    cands = list(range(F_))
    found = []
    for T in itertools.combinations(cands, m):
        if own is not None and own not in T:
            continue
        rest = [x for x in T if x != own] if own is not None else list(T)
        out = [y for y in cands if y not in T]
        ok = all(scores[a] > scores[b] or (scores[a] == scores[b] and a < b)
                 for a in rest for b in out)
        if ok:
            found.append(T)
    assert len(found) == 1, found
    return sorted(found[0]) + [-1] * (k - m)


@pytest.mark.parametrize("force_own", [False, True])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_matches_brute_force(force_own, seed):
    # 1 sequence of 10 blocks of 4 tokens, one query per position: F runs 1..10.
    prob = Problem("tiny", batch=1, n_q=40, max_kv=40, H=2, h=2, d=8, d_idx=4, block=4, topk=4,
                   causal=True, force_own=force_own)
    rng = np.random.default_rng(seed)
    # quantised scores so exact ties between blocks are common
    scores = rng.integers(-3, 4, size=(prob.n_q, prob.h, prob.nblk)).astype(np.float64)
    got = oracle.select(cfg_of(prob), scores)
    for t in range(prob.n_q):
        F_ = t // prob.block + 1
        for g in range(prob.h):
            want = brute_force_ids(scores[t, g], F_, prob.topk,
                                   own=(t // prob.block) if force_own else None)
            assert got[t, g].tolist() == want, (t, g)


def test_block_size_one_is_token_topk():
    # With one token per block, block scores are token scores and the selection
    # is the ordinary top-k of the causal token scores.
    prob = Problem("b1", batch=1, n_q=1, max_kv=300, H=4, h=2, d=8, d_idx=16, block=1, topk=20,
                   causal=True, seed=3)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    s = oracle.block_scores(cfg, x["q_idx"], x["k_idx"])
    ids = oracle.select(cfg, s)
    tok = torch.einsum("gd,ld->gl", x["q_idx"][0, 0].double(), x["k_idx"][0].double())
    for g in range(prob.h):
        want = torch.topk(tok[g], prob.topk).indices.sort().values.tolist()
        assert ids[0, g].tolist() == want


@pytest.mark.parametrize("force_own", [False, True])
def test_select_invariants(force_own):
    prob = SMALL.with_(n_q=200, max_kv=200, block=16, topk=5, force_own=force_own, seed=12)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    s = oracle.block_scores(cfg, x["q_idx"], x["k_idx"])
    ids = oracle.select(cfg, s)
    for row in range(ids.shape[0]):
        t = row % prob.n_q
        F_ = t // prob.block + 1
        for g in range(prob.h):
            r = ids[row, g]
            m = min(prob.topk, F_)
            assert (r[:m] >= 0).all() and (r[m:] == -1).all()
            assert (np.diff(r[:m]) > 0).all()
            assert (r[:m] < F_).all()
            if force_own:
                assert t // prob.block in r[:m]
    # A positive scale of the index query does not change the selection
    # (x2 is exact in bf16).
    x2 = dict(x)
    x2["q_idx"] = x["q_idx"] * 2
    ids2 = oracle.select(cfg, oracle.block_scores(cfg, x2["q_idx"], x2["k_idx"]))
    assert np.array_equal(ids, ids2)


@pytest.mark.parametrize("prob", [
    SMALL,
    SMALL.with_(causal=False, seed=13),
    SMALL.with_(n_q=1, max_kv=90, batch=3, len_range=(30, 90), seed=14),
])
def test_dense_matches_sdpa(prob):
    x = make_inputs(prob)
    sl = x["seq_lens"]
    mask = visible_mask(prob, sl)[:, :, None, :].expand(-1, -1, prob.H, -1)
    o_ref, lse_ref = torch_attn(prob, x, mask)
    o, lse = oracle.dense_attn(cfg_of(prob), x["q"], x["k"], x["v"], seq_lens=sl)
    np.testing.assert_allclose(o, o_ref.reshape(-1, prob.H, prob.d).numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.reshape(-1, prob.H).numpy(), atol=1e-12)


@pytest.mark.parametrize("prob", [
    SMALL.with_(topk=7),  # topk == number of blocks
    SMALL.with_(topk=9, causal=False, seed=15),
    SMALL.with_(topk=8, n_q=1, max_kv=120, batch=2, len_range=(50, 120), seed=16),
])
def test_full_topk_is_dense_attention(prob):
    # Attention runs on the raw K/V of the selected blocks, so selecting every
    # visible block is exactly dense GQA attention.
    x = make_inputs(prob)
    sl = x["seq_lens"]
    cfg = cfg_of(prob)
    ids = oracle.select(cfg, oracle.block_scores(cfg, x["q_idx"], x["k_idx"], seq_lens=sl),
                        seq_lens=sl)
    o, lse = oracle.sparse_attn(cfg, x["q"], x["k"], x["v"], ids, seq_lens=sl)
    mask = visible_mask(prob, sl)[:, :, None, :].expand(-1, -1, prob.H, -1)
    o_ref, lse_ref = torch_attn(prob, x, mask)
    np.testing.assert_allclose(o, o_ref.reshape(-1, prob.H, prob.d).numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.reshape(-1, prob.H).numpy(), atol=1e-12)


@pytest.mark.parametrize("seed", [17, 18])
def test_sparse_attn_matches_sdpa_under_block_mask(seed):
    prob = SMALL.with_(n_q=64, max_kv=64, block=8, topk=3, seed=seed)
    x = make_inputs(prob)
    rng = np.random.default_rng(seed)
    ids = np.full((prob.batch, prob.n_q, prob.h, prob.topk), -1, dtype=np.int32)
    for b in range(prob.batch):
        for t in range(prob.n_q):
            F_ = t // prob.block + 1
            for g in range(prob.h):
                m = rng.integers(1, min(prob.topk, F_) + 1)
                pick = rng.choice(F_, size=m, replace=False)
                pick[0] = t // prob.block  # keep at least one visible key
                pick = np.unique(pick)
                slots = rng.permutation(prob.topk)[:len(pick)]  # any order, -1 anywhere
                ids[b, t, g, slots] = pick
    o, lse = oracle.sparse_attn(cfg_of(prob), x["q"], x["k"], x["v"],
                                ids.reshape(-1, prob.h, prob.topk))
    o_ref, lse_ref = torch_attn(prob, x, ids_mask(prob, ids))
    np.testing.assert_allclose(o, o_ref.reshape(-1, prob.H, prob.d).numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.reshape(-1, prob.H).numpy(), atol=1e-12)


def test_topk1_own_block_is_block_local_attention():
    prob = SMALL.with_(n_q=96, max_kv=96, block=16, topk=1, force_own=True, seed=19)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    ids = oracle.select(cfg, oracle.block_scores(cfg, x["q_idx"], x["k_idx"]))
    o, _ = oracle.sparse_attn(cfg, x["q"], x["k"], x["v"], ids)
    t = torch.arange(prob.n_q)
    j = torch.arange(prob.max_kv)
    local = (j[None, :] // prob.block == t[:, None] // prob.block) & (j[None, :] <= t[:, None])
    mask = local[None, :, None, :].expand(prob.batch, -1, prob.H, -1)
    o_ref, _ = torch_attn(prob, x, mask)
    np.testing.assert_allclose(o, o_ref.reshape(-1, prob.H, prob.d).numpy(), atol=1e-12)


def test_id_order_does_not_matter():
    prob = SMALL.with_(topk=4, seed=20)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    ids = oracle.select(cfg, oracle.block_scores(cfg, x["q_idx"], x["k_idx"]))
    o1, l1 = oracle.sparse_attn(cfg, x["q"], x["k"], x["v"], ids)
    o2, l2 = oracle.sparse_attn(cfg, x["q"], x["k"], x["v"], ids[..., ::-1].copy())
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_golden_figure_head_to_group_mapping():
    # The pages' figure: 6 query heads, 2 index queries; Q1-Q3 use I1, Q4-Q6 use I2.
    with open(os.path.join(GOLDEN, "gqa_figure.json")) as f:
        fig = json.load(f)
    prob = Problem("fig", batch=1, n_q=32, max_kv=32, H=fig["H"], h=fig["h"], d=8, d_idx=8,
                   block=4, topk=2, causal=True, seed=21)
    x = make_inputs(prob)
    # group g selects {min(g, own), own}: the two groups differ wherever own >= 1
    ids = np.full((1, prob.n_q, prob.h, prob.topk), -1, dtype=np.int32)
    for t in range(prob.n_q):
        own = t // prob.block
        for g in range(prob.h):
            pick = sorted({min(g, own), own})
            ids[0, t, g, :len(pick)] = pick
    o, _ = oracle.sparse_attn(cfg_of(prob), x["q"], x["k"], x["v"], ids.reshape(-1, prob.h, 2))
    for hq, g in enumerate(fig["head_group"]):
        ids_g = ids[:, :, [g] * prob.h, :]  # every group takes group g's selection
        o_g, _ = torch_attn(prob, x, ids_mask(prob, ids_g))
        np.testing.assert_allclose(o[:, hq], o_g[0, :, hq].numpy(), atol=1e-12)


def test_planted_blocks_are_selected():
    # Decode with planted blocks (the recipe of the 128K decode workload, at
    # reduced length): every planted block of every group is in the top-k.
    prob = Problem("plant", batch=2, n_q=1, max_kv=8192, H=16, h=4, d=32, d_idx=128, block=64,
                   topk=16, causal=True, seed=22, plant_frac=0.04)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    ids = oracle.select(cfg, oracle.block_scores(cfg, x["q_idx"], x["k_idx"]))
    for b in range(prob.batch):
        for g in range(prob.h):
            planted = set(x["planted"][b, g].tolist())
            assert planted <= set(ids[b, g].tolist())


def test_forward_composes_the_stages():
    prob = SMALL.with_(seed=23, force_own=True)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    ids, o, lse = oracle.forward(cfg, x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"])
    ids2 = oracle.select(cfg, oracle.block_scores(cfg, x["q_idx"], x["k_idx"]))
    o2, l2 = oracle.sparse_attn(cfg, x["q"], x["k"], x["v"], ids2)
    assert np.array_equal(ids, ids2) and np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_row_subset_matches_full():
    prob = SMALL.with_(seed=24)
    x = make_inputs(prob)
    cfg = cfg_of(prob)
    full = oracle.block_scores(cfg, x["q_idx"], x["k_idx"])
    rows = [(1, 99), (0, 0), (1, 17)]
    sub = oracle.block_scores(cfg, x["q_idx"], x["k_idx"], rows=rows)
    for i, (b, t) in enumerate(rows):
        assert np.array_equal(sub[i], full[b * prob.n_q + t])
