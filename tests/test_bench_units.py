"""The benchmark's algorithmic units against closed forms (no GPU).

Every roofline fraction the bench reports divides these counts by a measured
time, so they are pinned here independently of the code that computes them:
decode bytes are K_idx read once per sequence plus the selected K/V blocks plus
q, q_idx and the output; prefill flops are 2*d_idx per visible (query, group,
key) for the index GEMM plus 4*d per (head, selected visible key) for the
attention.  With k at least the number of causal blocks the selection is every
causal block, so the attention count is dense causal attention's.
"""

import torch

import bench
from block_sparse_gqa_03_b200.inputs import WORKLOADS, Problem


def all_blocks(prob, n_q):
    """ids selecting blocks 0..topk-1 for every (sequence, query, group)."""
    ids = torch.arange(prob.topk, dtype=torch.int32)
    return ids.expand(prob.batch, n_q, prob.h, prob.topk).contiguous()


def test_decode_128k_bytes():
    p = WORKLOADS["decode_128k"]
    u = bench.work_units(p, {"seq_lens": None}, all_blocks(p, 1))
    kidx = 16 * 131072 * 128 * 2
    kv = 16 * 8 * 128 * 64 * 128 * 2 * 2  # 128 full blocks of K and V per (sequence, group)
    assert u["select"] == kidx + 16 * 8 * 128 * 2  # + q_idx
    assert u["attn"] == kv + 2 * 16 * 64 * 128 * 2  # + q and out
    assert abs((u["select"] + u["attn"]) / 1.074e9 - 1) < 1e-3  # 1.074 GB per step


def test_decode_bytes_follow_the_lengths_and_partial_blocks():
    p = Problem("lens", batch=2, n_q=1, max_kv=1000, H=4, h=2, d=64, d_idx=32, block=64, topk=16)
    lens = torch.tensor([1000, 130], dtype=torch.int32)
    ids = all_blocks(p, 1).clone()
    ids[1, :, :, 3:] = -1  # sequence 1 has 3 blocks: 64 + 64 + 2 visible tokens
    u = bench.work_units(p, {"seq_lens": lens}, ids)
    assert u["select"] == (1000 + 130) * 32 * 2 + 2 * 2 * 32 * 2
    vis = 2 * 1000 + 2 * 130  # per group: every visible token of each sequence
    assert u["attn"] == vis * 64 * 2 * 2 + 2 * 2 * 4 * 64 * 2


def test_prefill_flops_dense_when_k_covers_every_block():
    n = 1024
    p = Problem("dense", batch=1, n_q=n, max_kv=n, H=6, h=2, d=64, d_idx=32, block=64,
                topk=16, causal=True)
    u = bench.work_units(p, {"seq_lens": None}, all_blocks(p, n))
    causal_keys = n * (n + 1) // 2
    assert u["select"] == 2 * 32 * 2 * causal_keys == 67_174_400  # 6.72e7, the 1K config's index work
    assert u["attn"] == 4 * 64 * 6 * causal_keys


def test_prefill_index_flops_of_the_long_configs():
    for name, want in (("prefill_32k", 5.50e11), ("prefill_128k", 1.759e13)):
        p = WORKLOADS[name]
        _, lim = bench.positions(p, None, torch.device("cpu"))
        index = 2 * p.d_idx * p.h * int(lim.sum())
        assert index == 2 * p.d_idx * p.h * p.batch * p.n_q * (p.n_q + 1) // 2
        assert abs(index / want - 1) < 2e-3, (name, index)
