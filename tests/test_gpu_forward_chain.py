"""msa_forward chains its kernels as programmatic dependents and lets the top-k
kernel clear the attention's per-row merge counters (whose place in the workspace
depends on the shapes).  Interleaving fused and separate calls of different shapes
on one workspace must keep every result equal to the separate calls'."""

import pytest
import torch

from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    Problem("chain_a", batch=6, n_q=1, max_kv=20000, H=32, h=8, d=128, d_idx=128, block=64,
            topk=40, causal=True, seed=301, len_range=(9000, 20000)),
    Problem("chain_b", batch=2, n_q=1, max_kv=70000, H=16, h=2, d=64, d_idx=64, block=128,
            topk=200, causal=True, seed=302, len_range=(30000, 70000)),
]


def separate(prob, x, ws):
    kw = dict(block=prob.block, causal=prob.causal, seq_lens=x["seq_lens"], workspace=ws)
    ids = msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk, **kw)
    out, lse = msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, return_lse=True, **kw)
    return ids, out, lse


def fused(prob, x, ws):
    out, ids, lse = msa.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], topk=prob.topk,
                                    block=prob.block, causal=prob.causal, seq_lens=x["seq_lens"],
                                    return_ids=True, return_lse=True, workspace=ws)
    return ids, out, lse


def test_fused_and_separate_calls_interleaved_on_one_workspace():
    xs = [make_inputs(p, device="cuda") for p in SHAPES]
    ws = msa.Workspace("cuda")
    ref = [separate(p, x, msa.Workspace("cuda")) for p, x in zip(SHAPES, xs)]
    order = [0, 1, 0, 0, 1, 1, 0]
    for step, i in enumerate(order):
        p, x = SHAPES[i], xs[i]
        got = fused(p, x, ws) if step % 3 != 2 else separate(p, x, ws)
        for a, b in zip(got, ref[i]):
            assert torch.equal(a, b), (p.name, step)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
