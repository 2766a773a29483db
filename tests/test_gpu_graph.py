"""A decode step captured as a CUDA graph: pinned host -> device copy of the new
token's inputs, msa_append_kv, msa_forward (its kernels chained as programmatic
dependents, the top-k kernel clearing the attention's merge counters) and the
output read back, replayed several times with new inputs written into the pinned
buffer between replays.  Every replay must give bit for bit what the same calls
give issued one by one, and the device status must stay clean.
"""

import pytest
import torch

from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    Problem("graph_decode_g8", batch=4, n_q=1, max_kv=24000, H=64, h=8, d=128, d_idx=128,
            block=64, topk=32, causal=True, seed=501, len_range=(3000, 24000)),
    Problem("graph_decode_g16_d64", batch=3, n_q=1, max_kv=9000, H=16, h=1, d=64, d_idx=64,
            block=128, topk=9, causal=True, force_own=True, seed=502),
]


@pytest.mark.parametrize("prob", CASES, ids=lambda p: p.name)
def test_graph_replay_equals_eager_calls(prob):
    x = make_inputs(prob, device="cuda")
    L = (x["seq_lens"].cpu().tolist() if x["seq_lens"] is not None
         else [prob.max_kv] * prob.batch)
    g = torch.Generator().manual_seed(prob.seed)

    def new_inputs():
        # the next token's queries and K/V/K_idx rows (written at position L_b - 1)
        return {
            "q": torch.randn(x["q"].shape, generator=g).to(torch.bfloat16),
            "q_idx": torch.randn(x["q_idx"].shape, generator=g).to(torch.bfloat16),
            "k_new": torch.randn((prob.batch, 1, prob.h, prob.d), generator=g).to(torch.bfloat16),
            "v_new": torch.randn((prob.batch, 1, prob.h, prob.d), generator=g).to(torch.bfloat16),
            "k_idx_new": torch.randn((prob.batch, 1, prob.d_idx), generator=g).to(torch.bfloat16),
        }

    names = ["q", "q_idx", "k_new", "v_new", "k_idx_new"]
    host = {n: t.pin_memory() for n, t in new_inputs().items()}
    dev = {n: torch.empty_like(t, device="cuda") for n, t in host.items()}
    out_dev = torch.empty_like(x["q"])
    out_host = torch.empty(out_dev.shape, dtype=out_dev.dtype, pin_memory=True)
    ws = msa.Workspace("cuda")
    kw = dict(block=prob.block, causal=prob.causal, seq_lens=x["seq_lens"])

    def step():
        for n in names:
            dev[n].copy_(host[n], non_blocking=True)
        msa.msa_append_kv(x["k"], x["v"], x["k_idx"], dev["k_new"], dev["v_new"],
                          dev["k_idx_new"], block=prob.block, seq_lens=x["seq_lens"], workspace=ws)
        msa.msa_forward(dev["q"], x["k"], x["v"], dev["q_idx"], x["k_idx"], topk=prob.topk,
                        force_own_block=prob.force_own, out=out_dev, workspace=ws, **kw)
        out_host.copy_(out_dev, non_blocking=True)

    step()  # sizes the workspace and sets the kernels' attributes before the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    torch.cuda.synchronize()

    for _ in range(3):
        inputs = new_inputs()
        for n in names:
            host[n].copy_(inputs[n])
        graph.replay()
        torch.cuda.synchronize()
        got = out_host.clone()
        step()
        torch.cuda.synchronize()
        assert torch.equal(got, out_host)
        # and the rows really landed in the cache
        for b in range(prob.batch):
            assert torch.equal(x["k"][b, L[b] - 1].cpu(), inputs["k_new"][b, 0])
            assert torch.equal(x["k_idx"][b, L[b] - 1].cpu(), inputs["k_idx_new"][b, 0])
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
