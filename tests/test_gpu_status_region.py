"""The workspace's status region: the sticky status word and the decode
attention's per-row merge counters, which must be zero between calls.

* Calls of different decode shapes on one workspace leave the counters at zero
  (each row's merging CTA puts its counter back), so every result equals the
  result on a fresh workspace, call after call.
* A call that stopped early may leave counters set; the status word then holds
  the error, and msa_get_device_status clears the whole region.  The test sets the
  counters to garbage by hand, records an error with the bounded-wait self-test
  (a wait on a barrier nothing completes, 2 ms; no fault), reads the status back,
  and requires the next call to be exact again.
"""

import pytest
import torch

from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    Problem("status_a", batch=3, n_q=1, max_kv=20000, H=32, h=8, d=128, d_idx=128, block=64,
            topk=40, causal=True, seed=601, len_range=(5000, 20000)),
    Problem("status_b", batch=5, n_q=1, max_kv=9000, H=12, h=2, d=64, d_idx=64, block=32,
            topk=70, causal=True, seed=602, len_range=(1, 9000)),
]


def attn(prob, x, ids, ws):
    return msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, block=prob.block, causal=True,
                               seq_lens=x["seq_lens"], return_lse=True, workspace=ws)


@pytest.fixture(scope="module")
def cases():
    out = []
    for prob in SHAPES:
        x = make_inputs(prob, device="cuda")
        ids = msa.msa_index_select(x["q_idx"], x["k_idx"], block=prob.block, topk=prob.topk,
                                   seq_lens=x["seq_lens"])
        ref = attn(prob, x, ids, msa.Workspace("cuda"))
        out.append((prob, x, ids, ref))
    torch.cuda.synchronize()
    return out


def test_counters_return_to_zero_between_calls(cases):
    ws = msa.Workspace("cuda")
    for k in [0, 1, 1, 0, 1, 0, 0]:
        prob, x, ids, (ref_o, ref_l) = cases[k]
        o, l = attn(prob, x, ids, ws)
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
        # the counter words of the status region are all zero again
        assert int(ws.buf[256:msa.STATUS_BYTES].count_nonzero()) == 0
    assert msa.msa_get_device_status(ws) == msa.MSA_OK


def test_status_read_after_an_error_clears_the_counters(cases):
    prob, x, ids, (ref_o, ref_l) = cases[0]
    ws = msa.Workspace("cuda")
    attn(prob, x, ids, ws)  # sizes and initialises the workspace
    torch.cuda.synchronize()
    # counters as a call that stopped early could leave them
    ws.buf[256:msa.STATUS_BYTES] = torch.randint(0, 256, (msa.STATUS_BYTES - 256,),
                                                dtype=torch.uint8, device="cuda")
    assert msa.msa_selftest_wait_timeout(ws.buf, 2_000_000) == msa.MSA_OK
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_TIMEOUT
    assert int(ws.buf[:msa.STATUS_BYTES].count_nonzero()) == 0
    o, l = attn(prob, x, ids, ws)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
