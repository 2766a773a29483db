"""Out-of-bounds writes: canary-padded workspace and outputs.

Every buffer the library writes (the workspace, block ids, block scores, the
output and the log-sum-exps) is a view into a larger allocation whose bytes
before and after the view hold a fixed pattern.  After each call the pattern must
be intact, on the three attention paths (decode streaming kernel, KV-major
prefill, one CTA per row) and the index stage, so that no kernel writes outside
the sizes the library asked for.
"""

import pytest
import torch

from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import Problem, make_inputs

pytestmark = pytest.mark.gpu

PAD = 4096
PATTERN = 0xA5

CASES = [
    # decode: streaming scan, CTA top-k, streaming attention with split rows
    Problem("canary_decode", batch=3, n_q=1, max_kv=40000, H=32, h=8, d=128, d_idx=128, block=64,
            topk=100, causal=True, seed=801, len_range=(1000, 40000)),
    # prefill through the KV-major kernel (tcgen05 index GEMM, warp top-k)
    Problem("canary_kv", batch=1, n_q=1200, max_kv=1500, H=16, h=2, d=128, d_idx=64, block=64,
            topk=6, causal=True, force_own=True, seed=802),
    # prefill through the one-CTA-per-row kernel (block 32)
    Problem("canary_rows", batch=2, n_q=300, max_kv=400, H=8, h=2, d=64, d_idx=32, block=32,
            topk=4, causal=True, seed=803, len_range=(300, 400)),
]


class Padded:
    """`nbytes` usable bytes at offset PAD of an allocation padded on both sides."""

    def __init__(self, nbytes):
        self.nbytes = nbytes
        self.raw = torch.full((PAD + nbytes + PAD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.mid = self.raw[PAD:PAD + nbytes]

    def view(self, dtype, shape):
        return self.mid.view(dtype).view(shape)

    def intact(self):
        return bool(torch.all(self.raw[:PAD] == PATTERN)) and \
            bool(torch.all(self.raw[PAD + self.nbytes:] == PATTERN))


def padded_workspace(nbytes):
    p = Padded(nbytes)
    ws = msa.Workspace("cuda")
    ws.buf = p.mid
    assert msa.msa_workspace_init(p.mid) == msa.MSA_OK
    return p, ws


@pytest.mark.parametrize("prob", CASES, ids=lambda p: p.name)
def test_no_write_outside_the_buffers(prob):
    x = make_inputs(prob, device="cuda")
    sl = x["seq_lens"]
    p = msa.make_params(batch=prob.batch, n_q=prob.n_q, max_kv=prob.max_kv, H=prob.H, h=prob.h,
                        d=prob.d, d_idx=prob.d_idx, block=prob.block, topk=prob.topk,
                        causal=prob.causal, force_own_block=prob.force_own, seq_lens=sl,
                        q=x["q"], k=x["k"], v=x["v"], q_idx=x["q_idx"], k_idx=x["k_idx"],
                        out=x["q"])
    need = max(msa.msa_workspace_size(p, op)
               for op in (msa.MSA_OP_INDEX_SELECT, msa.MSA_OP_SPARSE_ATTN, msa.MSA_OP_FORWARD))
    wsp, ws = padded_workspace(need)
    nblk = -(-prob.max_kv // prob.block)
    rows = (prob.batch, prob.n_q, prob.h)
    ids_p = Padded(prob.batch * prob.n_q * prob.h * prob.topk * 4)
    sc_p = Padded(prob.batch * prob.n_q * prob.h * nblk * 4)
    out_p = Padded(x["q"].numel() * 2)
    lse_p = Padded(prob.batch * prob.n_q * prob.H * 4)
    ids = ids_p.view(torch.int32, rows + (prob.topk,))
    sc = sc_p.view(torch.float32, rows + (nblk,))
    out = out_p.view(torch.bfloat16, tuple(x["q"].shape))
    lse = lse_p.view(torch.float32, (prob.batch, prob.n_q, prob.H))
    kw = dict(block=prob.block, causal=prob.causal, seq_lens=sl, workspace=ws)
    bufs = [wsp, ids_p, sc_p, out_p, lse_p]

    msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk, force_own_block=prob.force_own,
                         block_ids=ids, block_scores=sc, **kw)
    torch.cuda.synchronize()
    assert all(b.intact() for b in bufs)
    msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, out=out, lse=lse, **kw)
    torch.cuda.synchronize()
    assert all(b.intact() for b in bufs)
    ref = out.clone()
    msa.msa_forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], topk=prob.topk,
                    force_own_block=prob.force_own, out=out, block_ids=ids, block_scores=sc,
                    lse=lse, **kw)
    torch.cuda.synchronize()
    assert all(b.intact() for b in bufs)
    assert torch.equal(out, ref)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    assert wsp.intact()
