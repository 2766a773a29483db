"""msa_sparse_attn_noalloc: the sparse branch for callers that cannot allocate
device memory (an engine's enqueue path, a real-time loop, a host framework that
owns every allocation).  Its intermediates live in the library's fixed device
array instead of a caller workspace.

Checked through the C ABI against msa_sparse_attn (which takes a caller
workspace), on two calls in a row each: a decode problem that runs in several
KV splits (the split partials use the fixed array) and the 1K prefill workload
(the KV-major kernel's inverted index and partial tiles use it).  This file is
collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_gqa_03_b200 import msa
from block_sparse_gqa_03_b200.inputs import WORKLOADS, Problem, make_inputs
from msa_check import OUT_MAX_ABS, OUT_MEAN_ABS

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    prob = Problem("noalloc", batch=4, n_q=1, max_kv=65536, H=64, h=8, d=128, d_idx=128,
                   block=64, topk=256, causal=True, seed=120, len_range=(30000, 65536))
    x = make_inputs(prob, device="cuda")
    kw = dict(block=prob.block, causal=True, seq_lens=x["seq_lens"])
    ids = msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk, **kw)
    ref, ref_lse = msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, return_lse=True, **kw)
    p = msa.make_params(batch=prob.batch, n_q=1, max_kv=prob.max_kv, H=prob.H, h=prob.h,
                        d=prob.d, d_idx=prob.d_idx, block=prob.block, topk=prob.topk,
                        seq_lens=x["seq_lens"], q=x["q"], k=x["k"], v=x["v"], out=ref)
    # the plan splits each row's blocks over several CTAs, so partials are needed
    assert msa.msa_workspace_size(p, msa.MSA_OP_SPARSE_ATTN) > msa.STATUS_BYTES
    lib = msa.load_library()
    stream = torch.cuda.current_stream().cuda_stream or None
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = lib.msa_sparse_attn_noalloc(ctypes.byref(p), x["q"].data_ptr(), x["k"].data_ptr(),
                                         x["v"].data_ptr(), ids.data_ptr(), out.data_ptr(),
                                         lse.data_ptr(), stream)
        assert rc == msa.MSA_OK, msa.msa_status_string(rc)
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs()
        assert float(err.max()) <= OUT_MAX_ABS and float(err.mean()) <= OUT_MEAN_ABS
        assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=2e-3)


def test_noalloc_kv_major_prefill_matches_workspace_entry_point_twice():
    # the 1K prefill workload (n 1024, H 6 / h 2, d 64, block 64, top-4) takes the
    # KV-major kernel, whose inverted index and partial tiles (about 3.8 MB) go to
    # the fixed array; the same kernels on the same inputs give identical bits
    prob = WORKLOADS["prefill_1k"]
    x = make_inputs(prob, device="cuda")
    kw = dict(block=prob.block, causal=prob.causal)
    ids = msa.msa_index_select(x["q_idx"], x["k_idx"], topk=prob.topk,
                               force_own_block=prob.force_own, **kw)
    ref, ref_lse = msa.msa_sparse_attn(x["q"], x["k"], x["v"], ids, return_lse=True, **kw)
    p = msa.make_params(batch=prob.batch, n_q=prob.n_q, max_kv=prob.max_kv, H=prob.H, h=prob.h,
                        d=prob.d, d_idx=prob.d_idx, block=prob.block, topk=prob.topk,
                        q=x["q"], k=x["k"], v=x["v"], out=ref)
    need = msa.msa_workspace_size(p, msa.MSA_OP_SPARSE_ATTN)
    assert msa.STATUS_BYTES + (1 << 20) < need < (8 << 20)
    lib = msa.load_library()
    stream = torch.cuda.current_stream().cuda_stream or None
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = lib.msa_sparse_attn_noalloc(ctypes.byref(p), x["q"].data_ptr(), x["k"].data_ptr(),
                                         x["v"].data_ptr(), ids.data_ptr(), out.data_ptr(),
                                         lse.data_ptr(), stream)
        assert rc == msa.MSA_OK, msa.msa_status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)


def test_noalloc_rejects_partials_beyond_its_scratch():
    # Find a shape whose split-KV partials exceed the fixed 8 MiB; the entry point
    # must refuse it on the host, before any launch.  The plan bounds the partials
    # by roughly (num_sms + 2 * rows) * G * (d + 1) * 4 bytes, so on some GPUs no
    # supported shape gets there.
    lib = msa.load_library()
    fake = torch.empty(16, device="cuda")
    for B, h, G in ((64, 9, 16), (40, 14, 16), (70, 8, 16), (36, 16, 16)):
        H, d, L = h * G, 128, 4096
        p = msa.make_params(batch=B, n_q=1, max_kv=L, H=H, h=h, d=d, d_idx=128, block=64,
                            topk=4096)
        p.q_strides[:] = [H * d, H * d, d]
        p.k_strides[:] = [L * h * d, h * d, d]
        p.v_strides[:] = [L * h * d, h * d, d]
        p.o_strides[:] = [H * d, H * d, d]
        if msa.msa_workspace_size(p, msa.MSA_OP_SPARSE_ATTN) > (8 << 20) + 4096:
            rc = lib.msa_sparse_attn_noalloc(ctypes.byref(p), fake.data_ptr(), fake.data_ptr(),
                                             fake.data_ptr(), fake.data_ptr(), fake.data_ptr(),
                                             None, None)
            assert rc == msa.MSA_ERR_WORKSPACE
            return
    pytest.skip("no supported shape needs more than the fixed scratch on this GPU")
