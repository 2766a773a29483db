"""The C ABI on a machine without a GPU: the library loads, exports every entry
point ``include/msa.h`` declares, and rejects bad arguments on the host before
anything is launched.  No compute call is made here."""

import ctypes
import os
import re

import pytest

from block_sparse_gqa_03_b200 import build as msa_build
from block_sparse_gqa_03_b200 import msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", text)


def test_header_declares_the_binding_names():
    names = declared_functions()
    assert sorted(names) == sorted(msa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(7):
        assert msa.msa_status_string(code)
    assert msa.msa_status_string(99) == "unknown status"


def valid_params(**kw):
    base = dict(batch=1, n_q=1024, max_kv=1024, H=6, h=2, d=64, d_idx=32, block=64, topk=4)
    base.update(kw)
    p = msa.make_params(**base)
    p.q_strides[:] = [1024 * 6 * 64, 6 * 64, 64]
    p.k_strides[:] = [1024 * 2 * 64, 2 * 64, 64]
    p.v_strides[:] = [1024 * 2 * 64, 2 * 64, 64]
    p.o_strides[:] = [1024 * 6 * 64, 6 * 64, 64]
    p.qi_strides[:] = [1024 * 2 * 32, 2 * 32, 32]
    p.ki_strides[:] = [1024 * 32, 32]
    return p


def test_workspace_size_host_only(lib):
    p = valid_params()
    sel = msa.msa_workspace_size(p, msa.MSA_OP_INDEX_SELECT)
    fwd = msa.msa_workspace_size(p, msa.MSA_OP_FORWARD)
    # status region + fp32 block scores [1, 1024, 2, 16] (+ ids for forward)
    assert sel >= msa.STATUS_BYTES + 1024 * 2 * 16 * 4
    assert fwd >= sel + 1024 * 2 * 4 * 4
    assert msa.msa_workspace_size(p, 99) == 0
    # the index scan alone, the candidate merge and the shard lengths need the
    # status region only; the candidates call needs what index select needs
    for op in (msa.MSA_OP_BLOCK_SCORES, msa.MSA_OP_SELECT_CANDIDATES, msa.MSA_OP_SHARD_LENGTHS,
               msa.MSA_OP_APPEND_KV):
        assert msa.msa_workspace_size(p, op) == msa.STATUS_BYTES
    assert msa.msa_workspace_size(p, msa.MSA_OP_INDEX_CANDIDATES) == sel


def test_sharded_decode_calls_validate_on_the_host(lib):
    p = valid_params(n_q=1)
    fake = 1 << 20  # never dereferenced: validation fails first
    ws_small = 128
    # candidate merge: empty or oversized lists, negative base, no output
    sc = lib.msa_select_candidates
    assert sc(ctypes.byref(p), 0, 4, 0, fake, fake, 0, 4, fake, None, fake, 4096,
              None) == msa.MSA_ERR_INVALID_ARG
    assert sc(ctypes.byref(p), 8, 4096, 0, fake, fake, 0, 4, fake, None, fake, 4096,
              None) == msa.MSA_ERR_UNSUPPORTED
    assert sc(ctypes.byref(p), 2, 4, 16, fake, fake, -1, 4, fake, None, fake, 4096,
              None) == msa.MSA_ERR_INVALID_ARG
    assert sc(ctypes.byref(p), 2, 4, 16, fake, fake, 0, 4, None, None, fake, 4096,
              None) == msa.MSA_ERR_INVALID_ARG
    assert sc(ctypes.byref(p), 2, 4, 16, fake, fake, 0, 4, fake, None, fake, ws_small,
              None) == msa.MSA_ERR_WORKSPACE
    # merge of partials: part count and alignment
    assert lib.msa_merge_partials(ctypes.byref(p), 0, fake, fake, fake, None,
                                  None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_merge_partials(ctypes.byref(p), 2, fake + 8, fake, fake, None,
                                  None) == msa.MSA_ERR_INVALID_ARG
    # shard lengths and the candidates call
    assert lib.msa_shard_lengths(ctypes.byref(p), -1, 10, fake, fake, 4096,
                                 None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_index_candidates(ctypes.byref(p), fake, fake, fake, None, fake, 1 << 30,
                                    None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_block_scores(ctypes.byref(p), fake, fake, None, fake, 4096,
                                None) == msa.MSA_ERR_INVALID_ARG
    assert msa.msa_launch_count(p, msa.MSA_OP_INDEX_CANDIDATES) == 2
    assert msa.msa_launch_count(p, msa.MSA_OP_SELECT_CANDIDATES) == 1


@pytest.mark.parametrize("bad,code", [
    (dict(H=7), msa.MSA_ERR_INVALID_ARG),          # H % h != 0
    (dict(d=96), msa.MSA_ERR_UNSUPPORTED),
    (dict(d_idx=48), msa.MSA_ERR_UNSUPPORTED),
    (dict(block=48), msa.MSA_ERR_UNSUPPORTED),
    (dict(topk=0), msa.MSA_ERR_INVALID_ARG),
    (dict(topk=5000), msa.MSA_ERR_UNSUPPORTED),
    (dict(n_q=2048), msa.MSA_ERR_INVALID_ARG),     # n_q > max_kv
    (dict(H=34, h=2), msa.MSA_ERR_UNSUPPORTED),    # G = 17
])
def test_bad_params_rejected_before_launch(lib, bad, code):
    p = valid_params(**bad)
    fake = 1 << 20  # never dereferenced: validation fails first
    rc = lib.msa_forward(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None, None, None,
                         fake, 1 << 30, None)
    assert rc == code
    assert msa.msa_workspace_size(p, msa.MSA_OP_FORWARD) == 0


def test_bad_pointers_and_workspace_rejected(lib):
    p = valid_params()
    fake = 1 << 20
    # null q
    assert lib.msa_forward(ctypes.byref(p), None, fake, fake, fake, fake, fake, None, None, None,
                           fake, 1 << 30, None) == msa.MSA_ERR_INVALID_ARG
    # misaligned k_idx
    assert lib.msa_index_select(ctypes.byref(p), fake, fake + 2, fake, None, fake, 1 << 30,
                                None) == msa.MSA_ERR_INVALID_ARG
    # workspace too small, or misaligned
    assert lib.msa_index_select(ctypes.byref(p), fake, fake, fake, None, fake, 512,
                                None) == msa.MSA_ERR_WORKSPACE
    assert lib.msa_index_select(ctypes.byref(p), fake, fake, fake, None, fake + 16, 1 << 30,
                                None) == msa.MSA_ERR_WORKSPACE
    # stride not a multiple of 8 elements
    p.k_strides[1] = 130
    assert lib.msa_sparse_attn(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, 1 << 30,
                               None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_selftest_wait_timeout(None, 4096, 1000, None) == msa.MSA_ERR_WORKSPACE
    assert lib.msa_selftest_wait_timeout(fake, 4096, 0, None) == msa.MSA_ERR_INVALID_ARG


def test_paged_params_validated(lib):
    p = valid_params()
    assert msa.msa_workspace_size(p, msa.MSA_OP_FORWARD) > 0
    fake = 1 << 20
    p.block_table, p.num_pages = fake, 64
    p.table_stride = 16  # = ceil(1024 / 64) blocks per sequence
    assert msa.msa_workspace_size(p, msa.MSA_OP_FORWARD) > 0
    p.table_stride = 15  # too short for max_kv
    assert msa.msa_workspace_size(p, msa.MSA_OP_FORWARD) == 0
    p.table_stride, p.num_pages = 16, 0  # empty pool
    assert msa.msa_workspace_size(p, msa.MSA_OP_FORWARD) == 0
    p.num_pages, p.block_table = 64, fake + 2  # misaligned table
    assert lib.msa_forward(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None, None, None,
                           fake, 1 << 30, None) == msa.MSA_ERR_INVALID_ARG


def test_append_args_validated(lib):
    p = valid_params()
    fake = 1 << 20
    assert msa.msa_workspace_size(p, msa.MSA_OP_APPEND_KV) == msa.STATUS_BYTES
    assert msa.msa_launch_count(p, msa.MSA_OP_APPEND_KV) == 1
    # new K rows without a K cache, misaligned new rows, a workspace without room
    # for the status region
    sb = msa.STATUS_BYTES
    assert lib.msa_append_kv(ctypes.byref(p), fake, None, None, None, None, None, fake, sb,
                             None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_append_kv(ctypes.byref(p), fake + 2, None, None, fake, None, None, fake, sb,
                             None) == msa.MSA_ERR_INVALID_ARG
    assert lib.msa_append_kv(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, sb - 256,
                             None) == msa.MSA_ERR_WORKSPACE
    p.ki_strides[1] = 16  # index-key rows closer than d_idx
    assert lib.msa_append_kv(ctypes.byref(p), None, None, fake, None, None, fake, fake, sb,
                             None) == msa.MSA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(msa, "LIB_PATH", "/nonexistent/libmsa.so")
    monkeypatch.setattr(msa, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        msa.load_library()


def test_prefill_chunk_plan_matches_the_library(lib):
    # the parity tests stratify their sampled prefill rows by the KV-major query
    # chunks; their restatement of the chunk plan must give the library's count
    # (five kernels per chunk)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from msa_check import kv_chunk_rows
    from block_sparse_gqa_03_b200.inputs import WORKLOADS
    for name in ("prefill_1k", "prefill_32k", "prefill_128k"):
        pr = WORKLOADS[name]
        p = msa.make_params(batch=pr.batch, n_q=pr.n_q, max_kv=pr.max_kv, H=pr.H, h=pr.h,
                            d=pr.d, d_idx=pr.d_idx, block=pr.block, topk=pr.topk)
        rows = pr.batch * pr.n_q
        nch = -(-rows // kv_chunk_rows(pr))
        assert msa.msa_launch_count(p, msa.MSA_OP_SPARSE_ATTN) == 5 * nch, name
