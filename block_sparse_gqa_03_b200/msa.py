"""Thin ctypes binding of ``libmsa.so`` (C ABI declared in ``include/msa.h``).

Argument marshalling only: every step of MSA runs in the library's CUDA kernels.
torch tensors provide device memory and the current stream.  The names follow
the C ABI: ``msa_index_select``, ``msa_sparse_attn``, ``msa_forward``,
``msa_workspace_size``, ``msa_get_device_status``, ``msa_workspace_init``,
``msa_selftest_wait_timeout``, ``msa_status_string``.

There is no fallback: if ``libmsa.so`` has not been built, or no CUDA device is
present, these functions raise.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")
STATUS_BYTES = 4096  # the workspace's status region (status word, decode merge counters)

MSA_OK = 0
MSA_ERR_INVALID_ARG = 1
MSA_ERR_UNSUPPORTED = 2
MSA_ERR_WORKSPACE = 3
MSA_ERR_CUDA = 4
MSA_ERR_TIMEOUT = 5
MSA_ERR_DEVICE_ASSERT = 6

MSA_OP_INDEX_SELECT = 0
MSA_OP_SPARSE_ATTN = 1
MSA_OP_FORWARD = 2
MSA_OP_APPEND_KV = 3
MSA_OP_BLOCK_SCORES = 4
MSA_OP_INDEX_CANDIDATES = 5
MSA_OP_SELECT_CANDIDATES = 6
MSA_OP_SHARD_LENGTHS = 7
MSA_OP_INDEX_TOPK = 8

EXPORTED = ("msa_workspace_size", "msa_index_select", "msa_sparse_attn", "msa_forward",
            "msa_get_device_status", "msa_workspace_init", "msa_selftest_wait_timeout",
            "msa_launch_count", "msa_sparse_attn_noalloc", "msa_status_string", "msa_append_kv",
            "msa_block_scores", "msa_index_candidates", "msa_select_candidates",
            "msa_merge_partials", "msa_shard_lengths", "msa_index_topk")


class MsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (status %d)" % (what, msa_status_string(code), code))
        self.code = code


class Params(ctypes.Structure):
    """Mirror of ``msa_params_t``."""

    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_q", "max_kv", "H", "h", "d", "d_idx", "block", "topk", "causal",
        "force_own_block")] + [
        ("softmax_scale", ctypes.c_float),
        ("seq_lens", ctypes.c_void_p),
        ("q_strides", ctypes.c_int64 * 3),
        ("k_strides", ctypes.c_int64 * 3),
        ("v_strides", ctypes.c_int64 * 3),
        ("qi_strides", ctypes.c_int64 * 3),
        ("ki_strides", ctypes.c_int64 * 2),
        ("o_strides", ctypes.c_int64 * 3),
        ("block_table", ctypes.c_void_p),
        ("table_stride", ctypes.c_int64),
        ("num_pages", ctypes.c_int64),
    ]


_lib = None
_lib_lock = threading.Lock()


def load_library():
    """Load ``libmsa.so``; raises if it has not been built."""
    global _lib
    with _lib_lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError("libmsa.so is not built (run __graft_entry__.build() or "
                                   "python -m block_sparse_gqa_03_b200.build)")
            lib = ctypes.CDLL(LIB_PATH)
            P, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
            lib.msa_workspace_size.argtypes = [P, I]
            lib.msa_workspace_size.restype = S
            lib.msa_index_select.argtypes = [P, P, P, P, P, P, S, P]
            lib.msa_index_select.restype = I
            lib.msa_sparse_attn.argtypes = [P, P, P, P, P, P, P, P, S, P]
            lib.msa_sparse_attn.restype = I
            lib.msa_forward.argtypes = [P, P, P, P, P, P, P, P, P, P, P, S, P]
            lib.msa_forward.restype = I
            lib.msa_append_kv.argtypes = [P, P, P, P, P, P, P, P, S, P]
            lib.msa_append_kv.restype = I
            lib.msa_get_device_status.argtypes = [P, P]
            lib.msa_get_device_status.restype = I
            lib.msa_workspace_init.argtypes = [P, S, P]
            lib.msa_workspace_init.restype = I
            lib.msa_selftest_wait_timeout.argtypes = [P, S, ctypes.c_uint64, P]
            lib.msa_selftest_wait_timeout.restype = I
            lib.msa_sparse_attn_noalloc.argtypes = [P, P, P, P, P, P, P, P]
            lib.msa_sparse_attn_noalloc.restype = I
            lib.msa_index_topk.argtypes = [P, P, P, P, P, P, S, P]
            lib.msa_index_topk.restype = I
            lib.msa_block_scores.argtypes = [P, P, P, P, P, S, P]
            lib.msa_block_scores.restype = I
            lib.msa_index_candidates.argtypes = [P, P, P, P, P, P, S, P]
            lib.msa_index_candidates.restype = I
            i32 = ctypes.c_int32
            lib.msa_select_candidates.argtypes = [P, i32, i32, i32, P, P, i32, i32, P, P, P, S, P]
            lib.msa_select_candidates.restype = I
            lib.msa_merge_partials.argtypes = [P, ctypes.c_int32, P, P, P, P, P]
            lib.msa_merge_partials.restype = I
            lib.msa_shard_lengths.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, P, S, P]
            lib.msa_shard_lengths.restype = I
            lib.msa_launch_count.argtypes = [P, I]
            lib.msa_launch_count.restype = I
            lib.msa_status_string.argtypes = [I]
            lib.msa_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def msa_status_string(code: int) -> str:
    return load_library().msa_status_string(int(code)).decode()


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream or None


def _outer(t: torch.Tensor, n: int):
    if t.stride(-1) != 1:
        raise ValueError("innermost axis must be contiguous")
    return list(t.stride()[:n])


def make_params(*, batch, n_q, max_kv, H, h, d, d_idx, block, topk, causal=True,
                force_own_block=False, softmax_scale=0.0, seq_lens=None, q=None, k=None, v=None,
                q_idx=None, k_idx=None, out=None, block_table=None, num_pages=0) -> Params:
    """With ``block_table`` (int32 [batch, table_stride]) k, v and k_idx are page pools
    ([num_pages, block, h, d] and [num_pages, block, d_idx]) and their strides are
    taken over (page, token in page, head)."""
    p = Params()
    p.batch, p.n_q, p.max_kv, p.H, p.h = batch, n_q, max_kv, H, h
    p.d, p.d_idx, p.block, p.topk = d, d_idx, block, topk
    p.causal, p.force_own_block = int(bool(causal)), int(bool(force_own_block))
    p.softmax_scale = float(softmax_scale)
    p.seq_lens = _ptr(seq_lens)
    if q is not None:
        p.q_strides[:] = _outer(q, 3)
    if k is not None:
        p.k_strides[:] = _outer(k, 3)
    if v is not None:
        p.v_strides[:] = _outer(v, 3)
    if q_idx is not None:
        p.qi_strides[:] = _outer(q_idx, 3)
    if k_idx is not None:
        p.ki_strides[:] = _outer(k_idx, 2)
    if out is not None:
        p.o_strides[:] = _outer(out, 3)
    if block_table is not None:
        p.block_table = _ptr(block_table)
        p.table_stride = block_table.stride(0)
        p.num_pages = int(num_pages)
    return p


class Workspace:
    """A device buffer for the library's workspace, grown on demand."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, STATUS_BYTES), dtype=torch.uint8, device=self.device)
            rc = load_library().msa_workspace_init(self.buf.data_ptr(), self.buf.numel(), _stream())
            if rc != MSA_OK:
                raise MsaError(rc, "msa_workspace_init")
        return self.buf


_default_ws: dict = {}


def _workspace(ws: Workspace | None, device) -> Workspace:
    if ws is not None:
        return ws
    key = torch.device(device).index
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def msa_workspace_size(params: Params, op: int) -> int:
    return int(load_library().msa_workspace_size(ctypes.byref(params), int(op)))


def msa_launch_count(params: Params, op: int) -> int:
    return int(load_library().msa_launch_count(ctypes.byref(params), int(op)))


def msa_get_device_status(workspace: Workspace | torch.Tensor, stream=None) -> int:
    buf = workspace.buf if isinstance(workspace, Workspace) else workspace
    return int(load_library().msa_get_device_status(buf.data_ptr(), _stream(stream)))


def msa_workspace_init(buf: torch.Tensor, stream=None) -> int:
    return int(load_library().msa_workspace_init(buf.data_ptr(), buf.numel(), _stream(stream)))


def msa_selftest_wait_timeout(buf: torch.Tensor, wait_ns: int, stream=None) -> int:
    return int(load_library().msa_selftest_wait_timeout(buf.data_ptr(), buf.numel(), int(wait_ns),
                                                        _stream(stream)))


def _check(rc: int, what: str):
    if rc != MSA_OK:
        raise MsaError(rc, what)


def _kv_extent(k, block_table, max_kv):
    """max_kv and the page count: the tensor's token axis, or for a page pool the
    caller's max_kv and the pool's first axis."""
    if block_table is None:
        return k.shape[1], 0
    if max_kv is None:
        raise ValueError("a paged KV cache needs max_kv")
    return int(max_kv), k.shape[0]


def msa_index_select(q_idx, k_idx, *, block, topk, causal=True, force_own_block=False,
                     seq_lens=None, return_scores=False, block_ids=None, block_scores=None,
                     block_table=None, max_kv=None, workspace: Workspace | None = None,
                     stream=None):
    """Stage 1: block ids int32 [b, n_q, h, topk] (and fp32 block scores if asked).
    With ``block_table``, ``k_idx`` is a page pool [num_pages, block, d_idx]."""
    b, n_q, h, d_idx = q_idx.shape
    max_kv, num_pages = _kv_extent(k_idx, block_table, max_kv)
    nblk = (max_kv + block - 1) // block
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=h, h=h, d=64, d_idx=d_idx, block=block,
                    topk=topk, causal=causal, force_own_block=force_own_block,
                    seq_lens=seq_lens, q_idx=q_idx, k_idx=k_idx, block_table=block_table,
                    num_pages=num_pages)
    dev = q_idx.device
    if block_ids is None:
        block_ids = torch.empty((b, n_q, h, topk), dtype=torch.int32, device=dev)
    if return_scores and block_scores is None:
        block_scores = torch.empty((b, n_q, h, nblk), dtype=torch.float32, device=dev)
    need = msa_workspace_size(p, MSA_OP_INDEX_SELECT)
    if need == 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_workspace_size")
    ws = _workspace(workspace, dev).get(need)
    _check(load_library().msa_index_select(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx),
                                           _ptr(block_ids), _ptr(block_scores), ws.data_ptr(),
                                           ws.numel(), _stream(stream)), "msa_index_select")
    return (block_ids, block_scores) if return_scores else block_ids


def msa_sparse_attn(q, k, v, block_ids, *, block, causal=True, seq_lens=None, softmax_scale=0.0,
                    return_lse=False, out=None, lse=None, block_table=None, max_kv=None,
                    workspace: Workspace | None = None, stream=None):
    """Stage 2: bf16 output [b, n_q, H, d] (and fp32 lse [b, n_q, H] if asked).
    With ``block_table``, ``k`` and ``v`` are page pools [num_pages, block, h, d]."""
    b, n_q, H, d = q.shape
    h = k.shape[2]
    max_kv, num_pages = _kv_extent(k, block_table, max_kv)
    topk = block_ids.shape[-1]
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((b, n_q, H), dtype=torch.float32, device=q.device)
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=H, h=h, d=d, d_idx=32, block=block,
                    topk=topk, causal=causal, softmax_scale=softmax_scale, seq_lens=seq_lens,
                    q=q, k=k, v=v, out=out, block_table=block_table, num_pages=num_pages)
    need = msa_workspace_size(p, MSA_OP_SPARSE_ATTN)
    if need == 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_workspace_size")
    ws = _workspace(workspace, q.device).get(need)
    _check(load_library().msa_sparse_attn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(block_ids), _ptr(out), _ptr(lse), ws.data_ptr(),
                                          ws.numel(), _stream(stream)), "msa_sparse_attn")
    return (out, lse) if return_lse else out


def msa_sparse_attn_noalloc(q, k, v, block_ids, *, block, causal=True, seq_lens=None,
                            softmax_scale=0.0, out=None, lse=None, stream=None):
    """Stage 2 without a workspace (the library's fixed device scratch holds the
    split-KV partials); for callers that cannot allocate device memory.  ``out``
    (and ``lse``, if wanted) should be preallocated by such callers."""
    b, n_q, H, d = q.shape
    max_kv, h = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=H, h=h, d=d, d_idx=32, block=block,
                    topk=block_ids.shape[-1], causal=causal, softmax_scale=softmax_scale,
                    seq_lens=seq_lens, q=q, k=k, v=v, out=out)
    _check(load_library().msa_sparse_attn_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                                  _ptr(block_ids), _ptr(out), _ptr(lse),
                                                  _stream(stream)), "msa_sparse_attn_noalloc")
    return out


def msa_append_kv(k, v, k_idx, k_new=None, v_new=None, k_idx_new=None, *, block,
                  seq_lens=None, block_table=None, max_kv=None,
                  workspace: Workspace | None = None, stream=None):
    """Writes the new tokens' rows into the cache: k_new / v_new [b, n_new, h, d] and
    k_idx_new [b, n_new, d_idx] (dense) go to positions L_b - n_new + t of k / v
    [b, max_kv, h, d] and k_idx [b, max_kv, d_idx] (or of the page pools, with
    ``block_table``).  Any of the new tensors may be None, and then its cache too
    (``k`` or ``v`` must be given for the shapes)."""
    ref = next(t for t in (k_new, v_new, k_idx_new) if t is not None)
    b, n_new = ref.shape[0], ref.shape[1]
    kv = k if k is not None else v
    h, d = kv.shape[2], kv.shape[3]
    max_kv, num_pages = _kv_extent(kv, block_table, max_kv)
    for t in (k_new, v_new, k_idx_new):
        if t is not None and not t.is_contiguous():
            raise ValueError("new rows must be dense")
    d_idx = k_idx.shape[-1] if k_idx is not None else 32
    p = make_params(batch=b, n_q=n_new, max_kv=max_kv, H=h, h=h, d=d, d_idx=d_idx,
                    block=block, topk=1, seq_lens=seq_lens, k=k, v=v, k_idx=k_idx,
                    block_table=block_table, num_pages=num_pages)
    need = msa_workspace_size(p, MSA_OP_APPEND_KV)
    if need == 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_workspace_size")
    ws = _workspace(workspace, kv.device).get(need)
    _check(load_library().msa_append_kv(ctypes.byref(p), _ptr(k_new), _ptr(v_new),
                                        _ptr(k_idx_new), _ptr(k), _ptr(v), _ptr(k_idx),
                                        ws.data_ptr(), ws.numel(), _stream(stream)),
           "msa_append_kv")


def msa_forward(q, k, v, q_idx, k_idx, *, block, topk, causal=True, force_own_block=False,
                seq_lens=None, softmax_scale=0.0, out=None, block_ids=None, block_scores=None,
                lse=None, return_ids=False, return_scores=False, return_lse=False,
                block_table=None, max_kv=None, workspace: Workspace | None = None, stream=None,
                params: Params | None = None):
    """Both stages; returns out, plus (ids, scores, lse) when asked, in that order.
    With ``block_table``, ``k``, ``v`` and ``k_idx`` are page pools."""
    b, n_q, H, d = q.shape
    h = k.shape[2]
    max_kv, num_pages = _kv_extent(k, block_table, max_kv)
    d_idx = q_idx.shape[-1]
    nblk = (max_kv + block - 1) // block
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if return_ids and block_ids is None:
        block_ids = torch.empty((b, n_q, h, topk), dtype=torch.int32, device=dev)
    if return_scores and block_scores is None:
        block_scores = torch.empty((b, n_q, h, nblk), dtype=torch.float32, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((b, n_q, H), dtype=torch.float32, device=dev)
    p = params or make_params(batch=b, n_q=n_q, max_kv=max_kv, H=H, h=h, d=d, d_idx=d_idx,
                              block=block, topk=topk, causal=causal,
                              force_own_block=force_own_block, softmax_scale=softmax_scale,
                              seq_lens=seq_lens, q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, out=out,
                              block_table=block_table, num_pages=num_pages)
    need = msa_workspace_size(p, MSA_OP_FORWARD)
    if need == 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_workspace_size")
    ws = _workspace(workspace, dev).get(need)
    _check(load_library().msa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx),
                                      _ptr(k_idx), _ptr(out), _ptr(block_ids), _ptr(block_scores),
                                      _ptr(lse), ws.data_ptr(), ws.numel(), _stream(stream)),
           "msa_forward")
    res = [out]
    if return_ids:
        res.append(block_ids)
    if return_scores:
        res.append(block_scores)
    if return_lse:
        res.append(lse)
    return res[0] if len(res) == 1 else tuple(res)


def msa_block_scores(q_idx, k_idx, *, block, causal=True, seq_lens=None, block_scores=None,
                     block_table=None, max_kv=None, workspace: Workspace | None = None,
                     stream=None):
    """Stage 1, first half: fp32 block scores [b, n_q, h, nblk] (-inf past the frontier)."""
    b, n_q, h, d_idx = q_idx.shape
    max_kv, num_pages = _kv_extent(k_idx, block_table, max_kv)
    nblk = (max_kv + block - 1) // block
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=h, h=h, d=64, d_idx=d_idx, block=block,
                    topk=1, causal=causal, seq_lens=seq_lens, q_idx=q_idx, k_idx=k_idx,
                    block_table=block_table, num_pages=num_pages)
    if block_scores is None:
        block_scores = torch.empty((b, n_q, h, nblk), dtype=torch.float32, device=q_idx.device)
    ws = _workspace(workspace, q_idx.device).get(msa_workspace_size(p, MSA_OP_BLOCK_SCORES))
    _check(load_library().msa_block_scores(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx),
                                           _ptr(block_scores), ws.data_ptr(), ws.numel(),
                                           _stream(stream)), "msa_block_scores")
    return block_scores


def msa_index_candidates(q_idx, k_idx, *, block, topk, causal=True, force_own_block=False,
                         seq_lens=None, block_ids=None, kept_scores=None, block_table=None,
                         max_kv=None, workspace: Workspace | None = None, stream=None):
    """msa_index_select plus the kept blocks' scores: (ids, scores), both [b, n_q, h, topk]."""
    b, n_q, h, d_idx = q_idx.shape
    max_kv, num_pages = _kv_extent(k_idx, block_table, max_kv)
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=h, h=h, d=64, d_idx=d_idx, block=block,
                    topk=topk, causal=causal, force_own_block=force_own_block,
                    seq_lens=seq_lens, q_idx=q_idx, k_idx=k_idx, block_table=block_table,
                    num_pages=num_pages)
    dev = q_idx.device
    if block_ids is None:
        block_ids = torch.empty((b, n_q, h, topk), dtype=torch.int32, device=dev)
    if kept_scores is None:
        kept_scores = torch.empty((b, n_q, h, topk), dtype=torch.float32, device=dev)
    need = msa_workspace_size(p, MSA_OP_INDEX_CANDIDATES)
    if need == 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_workspace_size")
    ws = _workspace(workspace, dev).get(need)
    _check(load_library().msa_index_candidates(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx),
                                               _ptr(block_ids), _ptr(kept_scores), ws.data_ptr(),
                                               ws.numel(), _stream(stream)),
           "msa_index_candidates")
    return block_ids, kept_scores


def msa_select_candidates(cand_scores, cand_ids, *, max_kv, block, topk, shard_blocks=0,
                          causal=True, force_own_block=False, seq_lens=None, block_base=0,
                          nblk_local=0, block_ids=None, local_ids=None, want_global=True,
                          want_local=False, workspace: Workspace | None = None, stream=None):
    """Global top-k from gathered candidate lists [nlists, b, n_q, h, len] (list r's ids
    local to the shard starting at block r * shard_blocks); returns the global ids and/or
    the ids local to the shard [block_base, block_base + nblk_local)."""
    nlists, b, n_q, h, llen = cand_ids.shape
    if not (cand_ids.is_contiguous() and cand_scores.is_contiguous()):
        raise ValueError("candidate lists must be dense")
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=h, h=h, d=64, d_idx=32, block=block,
                    topk=topk, causal=causal, force_own_block=force_own_block,
                    seq_lens=seq_lens)
    dev = cand_ids.device
    if want_global and block_ids is None:
        block_ids = torch.empty((b, n_q, h, topk), dtype=torch.int32, device=dev)
    if want_local and local_ids is None:
        local_ids = torch.empty((b, n_q, h, topk), dtype=torch.int32, device=dev)
    ws = _workspace(workspace, dev).get(msa_workspace_size(p, MSA_OP_SELECT_CANDIDATES))
    _check(load_library().msa_select_candidates(
        ctypes.byref(p), int(nlists), int(llen), int(shard_blocks), _ptr(cand_scores),
        _ptr(cand_ids), int(block_base), int(nblk_local),
        _ptr(block_ids if want_global else None), _ptr(local_ids if want_local else None),
        ws.data_ptr(), ws.numel(), _stream(stream)), "msa_select_candidates")
    return block_ids, local_ids


def msa_merge_partials(part_out, part_lse, *, out=None, lse=None, h=None, stream=None):
    """LSE merge of part_out bf16 [P, b, n_q, H, d] with part_lse fp32 [P, b, n_q, H].
    ``h`` (the KV heads) only has to make a valid head grouping of H."""
    P, b, n_q, H, d = part_out.shape
    if not (part_out.is_contiguous() and part_lse.is_contiguous()):
        raise ValueError("partials must be dense")
    if out is None:
        out = torch.empty((b, n_q, H, d), dtype=part_out.dtype, device=part_out.device)
    if h is None:
        h = next((c for c in range(1, 17) if H % c == 0 and H // c <= 16), 1)
    p = make_params(batch=b, n_q=n_q, max_kv=max(n_q, 1), H=H, h=h, d=d, d_idx=32, block=64,
                    topk=1, out=out)
    _check(load_library().msa_merge_partials(ctypes.byref(p), int(P), _ptr(part_out),
                                             _ptr(part_lse), _ptr(out), _ptr(lse),
                                             _stream(stream)), "msa_merge_partials")
    return out


def msa_shard_lengths(seq_lens, *, batch, max_kv, token_base, token_count, out=None,
                      workspace: Workspace | None = None, stream=None, device=None):
    """Per-sequence token counts inside the shard [token_base, token_base + token_count)."""
    dev = seq_lens.device if seq_lens is not None else torch.device(device or "cuda")
    if out is None:
        out = torch.empty((batch,), dtype=torch.int32, device=dev)
    p = make_params(batch=batch, n_q=1, max_kv=max_kv, H=1, h=1, d=64, d_idx=32, block=64,
                    topk=1, seq_lens=seq_lens)
    ws = _workspace(workspace, dev).get(msa_workspace_size(p, MSA_OP_SHARD_LENGTHS))
    _check(load_library().msa_shard_lengths(ctypes.byref(p), int(token_base), int(token_count),
                                            _ptr(out), ws.data_ptr(), ws.numel(),
                                            _stream(stream)), "msa_shard_lengths")
    return out


def msa_index_topk(q_idx, k_idx, *, block, topk, causal=True, force_own_block=False,
                   seq_lens=None, return_scores=False, block_ids=None, block_scores=None,
                   block_table=None, max_kv=None, workspace: Workspace | None = None,
                   stream=None):
    """Stage 1 for prefill in one kernel (the top-k kept in the index GEMM's epilogue):
    the ids of msa_index_select, and the block scores only if asked."""
    b, n_q, h, d_idx = q_idx.shape
    max_kv, num_pages = _kv_extent(k_idx, block_table, max_kv)
    nblk = (max_kv + block - 1) // block
    p = make_params(batch=b, n_q=n_q, max_kv=max_kv, H=h, h=h, d=64, d_idx=d_idx, block=block,
                    topk=topk, causal=causal, force_own_block=force_own_block,
                    seq_lens=seq_lens, q_idx=q_idx, k_idx=k_idx, block_table=block_table,
                    num_pages=num_pages)
    dev = q_idx.device
    if block_ids is None:
        block_ids = torch.empty((b, n_q, h, topk), dtype=torch.int32, device=dev)
    if return_scores and block_scores is None:
        block_scores = torch.empty((b, n_q, h, nblk), dtype=torch.float32, device=dev)
    ws = _workspace(workspace, dev).get(msa_workspace_size(p, MSA_OP_INDEX_TOPK))
    _check(load_library().msa_index_topk(ctypes.byref(p), _ptr(q_idx), _ptr(k_idx),
                                         _ptr(block_ids), _ptr(block_scores), ws.data_ptr(),
                                         ws.numel(), _stream(stream)), "msa_index_topk")
    return (block_ids, block_scores) if return_scores else block_ids

