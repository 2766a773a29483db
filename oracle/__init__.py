"""MSA oracle: float64 CPU statement of MiniMax Sparse Attention.

TEST INFRASTRUCTURE ONLY.  The library's product path never imports this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may use it.  It shares no code with the CUDA library.

The arithmetic lives in ``msa_oracle.cpp`` (plain loops, float64, OpenMP over
rows); this module builds it with the host C++ compiler and wraps it with
ctypes.  Inputs are host arrays: bf16 tensors travel as their raw uint16 bits
and are widened to float64 exactly inside the C++ code.

Sources: "MiniMax goes sparse" (atlascloud.ai) section 1, steps 1 and 2, and
"MiniMax M3 的 MSA 与阶跃 Step 3.7 Flash 的 MFA" (ai.air7.fun), section
"MSA：稀疏注意力的一种极简实现".  Parity status: every function is pinned by
the CPU tests in ``tests/test_oracle.py``; none is unpinned.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.cpp")
_LIB = os.path.join(_HERE, "libmsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmsa_oracle.so`` (g++, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["g++", "-std=c++17", "-O2", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_q", "max_kv", "H", "h", "d", "d_idx", "block", "topk", "causal",
        "force_own")] + [("scale", ctypes.c_double)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            for name, argt in {
                "oracle_block_scores": [P, P, P, P, I, P, P, P],
                "oracle_select": [P, P, P, I, P, P, P],
                "oracle_sparse_attn": [P, P, P, P, P, I, P, P, P, P, P],
                "oracle_dense_attn": [P, P, P, P, P, I, P, P, P, P],
                "oracle_forward": [P, P, P, P, P, P, P, I, P, P, P, P, P],
            }.items():
                fn = getattr(lib, name)
                fn.argtypes = argt
                fn.restype = I
            lib.oracle_num_threads.restype = I
            _lib = lib
    return _lib


@dataclass
class Config:
    """Shapes and flags of one MSA problem (the oracle's own copy)."""

    batch: int
    n_q: int
    max_kv: int
    H: int
    h: int
    d: int
    d_idx: int
    block: int
    topk: int
    causal: bool = True
    force_own: bool = False
    scale: float = 0.0  # 0 => 1/sqrt(d)

    @property
    def nblk(self) -> int:
        return (self.max_kv + self.block - 1) // self.block

    def _c(self) -> _Cfg:
        return _Cfg(self.batch, self.n_q, self.max_kv, self.H, self.h, self.d, self.d_idx,
                    self.block, self.topk, int(bool(self.causal)), int(bool(self.force_own)),
                    float(self.scale))


def _u16(a) -> np.ndarray:
    """Host bf16 data as a contiguous uint16 array (accepts torch or numpy)."""
    if hasattr(a, "detach"):
        import torch
        a = a.detach()
        if a.dtype == torch.bfloat16:
            a = a.contiguous().cpu().view(torch.int16)
        a = a.numpy()
    a = np.ascontiguousarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("oracle expects bf16 bits (uint16), got %s" % a.dtype)
    return a


def _i32(a) -> np.ndarray | None:
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _rows(cfg: Config, rows):
    """Rows are (b, t) pairs; None means every row of the problem."""
    if rows is None:
        bb, tt = np.meshgrid(np.arange(cfg.batch), np.arange(cfg.n_q), indexing="ij")
        rows = np.stack([bb.ravel(), tt.ravel()], axis=1)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
    return rows, np.ascontiguousarray(rows[:, 0]), np.ascontiguousarray(rows[:, 1])


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def block_scores(cfg: Config, q_idx, k_idx, seq_lens=None, rows=None) -> np.ndarray:
    """Block-max-pooled index scores, float64 [nrows, h, nblk]; -inf past the frontier."""
    lib = _load()
    rows, rb, rt = _rows(cfg, rows)
    qi, ki, sl = _u16(q_idx), _u16(k_idx), _i32(seq_lens)
    out = np.empty((len(rows), cfg.h, cfg.nblk), dtype=np.float64)
    c = cfg._c()
    lib.oracle_block_scores(ctypes.byref(c), _p(sl), _p(qi), _p(ki), len(rows), _p(rb), _p(rt),
                            _p(out))
    return out


def select(cfg: Config, scores: np.ndarray, seq_lens=None, rows=None) -> np.ndarray:
    """Top-k block ids, int32 [nrows, h, topk], ascending with -1 padding."""
    lib = _load()
    rows, rb, rt = _rows(cfg, rows)
    s = np.ascontiguousarray(scores, dtype=np.float64)
    assert s.shape == (len(rows), cfg.h, cfg.nblk), s.shape
    sl = _i32(seq_lens)
    ids = np.empty((len(rows), cfg.h, cfg.topk), dtype=np.int32)
    c = cfg._c()
    lib.oracle_select(ctypes.byref(c), _p(sl), _p(s), len(rows), _p(rb), _p(rt), _p(ids))
    return ids


def sparse_attn(cfg: Config, q, k, v, ids, seq_lens=None, rows=None):
    """Sparse-branch attention on given ids: (out float64 [nrows, H, d], lse [nrows, H])."""
    lib = _load()
    rows, rb, rt = _rows(cfg, rows)
    qq, kk, vv, sl = _u16(q), _u16(k), _u16(v), _i32(seq_lens)
    ii = _i32(ids)
    assert ii.shape == (len(rows), cfg.h, cfg.topk), ii.shape
    out = np.empty((len(rows), cfg.H, cfg.d), dtype=np.float64)
    lse = np.empty((len(rows), cfg.H), dtype=np.float64)
    c = cfg._c()
    lib.oracle_sparse_attn(ctypes.byref(c), _p(sl), _p(qq), _p(kk), _p(vv), len(rows), _p(rb),
                           _p(rt), _p(ii), _p(out), _p(lse))
    return out, lse


def dense_attn(cfg: Config, q, k, v, seq_lens=None, rows=None):
    """Textbook (causal) GQA softmax attention: (out [nrows, H, d], lse [nrows, H])."""
    lib = _load()
    rows, rb, rt = _rows(cfg, rows)
    qq, kk, vv, sl = _u16(q), _u16(k), _u16(v), _i32(seq_lens)
    out = np.empty((len(rows), cfg.H, cfg.d), dtype=np.float64)
    lse = np.empty((len(rows), cfg.H), dtype=np.float64)
    c = cfg._c()
    lib.oracle_dense_attn(ctypes.byref(c), _p(sl), _p(qq), _p(kk), _p(vv), len(rows), _p(rb),
                          _p(rt), _p(out), _p(lse))
    return out, lse


def forward(cfg: Config, q, k, v, q_idx, k_idx, seq_lens=None, rows=None):
    """Both stages for the given rows: (ids, out, lse)."""
    lib = _load()
    rows, rb, rt = _rows(cfg, rows)
    qq, kk, vv = _u16(q), _u16(k), _u16(v)
    qi, ki, sl = _u16(q_idx), _u16(k_idx), _i32(seq_lens)
    ids = np.empty((len(rows), cfg.h, cfg.topk), dtype=np.int32)
    out = np.empty((len(rows), cfg.H, cfg.d), dtype=np.float64)
    lse = np.empty((len(rows), cfg.H), dtype=np.float64)
    c = cfg._c()
    lib.oracle_forward(ctypes.byref(c), _p(sl), _p(qq), _p(kk), _p(vv), _p(qi), _p(ki), len(rows),
                       _p(rb), _p(rt), _p(ids), _p(out), _p(lse))
    return ids, out, lse
