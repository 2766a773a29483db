"""Agreement rules between the CUDA path and the float64 oracle.

Stage 1 (selection): block ids must be bit-exact, except on rows where the
oracle's last kept and first dropped candidates differ by less than 1e-3
relative; on those rows the GPU ids must be a valid top-k of the GPU's own fp32
block scores.  Block scores must match the oracle within 1e-3 relative, taken
relative to max(|S|, 1) (an fp32 sum of d_idx products carries an absolute
rounding error, so a score near zero is compared absolutely), with -inf matching
-inf.
Stage 2 (attention, same ids on both sides): max-abs error <= 2e-2 and
mean-abs error <= 2e-3 on the bf16 output; the log-sum-exp within 2e-3.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle

SCORE_RTOL = 1e-3
TIE_RTOL = 1e-3
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_ABS = 2e-3


def oracle_cfg(p) -> oracle.Config:
    return oracle.Config(p.batch, p.n_q, p.max_kv, p.H, p.h, p.d, p.d_idx, p.block, p.topk,
                         causal=p.causal, force_own=p.force_own)


def frontier(p, L, pos):
    nb = (L + p.block - 1) // p.block
    if not p.causal:
        return nb
    if pos < 0:
        return 0
    return min(nb, pos // p.block + 1)


def row_geometry(p, seq_lens, b, t):
    L = int(seq_lens[b]) if seq_lens is not None else p.max_kv
    pos = L - p.n_q + t
    F = frontier(p, L, pos)
    own = pos // p.block if (p.force_own and 0 <= pos and pos // p.block < F) else None
    return L, pos, F, own


def is_near_tie(scores_row, F, k, own):
    cands = [c for c in range(F) if c != own]
    kk = min(k, F) - (1 if own is not None else 0)
    if kk <= 0 or len(cands) <= kk:
        return False
    vals = np.sort(np.asarray([scores_row[c] for c in cands]))[::-1]
    a, b = vals[kk - 1], vals[kk]
    return (a - b) / max(abs(a), abs(b), 1e-6) < TIE_RTOL


def valid_topk(ids_row, scores_row, F, k, own):
    """ids form a valid top-k of scores: right count, ascending, -1 padded, in
    the frontier, own present when forced, and every kept score >= every dropped one."""
    m = min(k, F)
    kept = [int(x) for x in ids_row[:m]]
    if any(x < 0 or x >= F for x in kept) or any(int(x) != -1 for x in ids_row[m:]):
        return False
    if any(kept[i] >= kept[i + 1] for i in range(len(kept) - 1)):
        return False
    if own is not None and own not in kept:
        return False
    rest = [x for x in kept if x != own]
    dropped = [c for c in range(F) if c not in set(kept)]
    if not rest or not dropped:
        return True
    return min(scores_row[x] for x in rest) >= max(scores_row[x] for x in dropped)


def check_scores(gpu_scores, ora_scores, F_rows):
    """gpu/ora: [nrows, h, nblk]; only blocks before each row's frontier are compared
    numerically, later ones must be -inf on both sides where exposed."""
    g = np.asarray(gpu_scores, dtype=np.float64)
    o = np.asarray(ora_scores, dtype=np.float64)
    worst = 0.0
    for i, F in enumerate(F_rows):
        gi, oi = g[i, :, :F], o[i, :, :F]
        fin = np.isfinite(oi)
        assert np.array_equal(fin, np.isfinite(gi)), "finite pattern differs in row %d" % i
        if fin.any():
            err = np.abs(gi[fin] - oi[fin]) / np.maximum(np.abs(oi[fin]), 1.0)
            worst = max(worst, float(err.max()))
        assert np.all(np.isneginf(g[i, :, F:])), "row %d: blocks past the frontier not -inf" % i
    assert worst <= SCORE_RTOL, "block score relative error %g" % worst
    return worst


def check_ids(p, rows, seq_lens, gpu_ids, ora_ids, ora_scores, gpu_scores=None):
    """Returns (n_rows_checked, n_near_tie_rows)."""
    gi = np.asarray(gpu_ids)
    oi = np.asarray(ora_ids)
    near = 0
    for i, (b, t) in enumerate(rows):
        L, pos, F, own = row_geometry(p, seq_lens, b, t)
        for g in range(p.h):
            if np.array_equal(gi[i, g], oi[i, g]):
                continue
            assert is_near_tie(ora_scores[i, g], F, p.topk, own), \
                "ids differ on a row that is not a near tie: b=%d t=%d g=%d" % (b, t, g)
            assert gpu_scores is not None, "near-tie row needs the GPU scores"
            assert valid_topk(gi[i, g], gpu_scores[i, g], F, p.topk, own), \
                "GPU ids are not a valid top-k of the GPU scores: b=%d t=%d g=%d" % (b, t, g)
            near += 1
    return len(rows), near


def check_attn(gpu_out, gpu_lse, ora_out, ora_lse):
    go = np.asarray(gpu_out, dtype=np.float64)
    oo = np.asarray(ora_out, dtype=np.float64)
    err = np.abs(go - oo)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    assert max_abs <= OUT_MAX_ABS, "max-abs %g" % max_abs
    assert mean_abs <= OUT_MEAN_ABS, "mean-abs %g" % mean_abs
    if gpu_lse is not None:
        gl = np.asarray(gpu_lse, dtype=np.float64)
        ol = np.asarray(ora_lse, dtype=np.float64)
        assert np.array_equal(np.isneginf(gl), np.isneginf(ol))
        fin = np.isfinite(ol)
        if fin.any():
            lerr = float(np.abs(gl[fin] - ol[fin]).max())
            assert lerr <= LSE_ABS, "lse error %g" % lerr
    return max_abs, mean_abs


def take_rows(t: torch.Tensor, rows) -> np.ndarray:
    """t: [b, n_q, ...] device tensor -> host array [nrows, ...] for the (b, t) rows."""
    rb = torch.as_tensor([r[0] for r in rows], device=t.device, dtype=torch.long)
    rt = torch.as_tensor([r[1] for r in rows], device=t.device, dtype=torch.long)
    return t[rb, rt].cpu().numpy()


def sample_rows(p, n_rows: int, seed: int = 0):
    """Query rows for sampled checks: the first blocks, partial own blocks, the
    last queries and random ones, over every sequence."""
    rng = np.random.default_rng(seed)
    rows = set()
    B = p.block
    for b in range(p.batch):
        for t in (0, 1, B - 1, B, B + 1, 2 * B + 3, p.n_q // 2, p.n_q - 1, p.n_q - 2, p.n_q - B):
            if 0 <= t < p.n_q:
                rows.add((b, t))
        for t in range(max(0, p.n_q - 8), p.n_q):
            rows.add((b, t))
    while len(rows) < n_rows:
        rows.add((int(rng.integers(p.batch)), int(rng.integers(p.n_q))))
    return sorted(rows)


def kv_chunk_rows(p) -> int:
    """Query rows (flattened (b, t)) per chunk of the KV-major prefill attention.

    Restates the library's chunk plan: a chunk's partial tiles and per-slot
    records must fit a 6 GiB budget, next to one spare tile per (sequence,
    group, block) list; chunk-relative slot positions stay below 2^30.  A CPU
    test checks the resulting chunk count against msa_launch_count.
    """
    rows = p.batch * p.n_q
    row_bytes = 2 * p.d
    nj = p.batch * p.h * p.nblk
    qpt = 128 // p.G
    fixed = (nj + 1) * 128 * row_bytes
    per_bt = p.h * p.topk * (12 + p.G * 4 + (128 * row_bytes) // qpt + 1)
    budget = 6 << 30
    cr = (budget - fixed) // per_bt if fixed < budget else 1
    cr = max(cr, 1)
    if cr * p.h * p.topk > (1 << 30):
        cr = (1 << 30) // (p.h * p.topk)
    return min(cr, rows)


def sample_rows_chunked(p, n_rows: int, seed: int = 0, per_chunk_min: int = 64):
    """Query rows for sampled prefill checks, stratified over the KV-major query
    chunks: every chunk gets its first and last query, at least ``per_chunk_min``
    rows and an equal share of ``n_rows``; the special rows of ``sample_rows``
    (first blocks, partial own blocks, the last queries) are always included."""
    rng = np.random.default_rng(seed)
    rows = set(sample_rows(p, 0, seed))
    total = p.batch * p.n_q
    cr = kv_chunk_rows(p)
    nch = (total + cr - 1) // cr
    share = max(per_chunk_min, (n_rows - len(rows)) // nch)
    for c in range(nch):
        lo, hi = c * cr, min(total, (c + 1) * cr)
        chosen = {lo, hi - 1}
        want = min(share, hi - lo)
        while len(chosen) < want:
            chosen.add(int(rng.integers(lo, hi)))
        for bt in chosen:
            rows.add((bt // p.n_q, bt % p.n_q))
    return sorted(rows)


def page_pools(x, prob, spare: int = 5, seed: int = 0):
    """Scatters the contiguous k, v and k_idx of ``x`` into shuffled page pools of
    one block per page (plus ``spare`` unused pages of noise) on the tensors'
    device; returns (pools, block table int32 [batch, nblk])."""
    B, nb = prob.block, (prob.max_kv + prob.block - 1) // prob.block
    n_pages = prob.batch * nb + spare
    dev = x["k"].device
    g = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)
    table = perm[:prob.batch * nb].view(prob.batch, nb).to(torch.int32).to(dev)
    unused = perm[prob.batch * nb:].to(dev)
    gd = torch.Generator(device=dev).manual_seed(seed + 1)
    pools = {}
    for name in ("k", "v", "k_idx"):
        t = x[name]
        tail = tuple(t.shape[2:])
        pool = torch.empty((n_pages, B) + tail, dtype=t.dtype, device=dev)
        if spare:
            pool[unused] = torch.randn((spare, B) + tail, generator=gd, device=dev).to(t.dtype)
        for b in range(prob.batch):  # one sequence at a time bounds the staging memory
            padded = torch.zeros((nb * B,) + tail, dtype=t.dtype, device=dev)
            padded[:t.shape[1]] = t[b]
            pool[table[b].long()] = padded.view((nb, B) + tail)
            del padded
        pools[name] = pool
    return pools, table
