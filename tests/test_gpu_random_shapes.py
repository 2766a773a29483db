"""Seeded random shapes through every stage against the float64 oracle.

Decode and short prefill problems drawn from the supported space (G = 1..16,
d 64/128, d_idx 32/64/128, block 16..128, top-k up to the block count, variable
lengths, forced own block, causal or not, contiguous or paged cache), each checked
on every row by the same harness as the fixed cases.  The draw is seeded, so a
failure names a shape that can be rerun.
"""

import random

import pytest

from block_sparse_gqa_03_b200.inputs import Problem
from test_gpu_parity import run_and_check

pytestmark = pytest.mark.gpu


def draw(i):
    r = random.Random(7000 + i)
    h = r.choice([1, 2, 4, 8])
    G = r.choice([1, 2, 3, 4, 5, 6, 7, 8, 16]) if h <= 4 else r.choice([1, 2, 3, 4, 6, 8])
    d = r.choice([64, 128])
    d_idx = r.choice([32, 64, 128])
    block = r.choice([16, 32, 64, 128])
    decode = r.random() < 0.6
    batch = r.randint(1, 6)
    if decode:
        max_kv = r.randint(block, 40 * block)
        n_q = 1
    else:
        max_kv = r.randint(block, 12 * block)
        n_q = r.randint(1, max_kv)
    nblk = -(-max_kv // block)
    topk = r.randint(1, max(1, min(nblk, 96)))
    causal = decode or r.random() < 0.8
    lens = (max(n_q, 1) if not decode else 0, max_kv) if r.random() < 0.5 else None
    # keep the float64 oracle to a few seconds: attention and index-score work
    while (batch * n_q * (h * G * topk * block * d + h * max_kv * d_idx) > 4e8 and
           (batch > 1 or n_q > 1 or topk > 1)):
        if batch > 1:
            batch -= 1
        elif n_q > 1:
            n_q = max(1, n_q // 2)
        else:
            topk = max(1, topk // 2)
    return Problem("rand%d" % i, batch=batch, n_q=n_q, max_kv=max_kv, H=h * G, h=h, d=d,
                   d_idx=d_idx, block=block, topk=topk, causal=causal,
                   force_own=causal and r.random() < 0.3, seed=7100 + i, len_range=lens), \
        r.random() < 0.25


CASES = [draw(i) for i in range(40)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s%s" % (c[0].name, "_paged" if c[1] else ""))
def test_random_shape_all_rows(case):
    prob, paged = case
    run_and_check(prob, tail_fill=float("nan") if prob.len_range else None, paged=paged)
