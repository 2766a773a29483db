"""Decode-step cache write through the C ABI: the new tokens' K, V and K_idx rows
land at positions L_b - n_new + t of the contiguous cache or of the pages the
block table names, and nothing else changes.  The expected caches are built with
plain PyTorch indexing (the operation is a copy: bit-exact)."""

import pytest
import torch

from block_sparse_gqa_03_b200 import msa

pytestmark = pytest.mark.gpu


def rnd(*shape, g):
    return torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)


def setup(batch, max_kv, h, d, d_idx, n_new, seed, lens=None):
    g = torch.Generator(device="cuda").manual_seed(seed)
    k, v, ki = rnd(batch, max_kv, h, d, g=g), rnd(batch, max_kv, h, d, g=g), rnd(batch, max_kv, d_idx, g=g)
    kn, vn, kin = rnd(batch, n_new, h, d, g=g), rnd(batch, n_new, h, d, g=g), rnd(batch, n_new, d_idx, g=g)
    sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    return k, v, ki, kn, vn, kin, sl


@pytest.mark.parametrize("n_new,d,d_idx,varlen", [(1, 128, 128, True), (3, 64, 32, True),
                                                  (2, 128, 64, False)])
def test_append_contiguous(n_new, d, d_idx, varlen):
    batch, max_kv, h = 4, 700, 8
    lens = [700, 5, 333, 64] if varlen else None
    k, v, ki, kn, vn, kin, sl = setup(batch, max_kv, h, d, d_idx, n_new, seed=11, lens=lens)
    ek, ev, eki = k.clone(), v.clone(), ki.clone()
    for b in range(batch):
        L = lens[b] if varlen else max_kv
        for t in range(n_new):
            ek[b, L - n_new + t] = kn[b, t]
            ev[b, L - n_new + t] = vn[b, t]
            eki[b, L - n_new + t] = kin[b, t]
    ws = msa.Workspace("cuda")
    msa.msa_append_kv(k, v, ki, kn, vn, kin, block=64, seq_lens=sl, workspace=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_OK
    assert torch.equal(k, ek) and torch.equal(v, ev) and torch.equal(ki, eki)


def test_append_only_index_keys():
    k, v, ki, kn, vn, kin, sl = setup(2, 256, 8, 128, 128, 1, seed=12, lens=[256, 100])
    ek, ev, eki = k.clone(), v.clone(), ki.clone()
    eki[0, 255], eki[1, 99] = kin[0, 0], kin[1, 0]
    msa.msa_append_kv(k, v, ki, None, None, kin, block=64, seq_lens=sl)
    torch.cuda.synchronize()
    assert torch.equal(k, ek) and torch.equal(v, ev) and torch.equal(ki, eki)


def paged(x, block, table):
    """[batch, max_kv, ...] -> page pool with the given table (pages of `block` tokens)."""
    batch, max_kv = x.shape[:2]
    nb = max_kv // block
    pool = torch.zeros((int(table.max()) + 3, block) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    pool[table.long().view(-1)] = x.view((batch * nb, block) + tuple(x.shape[2:]))
    return pool


def test_append_paged_matches_contiguous():
    batch, max_kv, h, d, d_idx, block, n_new = 3, 512, 8, 128, 128, 64, 2
    lens = [512, 130, 65]
    k, v, ki, kn, vn, kin, sl = setup(batch, max_kv, h, d, d_idx, n_new, seed=13, lens=lens)
    g = torch.Generator(device="cpu").manual_seed(3)
    nb = max_kv // block
    table = torch.randperm(batch * nb + 4, generator=g)[:batch * nb].view(batch, nb).to(torch.int32).cuda()
    pk, pv, pki = paged(k, block, table), paged(v, block, table), paged(ki, block, table)
    msa.msa_append_kv(k, v, ki, kn, vn, kin, block=block, seq_lens=sl)
    msa.msa_append_kv(pk, pv, pki, kn, vn, kin, block=block, seq_lens=sl, block_table=table,
                      max_kv=max_kv)
    torch.cuda.synchronize()
    idx = table.long().view(-1)
    for pool, ref in ((pk, k), (pv, v), (pki, ki)):
        assert torch.equal(pool[idx].reshape(ref.shape), ref)


def test_append_bad_inputs_flagged():
    batch, max_kv, h, d, block = 2, 256, 8, 128, 64
    k, v, ki, kn, vn, kin, sl = setup(batch, max_kv, h, d, 128, 2, seed=14, lens=[1, 256])
    ek = k.clone()
    ws = msa.Workspace("cuda")
    # sequence 0 holds one token but two are appended: position -1 is not written
    msa.msa_append_kv(k, v, ki, kn, vn, kin, block=block, seq_lens=sl, workspace=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_ASSERT
    ek[0, 0] = kn[0, 1]
    ek[1, 254:256] = kn[1]
    assert torch.equal(k, ek)
    # a page outside the pool is recorded, not written
    table = torch.arange(batch * (max_kv // block), dtype=torch.int32, device="cuda").view(batch, -1)
    pk = paged(k, block, table)
    before = pk.clone()
    bad = table.clone()
    bad[1, -1] = 10_000
    sl2 = torch.tensor([256, 256], dtype=torch.int32, device="cuda")
    msa.msa_append_kv(pk, None, None, kn, None, None, block=block, seq_lens=sl2, block_table=bad,
                      max_kv=max_kv, workspace=ws)
    assert msa.msa_get_device_status(ws) == msa.MSA_ERR_DEVICE_ASSERT
    assert torch.equal(pk[int(table[1, -1])], before[int(table[1, -1])])  # sequence 1 not
    assert not torch.equal(pk[int(bad[0, -1])], before[int(bad[0, -1])])  # sequence 0 written
