"""Pins for the oracle's paged-cache gather (CPU only).

Logical key j of sequence b lives in page block_table[b][j // page_size], row
j % page_size ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1,
PagedAttention's logical-to-physical page table).
"""
import numpy as np
import pytest
import torch

import oracle


def _pool(seed, num_pages, H, P, d):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(num_pages, H, P, d, generator=g).to(torch.bfloat16)


def test_identity_table_is_a_reshape():
    """Pages laid out sequence after sequence with table[b][i] = b*pps + i: the
    logical cache is the pool reshaped [B, pps, H, P, d] -> [B, H, pps*P, d]."""
    B, H, P, pps, d = 3, 2, 16, 5, 64
    pool = _pool(1, B * pps, H, P, d)
    table = torch.arange(B * pps, dtype=torch.int32).view(B, pps)
    got = oracle.paged_gather(pool, table)
    want = pool.view(B, pps, H, P, d).permute(0, 2, 1, 3, 4).reshape(B, H, pps * P, d)
    assert torch.equal(got.view(torch.int16), want.contiguous().view(torch.int16))


def test_permuting_the_pool_with_the_table_changes_nothing():
    B, H, P, pps, d = 2, 3, 32, 4, 128
    n = 11
    pool = _pool(2, n, H, P, d)
    rng = np.random.default_rng(3)
    table = torch.from_numpy(rng.choice(n, size=(B, pps), replace=False).astype(np.int32))
    perm = rng.permutation(n)
    inv = np.argsort(perm)
    pool2 = pool[torch.from_numpy(perm)]                  # page i of pool2 = page perm[i] of pool
    table2 = torch.from_numpy(inv[table.numpy()].astype(np.int32))
    a = oracle.paged_gather(pool, table)
    b = oracle.paged_gather(pool2, table2)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_key_lookup_by_hand():
    """Element check: logical key j of (b, h) equals pool[table[b][j//P], h, j%P]."""
    B, H, P, pps, d = 2, 2, 16, 3, 64
    pool = _pool(4, 7, H, P, d)
    table = torch.tensor([[6, 0, 3], [2, 2, 5]], dtype=torch.int32)
    got = oracle.paged_gather(pool, table)
    for b in range(B):
        for h in range(H):
            for j in (0, 1, 15, 16, 31, 40, 47):
                assert torch.equal(got[b, h, j].view(torch.int16),
                                   pool[table[b, j // P], h, j % P].view(torch.int16))


def test_bad_page_id_is_rejected():
    pool = _pool(5, 4, 1, 16, 64)
    with pytest.raises(ValueError):
        oracle.paged_gather(pool, torch.tensor([[0, 4]], dtype=torch.int32))
