"""Pins of the oracle's score modifiers on the split-KV decode shape: per-sequence
key counts kv_lens with ALiBi or the relative-position table.

The modifier ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1:
score_mod(score, b, h, q_idx, kv_idx), with ALiBi, a position bias and a
learnable bias as examples) takes the query row's absolute position p; on the
decode shape row i of sequence b sits at p = kv_lens[b] - Lq + i and sees the
keys [0, kv_lens[b]).  Each pin builds the expected values without the
oracle's code: closed forms when Q = 0 (the scores are the bias alone), and
PyTorch's float64 SDPA with the bias and the key padding as an additive mask.
"""
import numpy as np
import torch

import oracle
from workloads import random_case


def _onehot_v(B, H, L, d):
    v = torch.zeros(B, H, L, d)
    v[:, :, torch.arange(L), torch.arange(L)] = 1.0  # key j -> column j (L <= d)
    return v.to(torch.bfloat16)


def test_alibi_with_kv_lens_closed_form():
    """Q = 0: row i of sequence b weighs key j < kv_lens[b] by exp(slope (j - p)),
    p = kv_lens[b] - Lq + i, so LSE = log sum_j exp(slope (j - p)) and, with V the
    one-hot columns, O[j] is that weight over the sum."""
    B, Hq, Hkv, Lq, L, d = 3, 2, 1, 4, 60, 64
    kv = torch.tensor([60, 17, 5], dtype=torch.int32)
    slopes = np.array([0.25, 0.03125])
    q = torch.zeros(B, Hq, Lq, d, dtype=torch.bfloat16)
    k = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    o, lse = oracle.attn_fwd(q, k, _onehot_v(B, Hkv, L, d), kv_lens=kv, alibi_slopes=slopes)
    for b in range(B):
        n = int(kv[b])
        for h, sl in enumerate(slopes):
            for i in range(Lq):
                p = n - Lq + i
                z = sl * (np.arange(n) - p)
                np.testing.assert_allclose(lse[b, h, i], np.log(np.exp(z).sum()), atol=1e-12)
                want = np.zeros(d)
                want[:n] = np.exp(z) / np.exp(z).sum()
                np.testing.assert_allclose(o[b, h, i], want, atol=1e-12)


def test_rel_bias_with_kv_lens_closed_form():
    """Q = 0: the scores are table[h, clamp(j - p, -R, R) + R] over j < kv_lens[b]."""
    B, Hq, Hkv, Lq, L, d, R = 2, 4, 2, 3, 50, 64, 7
    kv = torch.tensor([9, 50], dtype=torch.int32)
    table = np.random.default_rng(3).standard_normal((Hq, 2 * R + 1)) * 2.0
    q = torch.zeros(B, Hq, Lq, d, dtype=torch.bfloat16)
    k = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    o, lse = oracle.attn_fwd(q, k, _onehot_v(B, Hkv, L, d), kv_lens=kv, rel_bias=(table, R))
    for b in range(B):
        n = int(kv[b])
        for h in range(Hq):
            for i in range(Lq):
                p = n - Lq + i
                z = table[h, np.clip(np.arange(n) - p, -R, R) + R]
                np.testing.assert_allclose(lse[b, h, i], np.log(np.exp(z).sum()), atol=1e-12)
                np.testing.assert_allclose(o[b, h, i, :n], np.exp(z) / np.exp(z).sum(),
                                           atol=1e-12)


def _sdpa_f64(q, k, v, bias, scale):
    """float64 SDPA with an additive [B, Hq, Lq, Lk] bias (-inf = masked); GQA by
    repeating the KV heads.  Returns O and LSE (natural log)."""
    Hq, Hkv = q.shape[1], k.shape[1]
    k = k.double().repeat_interleave(Hq // Hkv, dim=1)
    v = v.double().repeat_interleave(Hq // Hkv, dim=1)
    q = q.double()
    s = torch.einsum("bhid,bhjd->bhij", q, k) * scale + bias
    lse = torch.logsumexp(s, dim=-1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=bias, scale=scale)
    return o.numpy(), lse.numpy()


def _padded_bias(kv, Hq, Lq, L, per_key):
    """[B, Hq, Lq, L]: per_key(h, j - p) for j < kv[b], -inf beyond."""
    B = len(kv)
    out = np.full((B, Hq, Lq, L), -np.inf)
    for b in range(B):
        n = int(kv[b])
        p = n - Lq + np.arange(Lq)
        dj = np.arange(n)[None, :] - p[:, None]
        for h in range(Hq):
            out[b, h, :, :n] = per_key(h, dj)
    return torch.from_numpy(out)


def test_alibi_with_kv_lens_equals_float64_sdpa():
    B, Hq, Hkv, Lq, L, d = 3, 8, 2, 16, 300, 64
    q, k, v, _, kv = random_case(11, B, Hq, Hkv, Lq, L, d, kv_len_range=(1, L))
    slopes = 2.0 ** (-np.arange(1, Hq + 1))
    scale = 0.125
    o, lse = oracle.attn_fwd(q, k, v, kv_lens=kv, alibi_slopes=slopes, scale=scale)
    bias = _padded_bias(kv.numpy(), Hq, Lq, L, lambda h, dj: slopes[h] * dj)
    want_o, want_lse = _sdpa_f64(q, k, v, bias, scale)
    np.testing.assert_allclose(lse, want_lse, atol=1e-10)
    np.testing.assert_allclose(o, want_o, atol=1e-10)


def test_rel_bias_with_kv_lens_equals_float64_sdpa():
    B, Hq, Hkv, Lq, L, d, R = 2, 4, 4, 5, 400, 128, 64
    q, k, v, _, kv = random_case(12, B, Hq, Hkv, Lq, L, d, kv_len_range=(100, L))
    table = np.random.default_rng(5).standard_normal((Hq, 2 * R + 1))
    o, lse = oracle.attn_fwd(q, k, v, kv_lens=kv, rel_bias=(table, R))
    bias = _padded_bias(kv.numpy(), Hq, Lq, L,
                        lambda h, dj: table[h, np.clip(dj, -R, R) + R])
    want_o, want_lse = _sdpa_f64(q, k, v, bias, 1.0 / np.sqrt(d))
    np.testing.assert_allclose(lse, want_lse, atol=1e-10)
    np.testing.assert_allclose(o, want_o, atol=1e-10)


def test_full_kv_lens_match_the_dense_entries():
    """kv_lens = Lk for every sequence: the same bits as the score-modifier
    entries without kv_lens (p = Lk - Lq + i in both)."""
    B, Hq, Hkv, Lq, L, d, R = 2, 4, 2, 6, 90, 64, 5
    q, k, v, _, _ = random_case(13, B, Hq, Hkv, Lq, L, d)
    kv = torch.full((B,), L, dtype=torch.int32)
    slopes = [0.5, 0.25, 0.125, 0.0625]
    a = oracle.attn_fwd(q, k, v, kv_lens=kv, alibi_slopes=slopes)
    b = oracle.attn_fwd(q, k, v, alibi_slopes=slopes)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    table = np.random.default_rng(7).standard_normal((Hq, 2 * R + 1))
    a = oracle.attn_fwd(q, k, v, kv_lens=kv, rel_bias=(table, R))
    b = oracle.attn_fwd(q, k, v, rel_bias=(table, R))
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
