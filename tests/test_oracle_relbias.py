"""Pins of the oracle's relative-position bias score modifier.

The modifier ("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1:
score_mod(score, b, h, q_idx, kv_idx) with a position bias or a learnable
bias as examples) adds table[h, clamp(j - p, -R, R) + R] to the scaled score
of query row i (absolute position p = Lk - Lq + i) and key j.  Each pin below
builds what the oracle should give without the oracle's code: a closed form
when the scores are the bias alone, PyTorch's float64 SDPA with the bias as an
additive mask, ALiBi when the table is affine, and a pure LSE shift when the
table is constant.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import random_case


def _bias_matrix(table, R, Lq, Lk):
    """[H, Lq, Lk] bias by a direct gather (numpy): delta = j - p clipped to [-R, R]."""
    p = np.arange(Lq)[:, None] + (Lk - Lq)
    j = np.arange(Lk)[None, :]
    idx = np.clip(j - p, -R, R) + R
    return np.asarray(table, dtype=np.float64)[:, idx]


def _table(seed, H, R, spread=2.0):
    g = np.random.default_rng(seed)
    return g.standard_normal((H, 2 * R + 1)) * spread


def test_bias_alone_gives_the_closed_form_softmax():
    """Q = 0: every score is the bias, so with V = one-hot columns O is the
    softmax of the causal rows' biases and LSE = log sum exp(bias)."""
    H, Lq, Lk, d, R = 2, 40, 64, 64, 9
    table = _table(1, H, R)
    q = torch.zeros(1, H, Lq, d, dtype=torch.bfloat16)
    k = torch.randn(1, H, Lk, d).to(torch.bfloat16)
    v = torch.zeros(1, H, Lk, d)
    v[0, :, np.arange(Lk), np.arange(Lk)] = 1.0
    v = v.to(torch.bfloat16)
    o, lse = oracle.attn_fwd(q, k, v, mask="causal", rel_bias=(table, R))
    bias = _bias_matrix(table, R, Lq, Lk)
    allowed = np.tril(np.ones((Lq, Lk), dtype=bool), k=Lk - Lq)
    z = np.where(allowed[None], bias, -np.inf)
    want_lse = np.log(np.exp(z).sum(-1))
    want_p = np.exp(z - want_lse[..., None])
    np.testing.assert_allclose(lse[0], want_lse, atol=1e-12)
    np.testing.assert_allclose(o[0, :, :, :Lk], want_p, atol=1e-12)


@pytest.mark.parametrize("mask,window,R", [("none", (-1, -1), 5), ("causal", (-1, -1), 30),
                                           ("causal", (7, 0), 3), ("none", (20, 11), 0)])
def test_equals_float64_sdpa_with_the_bias_as_additive_mask(mask, window, R):
    B, H, Hkv, Lq, Lk, d = 1, 4, 2, 33, 70, 32
    q, k, v, _, _ = random_case(7, B, H, Hkv, Lq, Lk, d)
    table = _table(2, H, R)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(q, k, v, scale=scale, mask=mask, window=window, rel_bias=(table, R))
    allowed = oracle.mask(1, Lq, Lk, mask=mask, window=window)[0]
    bias = _bias_matrix(table, R, Lq, Lk)
    add = torch.from_numpy(np.where(allowed[None], bias, -np.inf))[None]
    kk = k.double().repeat_interleave(H // Hkv, dim=1)
    vv = v.double().repeat_interleave(H // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), kk, vv, attn_mask=add,
                                                           scale=scale)
    s = scale * torch.einsum("bhid,bhjd->bhij", q.double(), kk) + add
    ref_lse = torch.logsumexp(s, dim=-1)
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-10)
    np.testing.assert_allclose(lse, ref_lse.numpy(), atol=1e-10)


def test_affine_table_is_alibi_inside_the_window():
    """table[delta + R] = slope * delta and a symmetric window of R: every visible
    key lies within R of its row, so the table is exactly ALiBi."""
    H, Lq, Lk, d, R = 3, 50, 90, 64, 12
    q, k, v, _, _ = random_case(11, 1, H, H, Lq, Lk, d)
    slopes = np.array([0.5, 0.125, 1.0 / 32])
    table = slopes[:, None] * np.arange(-R, R + 1)[None, :]
    o1, l1 = oracle.attn_fwd(q, k, v, window=(R, R), rel_bias=(table, R))
    o2, l2 = oracle.attn_fwd(q, k, v, window=(R, R), alibi_slopes=slopes)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


@pytest.mark.parametrize("R", [0, 4])
def test_constant_table_only_shifts_the_lse(R):
    H, Lq, Lk, d = 2, 20, 45, 64
    q, k, v, _, _ = random_case(13, 1, H, H, Lq, Lk, d)
    consts = np.array([0.75, -2.5])
    table = np.repeat(consts[:, None], 2 * R + 1, axis=1)
    o1, l1 = oracle.attn_fwd(q, k, v, mask="causal", rel_bias=(table, R))
    o0, l0 = oracle.attn_fwd(q, k, v, mask="causal")
    np.testing.assert_allclose(o1, o0, atol=1e-12)
    np.testing.assert_allclose(l1, l0 + consts[None, :, None], atol=1e-12)


def test_packed_sequences_apply_the_table_per_sequence():
    """Each packed sequence uses its own positions: equal to the dense call
    on that sequence alone."""
    H, d, R = 2, 64, 6
    table = _table(3, H, R)
    lens = [50, 1, 90]
    from workloads import packed_case
    q, k, v, cu_q, cu_k = packed_case(17, lens, lens, H, H, d)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, mask="causal", rel_bias=(table, R))
    s0 = 0
    for L in lens:
        qs = q[s0:s0 + L].permute(1, 0, 2)[None].contiguous()
        ks = k[s0:s0 + L].permute(1, 0, 2)[None].contiguous()
        vs = v[s0:s0 + L].permute(1, 0, 2)[None].contiguous()
        ro, rl = oracle.attn_fwd(qs, ks, vs, mask="causal", rel_bias=(table, R))
        np.testing.assert_allclose(o[s0:s0 + L], ro[0].transpose(1, 0, 2), atol=1e-12)
        np.testing.assert_allclose(lse[:, s0:s0 + L], rl[0], atol=1e-12)
        s0 += L
