"""Pins for the oracle's O and LSE (CPU only).

The pages print no numeric worked example, so the oracle is pinned by closed
forms, invariants and a library special case:
  - all keys equal      -> O is the mean of the allowed V rows, LSE = s + ln n;
  - one dominant score  -> O selects that key's V row;
  - V = one-hot columns -> O exposes P itself: rows of P sum to 1, P >= 0 and
                           P = 0 exactly where the mask forbids;
  - PyTorch's float64 scaled_dot_product_attention on CPU with a boolean mask
    (the page "FlashAttention 2 原理与 PyTorch 实战", section 二, uses SDPA as the
    reference call) agrees to 1e-12, GQA included;
  - split-KV: chunk-then-merge in double equals the unsplit result.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_mask import independent_mask
from workloads import random_case


def _bits(x):
    return x.to(torch.bfloat16)


def _sdpa64(q, k, v, allowed, scale):
    """float64 SDPA on CPU with a boolean mask; K/V heads repeated for GQA."""
    B, Hq, Lq, d = q.shape
    Hkv = k.shape[1]
    kk = k.double().repeat_interleave(Hq // Hkv, dim=1)
    vv = v.double().repeat_interleave(Hq // Hkv, dim=1)
    mask = torch.from_numpy(allowed)[:, None, :, :]
    o = torch.nn.functional.scaled_dot_product_attention(q.double(), kk, vv, attn_mask=mask,
                                                         scale=scale)
    s = torch.einsum("bhid,bhjd->bhij", q.double(), kk) * scale
    s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), lse.numpy()


CASES = [
    # (seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc)
    (0, 1, 2, 2, 16, 16, 64, "none", (-1, -1), 1, False),
    (1, 2, 4, 2, 33, 33, 64, "causal", (-1, -1), 1, False),
    (2, 1, 4, 1, 7, 45, 128, "causal", (-1, -1), 1, False),
    (3, 2, 2, 2, 40, 40, 64, "draft", (5, 5), 4, True),
    (4, 1, 3, 1, 19, 50, 64, "none", (3, 9), 1, True),
    (5, 2, 8, 2, 16, 70, 128, "draft", (20, 20), 16, False),
]


@pytest.mark.parametrize("case", CASES)
def test_matches_float64_sdpa(case):
    seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(q, k, v, scale=scale, mask=mask, window=window, draft_block=bd,
                             doc_ids=doc_ids)
    allowed = independent_mask(B, Lq, Lk, mask, window, bd,
                               None if doc_ids is None else doc_ids.numpy(), None)
    ro, rlse = _sdpa64(q, k, v, allowed, scale)
    has = allowed.any(-1)[:, None, :].repeat(Hq, axis=1)
    assert has.any()
    np.testing.assert_allclose(o[has], ro[has], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[has], rlse[has], rtol=0, atol=1e-12)


def test_all_keys_equal_gives_mean_of_allowed_v():
    B, H, Lq, Lk, d = 1, 2, 12, 30, 64
    q, k, v, _, _ = random_case(11, B, H, H, Lq, Lk, d)
    k = k[:, :, :1, :].expand(B, H, Lk, d).contiguous()      # every key identical
    scale = 0.125
    bd, window = 4, (7, 2)
    o, lse = oracle.attn_fwd(q, k, v, scale=scale, mask="draft", window=window, draft_block=bd)
    allowed = independent_mask(B, Lq, Lk, "draft", window, bd, None, None)[0]
    vd = v.double().numpy()
    for h in range(H):
        for i in range(Lq):
            n = int(allowed[i].sum())
            if n == 0:
                assert lse[0, h, i] == -np.inf and np.all(o[0, h, i] == 0)
                continue
            mean = vd[0, h, allowed[i]].mean(axis=0)
            np.testing.assert_allclose(o[0, h, i], mean, atol=1e-13)
            s = scale * float(np.dot(q[0, h, i].double().numpy(), k[0, h, 0].double().numpy()))
            assert abs(lse[0, h, i] - (s + math.log(n))) < 1e-12


def test_single_dominant_score_selects_one_row():
    d, Lk = 64, 40
    q = torch.zeros(1, 1, 1, d)
    q[0, 0, 0, 0] = 8.0
    k = torch.zeros(1, 1, Lk, d)
    jstar = 17
    k[0, 0, jstar, 0] = 8.0                                # score 64 at j*, 0 elsewhere
    v = torch.randn(1, 1, Lk, d, generator=torch.Generator().manual_seed(3))
    q, k, v = _bits(q), _bits(k), _bits(v)
    o, lse = oracle.attn_fwd(q, k, v, scale=1.0)
    gap = (Lk - 1) * math.exp(-64.0)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, jstar].double().numpy(), atol=4 * gap)
    assert abs(lse[0, 0, 0] - (64.0 + math.log1p(gap))) < 1e-12


@pytest.mark.parametrize("mask,window,bd", [("causal", (-1, -1), 1), ("draft", (6, 3), 5),
                                            ("none", (2, 2), 1)])
def test_onehot_v_exposes_probabilities(mask, window, bd):
    """V = identity rows: O[i, j] = P_ij.  Rows of P sum to 1, P >= 0, P = 0 where masked."""
    Lq = Lk = d = 64
    q, k, _, _, _ = random_case(21, 1, 1, 1, Lq, Lk, d)
    v = _bits(torch.eye(Lk, d)[None, None])
    o, lse = oracle.attn_fwd(q, k, v, scale=0.125, mask=mask, window=window, draft_block=bd)
    p = o[0, 0]
    allowed = independent_mask(1, Lq, Lk, mask, window, bd, None, None)[0]
    assert np.all(p[~allowed] == 0.0)
    assert np.all(p >= 0)
    rows = allowed.any(-1)
    np.testing.assert_allclose(p[rows].sum(-1), 1.0, atol=1e-13)
    # P_ij = exp(s_ij - LSE_i): the log of each visible entry plus LSE is the score
    s = 0.125 * (q[0, 0].double() @ k[0, 0].double().T).numpy()
    np.testing.assert_allclose(np.log(p[allowed]), (s - lse[0, 0][:, None])[allowed], atol=1e-11)


def test_fully_masked_rows_follow_the_convention():
    """Causal with more queries than keys: the first Lq - Lk rows see nothing."""
    q, k, v, _, _ = random_case(31, 1, 2, 2, 10, 4, 64)
    o, lse = oracle.attn_fwd(q, k, v, mask="causal")
    assert np.all(np.isneginf(lse[:, :, :6]))
    assert np.all(o[:, :, :6] == 0.0)
    assert np.all(np.isfinite(lse[:, :, 6:]))


def test_gqa_equals_repeated_kv_heads():
    q, k, v, _, _ = random_case(41, 2, 8, 2, 20, 33, 64)
    o1, l1 = oracle.attn_fwd(q, k, v, mask="causal")
    o2, l2 = oracle.attn_fwd(q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1),
                             mask="causal")
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_rows_subset_equals_full():
    q, k, v, doc, _ = random_case(51, 2, 4, 2, 24, 24, 64, doc_split=True)
    o, lse = oracle.attn_fwd(q, k, v, mask="draft", draft_block=3, window=(4, 4), doc_ids=doc)
    rows = np.array([0, 5, 23, 24, 100, 191])
    orr, lr = oracle.attn_fwd(q, k, v, mask="draft", draft_block=3, window=(4, 4), doc_ids=doc,
                              rows=rows)
    assert np.array_equal(orr, o.reshape(-1, 64)[rows])
    assert np.array_equal(lr, lse.reshape(-1)[rows])


def test_kv_lens_ignore_the_poisoned_tail():
    """Keys at or past kv_lens[b] never matter: NaN there leaves O finite and
    equal to the result on the truncated cache."""
    B, Hq, Hkv, Lq, Lk, d = 3, 4, 2, 2, 50, 64
    q, k, v, _, kv = random_case(61, B, Hq, Hkv, Lq, Lk, d, kv_len_range=(1, Lk))
    kp, vp = k.clone(), v.clone()
    for b in range(B):
        kp[b, :, kv[b]:] = float("nan")
        vp[b, :, kv[b]:] = float("nan")
    o, lse = oracle.attn_fwd(q, kp, vp, kv_lens=kv)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    for b in range(B):
        L = int(kv[b])
        ob, lb = oracle.attn_fwd(q[b:b + 1], k[b:b + 1, :, :L], v[b:b + 1, :, :L])
        assert np.array_equal(o[b], ob[0]) and np.array_equal(lse[b], lb[0])


@pytest.mark.parametrize("chunk", [1, 7, 16, 64, 1000])
def test_split_then_combine_equals_unsplit(chunk):
    B, Hq, Hkv, Lq, Lk, d = 3, 8, 2, 3, 100, 128
    q, k, v, _, kv = random_case(71, B, Hq, Hkv, Lq, Lk, d, kv_len_range=(1, Lk))
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, kv_lens=kv)
    op, lp = oracle.decode_partials(q, k, v, kv, chunk=chunk)
    o, lse = oracle.combine(op, lp)
    np.testing.assert_allclose(o, o_ref.reshape(-1, d), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref.reshape(-1), atol=1e-12, rtol=0)


def test_combine_of_empty_splits():
    op = np.zeros((3, 2, 4))
    lp = np.full((3, 2), -np.inf)
    lp[1, 0] = 0.5
    op[1, 0] = [1, 2, 3, 4]
    o, lse = oracle.combine(op, lp)
    assert lse[0] == 0.5 and np.array_equal(o[0], [1, 2, 3, 4])
    assert np.isneginf(lse[1]) and np.all(o[1] == 0)
