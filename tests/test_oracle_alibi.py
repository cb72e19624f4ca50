"""Pins of the oracle's ALiBi score_mod (S_ij += slope_h * (j - p)): closed forms
with all raw scores zero, invariance of O under the per-row constant, and the
zero slope."""
import numpy as np
import torch

import oracle
from workloads import random_case


def test_zero_scores_give_geometric_weights():
    """Q = 0: the causal row at position p sees keys 0..p with weights r^(p-j),
    r = exp(-slope), so LSE = log((1 - r^(p+1)) / (1 - r)) and, with V the
    one-hot columns, O[p, j] = r^(p-j) / sum_k r^k."""
    L, d = 48, 64
    slopes = np.array([0.25, 0.0625], dtype=np.float64)
    q = torch.zeros(1, 2, L, d, dtype=torch.bfloat16)
    k = torch.randn(1, 1, L, d, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    v = torch.zeros(1, 1, L, d)
    v[0, 0, torch.arange(L), torch.arange(L)] = 1.0   # key j -> column j (L <= d)
    o, lse = oracle.attn_fwd(q, k, v.to(torch.bfloat16), mask="causal", scale=0.1,
                             alibi_slopes=slopes)
    for h, sl in enumerate(slopes):
        r = np.exp(-sl)
        p = np.arange(L)
        np.testing.assert_allclose(lse[0, h], np.log((1 - r ** (p + 1)) / (1 - r)), rtol=0,
                                   atol=1e-12)
        for i in (0, 1, 17, L - 1):
            w = r ** (i - np.arange(i + 1))
            want = np.zeros(d)
            want[: i + 1] = w / w.sum()
            np.testing.assert_allclose(o[0, h, i], want, rtol=0, atol=1e-12)


def test_row_constant_cancels_in_o():
    """Without a mask the bias slope*j - slope*p differs between rows only by a
    per-row constant: equal query rows give equal O, and LSE drops by slope per
    position."""
    L, d = 40, 64
    q1, k, v, _, _ = random_case(3, 1, 1, 1, 1, L, d)
    q = q1.expand(1, 1, L, d).contiguous()
    o, lse = oracle.attn_fwd(q, k, v, alibi_slopes=[0.3])
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(o[0, 0, :1], (L, d)), atol=1e-12)
    np.testing.assert_allclose(np.diff(lse[0, 0]), -0.3, atol=1e-12)


def test_zero_slope_is_plain_attention():
    q, k, v, _, _ = random_case(4, 2, 4, 2, 37, 70, 64)
    a = oracle.attn_fwd(q, k, v, mask="causal", window=(9, 3), alibi_slopes=[0.0] * 4)
    b = oracle.attn_fwd(q, k, v, mask="causal", window=(9, 3))
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_bias_uses_the_row_position():
    """Lq = 1 over Lk keys, no mask, Q = 0: the row sits at p = Lk - 1, so the
    weights are r^(p-j) for every key (not r^(-j))."""
    L, d, sl = 30, 64, 0.2
    q = torch.zeros(1, 1, 1, d, dtype=torch.bfloat16)
    k = torch.randn(1, 1, L, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    v = torch.zeros(1, 1, L, d)
    v[0, 0, torch.arange(L), torch.arange(L)] = 1.0
    o, lse = oracle.attn_fwd(q, k, v.to(torch.bfloat16), alibi_slopes=[sl])
    r = np.exp(-sl)
    w = r ** (L - 1 - np.arange(L))
    np.testing.assert_allclose(lse[0, 0, 0], np.log(w.sum()), atol=1e-12)
    np.testing.assert_allclose(o[0, 0, 0, :L], w / w.sum(), atol=1e-12)
