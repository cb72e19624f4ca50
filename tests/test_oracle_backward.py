"""Pins of the backward oracle (oracle.attn_bwd): float64 autograd of PyTorch's
SDPA with an explicit mask, closed forms for uniform attention, the zero sum of
dK over keys (a shift of every key leaves the softmax unchanged), and GQA as the
sum over the query heads of a KV head."""
import numpy as np
import pytest
import torch

import oracle
from workloads import random_case


@pytest.mark.parametrize("mask,window,bd,doc", [("none", (-1, -1), 1, False),
                                                ("causal", (-1, -1), 1, False),
                                                ("causal", (6, 0), 1, True),
                                                ("draft", (5, 5), 4, False)])
def test_matches_float64_sdpa_autograd(mask, window, bd, doc):
    B, H, Lq, Lk, d = 2, 3, 24, 40, 16
    q, k, v, doc_ids, _ = random_case(11, B, H, H, Lq, Lk, d, doc_split=doc)
    do = torch.randn(B, H, Lq, d, generator=torch.Generator().manual_seed(2), dtype=torch.float64)
    vis = torch.from_numpy(oracle.mask(B, Lq, Lk, mask=mask, window=window, draft_block=bd,
                                       doc_ids=doc_ids))
    qd, kd, vd = (t.double().requires_grad_() for t in (q, k, v))
    # rows with no visible key: give them one harmless key so SDPA stays finite, then drop them
    has = vis.any(-1)
    vis_safe = vis.clone()
    vis_safe[~has] = True
    o = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=vis_safe[:, None],
                                                         scale=0.3)
    (o * do * has[:, None, :, None]).sum().backward()
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale=0.3, mask=mask, window=window,
                                 draft_block=bd, doc_ids=doc_ids)
    np.testing.assert_allclose(dq, qd.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dk, kd.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dv, vd.grad.numpy(), atol=1e-10, rtol=0)


def test_uniform_attention_closed_forms():
    """Q = 0 and no mask: every P_ij = 1/Lk, so dV_j = (1/Lk) sum_i dO_i; with all
    K rows equal, dS sums to zero against equal keys, so dQ = 0; dK = 0 since Q = 0."""
    B, H, Lq, Lk, d = 1, 2, 7, 9, 8
    q = torch.zeros(B, H, Lq, d, dtype=torch.bfloat16)
    k1 = torch.randn(1, 1, 1, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    k = k1.expand(B, H, Lk, d).contiguous()
    v = torch.randn(B, H, Lk, d, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    do = torch.randn(B, H, Lq, d, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale=0.5)
    want_dv = np.broadcast_to(do.numpy().sum(axis=2, keepdims=True) / Lk, dv.shape)
    np.testing.assert_allclose(dv, want_dv, atol=1e-12)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def test_dk_sums_to_zero_over_keys():
    q, k, v, _, _ = random_case(12, 1, 2, 2, 30, 30, 16)
    do = torch.randn(1, 2, 30, 16, generator=torch.Generator().manual_seed(6), dtype=torch.float64)
    _, dk, _ = oracle.attn_bwd(q, k, v, do, mask="causal", window=(8, 0))
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-10)


def test_gqa_adds_the_query_heads_of_a_kv_head():
    q, k, v, _, _ = random_case(13, 1, 4, 2, 20, 25, 16)
    do = torch.randn(1, 4, 20, 16, generator=torch.Generator().manual_seed(7), dtype=torch.float64)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, mask="causal")
    kr, vr = k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1)
    dq2, dk2, dv2 = oracle.attn_bwd(q, kr, vr, do, mask="causal")
    np.testing.assert_allclose(dq, dq2, atol=1e-12)
    np.testing.assert_allclose(dk, dk2.reshape(1, 2, 2, 25, 16).sum(axis=2), atol=1e-12)
    np.testing.assert_allclose(dv, dv2.reshape(1, 2, 2, 25, 16).sum(axis=2), atol=1e-12)
