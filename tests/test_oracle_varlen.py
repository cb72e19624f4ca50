"""Pins of the packed-sequence oracle (oracle.attn_fwd_varlen) against routes
that do not slice: the document-id mask of the dense oracle, a float64 SDPA
with an explicit mask, permutation of the sequences, and empty sequences."""
import numpy as np
import pytest
import torch

import oracle
from workloads import packed_case


def _dense_from_packed(x):
    """[total, H, d] -> [1, H, total, d]"""
    return x.permute(1, 0, 2).unsqueeze(0).contiguous()


@pytest.mark.parametrize("mask,window,bd", [("none", (-1, -1), 1), ("causal", (-1, -1), 1),
                                             ("causal", (5, 0), 1), ("none", (3, 7), 1),
                                             ("draft", (-1, -1), 4)])
def test_packing_equals_document_mask(mask, window, bd):
    """Self-attention sequences (Lq_b = Lk_b) packed back to back are the dense
    attention over the concatenation with one document id per sequence.  For
    the draft mask the lengths are multiples of the block, so local and global
    block indices agree."""
    lens = [8, 12, 4, 20] if mask == "draft" else [7, 13, 1, 30, 9]
    q, k, v, cu_q, cu_k = packed_case(3, lens, lens, 4, 2, 16)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, mask=mask, window=window, draft_block=bd)
    doc = torch.repeat_interleave(torch.arange(len(lens), dtype=torch.int32),
                                  torch.tensor(lens)).unsqueeze(0)
    od, ld = oracle.attn_fwd(_dense_from_packed(q), _dense_from_packed(k), _dense_from_packed(v),
                             mask=mask, window=window, draft_block=bd, doc_ids=doc)
    np.testing.assert_allclose(o, od[0].transpose(1, 0, 2), atol=1e-12, rtol=0)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(ld[0]))
    fin = np.isfinite(ld[0])
    np.testing.assert_allclose(lse[fin], ld[0][fin], atol=1e-12, rtol=0)


def test_query_shorter_than_keys_against_float64_sdpa():
    """Lq_b < Lk_b: rows sit at the end of their sequence (p = Lk_b - Lq_b + i)."""
    lq, lk = [3, 5], [9, 6]
    q, k, v, cu_q, cu_k = packed_case(5, lq, lk, 2, 1, 8)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, mask="causal", scale=0.3)
    for b in range(2):
        qs = q[cu_q[b]:cu_q[b + 1]].double().permute(1, 0, 2)
        ks = k[cu_k[b]:cu_k[b + 1]].double().permute(1, 0, 2).expand(2, -1, -1)
        vs = v[cu_k[b]:cu_k[b + 1]].double().permute(1, 0, 2).expand(2, -1, -1)
        i = torch.arange(lq[b])[:, None] + (lk[b] - lq[b])
        j = torch.arange(lk[b])[None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, attn_mask=j <= i,
                                                               scale=0.3)
        s = 0.3 * qs @ ks.transpose(-1, -2)
        s = s.masked_fill(~(j <= i), float("-inf"))
        np.testing.assert_allclose(o[cu_q[b]:cu_q[b + 1]], ref.permute(1, 0, 2).numpy(), atol=1e-12)
        np.testing.assert_allclose(lse[:, cu_q[b]:cu_q[b + 1]], torch.logsumexp(s, -1).numpy(),
                                   atol=1e-12)


def test_sequence_order_does_not_matter():
    lens_q, lens_k = [5, 11, 2], [5, 14, 9]
    q, k, v, cu_q, cu_k = packed_case(7, lens_q, lens_k, 2, 2, 8)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, mask="causal")
    perm = [2, 0, 1]
    cq, ck = cu_q.tolist(), cu_k.tolist()
    qp = torch.cat([q[cq[b]:cq[b + 1]] for b in perm])
    kp = torch.cat([k[ck[b]:ck[b + 1]] for b in perm])
    vp = torch.cat([v[ck[b]:ck[b + 1]] for b in perm])
    cqp = torch.tensor([0] + list(np.cumsum([lens_q[b] for b in perm])), dtype=torch.int32)
    ckp = torch.tensor([0] + list(np.cumsum([lens_k[b] for b in perm])), dtype=torch.int32)
    op, lp = oracle.attn_fwd_varlen(qp, kp, vp, cqp, ckp, mask="causal")
    rows = np.concatenate([np.arange(cq[b], cq[b + 1]) for b in perm])
    np.testing.assert_array_equal(op, o[rows])
    np.testing.assert_array_equal(lp, lse[:, rows])


def test_empty_sequences():
    """Lq_b = 0 contributes no rows; Lk_b = 0 gives rows with O = 0, LSE = -inf."""
    lens_q, lens_k = [3, 0, 2, 4], [3, 5, 0, 4]
    q, k, v, cu_q, cu_k = packed_case(9, lens_q, lens_k, 2, 1, 8)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k)
    rows_b2 = slice(3, 5)
    assert np.all(o[rows_b2] == 0.0) and np.all(np.isneginf(lse[:, rows_b2]))
    assert np.all(np.isfinite(lse[:, :3])) and np.all(np.isfinite(lse[:, 5:]))


def test_bad_cu_seqlens_rejected():
    q, k, v, cu_q, cu_k = packed_case(1, [2, 3], [2, 3], 1, 1, 8)
    with pytest.raises(ValueError):
        oracle.attn_fwd_varlen(q, k, v, torch.tensor([0, 3, 2], dtype=torch.int32), cu_k)
    with pytest.raises(ValueError):
        oracle.attn_fwd_varlen(q, k, v, cu_q, torch.tensor([0, 2, 6], dtype=torch.int32))
