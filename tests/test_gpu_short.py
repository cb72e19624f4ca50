"""GPU parity of the short-query prefill path (a cluster of CTAs splits the
keys of each query row tile and merges over distributed shared memory).

attn_fwd takes this path by itself when Lq <= 128, the row tiles of all
(b, kv head) are fewer than twice the SM count and the visible key range
spans at least 4 key tiles; it splits the range over up to 8 CTAs once each
gets 8 tiles or more.  The shapes below are chosen to land on both sides of
those choices (one CTA per row tile, and full 8-CTA clusters).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, to_dev
from workloads import random_case

pytestmark = pytest.mark.gpu


def _run(q, k, v, **kw):
    qd, kd, vd = to_dev(q, k, v)
    doc = kw.pop("doc_ids", None)
    docd = None if doc is None else doc.cuda().contiguous()
    o, lse = ab.attn_fwd(qd, kd, vd, doc_ids=docd, **kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    return o, lse


SHORT = [
    # seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc
    (31, 1, 4, 4, 16, 32768, 128, "none", (-1, -1), 1, False),     # 8-CTA clusters, 32 tiles each
    (32, 2, 32, 8, 8, 16384, 128, "causal", (-1, -1), 1, False),   # GQA 4: 32 rows per tile
    (33, 1, 2, 2, 100, 9000, 64, "causal", (-1, -1), 1, False),    # ragged Lk, d = 64
    (34, 2, 4, 4, 64, 20000, 128, "draft", (3000, 3000), 16, True),  # draft + window + documents
    (35, 1, 16, 1, 8, 5000, 64, "none", (700, 0), 1, True),         # GQA 16: 128 rows, one tile
    (36, 4, 8, 8, 16, 2064, 128, "draft", (512, 512), 16, True),    # the DFlash draft shape, smaller B*H
    (37, 1, 3, 3, 1, 70000, 64, "causal", (-1, -1), 1, False),      # a single query row
    (38, 1, 2, 1, 128, 4500, 128, "none", (2000, 2000), 1, False),  # 128 rows, both window sides
]


@pytest.mark.parametrize("case", SHORT, ids=lambda c: f"s{c[0]}_{c[7]}_lq{c[4]}_lk{c[5]}_d{c[6]}")
def test_short_query_parity(case):
    seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc, n_docs=6)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    o, lse = _run(q, k, v, doc_ids=doc_ids, **kw)
    ro, rl = oracle.attn_fwd(q, k, v, doc_ids=doc_ids, **kw)
    compare(o, lse, ro, rl, str(case))


def test_short_query_mask_recovered_bit_exactly():
    """Q = 0 and V = one-hot columns read the mask back through the cluster
    path (71 key tiles over 8 CTAs): O[i, c] != 0 exactly when key t*d + c is
    visible, and LSE = ln(count)."""
    d, Lq, Lk = 64, 32, 9000
    window = (5000, -1)
    _, _, _, doc_ids, _ = random_case(7, 1, 1, 1, Lq, Lk, d, doc_split=True, n_docs=5)
    want = oracle.mask(1, Lq, Lk, mask="causal", window=window, doc_ids=doc_ids)[0]
    q = torch.zeros(1, 1, Lq, d, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, Lk, d, dtype=torch.bfloat16)
    got = np.zeros((Lq, Lk), dtype=bool)
    lse_all = None
    for t in range((Lk + d - 1) // d):
        keys = np.arange(t * d, min((t + 1) * d, Lk))
        if not want[:, keys].any():
            continue
        v = torch.zeros(1, 1, Lk, d)
        v[0, 0, keys, keys - t * d] = 1.0
        o, lse = _run(q, k, v.to(torch.bfloat16), scale=0.125, mask="causal", window=window,
                      doc_ids=doc_ids)
        got[:, keys] = o[0, 0].float().cpu().numpy()[:, : len(keys)] != 0.0
        lse_all = lse[0, 0].cpu().numpy()
    assert np.array_equal(got, want)
    cnt = want.sum(-1)
    np.testing.assert_allclose(lse_all[cnt > 0], np.log(cnt[cnt > 0]), atol=1e-5)
    assert np.all(np.isneginf(lse_all[cnt == 0]))


def test_short_query_capturable_in_cuda_graph():
    q, k, v, _, _ = random_case(39, 1, 2, 2, 16, 12000, 128)
    qd, kd, vd = to_dev(q, k, v)
    o = torch.empty_like(qd)
    lse = torch.empty(1, 2, 16, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ab.attn_fwd(qd, kd, vd, o=o, lse=lse, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ab.attn_fwd(qd, kd, vd, o=o, lse=lse, stream=s)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(q, k, v)
    compare(o, lse, ro, rl, "short graph")


def test_short_query_repeated_calls_are_bit_identical():
    """The merge order over the cluster is fixed: same inputs, same bits."""
    q, k, v, _, _ = random_case(40, 1, 4, 2, 24, 20000, 64)
    qd, kd, vd = to_dev(q, k, v)
    o1, l1 = ab.attn_fwd(qd, kd, vd, mask="causal")
    o2, l2 = ab.attn_fwd(qd, kd, vd, mask="causal")
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
