"""GPU parity of attn_fwd (prefill) against the oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, to_dev
from workloads import (CAUSAL_4K, CAUSAL_32K_GQA, DRAFT_WINDOW_DOC, DRAFT_WINDOW_DOC_FULL, TINY,
                       make_inputs, random_case)

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


def test_tiny_config_full():
    """B=1, H=2, L=128, d=64, no mask, scale 1/8: every element."""
    inp = make_inputs(TINY)
    o, lse = _run(inp.q, inp.k, inp.v, scale=TINY.softmax_scale)
    ro, rl = oracle.attn_fwd(inp.q, inp.k, inp.v, scale=TINY.softmax_scale)
    compare(o, lse, ro, rl, "tiny")


RAGGED = [
    # seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc
    (1, 1, 2, 2, 1, 1, 64, "none", (-1, -1), 1, False),
    (2, 2, 3, 1, 200, 333, 64, "none", (-1, -1), 1, False),
    (3, 1, 4, 2, 300, 300, 128, "causal", (-1, -1), 1, False),
    (4, 2, 2, 2, 129, 257, 64, "causal", (-1, -1), 1, False),
    (5, 1, 2, 1, 385, 385, 128, "causal", (100, 0), 1, False),
    (6, 1, 2, 2, 260, 260, 64, "none", (37, 37), 1, False),
    (7, 2, 2, 2, 300, 300, 128, "draft", (-1, -1), 16, False),
    (8, 1, 4, 4, 16, 2064, 128, "draft", (512, 512), 16, True),
    (9, 2, 2, 2, 500, 500, 64, "causal", (-1, -1), 1, True),
    (10, 1, 2, 2, 600, 200, 64, "causal", (-1, -1), 1, False),   # Lq > Lk: empty rows
    (11, 1, 2, 2, 130, 1000, 128, "draft", (3, 200), 7, False),
    (12, 1, 8, 2, 256, 1024, 64, "causal", (-1, -1), 1, False),
    (13, 1, 16, 2, 1, 5000, 128, "causal", (-1, -1), 1, False),  # one query row
    (14, 2, 8, 1, 700, 1900, 128, "none", (-1, -1), 1, False),    # GQA 8, Lq < Lk
    (15, 1, 4, 4, 1000, 1000, 64, "causal", (-1, -1), 1, True),   # many documents
    (16, 1, 2, 2, 900, 900, 128, "draft", (70, 33), 48, True),    # block not a divisor of 128
    (17, 1, 2, 1, 383, 1150, 64, "causal", (200, 5), 1, False),   # causal + window, offset
    (18, 3, 3, 3, 129, 129, 128, "none", (0, 0), 1, False),       # each row sees one key
]


@pytest.mark.parametrize("case", RAGGED, ids=lambda c: f"s{c[0]}_{c[7]}_lq{c[4]}_lk{c[5]}_d{c[6]}")
def test_ragged_shapes_and_masks(case):
    seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc,
                                      n_docs=8 if seed == 15 else 3)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    o, lse = _run(q, k, v, doc_ids=doc_ids, **kw)
    ro, rl = oracle.attn_fwd(q, k, v, doc_ids=doc_ids, **kw)
    compare(o, lse, ro, rl, str(case))


@pytest.mark.parametrize("case", [
    (64, 257, 300, "causal", (-1, -1), 1, False),
    (128, 200, 700, "draft", (40, 40), 16, True),
    (64, 520, 520, "none", (130, 5), 1, True),
    (128, 16, 2064, "draft", (512, 512), 16, True),
])
def test_mask_recovered_bit_exactly(case):
    """Q = 0 makes every visible key equally likely; V = one-hot columns then
    reads the mask back: O[i, c] != 0 exactly when key t*d + c is visible for
    chunk t.  LSE = ln(count) checks the per-row counts."""
    d, Lq, Lk, mask, window, bd, doc = case
    _, _, _, doc_ids, _ = random_case(5, 1, 1, 1, Lq, Lk, d, doc_split=doc, n_docs=4)
    want = oracle.mask(1, Lq, Lk, mask=mask, window=window, draft_block=bd, doc_ids=doc_ids)[0]
    q = torch.zeros(1, 1, Lq, d, dtype=torch.bfloat16)
    k = torch.randn(1, 1, Lk, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    got = np.zeros((Lq, Lk), dtype=bool)
    lse_all = None
    for t in range((Lk + d - 1) // d):
        v = torch.zeros(1, 1, Lk, d)
        keys = np.arange(t * d, min((t + 1) * d, Lk))
        v[0, 0, keys, keys - t * d] = 1.0
        o, lse = _run(q, k * 0, v.to(torch.bfloat16), scale=0.125, mask=mask, window=window,
                      draft_block=bd, doc_ids=doc_ids)
        oc = o[0, 0].float().cpu().numpy()
        got[:, keys] = oc[:, : len(keys)] != 0.0
        lse_all = lse[0, 0].cpu().numpy()
    assert np.array_equal(got, want)
    cnt = want.sum(-1)
    has = cnt > 0
    assert np.all(np.isneginf(lse_all[~has]))
    np.testing.assert_allclose(lse_all[has], np.log(cnt[has]), atol=1e-5)


def test_output_guard_bytes_untouched():
    """Stores stay inside O and LSE: sentinel bytes after both survive."""
    B, H, L, d = 1, 2, 300, 64
    q, k, v, _, _ = random_case(3, B, H, H, L, L, d)
    qd, kd, vd = to_dev(q, k, v)
    n_o, n_l = B * H * L * d, B * H * L
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 1024,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[:n_o].view(B, H, L, d)
    lse = l_buf[:n_l].view(B, H, L)
    ab.attn_fwd(qd, kd, vd, mask="causal", o=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0) and torch.all(l_buf[n_l:] == 7.0)
    ro, rl = oracle.attn_fwd(q, k, v, mask="causal")
    compare(o, lse, ro, rl, "guard")


def test_config_causal_4k_full():
    """The headline workload, every row of every head against the oracle
    (about 7e10 double-precision flop on the host)."""
    cfg = CAUSAL_4K
    inp = make_inputs(cfg)
    o, lse = _run(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask)
    ro, rl = oracle.attn_fwd(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask)
    compare(o, lse, ro, rl, cfg.name)


def stratified_rows(B, H, L):
    """Every head; rows 0-255, every 64th row and the last 256 rows."""
    per = sorted(set(range(256)) | set(range(0, L, 64)) | set(range(L - 256, L)))
    per = np.array(per, dtype=np.int64)
    return np.concatenate([(bh * L) + per for bh in range(B * H)])


def test_config_causal_32k_gqa_stratified():
    cfg = CAUSAL_32K_GQA
    inp = make_inputs(cfg)
    o, lse = _run(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask)
    rows = stratified_rows(cfg.B, cfg.Hq, cfg.Lq)
    ro, rl = oracle.attn_fwd(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask=cfg.mask,
                             rows=rows)
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, cfg.d)[idx], lse.reshape(-1)[idx], ro, rl, cfg.name)


@pytest.mark.parametrize("cfg", [DRAFT_WINDOW_DOC, DRAFT_WINDOW_DOC_FULL], ids=lambda c: c.name)
def test_config_draft_window_doc_full(cfg):
    inp = make_inputs(cfg)
    kw = dict(scale=cfg.softmax_scale, mask=cfg.mask, window=cfg.window,
              draft_block=cfg.draft_block)
    o, lse = _run(inp.q, inp.k, inp.v, doc_ids=inp.doc_ids, **kw)
    ro, rl = oracle.attn_fwd(inp.q, inp.k, inp.v, doc_ids=inp.doc_ids, **kw)
    compare(o, lse, ro, rl, cfg.name)


def test_invalid_arguments_launch_nothing():
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 3, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ab.AttnError) as e:
        ab.attn_fwd(q, k, k)                        # Hq % Hkv != 0
    assert e.value.status == ab.ATTN_ERR_INVALID_ARG
    q96 = torch.zeros(1, 2, 8, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ab.AttnError) as e:
        ab.attn_fwd(q96, q96, q96)                  # d = 96 not built
    assert e.value.status == ab.ATTN_ERR_UNSUPPORTED
    with pytest.raises(ab.AttnError) as e:
        ab.attn_fwd(q, q, q, mask="draft", draft_block=0)
    assert e.value.status == ab.ATTN_ERR_INVALID_ARG


def test_capturable_in_cuda_graph():
    """The call allocates nothing and never synchronises, so it can be captured."""
    q, k, v, _, _ = random_case(9, 1, 2, 2, 256, 256, 64)
    qd, kd, vd = to_dev(q, k, v)
    o = torch.empty_like(qd)
    lse = torch.empty(1, 2, 256, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ab.attn_fwd(qd, kd, vd, mask="causal", o=o, lse=lse, stream=s)  # warm-up (attributes)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ab.attn_fwd(qd, kd, vd, mask="causal", o=o, lse=lse, stream=s)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(q, k, v, mask="causal")
    compare(o, lse, ro, rl, "graph")


def test_repeated_calls_are_bit_identical():
    """The persistent schedule is static: the same inputs give the same bits."""
    q, k, v, _, _ = random_case(19, 2, 4, 2, 777, 777, 64)
    qd, kd, vd = to_dev(q, k, v)
    o1, l1 = ab.attn_fwd(qd, kd, vd, mask="causal")
    o2, l2 = ab.attn_fwd(qd, kd, vd, mask="causal")
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
