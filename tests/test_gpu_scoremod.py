"""GPU parity of attn_fwd_score_mod (ALiBi) against the oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, sample_rows, to_dev
from workloads import random_case

pytestmark = pytest.mark.gpu


def slopes_for(H):
    """The usual ALiBi slopes 2^(-8 (h+1) / H)."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)


CASES = [
    # seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc
    (1, 1, 4, 4, 128, 128, 64, "causal", (-1, -1), 1, False),
    (2, 2, 8, 2, 300, 300, 64, "causal", (-1, -1), 1, False),
    (3, 1, 4, 1, 257, 700, 128, "none", (-1, -1), 1, False),
    (4, 1, 2, 2, 500, 500, 128, "causal", (100, 0), 1, True),
    (5, 2, 4, 4, 16, 2064, 128, "draft", (512, 512), 16, True),
    (6, 1, 8, 8, 1, 3000, 64, "causal", (-1, -1), 1, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c[0]}_{c[7]}_lq{c[4]}_lk{c[5]}_d{c[6]}")
def test_alibi_matches_oracle(case):
    seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc, n_docs=3)
    sl = slopes_for(Hq)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ab.attn_fwd_score_mod(qd, kd, vd, alibi_slopes=sl.cuda(),
                                   doc_ids=None if doc_ids is None else doc_ids.cuda(), **kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    ro, rl = oracle.attn_fwd(q, k, v, doc_ids=doc_ids, alibi_slopes=sl.double().numpy(), **kw)
    compare(o, lse, ro, rl, str(case))


def test_alibi_long_context_sampled():
    """Positions up to 16K: the bias reaches slope * 16K; sampled rows."""
    B, H, L, d = 1, 8, 16384, 128
    q, k, v, _, _ = random_case(21, B, H, H, L, L, d, factor=0.5)
    sl = slopes_for(H)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ab.attn_fwd_score_mod(qd, kd, vd, alibi_slopes=sl.cuda(), mask="causal")
    torch.cuda.synchronize()
    rows = sample_rows(B, H, L, 8, seed=5)
    ro, rl = oracle.attn_fwd(q, k, v, mask="causal", rows=rows, alibi_slopes=sl.double().numpy())
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, d)[idx], lse.reshape(-1)[idx], ro, rl, "alibi 16K")


def test_zero_slopes_match_plain_forward():
    q, k, v, _, _ = random_case(22, 1, 4, 2, 333, 333, 64)
    qd, kd, vd = to_dev(q, k, v)
    o1, l1 = ab.attn_fwd_score_mod(qd, kd, vd, alibi_slopes=torch.zeros(4, device="cuda"),
                                   mask="causal")
    o2, l2 = ab.attn_fwd(qd, kd, vd, mask="causal")
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def rel_table(seed, H, R, spread=1.5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(H, 2 * R + 1, generator=g) * spread).float()


REL_CASES = [
    # seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc, R
    (31, 1, 4, 4, 128, 128, 64, "causal", (-1, -1), 1, False, 16),
    (32, 2, 8, 2, 300, 300, 64, "causal", (-1, -1), 1, False, 200),   # R past a tile
    (33, 1, 4, 1, 257, 700, 128, "none", (-1, -1), 1, False, 64),     # both signs of j - p
    (34, 1, 2, 2, 500, 500, 128, "causal", (100, 0), 1, True, 7),
    (35, 2, 4, 4, 16, 2064, 128, "draft", (512, 512), 16, True, 32),
    (36, 1, 8, 8, 1, 3000, 64, "causal", (-1, -1), 1, False, 0),      # per-head constant
    (37, 1, 2, 2, 640, 640, 64, "none", (-1, -1), 1, False, 1000),    # R beyond every distance
]


@pytest.mark.parametrize("case", REL_CASES,
                         ids=lambda c: f"s{c[0]}_{c[7]}_lq{c[4]}_lk{c[5]}_d{c[6]}_R{c[11]}")
def test_relative_bias_matches_oracle(case):
    seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc, R = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc, n_docs=3)
    table = rel_table(seed, Hq, R)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ab.attn_fwd_score_mod(qd, kd, vd, rel_bias=(table.cuda(), R),
                                   doc_ids=None if doc_ids is None else doc_ids.cuda(), **kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    ro, rl = oracle.attn_fwd(q, k, v, doc_ids=doc_ids, rel_bias=(table.double().numpy(), R),
                             **kw)
    compare(o, lse, ro, rl, str(case))


@pytest.mark.parametrize("mod", ["alibi", "rel"])
def test_packed_sequences_with_a_score_modifier(mod):
    """attn_fwd_varlen_score_mod: each sequence's rows use their own positions."""
    from workloads import packed_case, packed_lengths
    H, d = 4, 64
    lens = packed_lengths(41, 6, 1, 700) + [128, 129]
    q, k, v, cu_q, cu_k = packed_case(41, lens, lens, H, H, d)
    kw = {}
    okw = {}
    if mod == "alibi":
        sl = slopes_for(H)
        kw["alibi_slopes"] = sl.cuda()
        okw["alibi_slopes"] = sl.double().numpy()
    else:
        table = rel_table(42, H, 40)
        kw["rel_bias"] = (table.cuda(), 40)
        okw["rel_bias"] = (table.double().numpy(), 40)
    qd, kd, vd, cqd, ckd = to_dev(q, k, v, cu_q, cu_k)
    o, lse = ab.attn_fwd_varlen(qd, kd, vd, cqd, ckd, max(lens), mask="causal", **kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    ro, rl = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, mask="causal", **okw)
    # packed LSE is [H, total]: compare token-major like O
    compare(o, lse.t(), ro, np.ascontiguousarray(rl.T), f"varlen {mod}")


def test_constant_table_matches_plain_forward():
    """R = 0 with one value per head: the same O, the LSE shifted by the value."""
    q, k, v, _, _ = random_case(43, 1, 4, 2, 333, 333, 128)
    qd, kd, vd = to_dev(q, k, v)
    consts = torch.tensor([[0.5], [-1.0], [2.0], [0.0]], dtype=torch.float32)
    o1, l1 = ab.attn_fwd_score_mod(qd, kd, vd, rel_bias=(consts.cuda(), 0), mask="causal")
    o2, l2 = ab.attn_fwd(qd, kd, vd, mask="causal")
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    shift = (l1 - l2).cpu()
    assert (shift - consts.view(1, 4, 1)).abs().max().item() <= 1e-3


def test_alibi_bench_workload_sampled_rows():
    """The benchmark's ALiBi leg: the causal 4K workload (B=2, H=16, d=64) with
    slopes 2^(-8 (h+1) / H), sampled rows against the oracle."""
    from workloads import CAUSAL_4K, make_inputs
    cfg = CAUSAL_4K
    inp = make_inputs(cfg)
    sl = slopes_for(cfg.Hq)
    qd, kd, vd = to_dev(inp.q, inp.k, inp.v)
    o, lse = ab.attn_fwd_score_mod(qd, kd, vd, alibi_slopes=sl.cuda(), scale=cfg.softmax_scale,
                                   mask="causal")
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    rows = sample_rows(cfg.B, cfg.Hq, cfg.Lq, 64, seed=7)
    ro, rl = oracle.attn_fwd(inp.q, inp.k, inp.v, scale=cfg.softmax_scale, mask="causal",
                             rows=rows, alibi_slopes=sl.double().numpy())
    idx = torch.from_numpy(rows).cuda()
    compare(o.reshape(-1, cfg.d)[idx], lse.reshape(-1)[idx], ro, rl, "alibi bench workload")


# ---------------------------------------------------------------- decode
DECODE_CASES = [
    # seed, B, Hq, Hkv, Lq, Lk_max, d, (lo, hi), num_splits, kind
    (31, 2, 8, 1, 1, 300, 128, (1, 300), 0, "alibi"),
    (32, 3, 16, 2, 16, 1000, 128, (1, 1000), 3, "alibi"),
    (33, 2, 4, 4, 3, 513, 64, (1, 513), 5, "rel"),
    (34, 2, 32, 2, 16, 640, 128, (100, 640), 2, "rel"),   # two row tiles per kv head
    (35, 1, 64, 8, 16, 2048, 128, (2048, 2048), 4, "alibi"),
    (36, 4, 8, 8, 1, 129, 64, (1, 129), 0, "rel"),
]


def _mod_args(kind, Hq, seed):
    """(device kwargs for the binding, oracle kwargs) of one score modifier."""
    if kind == "alibi":
        sl = slopes_for(Hq)
        return dict(alibi_slopes=sl.cuda()), dict(alibi_slopes=sl.double().numpy())
    R = 37
    table = torch.randn(Hq, 2 * R + 1, generator=torch.Generator().manual_seed(seed))
    return (dict(rel_bias=(table.cuda(), R)),
            dict(rel_bias=(table.double().numpy(), R)))


@pytest.mark.parametrize("case", DECODE_CASES,
                         ids=lambda c: f"s{c[0]}_{c[9]}_lq{c[4]}_lk{c[5]}_d{c[6]}")
def test_decode_score_mod_matches_oracle(case):
    """Split-KV decode with ALiBi or the relative-position table, query row i of
    sequence b at p = kv_lens[b] - Lq + i; K/V past kv_lens are NaN."""
    seed, B, Hq, Hkv, Lq, Lk, d, rng, ns, kind = case
    q, k, v, _, kv = random_case(seed, B, Hq, Hkv, Lq, Lk, d, kv_len_range=rng)
    kp, vp = k.clone(), v.clone()
    for b, L in enumerate(kv.tolist()):
        kp[b, :, L:] = float("nan")
        vp[b, :, L:] = float("nan")
    dev_kw, ora_kw = _mod_args(kind, Hq, seed)
    qd, kd, vd, kl = to_dev(q, kp, vp, kv)
    o, lse = ab.attn_decode_splitkv_score_mod(qd, kd, vd, kl, num_splits=ns, **dev_kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    ro, rl = oracle.attn_fwd(q, k, v, kv_lens=kv, **ora_kw)
    compare(o, lse, ro, rl, str(case))


@pytest.mark.parametrize("P,kind", [(128, "alibi"), (16, "rel")])
def test_paged_decode_score_mod_equals_contiguous(P, kind):
    """Identity page table: the paged and the contiguous score-modifier calls agree
    to the bit."""
    B, Hq, Hkv, Lq, d = 2, 16, 2, 4, 128
    pps = 1024 // P
    q, k, v, _, _ = random_case(41, B, Hq, Hkv, Lq, pps * P, d)
    kv = torch.tensor([700, 1024], dtype=torch.int32)
    kp = k.view(B, Hkv, pps, P, d).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, P, d).contiguous()
    vp = v.view(B, Hkv, pps, P, d).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, P, d).contiguous()
    table = torch.arange(B * pps, dtype=torch.int32).view(B, pps)
    dev_kw, _ = _mod_args(kind, Hq, 42)
    qd, kd, vd, kpd, vpd, td, kvd = to_dev(q, k, v, kp, vp, table, kv)
    o1, l1 = ab.attn_decode_splitkv_score_mod(qd, kd, vd, kvd, **dev_kw)
    o2, l2 = ab.attn_decode_paged_score_mod(qd, kpd, vpd, td, kvd, **dev_kw)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_alibi_full_size_sampled():
    """The Lq = 16 decode workload (B = 64, Hq = 64, Hkv = 8, kv_lens up to 32K,
    d = 128) with ALiBi slopes: 6 whole sequences (every head and query) against
    the oracle; biases reach slope * 32K."""
    from workloads import DECODE_LQ16, make_inputs
    cfg = DECODE_LQ16
    inp = make_inputs(cfg, device="cuda")
    sl = slopes_for(cfg.Hq)
    o, lse = ab.attn_decode_splitkv_score_mod(inp.q, inp.k, inp.v, inp.kv_lens,
                                              alibi_slopes=sl.cuda(), scale=cfg.softmax_scale)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    kv_host = inp.kv_lens.cpu()
    for b in np.random.default_rng(3).choice(cfg.B, 6, replace=False).tolist():
        L = int(kv_host[b])
        kvb = torch.tensor([L], dtype=torch.int32)
        ro, rl = oracle.attn_fwd(inp.q[b:b + 1].cpu(), inp.k[b:b + 1, :, :L].cpu(),
                                 inp.v[b:b + 1, :, :L].cpu(), scale=cfg.softmax_scale,
                                 kv_lens=kvb, alibi_slopes=sl.double().numpy())
        compare(o[b:b + 1], lse[b:b + 1], ro, rl, f"decode alibi b={b}")
