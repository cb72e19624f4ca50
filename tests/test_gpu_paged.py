"""GPU parity of attn_decode_paged against the oracle on the gathered cache."""
import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, to_dev

pytestmark = pytest.mark.gpu


def _case(seed, B, Hq, Hkv, Lq, P, pps, d, kv_lo, extra_pages=5):
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    n = B * pps + extra_pages
    q = torch.randn(B, Hq, Lq, d, generator=g).to(torch.bfloat16)
    kp = torch.randn(n, Hkv, P, d, generator=g).to(torch.bfloat16)
    vp = torch.randn(n, Hkv, P, d, generator=g).to(torch.bfloat16)
    table = torch.from_numpy(rng.permutation(n)[: B * pps].reshape(B, pps).astype(np.int32))
    kv = torch.from_numpy(rng.integers(kv_lo, pps * P + 1, size=B).astype(np.int32))
    return q, kp, vp, table, kv


CASES = [
    # seed, B, Hq, Hkv, Lq, page_size, pages_per_seq, d, min kv_len
    (1, 3, 16, 2, 1, 16, 40, 128, 1),
    (2, 2, 8, 1, 4, 32, 13, 128, 100),
    (3, 4, 8, 8, 1, 64, 9, 64, 1),
    (4, 2, 64, 8, 16, 128, 6, 128, 300),
    (5, 2, 16, 2, 1, 256, 5, 128, 1),
    (6, 1, 8, 1, 2, 16, 3, 64, 1),          # whole cache shorter than one 128-key tile
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"P{c[5]}_pps{c[6]}_lq{c[4]}_d{c[7]}")
def test_paged_decode_matches_gathered_oracle(case):
    seed, B, Hq, Hkv, Lq, P, pps, d, lo = case
    q, kp, vp, table, kv = _case(seed, B, Hq, Hkv, Lq, P, pps, d, lo)
    # pages that no sequence uses, and rows past kv_len, hold NaN: never read
    used = set(table.numpy().reshape(-1).tolist())
    kp_d, vp_d = kp.clone(), vp.clone()
    for page in range(kp.shape[0]):
        if page not in used:
            kp_d[page] = float("nan")
            vp_d[page] = float("nan")
    for b in range(B):
        L = int(kv[b])
        for i in range(pps):
            start = max(0, L - i * P)
            if start < P:
                kp_d[table[b, i], :, start:] = float("nan")
                vp_d[table[b, i], :, start:] = float("nan")
    qd, kpd, vpd, td, kvd = to_dev(q, kp_d, vp_d, table, kv)
    o, lse = ab.attn_decode_paged(qd, kpd, vpd, td, kvd)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    kc = oracle.paged_gather(kp, table)
    vc = oracle.paged_gather(vp, table)
    ro, rl = oracle.attn_fwd(q, kc, vc, kv_lens=kv)
    compare(o, lse, ro, rl, str(case))


@pytest.mark.parametrize("P,d", [(128, 128), (32, 128), (16, 128), (16, 64)])
def test_paged_equals_contiguous_entry_point(P, d):
    """Identity page table: the paged call and attn_decode_splitkv agree to the bit
    (pages shorter than a key tile are copied by the producer lanes, pages of 128
    by TMA; both must leave the same tile layout in shared memory)."""
    B, Hq, Hkv, Lq = 2, 16, 2, 1
    pps = 1024 // P
    g = torch.Generator().manual_seed(9)
    q = torch.randn(B, Hq, Lq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, pps * P, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, pps * P, d, generator=g).to(torch.bfloat16)
    kv = torch.tensor([700, 1024], dtype=torch.int32)
    kp = k.view(B, Hkv, pps, P, d).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, P, d).contiguous()
    vp = v.view(B, Hkv, pps, P, d).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, P, d).contiguous()
    table = torch.arange(B * pps, dtype=torch.int32).view(B, pps)
    qd, kd, vd, kpd, vpd, td, kvd = to_dev(q, k, v, kp, vp, table, kv)
    o1, l1 = ab.attn_decode_splitkv(qd, kd, vd, kvd)
    o2, l2 = ab.attn_decode_paged(qd, kpd, vpd, td, kvd)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_page_id_is_flagged_not_faulted():
    q, kp, vp, table, kv = _case(7, 2, 8, 1, 1, 64, 4, 128, 256)
    table[1, 2] = 10_000
    qd, kpd, vpd, td, kvd = to_dev(q, kp, vp, table, kv)
    ab.attn_decode_paged(qd, kpd, vpd, td, kvd)
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_ERR_INVALID_ARG and bits != 0
    assert ab.attn_get_device_error()[0] == ab.ATTN_OK


def test_bench_paged_workloads_equal_contiguous():
    """The benchmark's paged legs: the full Lq=1 decode cache (B=64, Hq=64, Hkv=8,
    32K keys, d=128) moved into a shuffled page pool of 128- and of 16-key pages
    exactly as the benchmark does; the paged call gives the contiguous call's O
    and LSE to the bit (the contiguous call is checked against the oracle in the
    full-size decode test)."""
    from workloads import DECODE_LQ1, make_inputs
    cfg = DECODE_LQ1
    inp = make_inputs(cfg, device="cuda")
    o_c, l_c = ab.attn_decode_splitkv(inp.q, inp.k, inp.v, inp.kv_lens, scale=cfg.softmax_scale)
    B, Hkv, L, d = inp.k.shape
    for page_size in (128, 16):
        pps = L // page_size
        g = torch.Generator(device="cuda")
        g.manual_seed(cfg.seed + 1000)
        perm = torch.randperm(B * pps, generator=g, device="cuda")

        def to_pool(x):
            pages = x.view(B, Hkv, pps, page_size, d).permute(0, 2, 1, 3, 4).reshape(
                B * pps, Hkv, page_size, d)
            pool = torch.empty_like(pages)
            pool[perm] = pages
            return pool
        kp, vp = to_pool(inp.k), to_pool(inp.v)
        table = perm.view(B, pps).to(torch.int32).contiguous()
        o_p, l_p = ab.attn_decode_paged(inp.q, kp, vp, table, inp.kv_lens,
                                        scale=cfg.softmax_scale)
        torch.cuda.synchronize()
        st, bits = ab.attn_get_device_error()
        assert st == ab.ATTN_OK, (st, bits)
        assert torch.equal(o_p, o_c) and torch.equal(l_p, l_c), page_size
        del kp, vp
        torch.cuda.empty_cache()
