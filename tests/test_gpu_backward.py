"""GPU parity of attn_bwd (dQ, dK, dV) against the double-precision backward oracle.

Tolerance: the kernel rounds P and dS to bf16 before the MMAs and writes bf16
gradients, so each gradient is compared against the oracle's with
max |d| <= 3e-2 * max|ref| and mean |d| <= 3e-3 * max|ref| (per tensor)."""
import math

import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import to_dev
from workloads import random_case

pytestmark = pytest.mark.gpu


def _check(got, ref, what):
    g = got.float().cpu().double().numpy()
    scale = max(1e-6, np.abs(ref).max())
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), what
    assert err.max() <= 3e-2 * scale and err.mean() <= 3e-3 * scale, \
        f"{what}: max {err.max():.3g} mean {err.mean():.3g} ref max {scale:.3g}"


CASES = [
    # seed, B, Hq, Hkv, Lq, Lk, mask, window, bd, doc, d
    (1, 1, 2, 2, 128, 128, "none", (-1, -1), 1, False, 64),
    (2, 1, 2, 2, 256, 256, "causal", (-1, -1), 1, False, 64),
    (3, 2, 4, 2, 200, 333, "causal", (-1, -1), 1, False, 64),
    (4, 1, 2, 1, 300, 300, "none", (40, 17), 1, True, 64),
    (5, 1, 2, 2, 160, 400, "draft", (-1, 64), 16, False, 64),
    (6, 1, 8, 2, 129, 129, "causal", (50, 0), 1, False, 64),
    (7, 1, 2, 2, 640, 640, "causal", (-1, -1), 1, False, 64),    # many query tiles per key tile
    (11, 1, 2, 2, 128, 128, "none", (-1, -1), 1, False, 128),
    (12, 1, 2, 2, 256, 256, "causal", (-1, -1), 1, False, 128),
    (13, 2, 4, 2, 200, 333, "causal", (-1, -1), 1, False, 128),
    (14, 1, 2, 1, 300, 300, "none", (40, 17), 1, True, 128),
    (15, 1, 2, 2, 160, 400, "draft", (-1, 64), 16, False, 128),
    (16, 1, 8, 2, 129, 129, "causal", (50, 0), 1, False, 128),
    (17, 1, 2, 2, 640, 640, "causal", (-1, -1), 1, False, 128),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c[0]}_{c[6]}_lq{c[4]}_lk{c[5]}_d{c[10]}")
def test_backward_matches_oracle(case):
    seed, B, Hq, Hkv, Lq, Lk, mask, window, bd, doc, d = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc, n_docs=3)
    do = torch.randn(B, Hq, Lq, d, generator=torch.Generator().manual_seed(seed + 100))
    do = do.to(torch.bfloat16)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    qd, kd, vd, dod = to_dev(q, k, v, do)
    docd = None if doc_ids is None else doc_ids.cuda()
    o, lse = ab.attn_fwd(qd, kd, vd, doc_ids=docd, **kw)
    dq, dk, dv = ab.attn_bwd(qd, kd, vd, o, lse, dod, doc_ids=docd, **kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    rq, rk, rv = oracle.attn_bwd(q, k, v, do, doc_ids=doc_ids, **kw)
    _check(dv, rv, f"dV {case}")
    _check(dk, rk, f"dK {case}")
    _check(dq, rq, f"dQ {case}")


def test_backward_rejects_on_host():
    q = torch.zeros(1, 2, 64, 96, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 2, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(ab.AttnError) as e:
        ab.attn_bwd(q, q, q, q, lse, q)               # d = 96 not built
    assert e.value.status == ab.ATTN_ERR_UNSUPPORTED


@pytest.mark.parametrize("d", [64, 128])
def test_backward_full_size_sampled_heads(d):
    """The benchmark's backward workload (causal, B=2, H=16, L=4096, d=64, and the
    same at d=128) on the inputs and dO the benchmark draws: whole heads of dQ,
    dK and dV compared with the oracle run on those heads alone (heads are
    independent without GQA)."""
    from workloads import CAUSAL_4K, make_inputs
    cfg = CAUSAL_4K.with_(d=d)
    inp = make_inputs(cfg)
    g = torch.Generator()
    g.manual_seed(cfg.seed + 1000)
    do = torch.randn(inp.q.shape, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = to_dev(inp.q, inp.k, inp.v, do)
    o, lse = ab.attn_fwd(qd, kd, vd, scale=cfg.softmax_scale, mask="causal")
    dq, dk, dv = ab.attn_bwd(qd, kd, vd, o, lse, dod, scale=cfg.softmax_scale, mask="causal")
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    for b, h in ((0, 3), (1, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = oracle.attn_bwd(inp.q[sl], inp.k[sl], inp.v[sl], do[sl],
                                     scale=cfg.softmax_scale, mask="causal")
        _check(dv[sl], rv, f"dV b{b} h{h} d{d}")
        _check(dk[sl], rk, f"dK b{b} h{h} d{d}")
        _check(dq[sl], rq, f"dQ b{b} h{h} d{d}")


def test_backward_capturable_in_cuda_graph():
    """attn_bwd (memset, D_i kernel, gradient kernel, dQ conversion) replays from
    a CUDA graph with the results of a direct call."""
    q, k, v, _, _ = random_case(31, 1, 4, 2, 300, 300, 64)
    do = torch.randn(1, 4, 300, 64, generator=torch.Generator().manual_seed(131)).to(torch.bfloat16)
    qd, kd, vd, dod = to_dev(q, k, v, do)
    o, lse = ab.attn_fwd(qd, kd, vd, mask="causal")
    ws = torch.empty(ab.load_library().attn_bwd_workspace_size(1, 4, 300, 64), dtype=torch.uint8,
                     device="cuda")
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    s = torch.cuda.Stream()
    kw = dict(mask="causal", workspace=ws, dq=dq, dk=dk, dv=dv, stream=s)
    with torch.cuda.stream(s):
        ab.attn_bwd(qd, kd, vd, o, lse, dod, **kw)           # set-up outside the capture
    s.synchronize()
    ref = (dq.clone(), dk.clone(), dv.clone())
    g = torch.cuda.CUDAGraph()
    dq.zero_(); dk.zero_(); dv.zero_()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        ab.attn_bwd(qd, kd, vd, o, lse, dod, **kw)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
    _check(dq, ref[0].float().cpu().double().numpy(), "dQ graph replay")
