"""attn_fwd_host: host buffers in and out, uploads / kernels / downloads
pipelined over chunks of (batch, kv head) pairs.  The chunks run the kernel one
attn_fwd call over the whole shape would, so the outputs match it bit for bit."""
import math

import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare
from workloads import random_case

pytestmark = pytest.mark.gpu

CASES = [
    # seed, B, Hq, Hkv, Lq, Lk, d, mask, window, draft_block, doc, pinned
    (1, 2, 8, 8, 1000, 1000, 64, "causal", (-1, -1), 1, False, True),     # 8 head chunks
    (2, 1, 8, 2, 700, 900, 128, "draft", (256, 256), 16, True, True),      # GQA, doc ids
    (3, 9, 2, 1, 300, 300, 64, "none", (-1, -1), 1, False, True),          # chunks of batches
    (4, 3, 4, 4, 257, 257, 128, "causal", (64, 0), 1, False, False),       # pageable memory
    (5, 1, 4, 4, 16, 2064, 128, "draft", (512, 512), 16, True, True),      # short queries
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c[0]}_b{c[1]}_lq{c[4]}_d{c[6]}")
def test_host_call_equals_device_call(case):
    seed, B, Hq, Hkv, Lq, Lk, d, mask, window, bd, doc, pinned = case
    q, k, v, doc_ids, _ = random_case(seed, B, Hq, Hkv, Lq, Lk, d, doc_split=doc, n_docs=3)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    hq, hk, hv = (t.pin_memory() if pinned else t for t in (q, k, v))
    hdoc = None if doc_ids is None else (doc_ids.pin_memory() if pinned else doc_ids)
    stream = torch.cuda.current_stream()
    o_h, l_h = ab.attn_fwd_host(hq, hk, hv, doc_ids=hdoc, **kw)
    stream.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    o_d, l_d = ab.attn_fwd(q.cuda(), k.cuda(), v.cuda(),
                           doc_ids=None if doc_ids is None else doc_ids.cuda(), **kw)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())
    ro, rl = oracle.attn_fwd(q, k, v, doc_ids=doc_ids, **kw)
    compare(o_h, l_h, ro, rl, str(case))


def test_host_call_reuses_workspace_and_outputs():
    """Two calls on one stream with the same workspace and output buffers:
    the second call's uploads wait for the first call's downloads."""
    q1, k1, v1, _, _ = random_case(11, 2, 4, 4, 512, 512, 64)
    q2, k2, v2, _, _ = random_case(12, 2, 4, 4, 512, 512, 64)
    ws = torch.empty(ab.attn_fwd_host_workspace_size(2, 4, 4, 512, 512, 64), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty(q1.shape, dtype=torch.bfloat16).pin_memory()
    lse = torch.empty(2, 4, 512, dtype=torch.float32).pin_memory()
    hs = [tuple(t.pin_memory() for t in trip) for trip in ((q1, k1, v1), (q2, k2, v2))]
    ab.attn_fwd_host(*hs[0], mask="causal", o=o, lse=lse, workspace=ws)
    torch.cuda.current_stream().synchronize()
    o_first = o.clone()
    ab.attn_fwd_host(*hs[0], mask="causal", o=o, lse=lse, workspace=ws)
    ab.attn_fwd_host(*hs[1], mask="causal", o=o, lse=lse, workspace=ws)
    torch.cuda.current_stream().synchronize()
    o2, l2 = ab.attn_fwd(q2.cuda(), k2.cuda(), v2.cuda(), mask="causal")
    torch.cuda.synchronize()
    assert torch.equal(o, o2.cpu()) and torch.equal(lse, l2.cpu())
    assert not torch.equal(o_first, o)


def test_host_call_rejects_a_small_workspace():
    q, k, v, _, _ = random_case(13, 1, 2, 2, 128, 128, 64)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(ab.AttnError) as e:
        ab.attn_fwd_host(q, k, v, workspace=ws)
    assert e.value.status == ab.ATTN_ERR_WORKSPACE
