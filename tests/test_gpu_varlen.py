"""GPU parity of attn_fwd_varlen (packed sequences) against the oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare as _compare
from workloads import packed_case

pytestmark = pytest.mark.gpu


def compare(o, lse, ro, rl, what):
    """O [total, Hq, d] and LSE [Hq, total]: compare row by row (LSE as [total, Hq])."""
    return _compare(o, lse.t(), ro, np.ascontiguousarray(rl.T), what)


def _run(q, k, v, cu_q, cu_k, max_q, **kw):
    qd, kd, vd = (t.cuda().contiguous() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))  # every row must be written
    lse = torch.full((q.shape[1], q.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
    ab.attn_fwd_varlen(qd, kd, vd, cu_q.cuda(), cu_k.cuda(), max_q, o=o, lse=lse, **kw)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    return o, lse


CASES = [
    # seed, lens_q, lens_k, Hq, Hkv, d, mask, window, bd
    (1, [128], [128], 2, 2, 64, "causal", (-1, -1), 1),
    (2, [1, 300, 77, 129, 1000], None, 4, 2, 64, "causal", (-1, -1), 1),
    (3, [500, 3, 256, 700], None, 2, 1, 128, "none", (-1, -1), 1),
    (4, [640, 130, 33], None, 2, 2, 128, "causal", (100, 0), 1),
    (5, [16, 16, 16, 48], [2064, 700, 16, 130], 4, 4, 128, "draft", (512, 512), 16),
    (6, [5, 260, 1], [900, 260, 300], 8, 2, 64, "causal", (-1, -1), 1),
    (7, [300, 451], None, 2, 2, 64, "none", (37, 37), 1),
    (8, [2, 0, 129, 7], [2, 5, 0, 300], 2, 1, 64, "causal", (-1, -1), 1),  # empty sequences
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c[0]}_{c[6]}_d{c[5]}")
def test_packed_sequences_match_oracle(case):
    seed, lq, lk, Hq, Hkv, d, mask, window, bd = case
    lk = lk or lq
    q, k, v, cu_q, cu_k = packed_case(seed, lq, lk, Hq, Hkv, d)
    kw = dict(scale=1.0 / math.sqrt(d), mask=mask, window=window, draft_block=bd)
    o, lse = _run(q, k, v, cu_q, cu_k, max(lq), **kw)
    ro, rl = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, **kw)
    compare(o, lse, ro, rl, str(case))


@pytest.mark.parametrize("d", [64, 128])
def test_equal_lengths_bit_identical_to_dense(d):
    """B sequences of one length packed back to back give the same bits as the
    [B, H, L, d] call: the tiles and their order of arithmetic are the same."""
    B, H, L = 3, 4, 333
    q, k, v, cu_q, cu_k = packed_case(11, [L] * B, [L] * B, H, H, d)
    o, lse = _run(q, k, v, cu_q, cu_k, L, mask="causal")
    dense = lambda t: t.reshape(B, L, H, d).permute(0, 2, 1, 3).contiguous().cuda()
    od, ld = ab.attn_fwd(dense(q), dense(k), dense(v), mask="causal")
    torch.cuda.synchronize()
    assert torch.equal(o.reshape(B, L, H, d).permute(0, 2, 1, 3), od)
    assert torch.equal(lse.reshape(H, B, L).permute(1, 0, 2), ld)


def test_output_guard_bytes_untouched():
    q, k, v, cu_q, cu_k = packed_case(12, [200, 57], [200, 57], 2, 2, 64)
    n_o, n_l = q.numel(), 2 * q.shape[0]
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 1024,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[:n_o].view(q.shape)
    lse = l_buf[:n_l].view(2, q.shape[0])
    ab.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(), 200,
                       mask="causal", o=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(o_buf[n_o:] == 7.0) and torch.all(l_buf[n_l:] == 7.0)
    ro, rl = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, mask="causal")
    compare(o, lse, ro, rl, "guard")


def test_bad_cu_seqlens_flagged_and_skipped():
    """A sequence with bounds out of order, or longer than max_seqlen_q, is
    skipped and reported; the other sequences are still right."""
    q, k, v, _, _ = packed_case(13, [100, 100, 100], [100, 100, 100], 2, 2, 64)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    good = torch.tensor([0, 100, 200, 300], dtype=torch.int32)
    ro, rl = oracle.attn_fwd_varlen(q, k, v, good, good, mask="causal")
    bad_q = torch.tensor([0, 100, 200, 150], dtype=torch.int32, device="cuda")  # sequence 2 reversed
    o = torch.zeros_like(qd)
    lse = torch.zeros(2, 300, dtype=torch.float32, device="cuda")
    ab.attn_fwd_varlen(qd, kd, vd, bad_q, good.cuda(), 100, mask="causal", o=o, lse=lse)
    torch.cuda.synchronize()
    st, _ = ab.attn_get_device_error()
    assert st == ab.ATTN_ERR_INVALID_ARG
    compare(o[:200], lse[:, :200], ro[:200], rl[:, :200], "sequences 0 and 1")
    ab.attn_fwd_varlen(qd, kd, vd, good.cuda(), good.cuda(), 64, mask="causal", o=o, lse=lse)
    torch.cuda.synchronize()
    st, _ = ab.attn_get_device_error()                    # every sequence longer than 64
    assert st == ab.ATTN_ERR_INVALID_ARG
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK and bits == 0


def test_bench_packed_workload_sampled_sequences():
    """The benchmark's packed workload (16 causal sequences of 128-4096 tokens,
    H=16, d=64, seed 5) in one call; the longest, the shortest and two more
    sequences checked whole against the oracle."""
    from workloads import packed_case, packed_lengths
    lens = packed_lengths(5, 16, 128, 4096)
    q, k, v, cu_q, cu_k = packed_case(5, lens, lens, 16, 16, 64)
    qd, kd, vd, cqd, ckd = (t.cuda() for t in (q, k, v, cu_q, cu_k))
    o, lse = ab.attn_fwd_varlen(qd, kd, vd, cqd, ckd, max(lens), mask="causal")
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    order = sorted(range(16), key=lambda i: lens[i])
    for b in sorted({order[0], order[-1], order[5], order[10]}):
        t0, t1 = int(cu_q[b]), int(cu_q[b + 1])
        one = torch.tensor([0, t1 - t0], dtype=torch.int32)
        ro, rl = oracle.attn_fwd_varlen(q[t0:t1], k[t0:t1], v[t0:t1], one, one, mask="causal")
        compare(o[t0:t1], lse[:, t0:t1], ro, rl, f"sequence {b}")
