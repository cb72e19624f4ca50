"""attn_decode_splitkv_noalloc: the decode entry point for callers that cannot
allocate device memory (a plugin whose host owns every device allocation, or
a decode loop where cudaMalloc is not allowed).  It must give the same result
as attn_decode_splitkv, which takes a caller-allocated workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, to_dev
from workloads import random_case


def _raw_call(q, k, v, kv, o, lse, num_splits=0):
    """Call the entry point through the C ABI directly (ctypes)."""
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    lib = ab.load_library()
    P = ctypes.c_void_p
    return lib.attn_decode_splitkv_noalloc(
        P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(o.data_ptr()), P(lse.data_ptr()),
        P(kv.data_ptr()), B, Hq, Hkv, Lq, Lk, d, ctypes.c_float(d ** -0.5), num_splits,
        P(torch.cuda.current_stream().cuda_stream))


def test_oversize_request_is_rejected_before_any_launch():
    """B=64, Hq=64, Lq=16, Lk_max=32768, d=128 needs ~270 MB of workspace: more
    than the fixed 32 MiB, so the call returns ATTN_ERR_WORKSPACE at once."""
    lib = ab.load_library()
    A = ctypes.c_void_p(0x10000)
    st = lib.attn_decode_splitkv_noalloc(A, A, A, A, A, A, 64, 64, 8, 16, 32768, 128,
                                         ctypes.c_float(0.088), 0, None)
    assert st == ab.ATTN_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    """Both entry points run the same kernels with the same split plan, so the
    results must be identical bit for bit.  The cases go small, large, small:
    the shared array then holds stale partials of another shape when the last
    case runs, which an exact comparison would catch if they leaked in."""
    cases = [
        # seed, B, Hq, Hkv, Lq, Lk_max, d, kv range
        (102, 3, 16, 2, 4, 1000, 64, (1, 1000)),
        (101, 8, 64, 8, 1, 32768, 128, (8192, 32768)),
        (103, 5, 32, 4, 2, 3000, 128, (1, 3000)),
    ]
    for seed, B, Hq, Hkv, Lq, Lk, d, rng in cases:
        q, k, v, _, kv = random_case(seed, B, Hq, Hkv, Lq, Lk, d, kv_len_range=rng)
        qd, kd, vd, kvd = to_dev(q, k, v, kv)
        o_ref, lse_ref = ab.attn_decode_splitkv(qd, kd, vd, kvd)
        torch.cuda.synchronize()
        ref_o = o_ref.float().cpu().double().numpy()
        ref_l = lse_ref.cpu().double().numpy()
        o = torch.empty_like(qd)
        lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device="cuda")
        for call in range(2):
            o.fill_(float("nan"))
            lse.fill_(float("nan"))
            st = _raw_call(qd, kd, vd, kvd, o, lse)
            assert st == ab.ATTN_OK, ab.attn_status_string(st)
            torch.cuda.synchronize()
            dev_st, bits = ab.attn_get_device_error()
            assert dev_st == ab.ATTN_OK, (dev_st, bits)
            compare(o, lse, ref_o, ref_l, f"noalloc seed={seed} call={call}")
            assert torch.equal(o, o_ref), f"noalloc seed={seed} call={call}: O differs"
            assert torch.equal(lse, lse_ref), f"noalloc seed={seed} call={call}: LSE differs"
