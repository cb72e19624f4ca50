"""Failure detection on the GPU without a fault: every wait in the kernels is
bounded; when one runs out the kernel records a timeout in the device error
word and returns.  The self-test kernel waits on an mbarrier that nothing
arrives on, so its wait must run out; the context must stay usable."""
import time

import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, to_dev
from workloads import random_case

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_timeout():
    st, _ = ab.attn_get_device_error()           # start from a clean error word
    assert st == ab.ATTN_OK
    t0 = time.time()
    ab.attn_selftest_wait_timeout()
    st, bits = ab.attn_get_device_error()        # synchronises the stream
    elapsed = time.time() - t0
    assert st == ab.ATTN_ERR_TIMEOUT and bits != 0
    assert elapsed < 30.0                         # the wait gave up by itself
    st, bits = ab.attn_get_device_error()        # read-and-clear
    assert st == ab.ATTN_OK and bits == 0


def test_context_usable_after_a_timeout():
    ab.attn_selftest_wait_timeout()
    ab.attn_get_device_error()
    q, k, v, _, _ = random_case(77, 1, 2, 2, 300, 300, 64)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ab.attn_fwd(qd, kd, vd, mask="causal")
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    ro, rl = oracle.attn_fwd(q, k, v, mask="causal")
    compare(o, lse, ro, rl, "after timeout")
