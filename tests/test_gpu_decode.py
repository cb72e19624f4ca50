"""GPU parity of attn_decode_splitkv (split-KV decode + combine) against the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import sm_attn_fwd_b200 as ab
from tests.gpu_helpers import compare, to_dev
from workloads import DECODE_LQ1, DECODE_LQ16, make_inputs, random_case

pytestmark = pytest.mark.gpu


def _poison_tail(k, v, kv_lens):
    """NaN past kv_lens[b]: the decode must never use those rows."""
    k, v = k.clone(), v.clone()
    for b, L in enumerate(kv_lens.tolist()):
        k[b, :, L:] = float("nan")
        v[b, :, L:] = float("nan")
    return k, v


def _decode(q, k, v, kv_lens, num_splits=0, scale=None):
    qd, kd, vd, kl = to_dev(q, k, v, kv_lens)
    o, lse = ab.attn_decode_splitkv(qd, kd, vd, kl, num_splits=num_splits, scale=scale)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    return o, lse


SMALL = [
    # seed, B, Hq, Hkv, Lq, Lk_max, d, (lo, hi), num_splits
    (1, 2, 8, 1, 1, 300, 128, (1, 300), 0),
    (2, 3, 16, 2, 1, 1000, 128, (1, 1000), 3),
    (3, 2, 16, 2, 16, 700, 128, (100, 700), 0),
    (4, 2, 4, 4, 3, 513, 64, (1, 513), 5),
    (5, 1, 64, 8, 16, 2048, 128, (2048, 2048), 4),
    (6, 4, 8, 8, 1, 129, 64, (1, 129), 0),
    (7, 2, 32, 2, 16, 640, 128, (1, 640), 2),          # 16 x 16 = 256 rows: two row tiles
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"s{c[0]}_lq{c[4]}_lk{c[5]}_d{c[6]}_ns{c[8]}")
def test_small_decode_with_poisoned_tail(case):
    seed, B, Hq, Hkv, Lq, Lk, d, rng, ns = case
    q, k, v, _, kv = random_case(seed, B, Hq, Hkv, Lq, Lk, d, kv_len_range=rng)
    kp, vp = _poison_tail(k, v, kv)
    o, lse = _decode(q, kp, vp, kv, num_splits=ns)
    ro, rl = oracle.attn_fwd(q, k, v, kv_lens=kv)
    compare(o, lse, ro, rl, str(case))


def test_partials_in_workspace_match_oracle_splits():
    """The documented workspace holds each split's normalised O_s and LSE_s."""
    B, Hq, Hkv, Lq, Lk, d = 2, 16, 2, 2, 900, 128
    q, k, v, _, kv = random_case(21, B, Hq, Hkv, Lq, Lk, d, kv_len_range=(1, Lk))
    ns, chunk = ab.attn_decode_num_splits(B, Hq, Hkv, Lq, Lk, d, 4)
    assert ns * chunk >= Lk and chunk % 128 == 0
    ws_bytes = ab.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, d, 4)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    qd, kd, vd, kl = to_dev(q, k, v, kv)
    ab.attn_decode_splitkv(qd, kd, vd, kl, num_splits=4, workspace=ws)
    torch.cuda.synchronize()
    nrows = B * Hq * Lq
    o_bytes = ns * nrows * d * 4
    off = (o_bytes + 255) // 256 * 256
    ws_o = ws[:o_bytes].view(torch.float32).view(ns, nrows, d)
    ws_l = ws[off:off + ns * nrows * 4].view(torch.float32).view(ns, nrows)
    ro, rl = oracle.decode_partials(q, k, v, kv, chunk=chunk, nsplit=ns)
    b_of_row = np.arange(nrows) // (Hq * Lq)
    for s in range(ns):
        used = (s * chunk) < kv.numpy()[b_of_row]
        compare(ws_o[s][torch.from_numpy(np.nonzero(used)[0]).cuda()],
                ws_l[s][torch.from_numpy(np.nonzero(used)[0]).cuda()],
                ro[s][used], rl[s][used], f"split {s}")


def test_split_count_does_not_change_the_result_beyond_rounding():
    B, Hq, Hkv, Lq, Lk, d = 2, 8, 1, 1, 1500, 128
    q, k, v, _, kv = random_case(31, B, Hq, Hkv, Lq, Lk, d, kv_len_range=(700, 1500))
    ro, rl = oracle.attn_fwd(q, k, v, kv_lens=kv)
    for ns in (1, 2, 5, 12):
        o, lse = _decode(q, k, v, kv, num_splits=ns)
        compare(o, lse, ro, rl, f"ns={ns}")


def test_workspace_too_small_is_rejected():
    q, k, v, _, kv = random_case(41, 1, 8, 1, 1, 256, 128, kv_len_range=(1, 256))
    qd, kd, vd, kl = to_dev(q, k, v, kv)
    need = ab.attn_decode_workspace_size(1, 8, 1, 1, 256, 128, 0)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ab.AttnError) as e:
        ab.attn_decode_splitkv(qd, kd, vd, kl, workspace=ws)
    assert e.value.status == ab.ATTN_ERR_WORKSPACE


def test_bad_kv_len_is_flagged_not_faulted():
    q, k, v, _, _ = random_case(51, 2, 8, 1, 1, 256, 128)
    kv = torch.tensor([100, 9999], dtype=torch.int32)
    qd, kd, vd, kl = to_dev(q, k, v, kv)
    ab.attn_decode_splitkv(qd, kd, vd, kl)
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_ERR_INVALID_ARG and bits != 0
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK and bits == 0


@pytest.mark.parametrize("cfg", [DECODE_LQ1, DECODE_LQ16], ids=lambda c: c.name)
def test_config_decode_full(cfg):
    """Full-size decode, every sequence and every head.  The 8.6 GB cache is
    drawn on the GPU with the workload recipe (the draws the bench times);
    each sequence's first kv_lens[b] keys are copied back and checked against
    the oracle."""
    inp = make_inputs(cfg, device="cuda")
    o, lse = ab.attn_decode_splitkv(inp.q, inp.k, inp.v, inp.kv_lens)
    torch.cuda.synchronize()
    st, bits = ab.attn_get_device_error()
    assert st == ab.ATTN_OK, (st, bits)
    kv_host = inp.kv_lens.cpu()
    for b in range(cfg.B):
        L = int(kv_host[b])
        qs = inp.q[b:b + 1].cpu()
        ks = inp.k[b:b + 1, :, :L].cpu()
        vs = inp.v[b:b + 1, :, :L].cpu()
        ro, rl = oracle.attn_fwd(qs, ks, vs, scale=cfg.softmax_scale)
        compare(o[b:b + 1], lse[b:b + 1], ro, rl, f"{cfg.name} b={b}")


def test_decode_capturable_in_cuda_graph():
    q, k, v, _, kv = random_case(61, 2, 16, 2, 1, 900, 128, kv_len_range=(100, 900))
    qd, kd, vd, kl = to_dev(q, k, v, kv)
    ws = torch.empty(ab.attn_decode_workspace_size(2, 16, 2, 1, 900, 128), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty_like(qd)
    lse = torch.empty(2, 16, 1, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ab.attn_decode_splitkv(qd, kd, vd, kl, workspace=ws, o=o, lse=lse, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        ab.attn_decode_splitkv(qd, kd, vd, kl, workspace=ws, o=o, lse=lse, stream=s)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(q, k, v, kv_lens=kv)
    compare(o, lse, ro, rl, "decode graph")
