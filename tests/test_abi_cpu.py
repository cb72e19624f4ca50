"""The C ABI without a GPU: the library loads, exports every function that
include/attn.h declares, and rejects invalid arguments on the host before
touching CUDA (so these calls are safe on a machine with no device)."""
import ctypes
import os
import re
import subprocess

import pytest

import sm_attn_fwd_b200 as ab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    assert set(declared_functions()) == set(ab.EXPORTED_SYMBOLS)


def test_binding_has_every_entry_point_under_its_name():
    """The Python binding offers each C entry point under the same name."""
    missing = [name for name in declared_functions()
               if not callable(getattr(ab, name, None)) or name not in ab.__all__]
    assert not missing, missing


def test_library_exports_every_declared_symbol():
    lib = ab.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", ab.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (attn_\w+)", out))
    assert set(declared_functions()) <= exported


def test_status_strings():
    names = {ab.ATTN_OK: "ATTN_OK", ab.ATTN_ERR_INVALID_ARG: "ATTN_ERR_INVALID_ARG",
             ab.ATTN_ERR_UNSUPPORTED: "ATTN_ERR_UNSUPPORTED",
             ab.ATTN_ERR_WORKSPACE: "ATTN_ERR_WORKSPACE", ab.ATTN_ERR_CUDA: "ATTN_ERR_CUDA",
             ab.ATTN_ERR_TIMEOUT: "ATTN_ERR_TIMEOUT"}
    for code, name in names.items():
        assert ab.attn_status_string(code) == name
    assert ab.attn_status_string(99) == "ATTN_ERR_UNKNOWN"


# Fake, 256-byte aligned addresses: validation must reject the call before
# any pointer is dereferenced or any CUDA call is made.
A = ctypes.c_void_p(0x10000)
M = ctypes.c_void_p(0x10008)  # misaligned for 16-byte operands


def _fwd(**kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, Hq=2, Hkv=1, Lq=8, Lk=8, d=64, scale=0.125,
                mask=0, wl=-1, wr=-1, bd=1, doc=None, stream=None)
    args.update(kw)
    return ab.load_library().attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"],
                                      args["B"], args["Hq"], args["Hkv"], args["Lq"], args["Lk"],
                                      args["d"], args["scale"], args["mask"], args["wl"],
                                      args["wr"], args["bd"], args["doc"], args["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), ab.ATTN_ERR_INVALID_ARG),
    (dict(o=M), ab.ATTN_ERR_INVALID_ARG),
    (dict(B=0), ab.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), ab.ATTN_ERR_INVALID_ARG),
    (dict(Lq=0), ab.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), ab.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), ab.ATTN_ERR_INVALID_ARG),
    (dict(mask=3), ab.ATTN_ERR_INVALID_ARG),
    (dict(wl=-2), ab.ATTN_ERR_INVALID_ARG),
    (dict(mask=2, bd=0), ab.ATTN_ERR_INVALID_ARG),
    (dict(doc=A, Lq=9, Lk=8), ab.ATTN_ERR_INVALID_ARG),
    (dict(d=96), ab.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), ab.ATTN_ERR_UNSUPPORTED),
    (dict(Lk=4096 * 128 + 1), ab.ATTN_ERR_UNSUPPORTED),
])
def test_attn_fwd_rejects_on_host(kw, status):
    assert _fwd(**kw) == status


def test_decode_split_plan_and_workspace_arithmetic():
    lib = ab.load_library()
    chunk = ctypes.c_int(0)
    # explicit split count: chunk = 128 * ceil(ceil(Lk / s) / 128)
    n = lib.attn_decode_num_splits(2, 16, 2, 1, 1000, 128, 3, ctypes.byref(chunk))
    assert (n, chunk.value) == (3, 384)
    n = lib.attn_decode_num_splits(2, 16, 2, 1, 1000, 128, 100, ctypes.byref(chunk))
    assert (n, chunk.value) == (8, 128)           # capped at ceil(1000 / 128)
    # library choice: chunks never exceed 8192 keys and cover Lk_max
    n = lib.attn_decode_num_splits(64, 64, 8, 1, 32768, 128, 0, ctypes.byref(chunk))
    assert chunk.value <= 12288 and chunk.value % 128 == 0 and n * chunk.value >= 32768
    assert (n, chunk.value) == (3, 11008)
    # few (b, kv head) units: at least two waves of CTAs over the SMs
    n = lib.attn_decode_num_splits(1, 8, 1, 1, 32768, 128, 0, ctypes.byref(chunk))
    assert n * 1 >= 2 * 148 or chunk.value == 128
    ws = lib.attn_decode_workspace_size(2, 16, 2, 1, 1000, 128, 3)
    nrows = 2 * 16 * 1
    o_bytes = 3 * nrows * 128 * 4
    assert ws == (o_bytes + 255) // 256 * 256 + 3 * nrows * 4
    assert lib.attn_decode_num_splits(2, 16, 3, 1, 1000, 128, 0, None) == -1
    assert lib.attn_decode_workspace_size(0, 16, 2, 1, 1000, 128, 0) == 0


def test_decode_rejects_on_host():
    lib = ab.load_library()
    args = [A, A, A, A, A, A, 2, 16, 2, 1, 1000, 128, 0.125, 0, A, 1 << 30, None]
    assert lib.attn_decode_splitkv(*args[:5], None, *args[6:]) == ab.ATTN_ERR_INVALID_ARG
    bad_d = list(args)
    bad_d[11] = 80
    assert lib.attn_decode_splitkv(*bad_d) == ab.ATTN_ERR_UNSUPPORTED
    small_ws = list(args)
    small_ws[15] = 64
    assert lib.attn_decode_splitkv(*small_ws) == ab.ATTN_ERR_WORKSPACE
    no_ws = list(args)
    no_ws[14] = None
    assert lib.attn_decode_splitkv(*no_ws) == ab.ATTN_ERR_WORKSPACE


def test_attn_fwd_varlen_rejects_on_host():
    lib = ab.load_library()
    #      q  k  v  o  lse cu_q cu_k B  Hq Hkv tq   tk   maxq d   scale mask wl  wr bd stream
    args = [A, A, A, A, A, A, A, 3, 8, 2, 500, 600, 300, 128, 0.125, 1, -1, -1, 1, None]

    def call(**over):
        a = list(args)
        for i, v in over.items():
            a[int(i[1:])] = v
        return lib.attn_fwd_varlen(*a)

    assert call(a5=None) == ab.ATTN_ERR_INVALID_ARG        # no cu_seqlens_q
    assert call(a6=ctypes.c_void_p(0x10002)) == ab.ATTN_ERR_INVALID_ARG  # cu_seqlens_k not int32-aligned
    assert call(a0=M) == ab.ATTN_ERR_INVALID_ARG           # q not 16-byte aligned
    assert call(a9=3) == ab.ATTN_ERR_INVALID_ARG           # Hq % Hkv != 0
    assert call(a12=0) == ab.ATTN_ERR_INVALID_ARG          # max_seqlen_q < 1
    assert call(a12=501) == ab.ATTN_ERR_INVALID_ARG        # max_seqlen_q > total_q
    assert call(a10=0) == ab.ATTN_ERR_INVALID_ARG          # total_q < 1
    assert call(a14=0.0) == ab.ATTN_ERR_INVALID_ARG        # scale
    assert call(a15=2, a18=0) == ab.ATTN_ERR_INVALID_ARG   # draft block < 1
    assert call(a16=-2) == ab.ATTN_ERR_INVALID_ARG         # window < -1
    assert call(a13=96) == ab.ATTN_ERR_UNSUPPORTED         # d


def test_attn_fwd_score_mod_rejects_on_host():
    lib = ab.load_library()
    #      q  k  v  o  lse B  Hq Hkv Lq   Lk   d   scale mask wl  wr bd doc  kind params stream
    args = [A, A, A, A, A, 2, 8, 2, 100, 100, 64, 0.125, 1, -1, -1, 1, None, 1, A, 0, None]
    assert lib.attn_fwd_score_mod(*args[:17], 7, A, 0, None) == ab.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_score_mod(*args[:17], 1, None, 0, None) == ab.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_score_mod(*args[:17], 1, ctypes.c_void_p(0x10002), 0, None) == \
        ab.ATTN_ERR_INVALID_ARG
    # relative-position table: R must be in [0, 2^20]
    assert lib.attn_fwd_score_mod(*args[:17], 2, A, -1, None) == ab.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_score_mod(*args[:17], 2, A, (1 << 20) + 1, None) == \
        ab.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_score_mod(*args[:17], 2, None, 4, None) == ab.ATTN_ERR_INVALID_ARG
    bad_d = list(args)
    bad_d[10] = 96
    assert lib.attn_fwd_score_mod(*bad_d) == ab.ATTN_ERR_UNSUPPORTED


def test_attn_bwd_rejects_on_host_and_sizes_its_workspace():
    lib = ab.load_library()
    B, Hq, Hkv, Lq, Lk, d = 2, 8, 2, 100, 130, 64
    need = lib.attn_bwd_workspace_size(B, Hq, Lq, d)
    rows = B * Hq * Lq
    assert need == (rows * d * 4 + 255) // 256 * 256 + rows * 4
    assert lib.attn_bwd_workspace_size(0, Hq, Lq, d) == 0
    #      q  k  v  o  lse dout dq dk dv
    ptrs = [A, A, A, A, A, A, A, A, A]
    tail = [B, Hq, Hkv, Lq, Lk, d, 0.125, 1, -1, -1, 1, None, A, need, None]
    assert lib.attn_bwd(*ptrs[:8], None, *tail) == ab.ATTN_ERR_INVALID_ARG       # no dv
    small = list(tail)
    small[13] = need - 1
    assert lib.attn_bwd(*ptrs, *small) == ab.ATTN_ERR_WORKSPACE
    d96 = list(tail)
    d96[5] = 96
    assert lib.attn_bwd(*ptrs, *d96) == ab.ATTN_ERR_UNSUPPORTED
    d128 = list(tail)                                  # d = 128 is built: its workspace is larger
    d128[5] = 128
    assert lib.attn_bwd(*ptrs, *d128) == ab.ATTN_ERR_WORKSPACE
    bad_ws = list(tail)
    bad_ws[12] = ctypes.c_void_p(0x10010)                                       # not 256-aligned
    assert lib.attn_bwd(*ptrs, *bad_ws) == ab.ATTN_ERR_INVALID_ARG


def test_attn_fwd_host_sizes_its_workspace_and_rejects_on_host():
    lib = ab.load_library()
    B, Hq, Hkv, Lq, Lk, d = 2, 8, 2, 100, 130, 64

    def up(x):
        return (x + 255) // 256 * 256
    qb, kb = B * Hq * Lq * d * 2, B * Hkv * Lk * d * 2
    base = up(qb) + 2 * up(kb) + up(qb) + up(B * Hq * Lq * 4)
    assert lib.attn_fwd_host_workspace_size(B, Hq, Hkv, Lq, Lk, d, 0) == base
    assert lib.attn_fwd_host_workspace_size(B, Hq, Hkv, Lq, Lk, d, 1) == base + up(B * Lk * 4)
    assert lib.attn_fwd_host_workspace_size(B, 7, Hkv, Lq, Lk, d, 0) == 0
    h = ctypes.c_void_p(0x1000)   # host pointers are only passed to copies; nothing is queued
    args = [h, h, h, h, h, B, Hq, Hkv, Lq, Lk, d, 0.125, 1, -1, -1, 1, None]
    assert lib.attn_fwd_host(*args, None, 0, None) == ab.ATTN_ERR_WORKSPACE
    assert lib.attn_fwd_host(*args, ctypes.c_void_p(0x10010), base, None) == ab.ATTN_ERR_WORKSPACE
    assert lib.attn_fwd_host(*args, A, base - 1, None) == ab.ATTN_ERR_WORKSPACE
    bad = list(args)
    bad[6] = 3                                                            # Hq % Hkv != 0
    assert lib.attn_fwd_host(*bad, A, base, None) == ab.ATTN_ERR_INVALID_ARG
    bad = list(args)
    bad[10] = 96                                                          # d
    assert lib.attn_fwd_host(*bad, A, 1 << 30, None) == ab.ATTN_ERR_UNSUPPORTED
    bad = list(args)
    bad[12] = 7                                                           # mask kind
    assert lib.attn_fwd_host(*bad, A, base, None) == ab.ATTN_ERR_INVALID_ARG
    with pytest.raises(ValueError, match="host"):
        import torch
        ab.attn_fwd_host(torch.zeros(1, 2, 8, 64, dtype=torch.float32),
                         torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16),
                         torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16))


def test_binding_checks_tensors_before_calling_the_library():
    """The Python binding rejects host tensors, wrong dtypes and wrong ranks itself."""
    import torch
    q4 = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)          # host tensor
    with pytest.raises(ValueError, match="CUDA"):
        ab.attn_fwd(q4, q4, q4)
    with pytest.raises(ValueError, match="CUDA"):
        ab.attn_fwd_score_mod(q4, q4, q4, alibi_slopes=torch.zeros(2))
    q3 = torch.zeros(8, 2, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 8], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        ab.attn_fwd_varlen(q3, q3, q3, cu, cu, 8)
    lse = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="CUDA"):
        ab.attn_bwd(q4, q4, q4, q4, lse, q4)


def test_decode_score_mod_rejects_on_host():
    lib = ab.load_library()
    #       q  k  v  o  lse kv B  Hq Hkv Lq Lk    d    scale  ns
    head = [A, A, A, A, A, A, 2, 16, 2, 1, 1000, 128, 0.125, 0]
    ws = ctypes.c_void_p(0x100000)
    need = lib.attn_decode_workspace_size(2, 16, 2, 1, 1000, 128, 0)
    tail = [ws, need, None]
    call = lib.attn_decode_splitkv_score_mod
    assert call(*head, 7, A, 0, *tail) == ab.ATTN_ERR_INVALID_ARG          # unknown kind
    assert call(*head, 1, None, 0, *tail) == ab.ATTN_ERR_INVALID_ARG       # no slopes
    assert call(*head, 2, A, -1, *tail) == ab.ATTN_ERR_INVALID_ARG         # R < 0
    assert call(*head, 2, A, (1 << 20) + 1, *tail) == ab.ATTN_ERR_INVALID_ARG
    assert call(*head, 1, A, 0, ws, need - 256, None) == ab.ATTN_ERR_WORKSPACE
    #        q  k  v  table o  lse kv B  Hq Hkv Lq P    pps np   d    scale  ns
    phead = [A, A, A, A, A, A, A, 2, 16, 2, 1, 16, 8, 16, 128, 0.125, 0]
    pcall = lib.attn_decode_paged_score_mod
    assert pcall(*phead, 9, A, 0, *tail) == ab.ATTN_ERR_INVALID_ARG
    assert pcall(*phead, 2, None, 3, *tail) == ab.ATTN_ERR_INVALID_ARG
    bad_page = list(phead)
    bad_page[11] = 24                                                     # not a power of two
    assert pcall(*bad_page, 1, A, 0, *tail) == ab.ATTN_ERR_INVALID_ARG


def test_decode_score_mod_binding_rejects_bad_modifiers():
    """The binding checks the modifier tensors before anything reaches the device."""
    import torch
    q = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    kv = torch.tensor([128], dtype=torch.int32)
    slopes = torch.ones(8)
    table = torch.zeros(8, 5)
    with pytest.raises(ValueError):   # both modifiers
        ab.attn_decode_splitkv_score_mod(q, k, k, kv, alibi_slopes=slopes, rel_bias=(table, 2))
    with pytest.raises(ValueError):   # slopes not on the device
        ab.attn_decode_splitkv_score_mod(q, k, k, kv, alibi_slopes=slopes)
    with pytest.raises(ValueError):   # table not [Hq, 2R + 1] on the device
        ab.attn_decode_paged_score_mod(q, k, k, kv.view(1, 1), kv, rel_bias=(table, 3))


def test_decode_split_plan_rule():
    """Without num_splits: at least two waves of CTAs over the SMs, and chunks of
    at most 12288 keys (a multiple of 128) covering Lk_max."""
    lib = ab.load_library()
    chunk = ctypes.c_int(0)
    # many (b, kv head) units: the chunk cap alone decides
    for lk, want in ((12288, 1), (12289, 2), (32768, 3), (65536, 6), (131072, 11)):
        n = lib.attn_decode_num_splits(64, 64, 8, 1, lk, 128, 0, ctypes.byref(chunk))
        assert n == want, (lk, n)
        assert chunk.value % 128 == 0 and chunk.value <= 12288 and n * chunk.value >= lk
        assert (n - 1) * chunk.value < lk  # no empty split
    # an explicit count is taken as given (up to one split per key tile)
    assert lib.attn_decode_num_splits(64, 64, 8, 1, 32768, 128, 5, None) == 5
    assert lib.attn_decode_num_splits(1, 8, 1, 1, 300, 128, 50, None) == 3
