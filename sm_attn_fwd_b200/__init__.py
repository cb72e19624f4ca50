"""Python binding of the B200 attention C ABI (``include/attn.h``).

Argument marshalling only: every step of the computation runs in the CUDA
library ``_lib/libattn_b200.so``.  PyTorch supplies device memory and the
current stream.  There is no fallback path: if the library is missing or the
tensors are not on a CUDA device, the calls raise.

Entry points (same names as the C ABI):
  attn_fwd(q, k, v, ...)                 -> (o, lse)
  attn_fwd_host(q, k, v, ...)            -> (o, lse)   host tensors in and out
  attn_decode_splitkv(q, k, v, kv_lens, ...) -> (o, lse)
  attn_decode_num_splits(...), attn_decode_workspace_size(...)
  attn_get_device_error(stream=None)     -> (status, raw_bits)
  attn_status_string(status)             -> str
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

__all__ = [
    "AttnError", "ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED",
    "ATTN_ERR_WORKSPACE", "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT",
    "MASK_NONE", "MASK_CAUSAL", "MASK_DRAFT_BLOCK", "lib_path", "load_library",
    "attn_fwd", "attn_fwd_score_mod", "attn_fwd_varlen", "attn_fwd_varlen_score_mod",
    "attn_bwd", "attn_bwd_workspace_size", "attn_decode_splitkv",
    "attn_fwd_host", "attn_fwd_host_workspace_size",
    "attn_decode_num_splits", "SCORE_MOD_NONE", "SCORE_MOD_ALIBI", "SCORE_MOD_REL_BIAS",
    "attn_decode_workspace_size", "attn_decode_paged", "attn_decode_splitkv_noalloc",
    "attn_decode_splitkv_score_mod", "attn_decode_paged_score_mod",
    "attn_get_device_error", "attn_selftest_wait_timeout", "attn_status_string",
    "EXPORTED_SYMBOLS",
]

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_WORKSPACE = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_DRAFT_BLOCK = 2
SCORE_MOD_NONE = 0
SCORE_MOD_ALIBI = 1
SCORE_MOD_REL_BIAS = 2
_MASKS = {"none": MASK_NONE, "causal": MASK_CAUSAL, "draft": MASK_DRAFT_BLOCK}

EXPORTED_SYMBOLS = (
    "attn_fwd", "attn_fwd_score_mod", "attn_fwd_varlen", "attn_fwd_varlen_score_mod",
    "attn_fwd_host_workspace_size", "attn_fwd_host",
    "attn_bwd_workspace_size", "attn_bwd",
    "attn_decode_num_splits", "attn_decode_workspace_size",
    "attn_decode_splitkv", "attn_decode_paged", "attn_decode_splitkv_noalloc",
    "attn_decode_splitkv_score_mod", "attn_decode_paged_score_mod",
    "attn_get_device_error", "attn_selftest_wait_timeout", "attn_status_string",
)

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "_lib", "libattn_b200.so")
_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {attn_status_string(status)}")


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the CUDA library (building it first if it is absent and nvcc exists)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            from . import build as _build
            _build.build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.attn_fwd.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, i32,
                                 i32, P, P]
        lib.attn_fwd.restype = i32
        lib.attn_fwd_score_mod.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32,
                                           i32, i32, i32, P, i32, P, i32, P]
        lib.attn_fwd_score_mod.restype = i32
        lib.attn_fwd_host_workspace_size.argtypes = [i32] * 7
        lib.attn_fwd_host_workspace_size.restype = sz
        lib.attn_fwd_host.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                      i32, i32, P, P, sz, P]
        lib.attn_fwd_host.restype = i32
        lib.attn_bwd_workspace_size.argtypes = [i32, i32, i32, i32]
        lib.attn_bwd_workspace_size.restype = sz
        lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32,
                                 i32, i32, i32, P, P, sz, P]
        lib.attn_bwd.restype = i32
        lib.attn_fwd_varlen.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32,
                                        i32, i32, i32, i32, P]
        lib.attn_fwd_varlen.restype = i32
        lib.attn_fwd_varlen_score_mod.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                  i32, i32, f32, i32, i32, i32, i32, i32, P, i32,
                                                  P]
        lib.attn_fwd_varlen_score_mod.restype = i32
        lib.attn_decode_num_splits.argtypes = [i32] * 7 + [ctypes.POINTER(ctypes.c_int)]
        lib.attn_decode_num_splits.restype = i32
        lib.attn_decode_workspace_size.argtypes = [i32] * 7
        lib.attn_decode_workspace_size.restype = sz
        lib.attn_decode_splitkv.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32,
                                            i32, P, sz, P]
        lib.attn_decode_splitkv.restype = i32
        lib.attn_decode_paged.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                          i32, f32, i32, P, sz, P]
        lib.attn_decode_paged.restype = i32
        lib.attn_decode_splitkv_score_mod.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                      i32, f32, i32, i32, P, i32, P, sz, P]
        lib.attn_decode_splitkv_score_mod.restype = i32
        lib.attn_decode_paged_score_mod.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                    i32, i32, i32, f32, i32, i32, P, i32, P, sz,
                                                    P]
        lib.attn_decode_paged_score_mod.restype = i32
        lib.attn_decode_splitkv_noalloc.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                                    i32, f32, i32, P]
        lib.attn_decode_splitkv_noalloc.restype = i32
        lib.attn_get_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
        lib.attn_get_device_error.restype = i32
        lib.attn_selftest_wait_timeout.argtypes = [P]
        lib.attn_selftest_wait_timeout.restype = i32
        lib.attn_status_string.argtypes = [i32]
        lib.attn_status_string.restype = ctypes.c_char_p
        _lib = lib
        return lib


def attn_status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check_bf16(name, t, layout="[B, H, L, D]"):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != layout.count(",") + 1 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {layout} tensor")


def attn_fwd(q, k, v, *, scale=None, mask="none", window=(-1, -1), draft_block=1,
             doc_ids=None, o=None, lse=None, stream=None):
    """Prefill attention forward (see ``attn_fwd`` in include/attn.h).

    q: [B, Hq, Lq, d], k/v: [B, Hkv, Lk, d], bf16 CUDA tensors.  Returns
    (o bf16 [B, Hq, Lq, d], lse fp32 [B, Hq, Lq]).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16(name, t)
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if doc_ids is not None:
        if doc_ids.dtype != torch.int32 or not doc_ids.is_cuda or not doc_ids.is_contiguous():
            raise ValueError("doc_ids must be a contiguous int32 CUDA tensor [B, Lk]")
    mk = mask if isinstance(mask, int) else _MASKS[mask]
    st = load_library().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq,
                                 Lk, d, float(scale), mk, int(window[0]), int(window[1]),
                                 int(draft_block), _ptr(doc_ids), _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd")
    return o, lse


def _check_host_bf16(name, t):
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bfloat16 [B, H, L, D] host tensor")


def attn_fwd_host_workspace_size(B, Hq, Hkv, Lq, Lk, d, with_doc_ids=False) -> int:
    return int(load_library().attn_fwd_host_workspace_size(B, Hq, Hkv, Lq, Lk, d,
                                                           int(bool(with_doc_ids))))


def attn_fwd_host(q, k, v, *, scale=None, mask="none", window=(-1, -1), draft_block=1,
                  doc_ids=None, o=None, lse=None, workspace=None, stream=None, device=None):
    """attn_fwd on host tensors (see ``attn_fwd_host`` in include/attn.h).

    q, k, v (and doc_ids) are contiguous CPU tensors, pinned for the copies to
    overlap the kernels; o and lse are CPU tensors (pinned ones are allocated
    when not given).  The copies and kernels are queued on ``stream``: the
    outputs are complete once it is synchronised (this wrapper does not wait).
    Returns (o, lse).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_host_bf16(name, t)
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32).pin_memory()
    if o.device.type != "cpu" or lse.device.type != "cpu":
        raise ValueError("o and lse must be host (CPU) tensors")
    if doc_ids is not None and (doc_ids.dtype != torch.int32 or doc_ids.device.type != "cpu"
                                or not doc_ids.is_contiguous()):
        raise ValueError("doc_ids must be a contiguous int32 host tensor [B, Lk]")
    need = attn_fwd_host_workspace_size(B, Hq, Hkv, Lq, Lk, d, doc_ids is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    mk = mask if isinstance(mask, int) else _MASKS[mask]
    st = load_library().attn_fwd_host(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lk, d, float(scale), mk,
        int(window[0]), int(window[1]), int(draft_block), _ptr(doc_ids), _ptr(workspace),
        workspace.numel(), _stream_handle(stream, dev))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_host")
    return o, lse


def _score_mod_args(Hq, alibi_slopes, rel_bias):
    """(kind, params tensor, arg) of the score modifier; at most one is given."""
    if alibi_slopes is not None and rel_bias is not None:
        raise ValueError("give alibi_slopes or rel_bias, not both")
    if alibi_slopes is not None:
        if (alibi_slopes.dtype != torch.float32 or not alibi_slopes.is_cuda
                or not alibi_slopes.is_contiguous() or alibi_slopes.numel() != Hq):
            raise ValueError("alibi_slopes must be a contiguous fp32 CUDA tensor [Hq]")
        return SCORE_MOD_ALIBI, alibi_slopes, 0
    if rel_bias is not None:
        table, rmax = rel_bias
        if (table.dtype != torch.float32 or not table.is_cuda or not table.is_contiguous()
                or tuple(table.shape) != (Hq, 2 * int(rmax) + 1)):
            raise ValueError("rel_bias table must be a contiguous fp32 CUDA tensor [Hq, 2R + 1]")
        return SCORE_MOD_REL_BIAS, table, int(rmax)
    return SCORE_MOD_NONE, None, 0


def attn_fwd_score_mod(q, k, v, *, alibi_slopes=None, rel_bias=None, scale=None, mask="none",
                       window=(-1, -1), draft_block=1, doc_ids=None, o=None, lse=None,
                       stream=None):
    """attn_fwd with a score modifier (see ``attn_fwd_score_mod`` in include/attn.h):
    ALiBi, S_ij += alibi_slopes[hq] * (j - p) (fp32 CUDA tensor [Hq]), or the
    relative-position bias rel_bias = (table, R), S_ij += table[hq, clamp(j - p, -R, R) + R]
    (fp32 CUDA tensor [Hq, 2R + 1])."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16(name, t)
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    kind, params, arg = _score_mod_args(Hq, alibi_slopes, rel_bias)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if doc_ids is not None:
        if doc_ids.dtype != torch.int32 or not doc_ids.is_cuda or not doc_ids.is_contiguous():
            raise ValueError("doc_ids must be a contiguous int32 CUDA tensor [B, Lk]")
    mk = mask if isinstance(mask, int) else _MASKS[mask]
    st = load_library().attn_fwd_score_mod(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                           Hkv, Lq, Lk, d, float(scale), mk, int(window[0]),
                                           int(window[1]), int(draft_block), _ptr(doc_ids),
                                           kind, _ptr(params), arg,
                                           _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_score_mod")
    return o, lse


def attn_bwd_workspace_size(B, Hq, Lq, d) -> int:
    """Bytes of workspace attn_bwd needs (see ``attn_bwd_workspace_size`` in include/attn.h)."""
    n = load_library().attn_bwd_workspace_size(B, Hq, Lq, d)
    if n == 0:
        raise AttnError(ATTN_ERR_INVALID_ARG, "attn_bwd_workspace_size")
    return int(n)


def attn_bwd(q, k, v, o, lse, dout, *, scale=None, mask="none", window=(-1, -1), draft_block=1,
             doc_ids=None, workspace=None, dq=None, dk=None, dv=None, stream=None):
    """Gradients of attn_fwd (see ``attn_bwd`` in include/attn.h): returns (dq, dk, dv).

    q, o, dout: [B, Hq, Lq, d]; k, v: [B, Hkv, Lk, d] bf16 CUDA tensors; lse: fp32
    [B, Hq, Lq] from attn_fwd with the same arguments.
    """
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_bf16(name, t)
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk, _ = k.shape
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, Hq, Lq]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    lib = load_library()
    need = lib.attn_bwd_workspace_size(B, Hq, Lq, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if doc_ids is not None:
        if doc_ids.dtype != torch.int32 or not doc_ids.is_cuda or not doc_ids.is_contiguous():
            raise ValueError("doc_ids must be a contiguous int32 CUDA tensor [B, Lk]")
    mk = mask if isinstance(mask, int) else _MASKS[mask]
    st = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                      _ptr(dk), _ptr(dv), B, Hq, Hkv, Lq, Lk, d, float(scale), mk, int(window[0]),
                      int(window[1]), int(draft_block), _ptr(doc_ids), _ptr(workspace),
                      workspace.numel() * workspace.element_size(),
                      _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, *, scale=None,
                    mask="none", window=(-1, -1), draft_block=1, alibi_slopes=None,
                    rel_bias=None, o=None, lse=None, stream=None):
    """Prefill forward over packed sequences (see ``attn_fwd_varlen`` and
    ``attn_fwd_varlen_score_mod`` in include/attn.h).

    q: [total_q, Hq, d], k/v: [total_k, Hkv, d] bf16 CUDA tensors (token-major);
    cu_seqlens_q/k: int32 CUDA tensors [B + 1].  Optional score modifier as in
    ``attn_fwd_score_mod``.  Returns (o bf16 [total_q, Hq, d], lse fp32 [Hq, total_q]).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16(name, t, "[total, H, D]")
    total_q, Hq, d = q.shape
    total_k, Hkv, _ = k.shape
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor [B + 1]")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 >= 2 entries")
    B = cu_seqlens_q.numel() - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    mk = mask if isinstance(mask, int) else _MASKS[mask]
    kind, params, arg = _score_mod_args(Hq, alibi_slopes, rel_bias)
    st = load_library().attn_fwd_varlen_score_mod(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B,
        Hq, Hkv, total_q, total_k, int(max_seqlen_q), d, float(scale), mk, int(window[0]),
        int(window[1]), int(draft_block), kind, _ptr(params), arg,
        _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_varlen")
    return o, lse


def attn_decode_num_splits(B, Hq, Hkv, Lq, Lk_max, d, num_splits=0):
    """(nsplit, chunk_keys) that attn_decode_splitkv uses for these arguments."""
    chunk = ctypes.c_int(0)
    n = load_library().attn_decode_num_splits(B, Hq, Hkv, Lq, Lk_max, d, num_splits,
                                              ctypes.byref(chunk))
    if n < 0:
        raise AttnError(ATTN_ERR_INVALID_ARG, "attn_decode_num_splits")
    return int(n), int(chunk.value)


def attn_fwd_varlen_score_mod(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, *,
                              alibi_slopes=None, rel_bias=None, **kw):
    """attn_fwd_varlen with a score modifier (see ``attn_fwd_varlen_score_mod`` in
    include/attn.h): ``alibi_slopes`` or ``rel_bias`` as in ``attn_fwd_score_mod``,
    each sequence's own positions; the other arguments as attn_fwd_varlen."""
    if alibi_slopes is None and rel_bias is None:
        raise ValueError("give alibi_slopes or rel_bias")
    return attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                           alibi_slopes=alibi_slopes, rel_bias=rel_bias, **kw)


def attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk_max, d, num_splits=0) -> int:
    n = load_library().attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk_max, d, num_splits)
    if n == 0:
        raise AttnError(ATTN_ERR_INVALID_ARG, "attn_decode_workspace_size")
    return int(n)


def attn_decode_splitkv(q, k_cache, v_cache, kv_lens, *, scale=None, num_splits=0,
                        workspace=None, o=None, lse=None, stream=None):
    """Split-KV decode (see ``attn_decode_splitkv`` in include/attn.h).

    q: [B, Hq, Lq, d]; k_cache/v_cache: [B, Hkv, Lk_max, d]; kv_lens: int32 [B]
    on the device.  ``workspace`` (uint8 CUDA tensor) is allocated here when
    not given.  Returns (o, lse).
    """
    return _decode(q, k_cache, v_cache, kv_lens, scale, num_splits, workspace, o, lse, stream,
                   None)


def attn_decode_splitkv_score_mod(q, k_cache, v_cache, kv_lens, *, alibi_slopes=None,
                                  rel_bias=None, scale=None, num_splits=0, workspace=None,
                                  o=None, lse=None, stream=None):
    """attn_decode_splitkv with a score modifier (see ``attn_decode_splitkv_score_mod``
    in include/attn.h): ``alibi_slopes`` (fp32 CUDA tensor [Hq]) or ``rel_bias`` =
    (table fp32 CUDA tensor [Hq, 2R + 1], R), with query row i of sequence b at
    position kv_lens[b] - Lq + i.  Returns (o, lse)."""
    mod = _score_mod_args(q.shape[1], alibi_slopes, rel_bias)
    return _decode(q, k_cache, v_cache, kv_lens, scale, num_splits, workspace, o, lse, stream,
                   mod)


def _decode(q, k_cache, v_cache, kv_lens, scale, num_splits, workspace, o, lse, stream, mod):
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_bf16(name, t)
    if kv_lens.dtype != torch.int32 or not kv_lens.is_cuda or not kv_lens.is_contiguous():
        raise ValueError("kv_lens must be a contiguous int32 CUDA tensor [B]")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk_max, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk_max, d, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    head = (_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), _ptr(kv_lens), B, Hq, Hkv,
            Lq, Lk_max, d, float(scale), int(num_splits))
    tail = (_ptr(workspace), ws_bytes, _stream_handle(stream, q.device))
    if mod is None:
        name = "attn_decode_splitkv"
        st = load_library().attn_decode_splitkv(*head, *tail)
    else:
        name = "attn_decode_splitkv_score_mod"
        kind, params, arg = mod
        st = load_library().attn_decode_splitkv_score_mod(*head, kind, _ptr(params), arg, *tail)
    if st != ATTN_OK:
        raise AttnError(st, name)
    return o, lse


def attn_decode_paged(q, k_pages, v_pages, block_table, kv_lens, *, scale=None, num_splits=0,
                      workspace=None, o=None, lse=None, stream=None):
    """Split-KV decode over a paged cache (see ``attn_decode_paged`` in include/attn.h).

    q: [B, Hq, Lq, d]; k_pages/v_pages: [num_pages, Hkv, page_size, d] bf16;
    block_table: int32 [B, pages_per_seq]; kv_lens: int32 [B] (device).
    """
    return _decode_paged(q, k_pages, v_pages, block_table, kv_lens, scale, num_splits, workspace,
                         o, lse, stream, None)


def attn_decode_paged_score_mod(q, k_pages, v_pages, block_table, kv_lens, *, alibi_slopes=None,
                                rel_bias=None, scale=None, num_splits=0, workspace=None, o=None,
                                lse=None, stream=None):
    """attn_decode_paged with a score modifier, as ``attn_decode_splitkv_score_mod``
    (see ``attn_decode_paged_score_mod`` in include/attn.h)."""
    mod = _score_mod_args(q.shape[1], alibi_slopes, rel_bias)
    return _decode_paged(q, k_pages, v_pages, block_table, kv_lens, scale, num_splits, workspace,
                         o, lse, stream, mod)


def _decode_paged(q, k_pages, v_pages, block_table, kv_lens, scale, num_splits, workspace, o,
                  lse, stream, mod):
    for name, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        _check_bf16(name, t)
    for name, t in (("block_table", block_table), ("kv_lens", kv_lens)):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    B, Hq, Lq, d = q.shape
    num_pages, Hkv, page_size, _ = k_pages.shape
    pages_per_seq = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = attn_decode_workspace_size(B, Hq, Hkv, Lq, pages_per_seq * page_size, d, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    head = (_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(o), _ptr(lse),
            _ptr(kv_lens), B, Hq, Hkv, Lq, page_size, pages_per_seq, num_pages, d, float(scale),
            int(num_splits))
    tail = (_ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream_handle(stream, q.device))
    if mod is None:
        name = "attn_decode_paged"
        st = load_library().attn_decode_paged(*head, *tail)
    else:
        name = "attn_decode_paged_score_mod"
        kind, params, arg = mod
        st = load_library().attn_decode_paged_score_mod(*head, kind, _ptr(params), arg, *tail)
    if st != ATTN_OK:
        raise AttnError(st, name)
    return o, lse


def attn_decode_splitkv_noalloc(q, k_cache, v_cache, kv_lens, *, scale=None, num_splits=0,
                                o=None, lse=None, stream=None):
    """Split-KV decode with the library's fixed device workspace (see
    ``attn_decode_splitkv_noalloc`` in include/attn.h): for callers that
    cannot allocate.  ``o`` and ``lse`` should be passed in by such callers;
    they are only allocated here as a convenience when omitted."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_bf16(name, t)
    if kv_lens.dtype != torch.int32 or not kv_lens.is_cuda or not kv_lens.is_contiguous():
        raise ValueError("kv_lens must be a contiguous int32 CUDA tensor [B]")
    B, Hq, Lq, d = q.shape
    _, Hkv, Lk_max, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    st = load_library().attn_decode_splitkv_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse), _ptr(kv_lens), B, Hq, Hkv,
        Lq, Lk_max, d, float(scale), int(num_splits), _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_decode_splitkv_noalloc")
    return o, lse


def attn_selftest_wait_timeout(stream=None):
    """Enqueue the failure-detection self-test kernel (see include/attn.h)."""
    dev = torch.cuda.current_device()
    st = load_library().attn_selftest_wait_timeout(_stream_handle(stream, dev))
    if st != ATTN_OK:
        raise AttnError(st, "attn_selftest_wait_timeout")


def attn_get_device_error(stream=None):
    """Synchronise the stream and read/clear the device error word: (status, raw_bits)."""
    bits = ctypes.c_int(0)
    dev = torch.cuda.current_device()
    st = load_library().attn_get_device_error(_stream_handle(stream, dev), ctypes.byref(bits))
    return int(st), int(bits.value)
