"""Attention oracle (CPU, double precision) — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it; this module only marshals arguments to the plain C
implementation in ``attn_oracle.c`` (built with gcc + OpenMP on first use).

Functions cite the passages they follow in ``attn_oracle.c``.  In short:
``attn_fwd`` is the plain definition softmax(mask(QK^T * scale)) V with a
two-pass softmax over each materialised score row ("FlashAttention 2 原理与
PyTorch 实战", sections 一 and 3.2); ``mask`` is the mask_mod predicate
("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", sections 1 and 3);
``decode_partials`` and ``combine`` are the split-KV decode written out as
chunk-then-merge (same page, section 1); ``paged_gather`` reads a paged cache
through its block table; ``attn_fwd_varlen`` applies the definition to each of
a batch of packed sequences; ``alibi_slopes`` adds the ALiBi score_mod (same
page, section 1); ``attn_bwd`` writes out the gradients dQ, dK, dV of the
definition on whole score rows (numpy, double).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle_attn.so")
_lock = threading.Lock()
_lib = None

_MASKS = {"none": 0, "causal": 1, "draft": 2}


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` into ``_build/liboracle_attn.so`` (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_mask.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P]
            lib.oracle_mask.restype = i32
            lib.oracle_count_pairs.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, i32]
            lib.oracle_count_pairs.restype = i64
            lib.oracle_attn_rows.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, i32, i32,
                                             i32, i32, P, P, P, i64, P, P, i32]
            lib.oracle_attn_rows.restype = i32
            lib.oracle_attn_rows_alibi.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, i32,
                                                   i32, i32, i32, P, P, P, i64, P, P, i32]
            lib.oracle_attn_rows_alibi.restype = i32
            lib.oracle_attn_rows_relbias.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64,
                                                     i32, i32, i32, i32, P, P, i32, P, i64, P, P,
                                                     i32]
            lib.oracle_attn_rows_relbias.restype = i32
            lib.oracle_attn_rows_mod.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, i32,
                                                 i32, i32, i32, P, P, P, P, i32, P, i64, P, P,
                                                 i32]
            lib.oracle_attn_rows_mod.restype = i32
            lib.oracle_decode_partials.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, f64,
                                                   i32, i32, P, P, i32]
            lib.oracle_decode_partials.restype = i32
            lib.oracle_combine.argtypes = [P, P, i32, i64, i32, P, P]
            lib.oracle_combine.restype = i32
            lib.oracle_paged_gather.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P]
            lib.oracle_paged_gather.restype = i32
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = i32
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _bf16_bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array of the bits."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("oracle expects bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError(f"oracle expects bf16 inputs, got {x.dtype}")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _i32(x):
    if x is None:
        return None
    if not isinstance(x, np.ndarray):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _mask_code(mask):
    return mask if isinstance(mask, int) else _MASKS[mask]


def mask(B, Lq, Lk, *, mask="none", window=(-1, -1), draft_block=1, doc_ids=None,
         kv_lens=None) -> np.ndarray:
    """Boolean mask [B, Lq, Lk]: entry (b, i, j) is True iff key j is visible to query row i."""
    out = np.zeros((B, Lq, Lk), dtype=np.uint8)
    doc = _i32(doc_ids)
    kl = _i32(kv_lens)
    rc = _load().oracle_mask(B, Lq, Lk, _mask_code(mask), int(window[0]), int(window[1]),
                             int(draft_block), _ptr(doc), _ptr(kl), _ptr(out))
    if rc:
        raise ValueError("oracle_mask: invalid arguments")
    return out.astype(bool)


_mask_matrix = mask  # the mask function above, for callers whose argument is named `mask`


def count_pairs(B, Lq, Lk, *, mask="none", window=(-1, -1), draft_block=1, doc_ids=None,
                kv_lens=None, nthreads=None) -> int:
    """Allowed (query row, key) pairs summed over the batch, for ONE head."""
    doc = _i32(doc_ids)
    kl = _i32(kv_lens)
    n = _load().oracle_count_pairs(B, Lq, Lk, _mask_code(mask), int(window[0]), int(window[1]),
                                   int(draft_block), _ptr(doc), _ptr(kl),
                                   int(nthreads or max_threads()))
    if n < 0:
        raise ValueError("oracle_count_pairs: invalid arguments")
    return int(n)


def attn_fwd(q, k, v, *, scale=None, mask="none", window=(-1, -1), draft_block=1,
             doc_ids=None, kv_lens=None, rows=None, nthreads=None, alibi_slopes=None,
             rel_bias=None):
    """Dense masked attention in double.

    q: [B, Hq, Lq, d] bf16; k, v: [B, Hkv, Lk, d] bf16.  Returns (O, LSE) as
    float64 numpy arrays, shaped [B, Hq, Lq, d] / [B, Hq, Lq], or [n, d] / [n]
    when ``rows`` (flat indices (b*Hq + hq)*Lq + i) is given.  Score modifiers
    (at most one): ``alibi_slopes`` ([Hq]) adds slope_h * (j - p) to every
    scaled score; ``rel_bias`` = (table [Hq, 2R + 1], R) adds
    table[h, clamp(j - p, -R, R) + R]; p = Lk_b - Lq + i, Lk_b = kv_lens[b] when
    kv_lens is given (the split-KV decode), else Lk.
    """
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, Hq, Lq, d = qb.shape
    Bk, Hkv, Lk, dk = kb.shape
    if vb.shape != kb.shape or Bk != B or dk != d:
        raise ValueError("shape mismatch between q, k, v")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    doc = _i32(doc_ids)
    kl = _i32(kv_lens)
    if rows is not None:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        n = rows.size
    else:
        n = B * Hq * Lq
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    if kl is not None and (rel_bias is not None or alibi_slopes is not None):
        if rel_bias is not None and alibi_slopes is not None:
            raise ValueError("rel_bias is not combined with alibi_slopes")
        sl = tb = None
        rmax = 0
        if alibi_slopes is not None:
            sl = np.ascontiguousarray(np.asarray(
                alibi_slopes.cpu().numpy() if hasattr(alibi_slopes, "cpu") else alibi_slopes,
                dtype=np.float64).reshape(-1))
            if sl.size != Hq:
                raise ValueError("alibi_slopes must have Hq entries")
        else:
            table, rmax = rel_bias
            tb = np.ascontiguousarray(np.asarray(
                table.cpu().numpy() if hasattr(table, "cpu") else table, dtype=np.float64))
            if tb.shape != (Hq, 2 * int(rmax) + 1):
                raise ValueError("rel_bias table must be [Hq, 2R + 1]")
        rc = _load().oracle_attn_rows_mod(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d,
                                          float(scale), _mask_code(mask), int(window[0]),
                                          int(window[1]), int(draft_block), _ptr(doc), _ptr(kl),
                                          _ptr(sl), _ptr(tb), int(rmax), _ptr(rows), n, _ptr(o),
                                          _ptr(lse), int(nthreads or max_threads()))
    elif rel_bias is not None:
        if alibi_slopes is not None:
            raise ValueError("rel_bias is not combined with alibi_slopes")
        table, rmax = rel_bias
        tb = np.ascontiguousarray(np.asarray(
            table.cpu().numpy() if hasattr(table, "cpu") else table, dtype=np.float64))
        if tb.shape != (Hq, 2 * int(rmax) + 1):
            raise ValueError("rel_bias table must be [Hq, 2R + 1]")
        rc = _load().oracle_attn_rows_relbias(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d,
                                              float(scale), _mask_code(mask), int(window[0]),
                                              int(window[1]), int(draft_block), _ptr(doc),
                                              _ptr(tb), int(rmax), _ptr(rows), n, _ptr(o),
                                              _ptr(lse), int(nthreads or max_threads()))
    elif alibi_slopes is not None:
        sl = np.ascontiguousarray(np.asarray(
            alibi_slopes.cpu().numpy() if hasattr(alibi_slopes, "cpu") else alibi_slopes,
            dtype=np.float64).reshape(-1))
        if sl.size != Hq:
            raise ValueError("alibi_slopes must have Hq entries")
        rc = _load().oracle_attn_rows_alibi(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d,
                                            float(scale), _mask_code(mask), int(window[0]),
                                            int(window[1]), int(draft_block), _ptr(doc), _ptr(sl),
                                            _ptr(rows), n, _ptr(o), _ptr(lse),
                                            int(nthreads or max_threads()))
    else:
        rc = _load().oracle_attn_rows(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Lq, Lk, d,
                                      float(scale), _mask_code(mask), int(window[0]),
                                      int(window[1]), int(draft_block), _ptr(doc), _ptr(kl),
                                      _ptr(rows), n, _ptr(o), _ptr(lse),
                                      int(nthreads or max_threads()))
    if rc:
        raise ValueError(f"oracle_attn_rows failed ({rc})")
    if rows is None:
        return o.reshape(B, Hq, Lq, d), lse.reshape(B, Hq, Lq)
    return o, lse


def decode_partials(q, k, v, kv_lens, *, chunk, nsplit=None, scale=None, nthreads=None):
    """Per-chunk partial (O_s, LSE_s) of the split-KV decode; shapes [S, B*Hq*Lq, d] / [S, B*Hq*Lq]."""
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, Hq, Lq, d = qb.shape
    _, Hkv, Lk, _ = kb.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if nsplit is None:
        nsplit = max(1, -(-Lk // chunk))
    kl = _i32(kv_lens)
    nrows = B * Hq * Lq
    o = np.zeros((nsplit, nrows, d), dtype=np.float64)
    lse = np.zeros((nsplit, nrows), dtype=np.float64)
    rc = _load().oracle_decode_partials(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(kl), B, Hq, Hkv, Lq,
                                        Lk, d, float(scale), int(chunk), int(nsplit), _ptr(o),
                                        _ptr(lse), int(nthreads or max_threads()))
    if rc:
        raise ValueError(f"oracle_decode_partials failed ({rc})")
    return o, lse


def combine(o_part, lse_part):
    """LSE-weighted merge of split partials: ([S, n, d], [S, n]) -> ([n, d], [n])."""
    o_part = np.ascontiguousarray(o_part, dtype=np.float64)
    lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
    S, n, d = o_part.shape
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = _load().oracle_combine(_ptr(o_part), _ptr(lse_part), S, n, d, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle_combine failed")
    return o, lse


def paged_gather(pages, block_table):
    """Logical cache [B, H, pages_per_seq * page_size, d] (bf16) from a page pool
    [num_pages, H, page_size, d] (bf16) and a block table [B, pages_per_seq]."""
    import torch
    pb = _bf16_bits(pages)
    num_pages, H, page_size, d = pb.shape
    bt = _i32(block_table)
    B, pps = bt.shape
    out = np.zeros((B, H, pps * page_size, d), dtype=np.uint16)
    rc = _load().oracle_paged_gather(_ptr(pb), _ptr(bt), B, H, page_size, pps, num_pages, d,
                                     _ptr(out))
    if rc:
        raise ValueError("oracle_paged_gather: page id out of range or bad shape")
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, *, scale=None, mask="none",
                    window=(-1, -1), draft_block=1, alibi_slopes=None, rel_bias=None):
    """Packed sequences: the plain definition applied to each sequence on its own.

    q: [total_q, Hq, d] bf16, k, v: [total_k, Hkv, d] bf16 (token-major);
    sequence b owns query tokens cu_seqlens_q[b]:cu_seqlens_q[b+1] and key tokens
    cu_seqlens_k[b]:cu_seqlens_k[b+1] ("FlexAttention 是什么，以及 DFlash2 之谜的完整
    侦破", section 1: a document mask at the packing level, ragged lengths without
    padding).  Each sequence is attention with Lq = Lq_b, Lk = Lk_b as in
    ``attn_fwd``; a row with no key gets O = 0, LSE = -inf.  Returns (O, LSE) as
    float64 numpy arrays shaped [total_q, Hq, d] and [Hq, total_q].
    """
    import torch
    cq = np.asarray(_i32(cu_seqlens_q), dtype=np.int64)
    ck = np.asarray(_i32(cu_seqlens_k), dtype=np.int64)
    if cq.shape != ck.shape or cq.ndim != 1 or cq.size < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    total_q, Hq, d = q.shape
    total_k, Hkv, _ = k.shape
    if cq[0] != 0 or ck[0] != 0 or cq[-1] != total_q or ck[-1] != total_k:
        raise ValueError("cu_seqlens must start at 0 and end at the token counts")
    if np.any(np.diff(cq) < 0) or np.any(np.diff(ck) < 0):
        raise ValueError("cu_seqlens must be non-decreasing")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((total_q, Hq, d), dtype=np.float64)
    lse = np.full((Hq, total_q), -np.inf, dtype=np.float64)
    for b in range(cq.size - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 == q0 or k1 == k0:
            continue  # no rows, or rows with no key (O = 0, LSE = -inf)
        qb = q[q0:q1].permute(1, 0, 2).unsqueeze(0).contiguous()
        kb = k[k0:k1].permute(1, 0, 2).unsqueeze(0).contiguous()
        vb = v[k0:k1].permute(1, 0, 2).unsqueeze(0).contiguous()
        ob, lb = attn_fwd(qb, kb, vb, scale=scale, mask=mask, window=window,
                          draft_block=draft_block, alibi_slopes=alibi_slopes, rel_bias=rel_bias)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[:, q0:q1] = lb[0]
    return o, lse


def attn_bwd(q, k, v, do, *, scale=None, mask="none", window=(-1, -1), draft_block=1,
             doc_ids=None):
    """Gradients of the forward above: (dQ, dK, dV) in double, for bf16 inputs.

    The backward of softmax attention ("FlashAttention 2 原理与 PyTorch 实战",
    section 3.2: the row statistics of the forward are recomputed, not stored
    as an N x N matrix), written out on whole score rows: with P the masked
    softmax of S = scale * Q K^T and O = P V,
        dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
        dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
    Rows with no visible key have P = 0 and contribute nothing.  Query heads of
    one KV head (GQA) add their dK and dV.  q: [B, Hq, Lq, d]; k, v: [B, Hkv, Lk, d];
    do: [B, Hq, Lq, d] (any float dtype, read as double).  Returns float64 numpy
    arrays shaped like q, k, v.
    """
    def as_f64(t):
        if isinstance(t, np.ndarray):
            return t.astype(np.float64)
        return t.detach().cpu().double().numpy()

    Q, K, V, dO = as_f64(q), as_f64(k), as_f64(v), as_f64(do)
    B, Hq, Lq, d = Q.shape
    _, Hkv, Lk, _ = K.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    group = Hq // Hkv
    allowed = _mask_matrix(B, Lq, Lk, mask=mask, window=window, draft_block=draft_block,
                           doc_ids=doc_ids)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(B):
        vis = allowed[b]
        for hq in range(Hq):
            hk = hq // group
            S = scale * Q[b, hq] @ K[b, hk].T
            S = np.where(vis, S, -np.inf)
            mx = S.max(axis=1, keepdims=True)
            has = np.isfinite(mx)
            E = np.where(vis, np.exp(S - np.where(has, mx, 0.0)), 0.0)
            l = E.sum(axis=1, keepdims=True)
            P = np.where(has, E / np.where(l > 0, l, 1.0), 0.0)
            O = P @ V[b, hk]
            dV[b, hk] += P.T @ dO[b, hq]
            dP = dO[b, hq] @ V[b, hk].T
            Dv = (dO[b, hq] * O).sum(axis=1, keepdims=True)
            dS = P * (dP - Dv)
            dQ[b, hq] = scale * dS @ K[b, hk]
            dK[b, hk] += scale * dS.T @ Q[b, hq]
    return dQ, dK, dV
