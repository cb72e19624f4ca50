"""Seeded synthetic inputs for the attention forward and split-KV decode.

This module only draws random numbers and packs them into tensors.  It holds
none of the attention arithmetic: the oracle (``oracle/``) and the CUDA path
(``sm_attn_fwd_b200``) both take their inputs from here and from nowhere else.

Recipe (all configurations): a ``torch.Generator`` on the requested device is
seeded with the configuration's seed; Q, K and V are drawn in that order with
``torch.randn(shape, dtype=float32)``, multiplied by the configuration's
factor, and rounded to bf16 (round-to-nearest-even, PyTorch's ``.to``).
Extra draws follow in this order: the document split point per sequence
(``randint(1, Lk)``), then the per-sequence KV lengths
(``randint(lo, hi + 1)``).  Shapes are contiguous [B, H, L, D].

The workloads follow the pages' shapes: the FlashAttention 2 article's SDPA
example (B=2, H=16, L=4096, d=64, causal; "FlashAttention 2 原理与 PyTorch 实战",
section 二), the block-diffusion draft call of the DFlash2 investigation
(non-causal + symmetric window, a handful of draft queries over a long
context; "FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 4,
experiment 1) and FlexDecoding's short-query / long-KV split-KV decode with
GQA (same page, section 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import torch

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_DRAFT_BLOCK = 2

_MASK_NAMES = {"none": MASK_NONE, "causal": MASK_CAUSAL, "draft": MASK_DRAFT_BLOCK}


def mask_code(mask) -> int:
    """Map "none" / "causal" / "draft" (or an int code) to the ABI's mask code."""
    if isinstance(mask, int):
        return mask
    return _MASK_NAMES[mask]


@dataclass(frozen=True)
class AttnConfig:
    """One prefill (``attn_fwd``) or decode (``attn_decode_splitkv``) workload."""

    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    d: int
    mask: str = "none"          # "none" | "causal" | "draft"
    window: tuple = (-1, -1)    # (w_left, w_right); -1 = unbounded side
    draft_block: int = 1
    doc_split: bool = False     # two documents per sequence, split at a drawn point
    factor: float = 1.0         # multiplies the N(0,1) draws before bf16 rounding
    decode: bool = False        # split-KV decode: per-sequence kv_lens drawn
    kv_len_range: Optional[tuple] = None  # (lo, hi) inclusive, decode only
    scale: Optional[float] = None         # None -> 1/sqrt(d)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / (self.d ** 0.5)

    @property
    def mask_kind(self) -> int:
        return mask_code(self.mask)

    def with_(self, **kw) -> "AttnConfig":
        return replace(self, **kw)


# The five workloads.  Sizes, seeds and distributions are fixed here.
TINY = AttnConfig("tiny_b1h2_l128_d64", seed=0, B=1, Hq=2, Hkv=2, Lq=128, Lk=128, d=64,
                  scale=1.0 / 8.0)
CAUSAL_4K = AttnConfig("causal_b2h16_l4096_d64", seed=1, B=2, Hq=16, Hkv=16, Lq=4096, Lk=4096,
                       d=64, mask="causal")
CAUSAL_32K_GQA = AttnConfig("causal_gqa_b1hq32hkv8_l32768_d128", seed=2, B=1, Hq=32, Hkv=8,
                            Lq=32768, Lk=32768, d=128, mask="causal", factor=0.5)
DRAFT_WINDOW_DOC = AttnConfig("draft16_win512_doc_b4h32_lq16_lk2064_d128", seed=3, B=4, Hq=32,
                              Hkv=32, Lq=16, Lk=2048 + 16, d=128, mask="draft",
                              window=(512, 512), draft_block=16, doc_split=True)
DRAFT_WINDOW_DOC_FULL = DRAFT_WINDOW_DOC.with_(
    name="draft16_win512_doc_b4h32_lq2064_lk2064_d128", Lq=2048 + 16)
DECODE_LQ1 = AttnConfig("decode_b64hq64hkv8_lq1_lk32768_d128", seed=4, B=64, Hq=64, Hkv=8,
                        Lq=1, Lk=32768, d=128, decode=True, kv_len_range=(8192, 32768))
DECODE_LQ16 = DECODE_LQ1.with_(name="decode_b64hq64hkv8_lq16_lk32768_d128", Lq=16)

CONFIGS = {c.name: c for c in (TINY, CAUSAL_4K, CAUSAL_32K_GQA, DRAFT_WINDOW_DOC,
                               DRAFT_WINDOW_DOC_FULL, DECODE_LQ1, DECODE_LQ16)}


@dataclass
class AttnInputs:
    cfg: AttnConfig
    q: torch.Tensor                       # bf16 [B, Hq, Lq, d]
    k: torch.Tensor                       # bf16 [B, Hkv, Lk, d]
    v: torch.Tensor                       # bf16 [B, Hkv, Lk, d]
    doc_ids: Optional[torch.Tensor] = None   # int32 [B, Lk]
    kv_lens: Optional[torch.Tensor] = None   # int32 [B]
    extra: dict = field(default_factory=dict)


def _randn_bf16(shape, g, device, factor):
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if factor != 1.0:
        x.mul_(factor)
    return x.to(torch.bfloat16)


def make_inputs(cfg: AttnConfig, device="cpu") -> AttnInputs:
    """Draw the inputs of ``cfg`` on ``device`` with the recipe in the module docstring."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    q = _randn_bf16((cfg.B, cfg.Hq, cfg.Lq, cfg.d), g, device, cfg.factor)
    k = _randn_bf16((cfg.B, cfg.Hkv, cfg.Lk, cfg.d), g, device, cfg.factor)
    v = _randn_bf16((cfg.B, cfg.Hkv, cfg.Lk, cfg.d), g, device, cfg.factor)
    doc_ids = kv_lens = None
    if cfg.doc_split:
        split = torch.randint(1, cfg.Lk, (cfg.B,), generator=g, device=device)
        pos = torch.arange(cfg.Lk, device=device)
        doc_ids = (pos[None, :] >= split[:, None]).to(torch.int32).contiguous()
    if cfg.decode:
        lo, hi = cfg.kv_len_range
        kv_lens = torch.randint(lo, hi + 1, (cfg.B,), generator=g, device=device).to(torch.int32)
    return AttnInputs(cfg, q, k, v, doc_ids, kv_lens)


def random_case(seed, B, Hq, Hkv, Lq, Lk, d, *, factor=1.0, device="cpu", doc_split=False,
                kv_len_range=None, n_docs=2):
    """Small ad-hoc cases for tests: same recipe, arbitrary shape.

    ``n_docs`` > 2 draws ``n_docs - 1`` sorted split points per sequence.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    q = _randn_bf16((B, Hq, Lq, d), g, device, factor)
    k = _randn_bf16((B, Hkv, Lk, d), g, device, factor)
    v = _randn_bf16((B, Hkv, Lk, d), g, device, factor)
    doc_ids = kv_lens = None
    if doc_split and Lk > 1:
        pos = torch.arange(Lk, device=device)
        splits = torch.randint(1, Lk, (B, max(1, n_docs - 1)), generator=g, device=device)
        splits, _ = torch.sort(splits, dim=1)
        doc_ids = (pos[None, :, None] >= splits[:, None, :]).sum(-1).to(torch.int32).contiguous()
    if kv_len_range is not None:
        lo, hi = kv_len_range
        kv_lens = torch.randint(lo, hi + 1, (B,), generator=g, device=device).to(torch.int32)
    return q, k, v, doc_ids, kv_lens


def packed_case(seed, lens_q, lens_k, Hq, Hkv, d, *, factor=1.0, device="cpu"):
    """Packed (token-major) sequences: Q [total_q, Hq, d], K and V [total_k, Hkv, d],
    bf16 from the same recipe (Q, K, V drawn in that order), and the int32
    cu_seqlens [B + 1] of both sides."""
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    q = _randn_bf16((tq, Hq, d), g, device, factor)
    k = _randn_bf16((tk, Hkv, d), g, device, factor)
    v = _randn_bf16((tk, Hkv, d), g, device, factor)
    cu_q = torch.tensor([0] + [int(x) for x in torch.tensor(lens_q).cumsum(0)], dtype=torch.int32,
                        device=device)
    cu_k = torch.tensor([0] + [int(x) for x in torch.tensor(lens_k).cumsum(0)], dtype=torch.int32,
                        device=device)
    return q, k, v, cu_q, cu_k


def packed_lengths(seed, n, lo, hi):
    """n sequence lengths drawn uniformly from [lo, hi] (the length mix of a
    packed batch of documents)."""
    g = torch.Generator()
    g.manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]
