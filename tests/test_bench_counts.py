"""The bench's work counts agree with the oracle on the inputs the bench times.

bench.py counts visible (query, key) pairs from the per-row key intervals of
the mask (no oracle on the product path); the mask-adjusted TFLOP/s it reports
is 4*d*Hq*pairs.  These CPU tests check that count against the oracle's
element-by-element mask on the same CPU-drawn inputs (the document split of
the draft workload comes from the generator), and the key-union byte count
against the oracle's mask.
"""
import numpy as np
import pytest

import bench
import oracle
from workloads import (CAUSAL_4K, CAUSAL_32K_GQA, DRAFT_WINDOW_DOC, DRAFT_WINDOW_DOC_FULL, TINY,
                       make_inputs)


@pytest.mark.parametrize("cfg", [TINY, CAUSAL_4K, CAUSAL_32K_GQA, DRAFT_WINDOW_DOC,
                                 DRAFT_WINDOW_DOC_FULL], ids=lambda c: c.name)
def test_bench_pair_count_equals_oracle(cfg):
    doc = make_inputs(cfg).doc_ids if cfg.doc_split else None
    want = oracle.count_pairs(cfg.B, cfg.Lq, cfg.Lk, mask=cfg.mask, window=cfg.window,
                              draft_block=cfg.draft_block, doc_ids=doc)
    got = bench.visible_pairs(cfg, doc_ids=None if doc is None else doc.numpy())
    assert got == want


def test_draft_workload_pair_count_value():
    """The Lq = 16 draft call (seed 3, CPU generator) has 27,440 visible pairs
    per head over the batch; without documents it would be 4 * 8,328."""
    cfg = DRAFT_WINDOW_DOC
    doc = make_inputs(cfg).doc_ids.numpy()
    assert bench.visible_pairs(cfg, doc_ids=doc) == 27440
    assert bench.visible_pairs(cfg) == 4 * sum(528 - i for i in range(16))


@pytest.mark.parametrize("cfg", [DRAFT_WINDOW_DOC, DRAFT_WINDOW_DOC_FULL, CAUSAL_4K],
                         ids=lambda c: c.name)
def test_bench_key_union_equals_oracle_mask(cfg):
    doc = make_inputs(cfg).doc_ids if cfg.doc_split else None
    if cfg.Lq * cfg.Lk * cfg.B > 2e8:
        cfg = cfg.with_(Lq=1024, Lk=1024)
    m = oracle.mask(cfg.B, cfg.Lq, cfg.Lk, mask=cfg.mask, window=cfg.window,
                    draft_block=cfg.draft_block, doc_ids=doc)
    want = int(m.any(axis=1).sum())
    got = bench.visible_keys(cfg, doc_ids=None if doc is None else doc.numpy())
    assert got == want
