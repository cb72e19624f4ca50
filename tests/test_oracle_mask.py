"""Pins for the oracle's mask predicate (CPU only).

The oracle evaluates mask_mod(b, q_idx, kv_idx) element by element
("FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 1).  Here the same
masks are built a second, independent way — numpy band matrices (tril/triu
with the bottom-right offset), a block-Kronecker lower triangle for the draft
mask, and an outer equality for document ids — and the two must agree bit for
bit, the way the page's section 3 diffed three independent mask
reproductions.
"""
import itertools

import numpy as np
import pytest

import oracle

MASKS = ("none", "causal", "draft")


def independent_mask(B, Lq, Lk, mask, window, draft_block, doc_ids, kv_lens):
    out = np.zeros((B, Lq, Lk), dtype=bool)
    for b in range(B):
        lkb = Lk if kv_lens is None else int(kv_lens[b])
        off = lkb - Lq                                    # query row i sits at p = i + off
        m = np.ones((Lq, Lk), dtype=bool)
        m[:, lkb:] = False                                # keys past the sequence end
        if mask == "causal":
            m &= np.tril(np.ones((Lq, Lk), dtype=bool), k=off)
        elif mask == "draft":
            bd = draft_block
            # block lower triangle over absolute positions, shifted by a multiple of
            # bd so that negative query positions stay representable
            shift = bd * ((max(0, -off) + bd - 1) // bd)
            npos = max(Lk, off + Lq) + shift
            nb = (npos + bd - 1) // bd
            full = np.kron(np.tril(np.ones((nb, nb), dtype=bool)), np.ones((bd, bd), dtype=bool))
            m &= full[off + shift: off + shift + Lq, shift: shift + Lk]
        wl, wr = window
        if wl >= 0:
            m &= np.triu(np.ones((Lq, Lk), dtype=bool), k=off - wl)
        if wr >= 0:
            m &= np.tril(np.ones((Lq, Lk), dtype=bool), k=off + wr)
        if doc_ids is not None:
            d = np.asarray(doc_ids[b])
            qdoc = np.full(Lq, -12345)
            valid = (np.arange(Lq) + off >= 0) & (np.arange(Lq) + off < Lk)
            qdoc[valid] = d[np.arange(Lq)[valid] + off]
            m &= (d[None, :] == qdoc[:, None]) & valid[:, None]
        out[b] = m
    return out


def _docs(rng, B, Lk, n_docs):
    docs = np.zeros((B, Lk), dtype=np.int32)
    for b in range(B):
        if Lk > 1:
            cuts = np.sort(rng.integers(1, Lk, size=n_docs - 1))
            docs[b] = np.searchsorted(cuts, np.arange(Lk), side="right")
    return docs


@pytest.mark.parametrize("mask", MASKS)
def test_mask_matches_independent_construction(mask):
    rng = np.random.default_rng(1234)
    shapes = [(1, 1), (1, 7), (7, 7), (16, 16), (5, 40), (40, 40), (33, 17), (3, 39)]
    blocks = (1, 2, 3, 4, 16) if mask == "draft" else (1,)
    windows = (-1, 0, 1, 3, 512)
    n_checked = 0
    for (Lq, Lk), bd, wl, wr in itertools.product(shapes, blocks, windows, windows):
        for variant in ("plain", "doc", "kvlens"):
            B = 2
            doc = _docs(rng, B, Lk, 3) if variant == "doc" else None
            if variant == "doc" and Lq > Lk:
                continue
            kv = None
            if variant == "kvlens":
                kv = rng.integers(0, Lk + 1, size=B).astype(np.int32)
            got = oracle.mask(B, Lq, Lk, mask=mask, window=(wl, wr), draft_block=bd,
                              doc_ids=doc, kv_lens=kv)
            want = independent_mask(B, Lq, Lk, mask, (wl, wr), bd, doc, kv)
            assert np.array_equal(got, want), (mask, Lq, Lk, bd, wl, wr, variant)
            n_checked += 1
    assert n_checked > 100


def test_causal_is_draft_block_of_one():
    """The causal mask is the draft-block mask with blocks of one token."""
    for Lq, Lk in [(1, 1), (9, 9), (5, 13), (13, 5)]:
        a = oracle.mask(1, Lq, Lk, mask="causal")
        b = oracle.mask(1, Lq, Lk, mask="draft", draft_block=1)
        assert np.array_equal(a, b)


def test_draft_block_hand_example():
    """Hand-enumerated draft mask, blocks of 2 over 6 tokens (golden fixture).

    Each token sees every earlier block and all of its own block in both
    directions, and nothing of a later block.
    """
    want = np.loadtxt(_golden("draft_block2_l6.txt"), dtype=int).astype(bool)
    got = oracle.mask(1, 6, 6, mask="draft", draft_block=2)[0]
    assert np.array_equal(got, want)


def test_symmetric_window_equals_block_diffusion_at_short_context():
    """Non-causal + symmetric window (w, w) equals the draft-block mask for the
    draft queries (the last block) while the whole context fits in the window,
    and stops being equal once it does not ("FlexAttention 是什么，以及 DFlash2
    之谜的完整侦破", section 3, finding 1)."""
    bd = 16
    for prefix in (0, 16, 64, 496):
        Lk = prefix + bd
        w = 512
        win = oracle.mask(1, bd, Lk, mask="none", window=(w, w))
        blk = oracle.mask(1, bd, Lk, mask="draft", draft_block=bd)
        assert np.array_equal(win, blk)
        assert blk.all()
    # beyond the window the symmetric window drops the far prefix
    Lk = 2048 + bd
    win = oracle.mask(1, bd, Lk, mask="none", window=(512, 512))
    blk = oracle.mask(1, bd, Lk, mask="draft", draft_block=bd)
    assert not np.array_equal(win, blk)
    assert blk.all() and not win.all()


def test_count_pairs_closed_forms():
    # causal, Lq = Lk = L: L (L + 1) / 2 per head
    for L in (1, 2, 127, 128, 129, 1000):
        assert oracle.count_pairs(1, L, L, mask="causal") == L * (L + 1) // 2
    # no mask: Lq * Lk
    assert oracle.count_pairs(3, 17, 29) == 3 * 17 * 29
    # draft queries (16) at the end of 2048 + 16 keys, window (512, 512), no docs:
    # row i (p = 2048 + i) sees [p - 512, 2063] -> 2064 - (1536 + i) = 528 - i keys
    n = oracle.count_pairs(1, 16, 2064, mask="draft", window=(512, 512), draft_block=16)
    assert n == sum(528 - i for i in range(16))
    # count equals the popcount of the mask
    rng = np.random.default_rng(7)
    doc = _docs(rng, 2, 50, 3)
    m = oracle.mask(2, 50, 50, mask="draft", window=(9, 4), draft_block=3, doc_ids=doc)
    assert oracle.count_pairs(2, 50, 50, mask="draft", window=(9, 4), draft_block=3,
                              doc_ids=doc) == int(m.sum())


def test_mask_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.mask(1, 4, 4, mask="draft", draft_block=0)
    with pytest.raises(ValueError):
        oracle.mask(1, 4, 4, window=(-2, 0))
    with pytest.raises(ValueError):
        oracle.mask(1, 4, 4, kv_lens=np.array([5], dtype=np.int32))


def _golden(name):
    import os
    return os.path.join(os.path.dirname(__file__), "golden", name)
