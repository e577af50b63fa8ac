"""Pins of the oracle's cross-scale list transfer (mask reuse; CPU only).

Sources: pith.science review of SparSTAR, "Extended reading notes / Core
claim" (a selection carried from one scale to another keeps less attention
mass than a fresh one; the method selects anew at every scale) and
Figure 1 (a carried-over mask can leave out blocks that matter at the new
scale).  The pages give
no map between the token positions of two scales.  The reading pinned here
resamples the block mask by nearest neighbour along each key segment (text,
image_ref, ref, cur):
- target offset p of segment g has as image the source offset
  floor(p * len_s[g] / len_t[g]);
- a block's centre is its token a + (n - 1) // 2;
- target query block i reads the list of the source block that holds the
  image of its centre query token;
- target key block j is kept when it is forced at the target, or when the
  image of its centre token lies in a listed source block.

Each test checks the oracle against something other than its own code:
- the identity map (the list comes back with the target's forced prefix);
- an exact 2x refinement with a closed form;
- the inverse formulation in plain Python on random ragged layouts: for
  every listed source block, the target offsets whose image falls in it form
  the integer interval [ceil(lo * lt / ls), ceil((hi + 1) * lt / ls) - 1],
  and the target blocks whose centre lies in one of those intervals are kept;
- single-block lists at every source block;
- the invariants of a valid list;
- the error returns.
"""
import numpy as np
import pytest

BLOCK = 128


def _nb(L):
    return (L + BLOCK - 1) // BLOCK


def _random_lists(rng, B, H, nQB, nKB, max_sel, p_invalid=0.0):
    idx = np.full((B, H, nQB, max_sel), -1, np.int32)
    cnt = np.zeros((B, H, nQB), np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                n = int(rng.integers(0, min(max_sel, nKB) + 1))
                chosen = np.sort(rng.choice(nKB, size=n, replace=False)).astype(np.int32)
                if p_invalid > 0 and n > 0:
                    bad = rng.random(n) < p_invalid
                    chosen[bad] = rng.choice([-1, nKB, nKB + 7, -100], size=int(bad.sum()))
                idx[b, h, i, :n] = chosen
                cnt[b, h, i] = n
    return idx, cnt


def _cdiv(a, b):
    return -(-a // b)


def _inverse(idx_s, cnt_s, len_s, len_t):
    """From the source side: the target blocks whose centre lies in the
    preimage of a listed source block (and the forced prefix)."""
    B, H, nQB_s, max_sel_s = idx_s.shape
    off_s = [int(x) for x in np.concatenate([[0], np.cumsum(len_s)[:-1]])]
    off_t = [int(x) for x in np.concatenate([[0], np.cumsum(len_t)[:-1]])]
    Lk_s, Lk_t = int(sum(len_s)), int(sum(len_t))
    nKB_s, nKB_t = _nb(Lk_s), _nb(Lk_t)
    nQB_t = _nb(len_t[3])
    nF_t = _nb(len_t[0] + len_t[1])
    ls_c, lt_c = int(len_s[3]), int(len_t[3])

    def centre(a, L):
        return a + (min(BLOCK, L - a) - 1) // 2

    # query side: source query block s covers target query offsets
    # [ceil(128 s lt / ls), ceil(128 (s+1) lt / ls) - 1]
    q_src = {}
    for i in range(nQB_t):
        c = centre(i * BLOCK, lt_c)
        for sblk in range(nQB_s):
            lo = _cdiv(sblk * BLOCK * lt_c, ls_c)
            hi = _cdiv(min((sblk + 1) * BLOCK, ls_c) * lt_c, ls_c) - 1
            if lo <= c <= hi:
                q_src[i] = sblk
    out = {}
    for b in range(B):
        for h in range(H):
            for i in range(nQB_t):
                si = q_src[i]
                n = min(int(cnt_s[b, h, si]), max_sel_s)
                listed = {int(x) for x in idx_s[b, h, si, :max(n, 0)] if 0 <= x < nKB_s}
                kept = set(range(nF_t))
                for sb in listed:
                    for g in range(4):
                        lo = max(sb * BLOCK, off_s[g]) - off_s[g]
                        hi = min(sb * BLOCK + BLOCK, off_s[g] + len_s[g]) - 1 - off_s[g]
                        if lo > hi or len_t[g] == 0:
                            continue
                        t_lo = off_t[g] + _cdiv(lo * len_t[g], len_s[g])
                        t_hi = off_t[g] + _cdiv((hi + 1) * len_t[g], len_s[g]) - 1
                        for j in range(nKB_t):
                            if t_lo <= centre(j * BLOCK, Lk_t) <= t_hi:
                                kept.add(j)
                out[(b, h, i)] = sorted(kept)
    return out


def _check_against(orc_out, expect):
    idx_t, cnt_t = orc_out
    for (b, h, i), kept in expect.items():
        assert cnt_t[b, h, i] == len(kept), ((b, h, i), cnt_t[b, h, i], kept)
        assert list(idx_t[b, h, i, :len(kept)]) == kept
        assert (idx_t[b, h, i, len(kept):] == -1).all()


def test_identity_map_returns_the_list_with_the_forced_prefix(orc):
    rng = np.random.default_rng(1)
    seg = [300, 0, 1000, 1100]  # straddling and partial blocks
    nKB, nQB = _nb(sum(seg)), _nb(seg[3])
    nF = _nb(seg[0] + seg[1])
    idx, cnt = _random_lists(rng, 1, 2, nQB, nKB, 8, p_invalid=0.2)
    idx_t, cnt_t = orc.transfer_lists(idx, cnt, seg, seg)
    for h in range(2):
        for i in range(nQB):
            n = cnt[0, h, i]
            want = sorted(set(range(nF)) | {int(x) for x in idx[0, h, i, :n] if 0 <= x < nKB})
            assert list(idx_t[0, h, i, :cnt_t[0, h, i]]) == want


def test_exact_2x_refinement_closed_form(orc):
    # text fills block 0; the cur segment doubles from m to 2m blocks.  Target
    # cur block q (global 1+q) has the image of source global block 1 + q//2,
    # and target query block i reads source query block i // 2.
    m = 6
    len_s, len_t = [128, 0, 0, 128 * m], [128, 0, 0, 256 * m]
    rng = np.random.default_rng(2)
    idx, cnt = _random_lists(rng, 1, 3, m, 1 + m, 5)
    idx_t, cnt_t = orc.transfer_lists(idx, cnt, len_s, len_t)
    for h in range(3):
        for i in range(2 * m):
            src = {int(x) for x in idx[0, h, i // 2, :cnt[0, h, i // 2]]}
            want = [0] + [1 + q for q in range(2 * m) if 1 + q // 2 in src]
            assert list(idx_t[0, h, i, :cnt_t[0, h, i]]) == want


@pytest.mark.parametrize("seed", range(16))
def test_matches_the_inverse_formulation_on_random_layouts(orc, seed):
    rng = np.random.default_rng(100 + seed)
    text = int(rng.integers(1, 300))
    img = int(rng.choice([0, int(rng.integers(1, 400))]))
    ref_s = int(rng.choice([0, int(rng.integers(50, 900))]))
    cur_s = int(rng.integers(60, 900))
    # ratios between 1/4 and 4, ragged everywhere
    ref_t = 0 if ref_s == 0 else max(1, int(ref_s * rng.uniform(0.25, 4.0)))
    cur_t = max(1, int(cur_s * rng.uniform(0.25, 4.0)))
    len_s, len_t = [text, img, ref_s, cur_s], [text, img, ref_t, cur_t]
    nKB_s, nQB_s = _nb(sum(len_s)), _nb(cur_s)
    idx, cnt = _random_lists(rng, 1, 2, nQB_s, nKB_s, max(1, nKB_s // 2), p_invalid=0.1)
    expect = _inverse(idx, cnt, len_s, len_t)
    _check_against(orc.transfer_lists(idx, cnt, len_s, len_t), expect)


def test_segment_absent_at_the_source_maps_to_nothing(orc):
    # The reference segment is empty at the source: a target block whose
    # centre is a reference token has no image and is never kept.
    len_s, len_t = [128, 0, 0, 512], [128, 0, 640, 512]
    nKB_s = _nb(sum(len_s))
    idx = np.tile(np.arange(nKB_s, dtype=np.int32), (1, 1, _nb(512), 1))
    cnt = np.full((1, 1, _nb(512)), nKB_s, np.int32)
    expect = _inverse(idx, cnt, len_s, len_t)
    _check_against(orc.transfer_lists(idx, cnt, len_s, len_t), expect)
    idx_t, cnt_t = orc.transfer_lists(idx, cnt, len_s, len_t)
    # target blocks 1..5 hold reference tokens only
    assert all(j not in range(1, 6) for j in idx_t[0, 0, 0, :cnt_t[0, 0, 0]])


def test_invariants_and_empty_source_lists(orc):
    rng = np.random.default_rng(7)
    len_s, len_t = [512, 3600, 4000, 4000], [512, 3600, 9000, 9000]
    nKB_s, nQB_s = _nb(sum(len_s)), _nb(len_s[3])
    nKB_t, nF_t = _nb(sum(len_t)), _nb(len_t[0] + len_t[1])
    idx, cnt = _random_lists(rng, 1, 2, nQB_s, nKB_s, 40, p_invalid=0.05)
    cnt[0, 1, :] = 0  # head 1: every source list empty
    idx_t, cnt_t = orc.transfer_lists(idx, cnt, len_s, len_t)
    for h in range(2):
        for i in range(idx_t.shape[2]):
            row = idx_t[0, h, i, :cnt_t[0, h, i]]
            assert (np.diff(row) > 0).all() and row.min() >= 0 and row.max() < nKB_t
            assert list(row[:nF_t]) == list(range(nF_t))
    assert (cnt_t[0, 1] == nF_t).all()


def test_error_returns(orc):
    # source cur block 1 maps onto target blocks 1..4: a row of 5 > stride 2
    idx = np.array([[[[1, 0]]]], np.int32)
    cnt = np.full((1, 1, 1), 2, np.int32)
    with pytest.raises(ValueError):
        orc.transfer_lists(idx, cnt, [128, 0, 0, 100], [128, 0, 0, 400], max_sel_t=2)
    idx_t, cnt_t = orc.transfer_lists(idx, cnt, [128, 0, 0, 100], [128, 0, 0, 400], max_sel_t=5)
    assert list(idx_t[0, 0, 0]) == [0, 1, 2, 3, 4] and cnt_t[0, 0, 0] == 5
    with pytest.raises(ValueError):  # no query tokens at the source
        orc.transfer_lists(np.zeros((1, 1, 0, 2), np.int32), np.zeros((1, 1, 0), np.int32),
                           [128, 0, 0, 0], [128, 0, 0, 400])


@pytest.mark.parametrize("layout", [
    ([100, 0, 700, 500], [100, 0, 420, 300]),
    ([100, 0, 252, 180], [100, 0, 420, 300]),
    ([100, 0, 735, 525], [100, 0, 420, 300]),
    ([100, 0, 559, 495], [100, 0, 435, 385]),
    ([1, 0, 127, 129], [1, 0, 1000, 1001]),
])
def test_single_block_lists_at_every_source_block(orc, layout):
    # Each source row lists one block; over the heads every source block is
    # listed alone, so every block boundary of the map is exercised.
    len_s, len_t = layout
    nKB_s, nQB_s = _nb(sum(len_s)), _nb(len_s[3])
    H = nKB_s
    idx = np.full((1, H, nQB_s, 1), -1, np.int32)
    for h in range(H):
        for i in range(nQB_s):
            idx[0, h, i, 0] = (h + 3 * i) % nKB_s
    cnt = np.ones((1, H, nQB_s), np.int32)
    expect = _inverse(idx, cnt, len_s, len_t)
    _check_against(orc.transfer_lists(idx, cnt, len_s, len_t), expect)
