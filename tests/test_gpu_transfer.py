"""Parity of the cross-scale list transfer (sparstar_transfer_lists, mask
reuse) with the oracle, bit for bit, and of attention over transferred lists.

Source: pith.science review of SparSTAR, "Extended reading notes / Core
claim" (a selection carried from one scale to another keeps less attention
mass than a fresh one) and Figure 1 (a carried-over mask can leave out blocks that
matter at the new scale).
The map between scales is the proportional per-segment reading that the
oracle's pins fix.

Source lists are either seeded random lists (with invalid entries, empty
rows and counts above the row stride) or the oracle's own fp32 selection of
synthetic source-scale inputs; no oracle input comes from the GPU.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_18_b200 import synth
import parity

pytestmark = pytest.mark.gpu

BLOCK = 128


@pytest.fixture(scope="module")
def sp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_attention_18_b200 import build
    build.build()
    from block_sparse_attention_18_b200 import sparstar
    return sparstar


def _nb(L):
    return (L + BLOCK - 1) // BLOCK


def _random_lists(rng, B, H, nQB, nKB, max_sel, count=None, p_invalid=0.0):
    idx = np.full((B, H, nQB, max_sel), -1, np.int32)
    cnt = np.zeros((B, H, nQB), np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                n = min(max_sel, nKB) if count is None else count
                n = int(rng.integers(0, n + 1)) if count is None else n
                chosen = np.sort(rng.choice(nKB, size=n, replace=False)).astype(np.int32)
                if p_invalid > 0 and n > 0:
                    bad = rng.random(n) < p_invalid
                    chosen[bad] = rng.choice([-1, nKB, nKB + 5, -77], size=int(bad.sum()))
                idx[b, h, i, :n] = chosen
                cnt[b, h, i] = n
    return idx, cnt


def _both(sp, orc, idx, cnt, len_s, len_t):
    got_idx, got_cnt = sp.sparstar_transfer_lists(torch.from_numpy(idx).cuda(),
                                                  torch.from_numpy(cnt).cuda(), len_s, len_t)
    torch.cuda.synchronize()
    stride = sp.sparstar_transfer_max_sel(len_s, len_t, idx.shape[-1])
    assert got_idx.shape[-1] == stride
    want_idx, want_cnt = orc.transfer_lists(idx, cnt, len_s, len_t, max_sel_t=stride)
    assert np.array_equal(got_cnt.cpu().numpy(), want_cnt)
    assert np.array_equal(got_idx.cpu().numpy(), want_idx)
    return want_idx, want_cnt


def _seg(w):
    return [w.text, w.image_ref, w.ref, w.cur]


# consecutive scales of the sweep (density schedule 0.625, 0.1875, 0.1875,
# 0.09375), both clip kinds, and the reverse direction
PAIRS = [("sweep_clip2_8000", "sweep_clip2_18000"), ("sweep_clip2_18000", "sweep_clip2_40500"),
         ("sweep_clip2_40500", "sweep_clip2_72000"), ("sweep_clip1_40500", "sweep_clip1_72000"),
         ("sweep_clip1_8000", "sweep_clip1_18000"), ("sweep_clip2_72000", "sweep_clip2_40500")]


@pytest.mark.parametrize("pair", PAIRS, ids=lambda p: "%s->%s" % p)
def test_sweep_scale_pairs_random_lists(sp, orc, pair):
    ws, wt = synth.WORKLOADS[pair[0]], synth.WORKLOADS[pair[1]]
    rng = np.random.default_rng(ws.Lk + 7 * wt.Lk)
    nF = _nb(ws.text + ws.image_ref)
    sel = nF + int(np.ceil(ws.density * (ws.nKB - nF)))
    idx, cnt = _random_lists(rng, 1, 2, ws.nQB, ws.nKB, sel, count=sel)
    _both(sp, orc, idx, cnt, _seg(ws), _seg(wt))


@pytest.mark.parametrize("seed", range(4))
def test_ragged_layouts_invalid_entries_and_batches(sp, orc, seed):
    rng = np.random.default_rng(500 + seed)
    text = int(rng.integers(1, 700))
    img = int(rng.choice([0, int(rng.integers(1, 3000))]))
    ref_s, cur_s = int(rng.integers(0, 5000)), int(rng.integers(1, 5000))
    ref_t = 0 if ref_s == 0 else max(1, int(ref_s * rng.uniform(0.3, 3.0)))
    cur_t = max(1, int(cur_s * rng.uniform(0.3, 3.0)))
    len_s, len_t = [text, img, ref_s, cur_s], [text, img, ref_t, cur_t]
    nKB_s, nQB_s = _nb(sum(len_s)), _nb(cur_s)
    idx, cnt = _random_lists(rng, 2, 3, nQB_s, nKB_s, max(1, nKB_s // 3), p_invalid=0.1)
    cnt[0, 0, 0] = idx.shape[-1] + 9  # a count above the stride reads as the stride
    cnt[1, 2, :] = 0  # empty source rows
    _both(sp, orc, idx, cnt, len_s, len_t)


def test_identity_and_exact_refinement(sp, orc):
    rng = np.random.default_rng(9)
    seg = [512, 3600, 9000, 9000]
    nKB, nQB = _nb(sum(seg)), _nb(seg[3])
    idx, cnt = _random_lists(rng, 1, 2, nQB, nKB, 60)
    _both(sp, orc, idx, cnt, seg, seg)
    len_s, len_t = [128, 0, 0, 128 * 40], [128, 0, 0, 256 * 40]
    idx, cnt = _random_lists(rng, 1, 2, 40, 41, 12)
    got_idx, got_cnt = _both(sp, orc, idx, cnt, len_s, len_t)
    src = {int(x) for x in idx[0, 1, 7, :cnt[0, 1, 7]]}
    assert list(got_idx[0, 1, 15, :got_cnt[0, 1, 15]]) == \
        [0] + [1 + q for q in range(80) if 1 + q // 2 in src]


def test_source_at_the_bitmap_limit(sp, orc):
    # 32768 source key blocks, the most the per-warp bitmap holds
    len_s = [128, 0, 32768 * 128 - 128 - 256, 256]
    len_t = [128, 0, 40000, 600]
    nKB_s = _nb(sum(len_s))
    assert nKB_s == 32768
    idx = np.array([[[[0, 5, 32766, 32767, 20000, -1], [0, 32767, 1, 2, 3, 4]]]], np.int32)
    cnt = np.array([[[5, 6]]], np.int32)
    _both(sp, orc, idx, cnt, len_s, len_t)


def test_attention_over_transferred_lists(sp, orc):
    # Fresh selection at the source scale (the oracle's fp32 path), carried
    # to the target scale, then the attention at the target over those lists.
    src = synth.custom(H=2, D=128, dtype="bf16", text=512, ref=2500, cur=2500, density=0.1875,
                       seed=31, offset_std=0.25)
    tgt = synth.custom(H=2, D=128, dtype="bf16", text=512, ref=5600, cur=5600, density=0.09375,
                       seed=32, offset_std=0.25)
    qs, ks, _ = synth.generate(src)
    _, _, _, sidx, scnt = orc.run_selection(synth.as_numpy(qs), synth.as_numpy(ks), src.text,
                                            src.image_ref, src.density)
    tidx, tcnt = _both(sp, orc, sidx, scnt, _seg(src), _seg(tgt))
    q, k, v = synth.generate(tgt)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    out, lse = sp.sparstar_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tidx).cuda(),
                                    torch.from_numpy(tcnt).cuda())
    torch.cuda.synchronize()
    rows = parity.sample_rows(tgt.B, tgt.H, tgt.Lq, seed=3)
    want, want_lse = orc.attn_rows_f64(qn, kn, vn, tidx, tcnt, rows)
    parity.check_out(parity.gather_rows(out, rows), want, "bf16")
    parity.check_lse(parity.gather_rows(lse, rows), want_lse, "bf16")
    # the transferred lists are longer than the target's own budget
    nF = _nb(tgt.text)
    sel_t = nF + int(np.ceil(tgt.density * (tgt.nKB - nF)))
    assert tcnt.mean() > sel_t


@pytest.mark.parametrize("pair", PAIRS[:3], ids=lambda p: "%s->%s" % p)
def test_worst_case_rows_reach_the_stride_bound(sp, orc, pair):
    # The bound is the forced prefix plus the largest per-source-block
    # counts.  The counts come from the oracle with single-block lists; a
    # row that lists the m blocks with the largest counts must reach it.
    ws, wt = synth.WORKLOADS[pair[0]], synth.WORKLOADS[pair[1]]
    seg_s, seg_t = _seg(ws), _seg(wt)
    nF_t = _nb(wt.text + wt.image_ref)
    one = np.tile(np.arange(ws.nKB, dtype=np.int32).reshape(1, ws.nKB, 1, 1), (1, 1, ws.nQB, 1))
    _, c1 = orc.transfer_lists(one, np.ones((1, ws.nKB, ws.nQB), np.int32), seg_s, seg_t)
    per_block = c1[0, :, 0] - nF_t  # target blocks kept through each source block
    m = 40
    top = np.sort(np.argsort(-per_block, kind="stable")[:m]).astype(np.int32)
    assert sp.sparstar_transfer_max_sel(seg_s, seg_t, m) == nF_t + int(np.sort(per_block)[-m:].sum())
    idx = np.tile(top, (1, 1, ws.nQB, 1))
    cnt = np.full((1, 1, ws.nQB), m, np.int32)
    got_idx, got_cnt = _both(sp, orc, idx, cnt, seg_s, seg_t)
    assert (got_cnt == got_idx.shape[-1]).all()


def test_target_at_the_block_map_limit(sp, orc):
    # 32768 target key blocks, the largest block map a CTA holds
    len_s = [128, 0, 50000, 700]
    len_t = [128, 0, 32768 * 128 - 128 - 900, 900]
    assert _nb(sum(len_t)) == 32768
    nKB_s = _nb(sum(len_s))
    rng = np.random.default_rng(77)
    idx, cnt = _random_lists(rng, 1, 2, _nb(len_s[3]), nKB_s, 60)
    _both(sp, orc, idx, cnt, len_s, len_t)
