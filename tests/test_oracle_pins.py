"""Pins of the CPU oracle against what the method's description and the
mathematics fix (CPU only).

Sources: SparSTAR (arXiv 2608.10519), pith.science review, "What carries the
argument" (128-token block means, S_ij = tau qbar_i^T kbar_j with
tau = D^-1/2, the block-average identity, forced text / Clip-1 reference,
joint Top-K under a density, forward-only sparse attention) and "Referee
Report" minor comment 5 (block-wise Top-K).

Each test checks the oracle against something other than itself: the
block-average identity evaluated by brute force, hand-derived fp32 values,
exhaustive subset enumeration, and torch's scaled_dot_product_attention in
fp64 as the textbook dense / masked special case.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from block_sparse_attention_18_b200 import synth
from conftest import GOLDEN

BLOCK = 128


def _bits_to_f32(h):
    return np.array([int(h, 16)], np.uint32).view(np.float32)[0]


def _read_cases(path):
    cases = []
    cur = None
    with open(path) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tok = line.split()
            if tok[0] == "case":
                cur = {"name": tok[1]}
                for kv in tok[2:]:
                    k, v = kv.split("=")
                    cur[k] = v
                cur["rows"] = {}
                cases.append(cur)
            else:
                cur["rows"][tok[0]] = tok[1:]
    return cases


# --------------------------------------------------------------- pooling

@pytest.mark.parametrize("case", _read_cases(os.path.join(GOLDEN, "pool_order.txt")),
                         ids=lambda c: c["name"])
def test_pool_f32_hand_derived(orc, case):
    L = int(case["L"])
    x = np.zeros((1, 1, L, 1), np.float32)
    for kv in case["rows"]["x"]:
        t, val = kv.split("=")
        x[0, 0, int(t), 0] = float(val)
    got = orc.pool_f32(x)[0, 0, int(case["block"]), 0]
    want = _bits_to_f32(case["expect"])
    assert got.view(np.uint32) == want.view(np.uint32), (got, want)


def test_pool_f64_partial_blocks_are_plain_means(orc):
    rng = np.random.default_rng(11)
    for L in (1, 127, 128, 129, 300, 515):
        x = rng.standard_normal((2, 3, L, 5)).astype(np.float32)
        got = orc.pool_f64(x)
        for blk in range(orc.nblocks(L)):
            seg = x[:, :, blk * BLOCK:min(L, (blk + 1) * BLOCK), :].astype(np.float64)
            np.testing.assert_allclose(got[:, :, blk], seg.mean(axis=2), rtol=1e-13, atol=1e-15)


def test_pool_f32_within_fp32_bound_of_f64(orc):
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((1, 2, 1000, 64)) * 3 + 1).astype(np.float32)
    m32 = orc.pool_f32(x).astype(np.float64)
    m64 = orc.pool_f64(x)
    # 16 sequential adds per stripe + 3 tree levels + 1 division: each
    # result is within (20 u) * mean|x| of the exact mean, u = 2^-24.
    absmean = np.abs(x.astype(np.float64))
    bound = 20 * 2.0 ** -24 * np.stack([absmean[:, :, b * BLOCK:(b + 1) * BLOCK].mean(axis=2)
                                        for b in range(orc.nblocks(1000))], axis=2)
    assert np.all(np.abs(m32 - m64) <= bound + 1e-30)


def test_pool_bf16_decoding_is_exact(orc):
    # bf16 inputs are widened exactly; pooling the bf16 tensor equals pooling
    # its exact fp32 widening (torch's conversion is the reference).
    g = torch.Generator().manual_seed(5)
    xb = torch.randn(1, 2, 333, 128, generator=g).to(torch.bfloat16)
    via_bf16 = orc.pool_f32(synth.as_numpy(xb))
    via_f32 = orc.pool_f32(xb.float().numpy())
    assert np.array_equal(via_bf16.view(np.uint32), via_f32.view(np.uint32))
    np.testing.assert_array_equal(orc.pool_f64(synth.as_numpy(xb)), orc.pool_f64(xb.float().numpy()))


# ----------------------------------------------------------------- score

def test_score_f32_hand_derived(orc):
    (case,) = _read_cases(os.path.join(GOLDEN, "score_order.txt"))
    D = int(case["D"])
    qbar = np.array([_bits_to_f32(h) for h in case["rows"]["qbar"]], np.float32).reshape(1, 1, 1, D)
    kbar = np.array([_bits_to_f32(h) for h in case["rows"]["kbar"]], np.float32).reshape(1, 1, 1, D)
    tau = np.float32(1.0 / math.sqrt(D))
    S = orc.score_f32(qbar, kbar, float(tau))
    want = _bits_to_f32(case["expect"])
    assert S[0, 0, 0, 0].view(np.uint32) == want.view(np.uint32)


@pytest.mark.parametrize("Lq,Lk,D", [(128, 128, 4), (200, 333, 16), (513, 1000, 64), (130, 1290, 128)])
def test_block_average_identity(orc, Lq, Lk, D):
    """qbar_i^T kbar_j equals the mean pairwise q.k over the two blocks, and
    S64 = tau times that, including partial blocks."""
    rng = np.random.default_rng(Lq * 7 + Lk)
    q = rng.standard_normal((1, 2, Lq, D)).astype(np.float32)
    k = rng.standard_normal((1, 2, Lk, D)).astype(np.float32)
    S64 = orc.score_f64(orc.pool_f64(q), orc.pool_f64(k))
    tau = 1.0 / math.sqrt(D)
    for h in range(2):
        for i in range(orc.nblocks(Lq)):
            Qi = q[0, h, i * BLOCK:min(Lq, (i + 1) * BLOCK)].astype(np.float64)
            for j in range(orc.nblocks(Lk)):
                Kj = k[0, h, j * BLOCK:min(Lk, (j + 1) * BLOCK)].astype(np.float64)
                pairwise = (Qi @ Kj.T).mean()
                assert abs(S64[0, h, i, j] - tau * pairwise) <= 1e-12 * max(1.0, abs(tau * pairwise))


def test_score_f32_within_bound_of_f64(orc):
    rng = np.random.default_rng(13)
    qbar = rng.standard_normal((1, 2, 9, 128)).astype(np.float32)
    kbar = rng.standard_normal((1, 2, 17, 128)).astype(np.float32)
    tau = np.float32(1.0 / math.sqrt(128))
    S32 = orc.score_f32(qbar, kbar, float(tau)).astype(np.float64)
    S64 = orc.score_f64(qbar.astype(np.float64), kbar.astype(np.float64))
    # fp32 tau differs from 1/sqrt(128) by < u; 128 sequential fma's
    bound = (130 * 2.0 ** -24) * tau * (np.abs(qbar).astype(np.float64) @ np.abs(kbar).astype(np.float64).transpose(0, 1, 3, 2))
    assert np.all(np.abs(S32 - S64) <= bound)


# ------------------------------------------------------------- selection

def _brute_force_select(scores, nF, k):
    """All k-subsets of the candidates; keep the one of largest exact sum,
    ties to the lexicographically smallest ascending index tuple (which is
    exactly 'top-k by score, ties to the lower index')."""
    nKB = len(scores)
    cands = range(nF, nKB)
    best, best_sum = None, None
    for sub in itertools.combinations(cands, k):
        s = sum((Fraction(float(scores[j])) for j in sub), Fraction(0))
        if best is None or s > best_sum or (s == best_sum and sub < best):
            best, best_sum = sub, s
    return list(range(nF)) + list(best)


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force(orc, seed):
    rng = np.random.default_rng(100 + seed)
    for trial in range(12):
        nKB = int(rng.integers(2, 13))
        nF = int(rng.integers(0, min(3, nKB - 1) + 1))
        C = nKB - nF
        density = float(rng.choice([1 / 8, 0.25, 0.3, 0.5, 0.625, 0.9, 1.0]))
        # coarse values force exact ties; +/-0 included
        vals = rng.choice(np.array([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 2.0, 3.5], np.float32), size=(1, 1, 3, nKB))
        if trial % 2:
            vals = rng.standard_normal((1, 1, 3, nKB)).astype(np.float32)
        k = min(C, math.ceil(density * C))
        for fn in (orc.select_f32, orc.select_f64):
            idx, cnt = fn(vals, nF, density)
            for i in range(3):
                assert cnt[0, 0, i] == nF + k
                assert list(idx[0, 0, i]) == _brute_force_select(vals[0, 0, i], nF, k)


def test_select_special_cases(orc):
    S = np.array([[[[5.0, 1.0, 2.0, 2.0, 0.0, -0.0, 2.0, 7.0]]]], np.float32)
    # k = C keeps everything (density 1)
    idx, cnt = orc.select_f32(S, 1, 1.0)
    assert list(idx[0, 0, 0]) == list(range(8)) and cnt[0, 0, 0] == 8
    # k = 1: the maximum candidate (block 7); the forced block 0 is not ranked
    idx, _ = orc.select_f32(S, 1, 1 / 7)
    assert list(idx[0, 0, 0]) == [0, 7]
    # three-way tie at 2.0 (blocks 2, 3, 6) with k = 3 -> 7 then the two lower tied blocks
    idx, _ = orc.select_f32(S, 1, 3 / 7)
    assert list(idx[0, 0, 0]) == [0, 2, 3, 7]
    # +0 and -0 are equal: the lower index (4) wins
    S2 = np.array([[[[9.0, -0.0, 0.0, -1.0]]]], np.float32)
    idx, _ = orc.select_f32(S2, 1, 1 / 3)
    assert list(idx[0, 0, 0]) == [0, 1]
    # all-equal scores: the k lowest candidates
    S3 = np.full((1, 1, 1, 10), 0.5, np.float32)
    idx, _ = orc.select_f32(S3, 2, 0.5)
    assert list(idx[0, 0, 0]) == [0, 1, 2, 3, 4, 5]
    # unused slots of a wider list are -1
    idx, cnt = orc.select_f32(S3, 2, 0.5, max_sel=8)
    assert list(idx[0, 0, 0]) == [0, 1, 2, 3, 4, 5, -1, -1] and cnt[0, 0, 0] == 6


def test_select_counts_golden(orc):
    rows = []
    with open(os.path.join(GOLDEN, "select_counts.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                rows.append(line.split())
    assert len(rows) == len(synth.WORKLOADS)
    for name, Lk, nKB, nF, C, dens, k, sel in rows:
        w = synth.WORKLOADS[name]
        assert w.Lk == int(Lk) and w.nKB == int(nKB) and w.density == float(dens)
        assert orc.forced_blocks(w.text, w.image_ref) == int(nF)
        assert int(nKB) - int(nF) == int(C)
        assert orc.select_count(w.nKB, int(nF), w.density) == int(sel)


def test_select_count_rejects_bad_arguments(orc):
    assert orc.select_count(10, 2, 0.0) == -1
    assert orc.select_count(10, 2, 1.5) == -1
    assert orc.select_count(10, 11, 0.5) == -1
    assert orc.select_count(0, 0, 0.5) == -1
    assert orc.select_count(10, 10, 0.5) == 10  # nothing left to rank


def test_forced_blocks_straddling(orc):
    # Clip 1: text 512 + image reference 3600 = 4112 tokens -> block 32 holds
    # tokens 4096..4223 and is forced.
    assert orc.forced_blocks(512, 3600) == 33
    assert orc.forced_blocks(512, 0) == 4
    assert orc.forced_blocks(0, 0) == 0
    assert orc.forced_blocks(1, 0) == 1


def test_fp32_selection_agrees_with_fp64_off_near_ties(orc):
    w = synth.custom(H=4, D=128, text=256, ref=1500, cur=1500, density=0.1875, seed=21)
    q, k, _ = synth.generate(w)
    qn, kn = synth.as_numpy(q), synth.as_numpy(k)
    _, _, _, idx32, _ = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    nF = orc.forced_blocks(w.text, w.image_ref)
    S64 = orc.score_f64(orc.pool_f64(qn), orc.pool_f64(kn))
    idx64, _ = orc.select_f64(S64, nF, w.density)
    kk = orc.select_count(w.nKB, nF, w.density) - nF
    gap, scale = orc.near_tie_gaps(S64, nF, kk)
    differ = np.any(idx32 != idx64, axis=-1)
    near = gap < 1e-6 * scale
    assert not np.any(differ & ~near)


# The near-tie rule: with a row's candidate scores sorted descending
# s(1) >= s(2) >= ..., the row's gap is s(k) - s(k+1) and its scale is the
# largest |S| over the candidates (forced blocks are not ranked, so they take
# no part).  Each row below is built so that its gap and scale are known
# without sorting anything.

def _gaps(orc, rows, nF, k):
    S = np.array(rows, np.float64)
    return orc.near_tie_gaps(S, nF, k)


def test_near_tie_gap_hand_built_rows(orc):
    # nF = 2 forced blocks hold the row's largest |S| (-200, 100): they must
    # not enter the scale.  Candidates (after the forced prefix):
    #   row 0: 3, 1, 7, 5     -> descending 7 5 | 3 1      gap 5 - 3 = 2, scale 7
    #   row 1: 4, 2, 4, 1     -> descending 4 4 | 2 1      gap 4 - 2 = 2, scale 4
    #   row 2: -3, -1, -7, -2 -> descending -1 -2 | -3 -7  gap 1, scale 7
    #   row 3: 9, 4.5, 10, 5  -> descending 10 9 | 5 4.5   gap 4 (the steps
    #          before and after it are 1 and 0.5, so an index off by one
    #          on either side gives another value)
    rows = [[100.0, -200.0, 3.0, 1.0, 7.0, 5.0],
            [-200.0, 100.0, 4.0, 2.0, 4.0, 1.0],
            [100.0, -200.0, -3.0, -1.0, -7.0, -2.0],
            [-200.0, 100.0, 9.0, 4.5, 10.0, 5.0]]
    gap, scale = _gaps(orc, rows, 2, 2)
    assert gap.tolist() == [2.0, 2.0, 1.0, 4.0]
    assert scale.tolist() == [7.0, 4.0, 7.0, 10.0]


def test_near_tie_gap_exact_tie_at_the_boundary(orc):
    # k = 1 with two equal leaders: s(1) = s(2) = 4, gap exactly 0.
    gap, scale = _gaps(orc, [[9.0, 2.0, 4.0, 1.0, 4.0]], 1, 1)
    assert gap[0] == 0.0 and scale[0] == 4.0
    # k = 2 on the same row: descending 4 4 | 2 1, gap 2.
    gap, _ = _gaps(orc, [[9.0, 2.0, 4.0, 1.0, 4.0]], 1, 2)
    assert gap[0] == 2.0


def test_near_tie_gap_is_infinite_when_nothing_or_everything_is_kept(orc):
    rows = [[5.0, 3.0, 1.0, 2.0], [0.0, -1.0, -1.0, -1.0]]
    for k in (0, 3):  # C = 3 candidates after nF = 1
        gap, scale = _gaps(orc, rows, 1, k)
        assert np.all(np.isposinf(gap))
        assert scale.tolist() == [3.0, 1.0]


def test_near_tie_gap_on_shuffled_rows_with_distinct_steps(orc):
    # Each row is a shuffle of v_1 > v_2 > ... whose steps v_i - v_{i+1}
    # are distinct powers of two (exact in fp64), so the gap at k is the
    # k-th step and nothing else; the rows differ, which also pins the row
    # stride.  Forced blocks carry values far outside the candidates.
    rng = np.random.default_rng(7)
    C, nF, nrow = 11, 3, 6
    rows, want_gap, want_scale = [], {}, []
    for r in range(nrow):
        steps = [2.0 ** e for e in rng.permutation(C - 1)]
        top = float(rng.integers(-40, 40))
        vals = [top]
        for s in steps:
            vals.append(vals[-1] - s)
        want_scale.append(max(abs(vals[0]), abs(vals[-1])))
        for k in range(1, C):
            want_gap[(r, k)] = steps[k - 1]
        forced = [1e6 * (1 + r), -2e6, 3e6]
        rows.append(forced + [vals[i] for i in rng.permutation(C)])
    for k in range(1, C):
        gap, scale = _gaps(orc, rows, nF, k)
        assert gap.tolist() == [want_gap[(r, k)] for r in range(nrow)], k
        assert scale.tolist() == want_scale


def test_near_tie_rule_flags_exactly_the_close_rows(orc):
    # The decision the GPU tests take from these values: gap < 1e-6 * scale.
    # Candidates 0.5, 0.5 - d, 0.25 with k = 1, so the scale is 0.5.
    # Row 0: d = 1e-7 -> near.  Row 1: d = 1e-5 -> not near.
    # Row 2: an exact tie -> near.  Row 3: k = C -> never near.
    rows = [[1.0, 0.5, 0.5 - 1e-7, 0.25], [1.0, 0.5, 0.5 - 1e-5, 0.25],
            [1.0, 0.5, 0.5, 0.25]]
    gap, scale = _gaps(orc, rows, 1, 1)
    near = gap < 1e-6 * scale
    assert near.tolist() == [True, False, True]
    gap, scale = _gaps(orc, rows, 1, 3)
    assert not np.any(gap < 1e-6 * scale)


# ------------------------------------------------------------- attention

def _to_f64(x):
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def _mask_from_lists(kv_idx, kv_cnt, Lq, Lk):
    B, H, nQB, _ = kv_idx.shape
    m = torch.zeros(B, H, Lq, Lk, dtype=torch.bool)
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                for j in kv_idx[b, h, i, :kv_cnt[b, h, i]]:
                    m[b, h, i * BLOCK:(i + 1) * BLOCK, j * BLOCK:(j + 1) * BLOCK] = True
    return m


@pytest.mark.parametrize("dtype,Lq,Lk,D", [("f32", 300, 421, 64), ("bf16", 128, 256, 128),
                                           ("bf16", 257, 1000, 128), ("f32", 1, 129, 64)])
def test_attention_density_one_is_dense_sdpa(orc, dtype, Lq, Lk, D):
    w = synth.custom(H=2, D=D, dtype=dtype, text=0, ref=Lk - Lq, cur=Lq, density=1.0, seed=Lq + Lk)
    q, k, v = synth.generate(w)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    _, _, _, idx, cnt = orc.run_selection(qn, kn, w.text, w.image_ref, 1.0)
    assert np.all(cnt == w.nKB)
    out, lse = orc.attn_rows_f64(qn, kn, vn, idx, cnt)
    q64, k64, v64 = (torch.from_numpy(_to_f64(t)) for t in (qn, kn, vn))
    ref = torch.nn.functional.scaled_dot_product_attention(q64, k64, v64)
    np.testing.assert_allclose(out.reshape(ref.shape), ref.numpy(), rtol=1e-11, atol=1e-12)
    ref_lse = torch.logsumexp((q64 @ k64.transpose(-1, -2)) / math.sqrt(D), dim=-1)
    np.testing.assert_allclose(lse.reshape(ref_lse.shape), ref_lse.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype,text,ref,cur,density", [("bf16", 128, 600, 650, 0.25),
                                                         ("f32", 200, 0, 700, 0.5),
                                                         ("bf16", 512, 300, 260, 0.1875)])
def test_attention_sparse_is_masked_sdpa(orc, dtype, text, ref, cur, density):
    w = synth.custom(H=2, D=64, dtype=dtype, text=text, ref=ref, cur=cur, density=density, seed=cur)
    q, k, v = synth.generate(w)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    _, _, _, idx, cnt = orc.run_selection(qn, kn, w.text, w.image_ref, density)
    out, lse = orc.attn_rows_f64(qn, kn, vn, idx, cnt)
    mask = _mask_from_lists(idx, cnt, w.Lq, w.Lk)
    q64, k64, v64 = (torch.from_numpy(_to_f64(t)) for t in (qn, kn, vn))
    ref_out = torch.nn.functional.scaled_dot_product_attention(q64, k64, v64, attn_mask=mask)
    np.testing.assert_allclose(out.reshape(ref_out.shape), ref_out.numpy(), rtol=1e-11, atol=1e-12)
    s = (q64 @ k64.transpose(-1, -2)) / math.sqrt(64)
    ref_lse = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(lse.reshape(ref_lse.shape), ref_lse.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_row_sampling_matches_full(orc):
    w = synth.custom(H=3, D=64, dtype="bf16", text=128, ref=300, cur=333, density=0.5, seed=3)
    q, k, v = synth.generate(w)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    _, _, _, idx, cnt = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    full, lse_full = orc.attn_rows_f64(qn, kn, vn, idx, cnt)
    rows = np.array([0, 5, 332, 333, 700, 998], np.int64)
    part, lse_part = orc.attn_rows_f64(qn, kn, vn, idx, cnt, rows)
    np.testing.assert_array_equal(part, full[rows])
    np.testing.assert_array_equal(lse_part, lse_full[rows])


def test_attention_empty_list_gives_zero_and_minus_inf(orc):
    q = np.ones((1, 1, 4, 64), np.float32)
    k = np.ones((1, 1, 200, 64), np.float32)
    idx = np.full((1, 1, 1, 2), -1, np.int32)
    cnt = np.zeros((1, 1, 1), np.int32)
    out, lse = orc.attn_rows_f64(q, k, k, idx, cnt)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
