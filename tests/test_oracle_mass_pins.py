"""Pins of the oracle's retained-attention-mass diagnostic (CPU only).

Sources: pith.science review of SparSTAR, "Extended reading notes / Core
claim" (block-wise Top-K recomputed at every scale stays close to the
token-wise upper bound in retained attention mass) and "What would settle
it" (the exact token-wise Top-K at the same densities as the comparison).

Reading: retained mass of a mask for one query row = the sum of the row's
dense softmax weights over the kept keys; the token-wise bound keeps the
forced blocks and spends the block list's candidate-token budget M on the
M largest candidate weights.

Each test checks the oracle against something other than its own code:
density 1 (mass exactly 1), uniform scores (token-count ratios), a two-level
score construction with a closed form, brute force over every pair of
candidate tokens with weights from torch.softmax, and the identity
mass_block = exp(lse_sparse - lse_dense) against the oracle's separate
attention routine.
"""
import math

import numpy as np
import torch

from block_sparse_attention_18_b200 import synth

BLOCK = 128


def _full_lists(nQB, nKB, B=1, H=1):
    idx = np.tile(np.arange(nKB, dtype=np.int32), (B, H, nQB, 1))
    cnt = np.full((B, H, nQB), nKB, np.int32)
    return idx, cnt


def _fixed_lists(blocks, nQB, B=1, H=1):
    idx = np.tile(np.array(blocks, np.int32), (B, H, nQB, 1))
    cnt = np.full((B, H, nQB), len(blocks), np.int32)
    return idx, cnt


def test_density_one_retains_everything(orc):
    w = synth.custom(H=2, D=64, dtype="f32", text=128, ref=500, cur=300, density=1.0, seed=3)
    q, k, _ = synth.generate(w)
    qn, kn = synth.as_numpy(q), synth.as_numpy(k)
    nF = orc.forced_blocks(w.text, w.image_ref)
    idx, cnt = _full_lists(w.nQB, w.nKB, H=w.H)
    rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)[::7]
    m = orc.retained_mass_f64(qn, kn, idx, cnt, nF, rows)
    assert np.allclose(m["mass_block"], 1.0, rtol=0, atol=1e-12)
    assert np.allclose(m["mass_tok"], 1.0, rtol=0, atol=1e-12)


def test_uniform_scores_give_token_count_ratios(orc):
    # q = 0: every score is 0 and every dense weight is 1 / Lk.
    w = synth.custom(H=1, D=64, dtype="f32", text=200, ref=300, cur=260, density=0.5, seed=4)
    _, k, _ = synth.generate(w)
    q = torch.zeros(w.B, w.H, w.Lq, w.D)
    qn, kn = synth.as_numpy(q), synth.as_numpy(k)
    nF = orc.forced_blocks(w.text, w.image_ref)  # 2 blocks: tokens 0..255
    blocks = [0, 1, 3, w.nKB - 1]                # the last block is partial
    idx, cnt = _fixed_lists(blocks, w.nQB)
    rows = np.arange(w.Lq, dtype=np.int64)
    m = orc.retained_mass_f64(qn, kn, idx, cnt, nF, rows)
    Lk = w.Lk
    tokens = lambda j: min(BLOCK, Lk - BLOCK * j)  # noqa: E731
    kept = sum(tokens(j) for j in blocks)
    forced = sum(tokens(j) for j in range(nF))
    assert np.allclose(m["lse_dense"], math.log(Lk), rtol=0, atol=1e-12)
    assert np.allclose(m["mass_block"], kept / Lk, rtol=0, atol=1e-12)
    assert np.allclose(m["mass_forced"], forced / Lk, rtol=0, atol=1e-12)
    assert np.allclose(m["mass_tok"], kept / Lk, rtol=0, atol=1e-12)


def test_two_level_scores_closed_form(orc):
    # Scores take two values: tau*c on a "hot" token set, 0 elsewhere, so
    # every mass is a ratio of counts weighted by e^(tau c).
    D, c = 64, 24.0
    tau = 1.0 / math.sqrt(D)
    text, ref, cur = 128, 700, 140
    Lk, Lq = text + ref + cur, cur
    rng = np.random.default_rng(7)
    k = rng.standard_normal((1, 1, Lk, D)).astype(np.float32)
    hot = np.zeros(Lk, bool)
    hot[rng.choice(Lk, 90, replace=False)] = True
    k[0, 0, :, 0] = np.where(hot, 1.0, 0.0)
    q = np.zeros((1, 1, Lq, D), np.float32)
    q[..., 0] = c
    nF = 1
    nQB, nKB = (Lq + BLOCK - 1) // BLOCK, (Lk + BLOCK - 1) // BLOCK
    blocks = [0, 2, 5, nKB - 1]
    idx, cnt = _fixed_lists(blocks, nQB)
    m = orc.retained_mass_f64(q, k, idx, cnt, nF, np.array([0, 77, Lq - 1], np.int64))
    e = math.exp(tau * c)
    Z = hot.sum() * e + (Lk - hot.sum())
    in_block = np.zeros(Lk, bool)
    for j in blocks:
        in_block[j * BLOCK:(j + 1) * BLOCK] = True
    forced = np.zeros(Lk, bool)
    forced[:nF * BLOCK] = True
    mass = lambda sel: (hot[sel].sum() * e + (~hot[sel]).sum()) / Z  # noqa: E731
    M = int((in_block & ~forced).sum())
    hot_cand = int((hot & ~forced).sum())
    top = (min(M, hot_cand) * e + max(0, M - hot_cand)) / Z
    assert np.allclose(m["lse_dense"], math.log(Z), rtol=0, atol=1e-12)
    assert np.allclose(m["mass_block"], mass(in_block), rtol=0, atol=1e-12)
    assert np.allclose(m["mass_forced"], mass(forced), rtol=0, atol=1e-12)
    assert np.allclose(m["mass_tok"], mass(forced) + top, rtol=0, atol=1e-12)


def test_token_bound_is_the_best_pair_by_brute_force(orc):
    # Keys [text 128 | ref 256 | cur 130]: Lk = 514, so the last key block
    # holds 2 tokens.  Listing the forced block and that tail gives a
    # candidate budget of 2, and the bound adds the best pair of candidate
    # weights, found here over every pair.
    D = 64
    w = synth.custom(H=1, D=D, dtype="f32", text=128, ref=256, cur=130, density=0.5,
                     offset_std=0.7, seed=9)
    q, k, _ = synth.generate(w)
    assert w.Lk == 514 and w.nKB == 5
    idx, cnt = _fixed_lists([0, w.nKB - 1], w.nQB)
    rows = np.array([0, 5, w.Lq - 1], np.int64)
    m = orc.retained_mass_f64(synth.as_numpy(q), synth.as_numpy(k), idx, cnt, 1, rows)
    for n, r in enumerate(rows):
        s = (q[0, 0, r].double() @ k[0, 0].double().T) / math.sqrt(D)
        p = torch.softmax(s, dim=0).numpy()
        cand = p[BLOCK:]
        pair = cand[:, None] + cand[None, :]
        np.fill_diagonal(pair, -np.inf)
        assert abs(m["mass_forced"][n] - p[:BLOCK].sum()) <= 1e-12
        assert abs(m["mass_block"][n] - (p[:BLOCK].sum() + p[512:].sum())) <= 1e-12
        assert abs(m["mass_tok"][n] - (p[:BLOCK].sum() + pair.max())) <= 1e-12
        assert abs(m["lse_dense"][n] - torch.logsumexp(s, 0).item()) <= 1e-12


def test_invariants_and_lse_identity(orc):
    w = synth.custom(H=2, D=128, dtype="bf16", text=300, ref=900, cur=700, density=0.3,
                     seed=12)
    q, k, v = synth.generate(w)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    _, _, _, idx, cnt = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    nF = orc.forced_blocks(w.text, w.image_ref)
    rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)[::11]
    m = orc.retained_mass_f64(qn, kn, idx, cnt, nF, rows)
    _, lse_sparse = orc.attn_rows_f64(qn, kn, vn, idx, cnt, rows)
    eps = 1e-12
    assert np.all(m["mass_forced"] <= m["mass_block"] + eps)
    assert np.all(m["mass_block"] <= m["mass_tok"] + eps)
    assert np.all(m["mass_tok"] <= 1.0 + eps)
    assert np.allclose(m["mass_block"], np.exp(lse_sparse - m["lse_dense"]), rtol=1e-10,
                       atol=0)
