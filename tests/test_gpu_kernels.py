"""GPU parity of each step against the CPU oracle, through the C ABI.

Pool, score and select must match the oracle bit for bit (same fixed fp32
orders; integer lists exactly).  Attention must be within the stated
tolerance of the oracle's fp64 attention given the same block lists.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_18_b200 import synth
import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_attention_18_b200 import build
    build.build()
    from block_sparse_attention_18_b200 import sparstar
    return sparstar


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


# ------------------------------------------------------------------ pool

@pytest.mark.parametrize("dtype,L,D", [("bf16", 128, 128), ("bf16", 1000, 128), ("bf16", 1, 128),
                                       ("bf16", 4097, 64), ("f32", 777, 64), ("f32", 300, 128)])
def test_pool_bit_exact(sp, orc, dtype, L, D):
    w = synth.custom(H=3, D=D, dtype=dtype, cur=L, seed=L + D)
    q, _, _ = synth.generate(w)
    got = sp.sparstar_block_pool(q.cuda()).cpu().numpy()
    want = orc.pool_f32(synth.as_numpy(q))
    assert np.array_equal(_bits(got), _bits(want))


def test_pool_order_fixture_cases(sp, orc):
    # values where any other summation order changes the fp32 result
    x = torch.zeros(1, 1, 133, 64)
    x[0, 0, 0, :] = 2.0 ** 24
    x[0, 0, 1, :8] = 1.0
    x[0, 0, 9, :8] = 1.0
    x[0, 0, 2, 8:16] = 1.0
    x[0, 0, 3, 8:16] = 1.0
    x[0, 0, 4, 16:24] = 1.0
    x[0, 0, 5, 16:24] = 1.0
    x[0, 0, 128:133, :] = torch.tensor([1.0, 2.0, 4.0, 0.0, 3.0])[:, None]
    x[0, 0, 130, 30] = -0.0
    got = sp.sparstar_block_pool(x.cuda()).cpu().numpy()
    want = orc.pool_f32(x.numpy())
    assert np.array_equal(_bits(got), _bits(want))


# ----------------------------------------------------------------- score

@pytest.mark.parametrize("Lq,Lk,D", [(1000, 3000, 128), (128, 128, 64), (9000, 20000, 128)])
def test_score_bit_exact(sp, orc, Lq, Lk, D):
    w = synth.custom(H=2, D=D, dtype="bf16", ref=Lk - Lq, cur=Lq, seed=Lk)
    q, k, _ = synth.generate(w)
    tau = np.float32(1.0 / np.sqrt(np.float64(D)))
    S = sp.sparstar_block_score(sp.sparstar_block_pool(q.cuda()), sp.sparstar_block_pool(k.cuda()),
                                float(tau)).cpu().numpy()
    Sw = orc.score_f32(orc.pool_f32(synth.as_numpy(q)), orc.pool_f32(synth.as_numpy(k)), float(tau))
    assert np.array_equal(_bits(S), _bits(Sw))


# ---------------------------------------------------------------- select

def _select_both(sp, orc, S, nF, density, max_sel=None):
    idx, cnt = sp.sparstar_select(torch.from_numpy(S).cuda(), nF, density, max_sel=max_sel)
    widx, wcnt = orc.select_f32(S, nF, density, max_sel=max_sel)
    return idx.cpu().numpy(), cnt.cpu().numpy(), widx, wcnt


@pytest.mark.parametrize("nKB", [2, 9, 40, 100, 200, 400, 900, 1129, 1158, 1600, 2100, 3000])
@pytest.mark.parametrize("density", [0.09375, 0.1875, 0.625, 1.0])
def test_select_bit_exact_random(sp, orc, nKB, density):
    rng = np.random.default_rng(nKB)
    S = rng.standard_normal((1, 2, 5, nKB)).astype(np.float32)
    nF = min(4, nKB - 1)
    idx, cnt, widx, wcnt = _select_both(sp, orc, S, nF, density)
    assert np.array_equal(cnt, wcnt)
    assert np.array_equal(idx, widx)


@pytest.mark.parametrize("nKB", [37, 300, 2500])
def test_select_ties_and_signed_zeros(sp, orc, nKB):
    rng = np.random.default_rng(7)
    vals = np.array([-2.0, -0.0, 0.0, 0.5, 0.5, 1.0, 3.0], np.float32)
    S = rng.choice(vals, size=(2, 1, 3, nKB)).astype(np.float32)
    S[0, 0, 0, :] = 0.25                      # all equal
    S[0, 0, 1, ::2] = -0.0                    # +0 / -0 mixture
    S[0, 0, 1, 1::2] = 0.0
    for nF in (0, 1, 33):
        for density in (1 / 3, 0.5, 0.9):
            idx, cnt, widx, wcnt = _select_both(sp, orc, S, nF, density, max_sel=nKB)
            assert np.array_equal(cnt, wcnt) and np.array_equal(idx, widx)


def test_select_k_equals_one_and_all_forced(sp, orc):
    S = np.random.default_rng(3).standard_normal((1, 1, 4, 50)).astype(np.float32)
    idx, cnt, widx, wcnt = _select_both(sp, orc, S, 2, 1 / 48)   # k = 1
    assert np.array_equal(idx, widx) and np.all(cnt == 3)
    idx, cnt, widx, wcnt = _select_both(sp, orc, S, 50, 0.5)     # C = 0: forced only
    assert np.array_equal(idx, widx) and np.all(cnt == 50)
