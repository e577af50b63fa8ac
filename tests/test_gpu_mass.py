"""Parity of the retained-attention-mass diagnostic (sparstar_retained_mass)
with the fp64 oracle.

Source: pith.science review of SparSTAR, "Extended reading notes / Core
claim" (retained attention mass of block-wise Top-K against the token-wise
upper bound) and "What would settle it" (token-wise Top-K at the same
densities).

The GPU scores are fp32 (q.k accumulated with fp32 FMAs) and every sum is
fp64, so against the fp64 oracle the masses agree to ~1e-6; the test bounds
are 2e-5 on masses and 1e-4 on the dense LSE.  The block mass is also
checked against exp(lse_sparse - lse_dense), with lse_sparse from the
attention kernel (relative 1e-3).
"""
import json

import numpy as np
import pytest
import torch

from block_sparse_attention_18_b200 import synth
import parity

pytestmark = pytest.mark.gpu

MASS_TOL = 2e-5
LSE_TOL = 1e-4


@pytest.fixture(scope="module")
def sp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_attention_18_b200 import build
    build.build()
    from block_sparse_attention_18_b200 import sparstar
    return sparstar


def _run(sp, orc, w, rows, q=None, k=None, v=None):
    if q is None:
        q, k, v = synth.generate(w)
    qn, kn = synth.as_numpy(q), synth.as_numpy(k)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse, ws = sp.sparstar_forward_fused(qd, kd, vd, w.text, w.image_ref, w.ref, w.cur,
                                             w.density)
    got = sp.sparstar_retained_mass(qd, kd, ws.kv_idx, ws.kv_cnt, ws.n_forced,
                                    torch.from_numpy(rows).cuda())
    torch.cuda.synchronize()
    got = {n: t.cpu().numpy() for n, t in got.items()}
    # The oracle gets its own lists (its fp32 selection), which the GPU's
    # lists must equal bit for bit; no oracle input comes from the GPU.
    _, _, _, oidx, ocnt = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    gidx, sel = ws.kv_idx.cpu().numpy(), oidx.shape[-1]
    assert np.array_equal(gidx[..., :sel], oidx) and (gidx[..., sel:] == -1).all()
    assert np.array_equal(ws.kv_cnt.cpu().numpy(), ocnt)
    want = orc.retained_mass_f64(qn, kn, oidx, ocnt, ws.n_forced, rows)
    for n in ("mass_block", "mass_tok", "mass_forced"):
        err = float(np.max(np.abs(got[n] - want[n])))
        assert err <= MASS_TOL, "%s: max err %.3g" % (n, err)
    err = float(np.max(np.abs(got["lse_dense"] - want["lse_dense"])))
    assert err <= LSE_TOL, "lse_dense: max err %.3g" % err
    # the block mass from the attention kernel's own LSE
    lse_sparse = parity.gather_rows(lse, rows)
    from_lse = np.exp(lse_sparse - got["lse_dense"])
    assert np.allclose(from_lse, got["mass_block"], rtol=1e-3, atol=0)
    eps = 1e-9
    assert np.all(got["mass_forced"] <= got["mass_block"] + eps)
    assert np.all(got["mass_block"] <= got["mass_tok"] + eps)
    assert np.all(got["mass_tok"] <= 1.0 + eps)
    return got


@pytest.mark.parametrize("name", ["tiny", "mid", "partial_tail", "sweep_clip1_18000"])
def test_mass_matches_oracle(sp, orc, name):
    w = synth.WORKLOADS[name]
    if name == "tiny":
        rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)
    else:
        rows = parity.sample_rows(w.B, w.H, w.Lq, per_head_blocks=2, rows_per_block=3,
                                  seed=w.seed)
    got = _run(sp, orc, w, rows)
    print(json.dumps({"workload": name, "rows": int(rows.size),
                      "mass_block": float(got["mass_block"].mean()),
                      "mass_tok": float(got["mass_tok"].mean())}))


def test_mass_largest_sampled_rows(sp, orc):
    w = synth.WORKLOADS["largest"]
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(w.B * w.H * w.Lq, 24, replace=False)).astype(np.int64)
    rows[0] = 0
    rows[-1] = w.B * w.H * w.Lq - 1  # the partial last query block of the last head
    _run(sp, orc, w, rows)


def test_mass_density_one_and_no_forced_blocks(sp, orc):
    w = synth.custom(H=2, D=128, dtype="bf16", text=0, ref=900, cur=1000, density=1.0, seed=8)
    rows = np.arange(0, w.B * w.H * w.Lq, 37, dtype=np.int64)
    got = _run(sp, orc, w, rows)
    assert np.allclose(got["mass_block"], 1.0, atol=1e-9)
    assert np.allclose(got["mass_tok"], 1.0, atol=1e-9)
    assert np.all(got["mass_forced"] == 0.0)


def test_mass_rows_outside_the_tensor_are_nan(sp):
    w = synth.custom(H=1, D=128, dtype="bf16", text=128, ref=300, cur=300, density=0.5, seed=2)
    q, k, _ = (t.cuda() for t in synth.generate(w))
    nF = sp.sparstar_forced_blocks(w.text, w.image_ref)
    qbar, kbar = sp.sparstar_block_pool_qk(q, k)
    idx, cnt = sp.sparstar_score_select(qbar, kbar, nF, w.density)
    rows = torch.tensor([-1, 0, w.Lq, 5], dtype=torch.int64, device="cuda")
    got = sp.sparstar_retained_mass(q, k, idx, cnt, nF, rows)
    torch.cuda.synchronize()
    mb = got["mass_block"].cpu().numpy()
    assert np.isnan(mb[0]) and np.isnan(mb[2])
    assert np.isfinite(mb[1]) and np.isfinite(mb[3])
