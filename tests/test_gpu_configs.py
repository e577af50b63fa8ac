"""End-to-end parity on every workload at full size, in the launch
configuration the benchmark times (``sparstar_forward``: pool Q, pool K,
score, select, attention on one stream).

- Block lists: bit-exact against the oracle's fp32 selection on every row.
- Near ties (fp64 gap s(k) - s(k+1) < 1e-6 * max|S|) are logged; any row
  where the fp32 selection differs from the fp64 selection must be one.
- Attention: on sampled rows (first and last query block of every head,
  random blocks, first / last / random rows), within tolerance of the
  oracle's fp64 attention run on the oracle's own block lists.  Tiny is
  compared on every row.
"""
import json

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


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_end_to_end(sp, orc, name):
    w = synth.WORKLOADS[name]
    q, k, v = synth.generate(w)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, ws = sp.sparstar_forward(q.cuda(), k.cuda(), v.cuda(), w.text, w.image_ref, w.ref,
                                       w.cur, w.density, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    # selection: bit-exact
    _, _, _, idx32, cnt32 = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    assert np.array_equal(ws.kv_cnt.cpu().numpy(), cnt32)
    gidx = ws.kv_idx.cpu().numpy()
    mismatch = np.any(gidx != idx32, axis=-1)
    assert not mismatch.any(), "%d rows differ" % int(mismatch.sum())

    # near ties against the fp64 selection
    nF = orc.forced_blocks(w.text, w.image_ref)
    kk = orc.select_count(w.nKB, nF, w.density) - nF
    S64 = orc.score_f64(orc.pool_f64(qn), orc.pool_f64(kn))
    idx64, _ = orc.select_f64(S64, nF, w.density)
    gap, scale = orc.near_tie_gaps(S64, nF, kk)
    near = gap < parity.NEAR_TIE_REL * scale
    differ = np.any(idx32 != idx64, axis=-1)
    print(json.dumps({"workload": name, "rows": int(near.size), "near_tie_rows": int(near.sum()),
                      "fp32_vs_fp64_differ": int(differ.sum())}))
    assert not np.any(differ & ~near)

    # attention
    if name == "tiny":
        rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)
    else:
        rows = parity.sample_rows(w.B, w.H, w.Lq, seed=w.seed)
    want, want_lse = orc.attn_rows_f64(qn, kn, vn, idx32, cnt32, rows)
    max_abs, rel_l2 = parity.check_out(parity.gather_rows(out, rows), want, w.dtype)
    parity.check_lse(parity.gather_rows(lse, rows), want_lse, w.dtype)
    print(json.dumps({"workload": name, "rows_checked": int(rows.size), "max_abs": max_abs,
                      "rel_l2": rel_l2}))
