"""Parity of the fused selection front-end (sparstar_block_pool_qk,
sparstar_score_select, sparstar_forward_fused) with the oracle.

- Block means: bit-exact against the oracle's fixed-order fp32 pooling.
- Block lists: bit-exact against the oracle's fp32 selection on every row,
  on every workload at full size and on edge cases: ragged query and key
  tails, query-block counts that are not a multiple of the 16 rows a CTA
  scores, key-block counts at and around the 128-wide staging tile, exact
  ties (duplicated key blocks, all-zero query blocks), k = 1, k = C, C = 0,
  long rows whose threshold search gallops up from the smallest key or spans
  many binades, D = 64, fp32 inputs, and the largest nKB the fused kernel
  accepts.
- The whole fused chain, eager and replayed from a captured CUDA graph,
  against the oracle's attention on sampled rows.
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


def _selection_parity(sp, orc, w, q, k):
    """Pool + fused score/select on the GPU against the oracle's fp32 path."""
    qn, kn = synth.as_numpy(q), synth.as_numpy(k)
    qbar, kbar = sp.sparstar_block_pool_qk(q.cuda(), k.cuda())
    nF = sp.sparstar_forced_blocks(w.text, w.image_ref)
    kv_idx, kv_cnt = sp.sparstar_score_select(qbar, kbar, nF, w.density)
    torch.cuda.synchronize()
    oq, ok_, _, idx32, cnt32 = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    assert np.array_equal(qbar.cpu().numpy().view(np.uint32), oq.view(np.uint32))
    assert np.array_equal(kbar.cpu().numpy().view(np.uint32), ok_.view(np.uint32))
    assert np.array_equal(kv_cnt.cpu().numpy(), cnt32)
    gidx = kv_idx.cpu().numpy()
    bad = np.any(gidx != idx32, axis=-1)
    assert not bad.any(), "%d of %d rows differ" % (int(bad.sum()), bad.size)
    return qbar, kbar, kv_idx, kv_cnt


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_fused_selection_every_workload(sp, orc, name):
    w = synth.WORKLOADS[name]
    q, k, _ = synth.generate(w)
    _selection_parity(sp, orc, w, q, k)


EDGE = {
    # nQB = 17 (one row past a CTA's 16), ragged query and key tails
    "rows17_ragged": dict(H=2, text=300, ref=1000, cur=17 * 128 - 50, density=0.3),
    # nKB = 128 exactly (one full staging tile), then 129 (a one-block tail tile)
    "nkb128": dict(H=2, text=128, ref=64 * 128, cur=63 * 128, density=0.2),
    "nkb129": dict(H=2, text=128, ref=64 * 128 + 1, cur=63 * 128, density=0.2),
    # k = 1 and k = C
    "k1": dict(H=2, text=512, ref=3000, cur=4000, density=1e-3),
    "kC": dict(H=2, text=512, ref=3000, cur=4000, density=1.0),
    # no candidates at all: the forced text block is the only key block
    "c0": dict(H=2, text=100, cur=20, density=0.5),
    # D = 64 and fp32 inputs
    "d64_bf16": dict(H=2, D=64, text=256, ref=2000, cur=2100, density=0.25),
    "f32_d128": dict(H=2, dtype="f32", text=256, ref=2000, cur=2100, density=0.25),
    # Clip-1 layout: a forced prefix that ends inside a block
    "clip1": dict(H=2, text=512, image_ref=3600, ref=2000, cur=2000, density=0.1875),
    # the column kernel at its key-column boundaries: nKB = 256 (one column
    # per thread), 257 (two), 1536 (its largest), then 1537 (the TMA-tiled
    # kernel's first)
    "cols_nkb256": dict(H=2, text=128, ref=127 * 128, cur=128 * 128, density=0.15),
    "cols_nkb257": dict(H=2, text=128, ref=127 * 128 + 1, cur=128 * 128, density=0.15),
    "cols_max": dict(H=1, text=512, ref=1536 * 128 - 512 - 10 * 128, cur=10 * 128,
                     density=0.1),
    "tiled_min": dict(H=1, text=512, ref=1536 * 128 - 512 - 10 * 128 + 1, cur=10 * 128,
                      density=0.1),
    # the column kernel with crowded buckets (lists longer than 64 keys)
    "cols_one_bucket": dict(H=2, text=256, ref=40000, cur=38000, density=0.3,
                            offset_std=1e-3),
    # long rows: the threshold's binade found by galloping up from the
    # smallest key (k > C/2), and scores spread over many binades
    "cols_gallop_up": dict(H=2, text=256, ref=40000, cur=38000, density=0.8),
    "cols_wide_range": dict(H=2, text=256, ref=40000, cur=38000, density=0.2,
                            offset_std=50.0),
    # the TMA-tiled kernel's largest nKB (1664), then the first wide one (1665)
    "tiled_max": dict(H=1, text=512, ref=1650 * 128, cur=10 * 128, density=0.1),
    "wide_min": dict(H=1, text=512, ref=1650 * 128 + 1, cur=10 * 128, density=0.1),
    # the wide kernel with D = 64, 17 query blocks and ragged tails
    "wide_d64": dict(H=1, D=64, text=300, ref=1700 * 128, cur=17 * 128 - 9, density=0.1),
    # scores squeezed into one histogram bucket (offsets and noise tiny):
    # the bucket list holds whole rows
    "one_bucket": dict(H=2, text=256, ref=3000, cur=3000, density=0.2, offset_std=1e-3),
    # the same on the wide kernel with D = 64, where the bucket outgrows the
    # warp's scratch and the whole-row radix select takes over
    "wide_radix": dict(H=1, D=64, text=300, ref=1700 * 128, cur=17 * 128 - 9, density=0.1,
                       offset_std=1e-3),
}


@pytest.mark.parametrize("case", list(EDGE))
def test_fused_selection_edge_cases(sp, orc, case):
    kw = dict(EDGE[case])
    w = synth.custom(seed=11, **kw)
    q, k, _ = synth.generate(w)
    _, _, kv_idx, kv_cnt = _selection_parity(sp, orc, w, q, k)
    nF = sp.sparstar_forced_blocks(w.text, w.image_ref)
    sel = sp.sparstar_select_count(w.nKB, nF, w.density)
    assert int(kv_cnt.min()) == int(kv_cnt.max()) == sel


def test_fused_selection_exact_ties(sp, orc):
    """Duplicated key blocks give bit-equal scores; zero query blocks score 0
    against everything.  Both must resolve to the lower block index."""
    w = synth.custom(H=2, text=256, ref=2048, cur=3000, density=0.3, seed=5)
    q, k, _ = synth.generate(w)
    nF = sp.sparstar_forced_blocks(w.text, w.image_ref)
    # copy key blocks nF..nF+7 over every 3rd later block: many exact ties
    for j in range(nF + 8, w.nKB - 1, 3):
        src = nF + (j % 8)
        k[:, :, j * 128:(j + 1) * 128] = k[:, :, src * 128:(src + 1) * 128]
    q[:, :, 0:128] = 0          # first query block: every score is +0
    q[:, 1, 5 * 128:6 * 128] = 0
    _selection_parity(sp, orc, w, q, k)


def test_fused_selection_at_the_nkb_limit(sp, orc):
    limit = sp.sparstar_score_select_max_nkb(128)
    w = synth.custom(H=1, text=512, ref=(limit - 24) * 128, cur=20 * 128 - 7, density=0.05,
                     seed=6)
    assert w.nKB == limit
    q, k, _ = synth.generate(w)
    _selection_parity(sp, orc, w, q, k)


def test_fused_matches_separate_calls_bitwise(sp):
    """Same inputs through the five-launch chain and the three-launch chain:
    identical block lists, outputs and LSE."""
    w = synth.WORKLOADS["partial_tail"]
    q, k, v = (t.cuda() for t in synth.generate(w))
    out_a, lse_a, ws_a = sp.sparstar_forward(q, k, v, w.text, w.image_ref, w.ref, w.cur,
                                             w.density)
    out_b, lse_b, ws_b = sp.sparstar_forward_fused(q, k, v, w.text, w.image_ref, w.ref, w.cur,
                                                   w.density)
    torch.cuda.synchronize()
    assert ws_b.S is None
    assert torch.equal(ws_a.qbar, ws_b.qbar) and torch.equal(ws_a.kbar, ws_b.kbar)
    assert torch.equal(ws_a.kv_idx, ws_b.kv_idx) and torch.equal(ws_a.kv_cnt, ws_b.kv_cnt)
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)


@pytest.mark.parametrize("name", ["mid", "partial_tail"])
def test_fused_chain_in_a_cuda_graph(sp, orc, name):
    """Capture the fused chain once, replay it on two different inputs copied
    into the captured buffers; each replay matches the oracle."""
    w = synth.WORKLOADS[name]
    inputs = [synth.generate(w), synth.generate(synth.with_seed(w, w.seed + 100))]
    q, k, v = (t.cuda() for t in inputs[0])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # first call outside the capture (kernel attributes, driver entry points)
    out, lse, ws = sp.sparstar_forward_fused(q, k, v, w.text, w.image_ref, w.ref, w.cur,
                                             w.density, status=status)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            sp.sparstar_forward_fused(q, k, v, w.text, w.image_ref, w.ref, w.cur, w.density,
                                      workspace=ws, out=out, lse=lse, status=status)
    torch.cuda.current_stream().wait_stream(side)
    for qh, kh, vh in inputs:
        q.copy_(qh)
        k.copy_(kh)
        v.copy_(vh)
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        qn, kn, vn = (synth.as_numpy(t) for t in (qh, kh, vh))
        _, _, _, idx32, cnt32 = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
        assert np.array_equal(ws.kv_idx.cpu().numpy(), idx32)
        assert np.array_equal(ws.kv_cnt.cpu().numpy(), cnt32)
        rows = parity.sample_rows(w.B, w.H, w.Lq, per_head_blocks=3, rows_per_block=8,
                                  seed=w.seed)
        want, want_lse = orc.attn_rows_f64(qn, kn, vn, idx32, cnt32, rows)
        max_abs, rel_l2 = parity.check_out(parity.gather_rows(out, rows), want, w.dtype)
        parity.check_lse(parity.gather_rows(lse, rows), want_lse, w.dtype)
        print(json.dumps({"workload": name, "graph_replay": True, "max_abs": max_abs,
                          "rel_l2": rel_l2}))
    del graph


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f32", 128), ("bf16", 64)])
def test_fused_chain_on_the_simt_attention_path(sp, orc, dtype, D):
    """The three-launch chain where attention runs on the fp32 SIMT kernel
    (fp32 inputs, or D = 64): lists bit-exact, outputs within tolerance."""
    w = synth.custom(H=2, D=D, dtype=dtype, text=300, ref=700, cur=600, density=0.4, seed=21)
    q, k, v = synth.generate(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, ws = sp.sparstar_forward_fused(q.cuda(), k.cuda(), v.cuda(), w.text, w.image_ref,
                                             w.ref, w.cur, w.density, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    _, _, _, idx32, cnt32 = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    assert np.array_equal(ws.kv_idx.cpu().numpy(), idx32)
    assert np.array_equal(ws.kv_cnt.cpu().numpy(), cnt32)
    rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)
    want, want_lse = orc.attn_rows_f64(qn, kn, vn, idx32, cnt32, rows)
    parity.check_out(parity.gather_rows(out, rows), want, w.dtype)
    parity.check_lse(parity.gather_rows(lse, rows), want_lse, w.dtype)
