"""GPU attention over block lists against the oracle's fp64 attention,
given the same lists (the oracle's own selection, or lists built by the
test): the tcgen05 kernel (bf16, D = 128) and the fp32 SIMT kernel."""
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


def _run(sp, orc, w, idx=None, cnt=None, scale=1.0, rows=None, expect_status=0):
    q, k, v = synth.generate(w)
    if scale != 1.0:
        q = (q.float() * scale).to(q.dtype)
        k = (k.float() * scale).to(k.dtype)
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    if idx is None:
        _, _, _, idx, cnt = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = sp.sparstar_attn_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda(),
                                    torch.from_numpy(cnt).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == expect_status
    if rows is None:
        rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)
    want, want_lse = orc.attn_rows_f64(qn, kn, vn, idx, cnt, rows)
    got = parity.gather_rows(out, rows)
    got_lse = parity.gather_rows(lse, rows)
    errs = parity.check_out(got, want, w.dtype)
    parity.check_lse(got_lse, want_lse, w.dtype)
    return errs


TC_CASES = [  # bf16, D = 128: the tcgen05 kernel
    dict(text=128, ref=256, cur=256, density=1.0),      # dense, all tiles full
    dict(text=0, ref=1, cur=128, density=1.0),          # Lk = 129: one real key in the tail tile
    dict(text=512, ref=700, cur=300, density=0.5),      # ragged Lq and Lk
    dict(text=512, ref=4000, cur=4000, density=0.1875),
    dict(text=100, ref=0, cur=1, density=1.0),          # one query row
    dict(text=512, ref=8192, cur=8192, density=0.625, H=2),  # long lists (> ring depth)
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "%d_%d_%d_%g" % (
    c["text"], c["ref"], c["cur"], c["density"]))
def test_tcgen05_attention_matches_oracle(sp, orc, case):
    w = synth.custom(H=case.get("H", 3), D=128, dtype="bf16", text=case["text"], ref=case["ref"],
                     cur=case["cur"], density=case["density"], seed=case["cur"] + case["ref"])
    _run(sp, orc, w)


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f32", 128), ("bf16", 64)])
@pytest.mark.parametrize("text,ref,cur,density", [(128, 0, 1024, 0.5), (200, 333, 517, 0.3)])
def test_simt_attention_matches_oracle(sp, orc, dtype, D, text, ref, cur, density):
    w = synth.custom(H=2, D=D, dtype=dtype, text=text, ref=ref, cur=cur, density=density,
                     seed=cur + D)
    _run(sp, orc, w)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_rescale_path_with_wide_score_range(sp, orc, dtype, D):
    # Q and K scaled up so the running max jumps by far more than the
    # rescale threshold from tile to tile; lists ordered by ascending score.
    w = synth.custom(H=2, D=D, dtype=dtype, text=0, ref=1024, cur=512, density=1.0,
                     offset_std=1.5, seed=99)
    q, k, _ = synth.generate(w)
    nQB, nKB = w.nQB, w.nKB
    S = orc.score_f64(orc.pool_f64(synth.as_numpy(q)), orc.pool_f64(synth.as_numpy(k)))
    idx = np.argsort(S, axis=-1, kind="stable").astype(np.int32)  # ascending score
    cnt = np.full((1, 2, nQB), nKB, np.int32)
    _run(sp, orc, w, idx=np.ascontiguousarray(idx), cnt=cnt, scale=2.0)


def test_empty_lists_duplicates_and_bad_indices(sp, orc):
    w = synth.custom(H=2, D=128, dtype="bf16", text=128, ref=300, cur=400, density=1.0, seed=5)
    nQB, nKB = w.nQB, w.nKB
    idx = np.full((1, 2, nQB, 6), -1, np.int32)
    cnt = np.zeros((1, 2, nQB), np.int32)
    idx[0, 0, 0, :3] = [0, 4, 2]          # unsorted list
    cnt[0, 0, 0] = 3
    idx[0, 0, 1, :2] = [1, 1]             # the same tile twice
    cnt[0, 0, 1] = 2
    # [0,0,2] and [0,1,*] except below stay empty: out = 0, lse = -inf
    idx[0, 1, 3, :4] = [3, nKB + 3, -7, nKB - 1]   # two bad entries are skipped
    cnt[0, 1, 3] = 4
    _run(sp, orc, w, idx=idx, cnt=cnt, expect_status=sp.STATUS_BAD_INDEX)


def test_for_fp32_simt_bad_indices_flagged(sp, orc):
    w = synth.custom(H=1, D=64, dtype="f32", text=0, ref=200, cur=256, density=1.0, seed=6)
    idx = np.array([[[[0, 9], [2, 1]]]], np.int32)
    cnt = np.array([[[2, 2]]], np.int32)
    _run(sp, orc, w, idx=idx, cnt=cnt, expect_status=sp.STATUS_BAD_INDEX)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_uneven_list_lengths_within_pairs(sp, orc, seed):
    """Query blocks run in pairs (2p, 2p+1), each with its own list: random
    lengths from 0 to every key block (so the pairs see every mix of equal,
    unequal, empty and longer-than-the-ring lists), random order, invalid
    entries mixed in, an odd number of query blocks (the last pair has no
    second block) and a partial last key block."""
    rng = np.random.default_rng(seed)
    w = synth.custom(H=2, D=128, dtype="bf16", text=256, ref=1900, cur=9 * 128 - 40,
                     density=1.0, seed=40 + seed)
    nQB, nKB = w.nQB, w.nKB
    assert nQB % 2 == 1
    max_sel = nKB + 4
    idx = np.full((1, w.H, nQB, max_sel), -1, np.int32)
    cnt = np.zeros((1, w.H, nQB), np.int32)
    bad = False
    for h in range(w.H):
        for i in range(nQB):
            n = int(rng.integers(0, nKB + 1))
            lst = rng.permutation(nKB)[:n].tolist()
            if n and rng.random() < 0.3:  # invalid entries are skipped
                lst.insert(int(rng.integers(0, n)), int(rng.choice([-3, nKB, nKB + 9])))
                bad = True
            idx[0, h, i, :len(lst)] = lst
            cnt[0, h, i] = len(lst)
    _run(sp, orc, w, idx=idx, cnt=cnt, expect_status=sp.STATUS_BAD_INDEX if bad else 0)


def test_every_list_length_pair_up_to_12(sp, orc):
    """Every pair of list lengths (nA, nB) with 0 <= nA, nB <= 12 in one
    launch: 19 heads x 9 query-block pairs, the pair (A, B) of head h, pair p
    taking combination 9h + p.  These are the pairs the ring's happens-before
    model covers (tests/test_ring_protocol.py); on the GPU each runs the
    producer order, the slot closed forms and the alternating full barriers
    through its own mix of key and value tiles."""
    w = synth.custom(H=19, D=128, dtype="bf16", text=128, ref=640, cur=18 * 128,
                     density=1.0, seed=77)
    nQB, nKB = w.nQB, w.nKB
    assert nQB == 18 and nKB >= 12
    rng = np.random.default_rng(12)
    combos = [(a, b) for a in range(13) for b in range(13)]
    idx = np.full((1, w.H, nQB, 12), -1, np.int32)
    cnt = np.zeros((1, w.H, nQB), np.int32)
    for c, (na, nb) in enumerate(combos):
        h, p = divmod(c, 9)
        for i, n in ((2 * p, na), (2 * p + 1, nb)):
            lst = np.sort(rng.choice(nKB, size=n, replace=False))
            idx[0, h, i, :n] = lst
            cnt[0, h, i] = n
    rows = parity.sample_rows(w.B, w.H, w.Lq, per_head_blocks=18, rows_per_block=4, seed=5)
    _run(sp, orc, w, idx=idx, cnt=cnt, rows=rows)


def test_many_pairs_with_uneven_lists(sp, orc):
    """More query-block pairs than SMs (16 heads x 24 pairs = 384), each
    block with a random list length in 0..7: pairs where one block has
    several more tiles than the other (a run of one block's P hand-offs at
    the end of the pair), blocks without tiles beside blocks with tiles, and
    consecutive pairs of a head with different mixes."""
    w = synth.custom(H=16, D=128, dtype="bf16", text=128, ref=1024, cur=48 * 128,
                     density=1.0, seed=91)
    nQB, nKB = w.nQB, w.nKB
    assert nQB == 48 and nKB >= 8
    rng = np.random.default_rng(4)
    idx = np.full((1, w.H, nQB, 7), -1, np.int32)
    cnt = np.zeros((1, w.H, nQB), np.int32)
    for h in range(w.H):
        for i in range(nQB):
            n = int(rng.integers(0, 8))
            idx[0, h, i, :n] = np.sort(rng.choice(nKB, size=n, replace=False))
            cnt[0, h, i] = n
    # uneven pairs (one block at least two tiles longer) are common
    pairs = cnt.reshape(w.H, nQB // 2, 2)
    assert (np.abs(pairs[..., 0] - pairs[..., 1]) >= 2).sum() > 100
    rows = parity.sample_rows(w.B, w.H, w.Lq, per_head_blocks=48, rows_per_block=2, seed=6)
    _run(sp, orc, w, idx=idx, cnt=cnt, rows=rows)
