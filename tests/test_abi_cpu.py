"""The C-ABI library on a host without a GPU: it loads, exports every entry
point include/sparstar.h declares, computes its host-only helpers, and
rejects bad arguments with a status code before launching anything."""
import ctypes
import os
import re

import pytest
import torch

from block_sparse_attention_18_b200 import synth
from conftest import GOLDEN, ROOT

HEADER = os.path.join(ROOT, "include", "sparstar.h")


@pytest.fixture(scope="module")
def sp():
    from block_sparse_attention_18_b200 import build
    build.build()
    from block_sparse_attention_18_b200 import sparstar
    return sparstar


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\S.*?\b(sparstar_[a-z_0-9]+)\s*\(", text, re.M)))


def test_header_declares_the_four_steps():
    names = _declared_symbols()
    for n in ("sparstar_block_pool", "sparstar_block_score", "sparstar_select",
              "sparstar_attn_fwd", "sparstar_select_count", "sparstar_forced_blocks",
              "sparstar_forward", "sparstar_strerror", "sparstar_version"):
        assert n in names


def test_library_exports_every_declared_symbol(sp):
    lib = ctypes.CDLL(sp.LIB_PATH)
    missing = [n for n in _declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_strerror(sp):
    assert sp.lib.sparstar_version() >= 10000
    for code in range(6):
        assert sp.lib.sparstar_strerror(code)
    assert sp.lib.sparstar_strerror(99) == b"unknown status"


def test_select_count_matches_golden(sp):
    with open(os.path.join(GOLDEN, "select_counts.txt")) as fh:
        rows = [l.split() for l in fh if l.strip() and not l.startswith("#")]
    for name, Lk, nKB, nF, C, dens, k, sel in rows:
        w = synth.WORKLOADS[name]
        assert sp.sparstar_forced_blocks(w.text, w.image_ref) == int(nF)
        assert sp.sparstar_select_count(int(nKB), int(nF), float(dens)) == int(sel)


def test_select_count_and_forced_blocks_reject_bad_arguments(sp):
    assert sp.sparstar_select_count(10, 2, 0.0) == -1
    assert sp.sparstar_select_count(10, 2, 1.0000001) == -1
    assert sp.sparstar_select_count(10, 2, float("nan")) == -1
    assert sp.sparstar_select_count(10, 11, 0.5) == -1
    assert sp.sparstar_select_count(0, 0, 0.5) == -1
    assert sp.sparstar_select_count(10, 10, 0.5) == 10
    assert sp.sparstar_forced_blocks(-1, 0) == -1
    assert sp.sparstar_forced_blocks(512, 3600) == 33


# Fake device addresses: every call below fails its argument check before
# any CUDA call, so no address is ever dereferenced.
A = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10004)  # not 16-byte aligned
NUL = None


def test_pool_argument_errors(sp):
    L = sp.lib
    assert L.sparstar_block_pool(A, 7, 1, 1, 128, 128, A, NUL) == sp.EDTYPE
    assert L.sparstar_block_pool(NUL, 0, 1, 1, 128, 128, A, NUL) == sp.EINVAL
    assert L.sparstar_block_pool(A, 0, 1, 1, 128, 96, A, NUL) == sp.EINVAL
    assert L.sparstar_block_pool(A, 0, 1, 1, 0, 128, A, NUL) == sp.EINVAL
    assert L.sparstar_block_pool(MIS, 0, 1, 1, 128, 128, A, NUL) == sp.EINVAL


def test_score_argument_errors(sp):
    L = sp.lib
    assert L.sparstar_block_score(A, A, 1, 1, 4, 4, 128, float("inf"), A, NUL) == sp.EINVAL
    assert L.sparstar_block_score(A, NUL, 1, 1, 4, 4, 128, 0.1, A, NUL) == sp.EINVAL
    assert L.sparstar_block_score(A, A, 1, 1, 4, 4, 32, 0.1, A, NUL) == sp.EINVAL
    assert L.sparstar_block_score(A, A, 1, 70000, 4, 4, 128, 0.1, A, NUL) == sp.EINVAL


def test_select_argument_errors(sp):
    L = sp.lib
    assert L.sparstar_select(A, 1, 1, 4, 10, 2, 0.0, A, A, 10, NUL) == sp.EINVAL
    assert L.sparstar_select(A, 1, 1, 4, 10, 11, 0.5, A, A, 10, NUL) == sp.EINVAL
    assert L.sparstar_select(A, 1, 1, 4, 10, 2, 0.5, A, A, 5, NUL) == sp.ESIZE
    assert L.sparstar_select(NUL, 1, 1, 4, 10, 2, 0.5, A, A, 10, NUL) == sp.EINVAL


def test_attn_argument_errors(sp):
    L = sp.lib
    args = lambda **kw: [kw.get("q", A), A, A, kw.get("dtype", 0), 1, 1, kw.get("Lq", 128),
                         kw.get("Lk", 256), kw.get("D", 128), kw.get("tau", 0.088), A, A,
                         kw.get("max_sel", 2), kw.get("out", A), NUL, NUL, NUL]
    assert L.sparstar_attn_fwd(*args(dtype=3)) == sp.EDTYPE
    assert L.sparstar_attn_fwd(*args(q=NUL)) == sp.EINVAL
    assert L.sparstar_attn_fwd(*args(q=MIS)) == sp.EINVAL
    assert L.sparstar_attn_fwd(*args(out=MIS)) == sp.EINVAL
    assert L.sparstar_attn_fwd(*args(D=256)) == sp.EINVAL
    assert L.sparstar_attn_fwd(*args(Lk=0)) == sp.EINVAL
    assert L.sparstar_attn_fwd(*args(max_sel=-1)) == sp.EINVAL
    assert L.sparstar_attn_fwd(*args(tau=float("nan"))) == sp.EINVAL


def test_forward_checks_the_chain_first(sp):
    L = sp.lib
    # density outside (0, 1]
    assert L.sparstar_forward(A, A, A, 0, 1, 1, 128, 128, 0, 256, 256, 1.5, A, A, A, A, A, 8, A,
                              NUL, NUL, NUL) == sp.EINVAL
    # max_sel too small for ceil(0.5 * 4) + 1
    assert L.sparstar_forward(A, A, A, 0, 1, 1, 128, 128, 0, 256, 256, 0.5, A, A, A, A, A, 2, A,
                              NUL, NUL, NUL) == sp.ESIZE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_no_device_is_reported_not_crashed(sp):
    L = sp.lib
    assert L.sparstar_block_pool(A, 0, 1, 1, 128, 128, A, NUL) == sp.ENODEV
    assert L.sparstar_attn_fwd(A, A, A, 0, 1, 1, 128, 256, 128, 0.088, A, A, 2, A, NUL, NUL,
                               NUL) == sp.ENODEV


def test_fused_front_end_limits_and_argument_errors(sp):
    L = sp.lib
    # 16 score rows of stride ceil(nKB/128)*128 floats plus the staged tiles
    # must fit 227 KB of shared memory.
    assert sp.sparstar_score_select_max_nkb(128) == 2432
    assert sp.sparstar_score_select_max_nkb(64) == 2944
    assert sp.sparstar_score_select_max_nkb(96) == -1
    # every config of the scope table fits (largest: nKB 1158)
    for w in synth.WORKLOADS.values():
        assert w.nKB <= sp.sparstar_score_select_max_nkb(w.D)
    ss = lambda nKB, max_sel=4000, D=128, dens=0.5, q=A: L.sparstar_score_select(
        q, A, 1, 1, 4, nKB, D, 0.088, 2, dens, A, A, max_sel, NUL, NUL)
    assert ss(2433) == sp.ESIZE
    assert ss(10, max_sel=5) == sp.ESIZE
    assert ss(10, dens=0.0) == sp.EINVAL
    assert ss(10, D=32) == sp.EINVAL
    assert ss(10, q=MIS) == sp.EINVAL
    assert ss(10, q=NUL) == sp.EINVAL
    assert L.sparstar_block_pool_qk(A, A, 5, 1, 1, 128, 256, 128, A, A, NUL) == sp.EDTYPE
    assert L.sparstar_block_pool_qk(A, MIS, 0, 1, 1, 128, 256, 128, A, A, NUL) == sp.EINVAL
    assert L.sparstar_block_pool_qk(A, A, 0, 1, 1, 0, 256, 128, A, A, NUL) == sp.EINVAL
    assert L.sparstar_block_pool_qk(A, A, 0, 1, 1, 128, 256, 128, A, NUL, NUL) == sp.EINVAL
    # the fused chain is checked before anything launches
    fwd = lambda ref, max_sel, dens=0.5: L.sparstar_forward_fused(
        A, A, A, 0, 1, 1, 128, 128, 0, ref, 256, dens, A, A, A, A, max_sel, A, NUL, NUL, NUL)
    assert fwd(256, 2) == sp.ESIZE
    assert fwd(256, 8, dens=2.0) == sp.EINVAL
    assert fwd(2432 * 128, 4000) == sp.ESIZE  # nKB above the fused limit


def test_retained_mass_argument_errors(sp):
    L = sp.lib
    args = lambda **kw: [kw.get("q", A), A, kw.get("dtype", 0), 1, 1, 256, 640,  # noqa: E731
                         kw.get("D", 128), 0.088, kw.get("nF", 1), A, A, 4, A,
                         kw.get("n", 8), kw.get("scratch", A), A, A, A, A, NUL]
    assert L.sparstar_retained_mass(*args(dtype=9)) == sp.EDTYPE
    assert L.sparstar_retained_mass(*args(q=MIS)) == sp.EINVAL
    assert L.sparstar_retained_mass(*args(D=80)) == sp.EINVAL
    assert L.sparstar_retained_mass(*args(nF=6)) == sp.EINVAL  # nKB is 5
    assert L.sparstar_retained_mass(*args(nF=-1)) == sp.EINVAL
    assert L.sparstar_retained_mass(*args(n=0)) == sp.EINVAL
    assert L.sparstar_retained_mass(*args(scratch=NUL)) == sp.EINVAL


def test_transfer_lists_argument_errors(sp):
    L = sp.lib
    seg = lambda *v: (ctypes.c_int64 * 4)(*v)  # noqa: E731
    src, dst = seg(128, 0, 256, 256), seg(128, 0, 512, 512)  # nKB_t = 9

    def call(**kw):
        return L.sparstar_transfer_lists(kw.get("idx", A), A, kw.get("src_max_sel", 4),
                                         kw.get("B", 1), 1, kw.get("src", src),
                                         kw.get("dst", dst), kw.get("out", A), A,
                                         kw.get("dst_max_sel", 9), NUL)
    assert call(idx=NUL) == sp.EINVAL
    assert call(out=NUL) == sp.EINVAL
    assert call(B=0) == sp.EINVAL
    assert call(src_max_sel=0) == sp.EINVAL
    assert call(src=NUL) == sp.EINVAL
    assert call(src=seg(128, 0, -1, 256)) == sp.EINVAL
    assert call(src=seg(128, 0, 256, 0)) == sp.EINVAL  # target queries without a source
    # Hand-derived stride bound: nF_t = 1; the 8 other target blocks have
    # their centre images two by two in source blocks 1, 2, 3, 4.
    assert sp.sparstar_transfer_max_sel([128, 0, 256, 256], [128, 0, 512, 512], 4) == 9
    assert sp.sparstar_transfer_max_sel([128, 0, 256, 256], [128, 0, 512, 512], 2) == 5
    assert sp.sparstar_transfer_max_sel([128, 0, 256, 256], [128, 0, 512, 512], 1) == 3
    assert sp.sparstar_transfer_max_sel([128, 0, 256, 0], [128, 0, 512, 512], 1) == -1
    assert call(dst_max_sel=8) == sp.ESIZE  # below the bound (9)
    assert call(src=seg(128, 0, 32768 * 128, 256)) == sp.ESIZE  # source bitmap limit
    assert call(dst=seg(128, 0, 32768 * 128, 512)) == sp.ESIZE  # target block-map limit
    # no target rows: nothing to do, nothing launched, even without a device
    assert call(dst=seg(128, 0, 512, 0), dst_max_sel=9) == sp.OK
