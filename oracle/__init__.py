"""CPU oracle for SparSTAR's per-scale block-sparse attention forward.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import this package.  It is a
thin ctypes wrapper over ``sparstar_oracle.c`` (plain C, fp64 attention and
an fp32 selection path in a fixed, stated order) and shares nothing with the
CUDA path.

Every function takes and returns numpy arrays on the host.  Tensors are
[B, H, L, D] row-major; bf16 tensors are passed as uint16 bit patterns.

Method passages each function follows (SparSTAR, arXiv 2608.10519; pith.science
review, "What carries the argument"): 128-token block means, the score
S_ij = tau * qbar_i^T kbar_j with tau = D^-1/2, forced text / Clip-1 image
reference blocks, joint Top-K of the remaining blocks under a density, and
attention over the selected blocks only.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(block-average identity, hand-derived order fixtures, brute-force top-k,
dense-attention and masked-attention special cases against torch's
scaled_dot_product_attention), ``tests/test_oracle_mass_pins.py`` (retained
mass) and ``tests/test_oracle_transfer_pins.py`` (lists carried across scales:
identity, a 2x closed form, the inverse formulation).  No function is
parity unpinned.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
BLOCK = 128


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        vp = ctypes.c_void_p
        L.orc_num_threads.restype = i32
        L.orc_forced_blocks.argtypes = [i64, i64]
        L.orc_forced_blocks.restype = i64
        L.orc_select_count.argtypes = [i64, i64, f64]
        L.orc_select_count.restype = i64
        L.orc_pool_f32.argtypes = [vp, i32, i64, i64, i64, i64, vp]
        L.orc_pool_f64.argtypes = [vp, i32, i64, i64, i64, i64, vp]
        L.orc_score_f32.argtypes = [vp, vp, i64, i64, i64, i64, i64, f32, vp]
        L.orc_score_f64.argtypes = [vp, vp, i64, i64, i64, i64, i64, vp]
        L.orc_select_f32.argtypes = [vp, i64, i64, i64, i64, i64, f64, vp, vp, i64]
        L.orc_select_f32.restype = i32
        L.orc_select_f64.argtypes = [vp, i64, i64, i64, i64, i64, f64, vp, vp, i64]
        L.orc_select_f64.restype = i32
        L.orc_near_tie_gaps.argtypes = [vp, i64, i64, i64, i64, vp, vp]
        L.orc_attn_rows_f64.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64,
                                        vp, vp, i64, i64, vp, vp, vp]
        L.orc_retained_mass_f64.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, i64,
                                            vp, vp, i64, i64, vp, vp, vp, vp, vp]
        L.orc_transfer_lists.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp, i64]
        L.orc_transfer_lists.restype = i32
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return 0
    if x.dtype == np.float32:
        return 1
    raise TypeError("oracle inputs are bf16 bit patterns (uint16) or float32, got %s" % x.dtype)


def nblocks(L: int) -> int:
    return (L + BLOCK - 1) // BLOCK


def num_threads() -> int:
    return lib().orc_num_threads()


def forced_blocks(text_len: int, image_ref_len: int) -> int:
    return lib().orc_forced_blocks(text_len, image_ref_len)


def select_count(nKB: int, nF: int, density: float) -> int:
    return lib().orc_select_count(nKB, nF, density)


def pool_f32(x: np.ndarray) -> np.ndarray:
    """fp32 block means in the fixed stripe order; x: [B,H,L,D]."""
    x = np.ascontiguousarray(x)
    B, H, L, D = x.shape
    out = np.empty((B, H, nblocks(L), D), np.float32)
    lib().orc_pool_f32(_ptr(x), _dtype_code(x), B, H, L, D, _ptr(out))
    return out


def pool_f64(x: np.ndarray) -> np.ndarray:
    """fp64 block means (plain definition); x: [B,H,L,D]."""
    x = np.ascontiguousarray(x)
    B, H, L, D = x.shape
    out = np.empty((B, H, nblocks(L), D), np.float64)
    lib().orc_pool_f64(_ptr(x), _dtype_code(x), B, H, L, D, _ptr(out))
    return out


def score_f32(qbar: np.ndarray, kbar: np.ndarray, tau: float) -> np.ndarray:
    qbar = np.ascontiguousarray(qbar, np.float32)
    kbar = np.ascontiguousarray(kbar, np.float32)
    B, H, nQB, D = qbar.shape
    nKB = kbar.shape[2]
    S = np.empty((B, H, nQB, nKB), np.float32)
    lib().orc_score_f32(_ptr(qbar), _ptr(kbar), B, H, nQB, nKB, D, tau, _ptr(S))
    return S


def score_f64(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    qbar = np.ascontiguousarray(qbar, np.float64)
    kbar = np.ascontiguousarray(kbar, np.float64)
    B, H, nQB, D = qbar.shape
    nKB = kbar.shape[2]
    S = np.empty((B, H, nQB, nKB), np.float64)
    lib().orc_score_f64(_ptr(qbar), _ptr(kbar), B, H, nQB, nKB, D, _ptr(S))
    return S


def _select(fn, S, nF, density, max_sel):
    B, H, nQB, nKB = S.shape
    sel = select_count(nKB, nF, density)
    if sel < 0:
        raise ValueError("bad selection arguments")
    if max_sel is None:
        max_sel = sel
    kv_idx = np.empty((B, H, nQB, max_sel), np.int32)
    kv_cnt = np.empty((B, H, nQB), np.int32)
    rc = fn(_ptr(S), B, H, nQB, nKB, nF, density, _ptr(kv_idx), _ptr(kv_cnt), max_sel)
    if rc != 0:
        raise ValueError("oracle select failed (%d)" % rc)
    return kv_idx, kv_cnt


def select_f32(S: np.ndarray, nF: int, density: float, max_sel=None):
    return _select(lib().orc_select_f32, np.ascontiguousarray(S, np.float32), nF, density, max_sel)


def select_f64(S: np.ndarray, nF: int, density: float, max_sel=None):
    return _select(lib().orc_select_f64, np.ascontiguousarray(S, np.float64), nF, density, max_sel)


def near_tie_gaps(S64: np.ndarray, nF: int, k: int):
    S64 = np.ascontiguousarray(S64, np.float64)
    nKB = S64.shape[-1]
    nrow = S64.size // nKB
    gap = np.empty(nrow, np.float64)
    scale = np.empty(nrow, np.float64)
    lib().orc_near_tie_gaps(_ptr(S64), nrow, nKB, nF, k, _ptr(gap), _ptr(scale))
    return gap.reshape(S64.shape[:-1]), scale.reshape(S64.shape[:-1])


def attn_rows_f64(q, k, v, kv_idx, kv_cnt, rows=None):
    """fp64 attention over the listed blocks for the given flat rows
    (bh * Lq + r); all rows when ``rows`` is None.  Returns (out, lse)."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    code = _dtype_code(q)
    assert _dtype_code(k) == code and _dtype_code(v) == code
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    kv_idx = np.ascontiguousarray(kv_idx, np.int32)
    kv_cnt = np.ascontiguousarray(kv_cnt, np.int32)
    max_sel = kv_idx.shape[-1]
    if rows is None:
        rows = np.arange(B * H * Lq, dtype=np.int64)
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.empty((rows.size, D), np.float64)
    lse = np.empty(rows.size, np.float64)
    lib().orc_attn_rows_f64(_ptr(q), _ptr(k), _ptr(v), code, B, H, Lq, Lk, D,
                            _ptr(kv_idx), _ptr(kv_cnt), max_sel, rows.size, _ptr(rows),
                            _ptr(out), _ptr(lse))
    return out, lse


def retained_mass_f64(q, k, kv_idx, kv_cnt, nF, rows):
    """Retained attention mass of the block lists and the token-wise bound at
    the same candidate-token budget, in fp64, for the flat rows given.
    Returns a dict of arrays: lse_dense, mass_block, mass_tok, mass_forced."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    code = _dtype_code(q)
    assert _dtype_code(k) == code
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    kv_idx = np.ascontiguousarray(kv_idx, np.int32)
    kv_cnt = np.ascontiguousarray(kv_cnt, np.int32)
    rows = np.ascontiguousarray(rows, np.int64)
    out = {n: np.empty(rows.size, np.float64)
           for n in ("lse_dense", "mass_block", "mass_tok", "mass_forced")}
    lib().orc_retained_mass_f64(_ptr(q), _ptr(k), code, B, H, Lq, Lk, D, nF, _ptr(kv_idx),
                                _ptr(kv_cnt), kv_idx.shape[-1], rows.size, _ptr(rows),
                                _ptr(out["lse_dense"]), _ptr(out["mass_block"]),
                                _ptr(out["mass_tok"]), _ptr(out["mass_forced"]))
    return out


def transfer_lists(kv_idx, kv_cnt, len_s, len_t, max_sel_t=None):
    """Block lists of a source scale carried to a target scale by position
    (the mask reuse the method argues against).  kv_idx [B,H,nQB_s,max_sel_s],
    kv_cnt [B,H,nQB_s]; len_s, len_t: the four segment lengths (text,
    image_ref, ref, cur) at each scale.  Returns (kv_idx_t, kv_cnt_t) with
    max_sel_t = nKB_t unless given."""
    kv_idx = np.ascontiguousarray(kv_idx, np.int32)
    kv_cnt = np.ascontiguousarray(kv_cnt, np.int32)
    B, H, _, max_sel_s = kv_idx.shape
    ls = np.ascontiguousarray(len_s, np.int64)
    lt = np.ascontiguousarray(len_t, np.int64)
    assert ls.shape == (4,) and lt.shape == (4,)
    assert kv_idx.shape[2] == nblocks(int(ls[3])) and kv_cnt.shape == kv_idx.shape[:3]
    nKB_t = nblocks(int(lt.sum()))
    nQB_t = nblocks(int(lt[3]))
    if max_sel_t is None:
        max_sel_t = nKB_t
    idx_t = np.empty((B, H, nQB_t, max_sel_t), np.int32)
    cnt_t = np.empty((B, H, nQB_t), np.int32)
    rc = lib().orc_transfer_lists(_ptr(kv_idx), _ptr(kv_cnt), max_sel_s, B, H, _ptr(ls),
                                  _ptr(lt), _ptr(idx_t), _ptr(cnt_t), max_sel_t)
    if rc != 0:
        raise ValueError("orc_transfer_lists: bad arguments (code %d)" % rc)
    return idx_t, cnt_t


def run_selection(q, k, text_len, image_ref_len, density):
    """The fp32 selection path end to end (pool Q, pool K, score, select).
    Returns (qbar, kbar, S, kv_idx, kv_cnt)."""
    D = q.shape[-1]
    tau = np.float32(1.0 / np.sqrt(np.float64(D)))
    qbar = pool_f32(q)
    kbar = pool_f32(k)
    S = score_f32(qbar, kbar, float(tau))
    nF = forced_blocks(text_len, image_ref_len)
    kv_idx, kv_cnt = select_f32(S, nF, density)
    return qbar, kbar, S, kv_idx, kv_cnt
