"""Python binding of libsparstar (C ABI in include/sparstar.h).

Argument marshalling only: every function reads device pointers, shapes and
the current CUDA stream from torch tensors, allocates missing outputs with
torch, and calls the entry point of the same name.  Every step of the path
runs in the library's kernels; there is no Python or CPU path.  Importing
this module fails when the library has not been built.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparstar.so")
BLOCK = 128

OK, EINVAL, EDTYPE, ECUDA, ESIZE, ENODEV = range(6)
STATUS_BAD_INDEX = 0x1
STATUS_TIMEOUT = 0x2

_DTYPE = {torch.bfloat16: 0, torch.float32: 1}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libsparstar.so is not built (run block_sparse_attention_18_b200/build.py "
                          "or __graft_entry__.build()); there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    i64, i32, f32, f64, vp = (ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double,
                              ctypes.c_void_p)
    L.sparstar_block_pool.argtypes = [vp, i32, i64, i64, i64, i64, vp, vp]
    L.sparstar_block_score.argtypes = [vp, vp, i64, i64, i64, i64, i64, f32, vp, vp]
    L.sparstar_forced_blocks.argtypes = [i64, i64]
    L.sparstar_forced_blocks.restype = i64
    L.sparstar_select_count.argtypes = [i64, i64, f64]
    L.sparstar_select_count.restype = i64
    L.sparstar_select.argtypes = [vp, i64, i64, i64, i64, i64, f64, vp, vp, i64, vp]
    L.sparstar_attn_fwd.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, f32, vp, vp, i64,
                                    vp, vp, vp, vp]
    L.sparstar_forward.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, i64, i64, f64, vp,
                                   vp, vp, vp, vp, i64, vp, vp, vp, vp]
    L.sparstar_forward_static.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, i64, i64, f64,
                                          vp, vp, vp, vp]
    L.sparstar_forward_static.restype = i32
    L.sparstar_block_pool_qk.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, vp, vp, vp]
    L.sparstar_score_select.argtypes = [vp, vp, i64, i64, i64, i64, i64, f32, i64, f64, vp, vp,
                                        i64, vp, vp]
    L.sparstar_score_select_max_nkb.argtypes = [i64]
    L.sparstar_score_select_max_nkb.restype = i64
    L.sparstar_forward_fused.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, i64, i64, f64,
                                         vp, vp, vp, vp, i64, vp, vp, vp, vp]
    L.sparstar_retained_mass.argtypes = [vp, vp, i32, i64, i64, i64, i64, i64, f32, i64, vp, vp,
                                         i64, vp, i64, vp, vp, vp, vp, vp, vp]
    L.sparstar_transfer_lists.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp, i64, vp]
    L.sparstar_transfer_max_sel.argtypes = [vp, vp, i64]
    L.sparstar_transfer_max_sel.restype = i64
    L.sparstar_test_attn_timeout.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, vp, i64, vp, vp,
                                             vp]
    L.sparstar_test_attn_timeout.restype = i32
    L.sparstar_strerror.argtypes = [i32]
    L.sparstar_strerror.restype = ctypes.c_char_p
    L.sparstar_version.restype = i32
    for name in ("sparstar_block_pool", "sparstar_block_score", "sparstar_select",
                 "sparstar_attn_fwd", "sparstar_forward", "sparstar_block_pool_qk",
                 "sparstar_score_select", "sparstar_forward_fused", "sparstar_retained_mass",
                 "sparstar_transfer_lists"):
        getattr(L, name).restype = i32
    return L


lib = _load()


class SparstarError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s: %s (%d)" % (where, lib.sparstar_strerror(code).decode(), code))


def _check(code: int, where: str):
    if code != OK:
        raise SparstarError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return t


def nblocks(L: int) -> int:
    return (L + BLOCK - 1) // BLOCK


def default_tau(D: int) -> float:
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def sparstar_forced_blocks(text_len: int, image_ref_len: int) -> int:
    return lib.sparstar_forced_blocks(text_len, image_ref_len)


def sparstar_select_count(nKB: int, n_forced_blocks: int, density: float) -> int:
    return lib.sparstar_select_count(nKB, n_forced_blocks, density)


def sparstar_block_pool(x: torch.Tensor, xbar: torch.Tensor = None, stream=None) -> torch.Tensor:
    _dev(x, "x")
    B, H, L, D = x.shape
    if xbar is None:
        xbar = torch.empty(B, H, nblocks(L), D, device=x.device, dtype=torch.float32)
    _dev(xbar, "xbar", torch.float32)
    _check(lib.sparstar_block_pool(_ptr(x), _DTYPE.get(x.dtype, -1), B, H, L, D, _ptr(xbar),
                                   _stream(stream)), "sparstar_block_pool")
    return xbar


def sparstar_block_score(qbar: torch.Tensor, kbar: torch.Tensor, tau: float = None,
                         S: torch.Tensor = None, stream=None) -> torch.Tensor:
    _dev(qbar, "qbar", torch.float32)
    _dev(kbar, "kbar", torch.float32)
    B, H, nQB, D = qbar.shape
    nKB = kbar.shape[2]
    if tau is None:
        tau = default_tau(D)
    if S is None:
        S = torch.empty(B, H, nQB, nKB, device=qbar.device, dtype=torch.float32)
    _dev(S, "S", torch.float32)
    _check(lib.sparstar_block_score(_ptr(qbar), _ptr(kbar), B, H, nQB, nKB, D, tau, _ptr(S),
                                    _stream(stream)), "sparstar_block_score")
    return S


def sparstar_select(S: torch.Tensor, n_forced_blocks: int, density: float, max_sel: int = None,
                    kv_idx: torch.Tensor = None, kv_cnt: torch.Tensor = None, stream=None):
    _dev(S, "S", torch.float32)
    B, H, nQB, nKB = S.shape
    if max_sel is None:
        max_sel = kv_idx.shape[-1] if kv_idx is not None else \
            sparstar_select_count(nKB, n_forced_blocks, density)
        if max_sel < 0:
            raise SparstarError(EINVAL, "sparstar_select")
    if kv_idx is None:
        kv_idx = torch.empty(B, H, nQB, max_sel, device=S.device, dtype=torch.int32)
    if kv_cnt is None:
        kv_cnt = torch.empty(B, H, nQB, device=S.device, dtype=torch.int32)
    _dev(kv_idx, "kv_idx", torch.int32)
    _dev(kv_cnt, "kv_cnt", torch.int32)
    _check(lib.sparstar_select(_ptr(S), B, H, nQB, nKB, n_forced_blocks, density, _ptr(kv_idx),
                               _ptr(kv_cnt), max_sel, _stream(stream)), "sparstar_select")
    return kv_idx, kv_cnt


def sparstar_attn_fwd(q, k, v, kv_idx, kv_cnt, tau: float = None, out=None, lse=None,
                      status=None, want_lse: bool = True, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    _dev(kv_idx, "kv_idx", torch.int32)
    _dev(kv_cnt, "kv_cnt", torch.int32)
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    if tau is None:
        tau = default_tau(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, Lq, device=q.device, dtype=torch.float32)
    _check(lib.sparstar_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _DTYPE.get(q.dtype, -1), B, H, Lq,
                                 Lk, D, tau, _ptr(kv_idx), _ptr(kv_cnt), kv_idx.shape[-1],
                                 _ptr(out), _ptr(lse), _ptr(status), _stream(stream)),
           "sparstar_attn_fwd")
    return out, lse


class Workspace:
    """Caller-owned device buffers for one scale of ``sparstar_forward``."""

    def __init__(self, B, H, D, text_len, image_ref_len, ref_len, cur_len, density, device,
                 scores: bool = True):
        Lk = text_len + image_ref_len + ref_len + cur_len
        self.nQB, self.nKB = nblocks(cur_len), nblocks(Lk)
        self.n_forced = sparstar_forced_blocks(text_len, image_ref_len)
        self.max_sel = sparstar_select_count(self.nKB, self.n_forced, density)
        if self.max_sel < 0:
            raise SparstarError(EINVAL, "Workspace")
        f32, i32 = torch.float32, torch.int32
        self.qbar = torch.empty(B, H, self.nQB, D, device=device, dtype=f32)
        self.kbar = torch.empty(B, H, self.nKB, D, device=device, dtype=f32)
        # The fused front-end keeps the scores on chip and needs no S.
        self.S = torch.empty(B, H, self.nQB, self.nKB, device=device, dtype=f32) \
            if scores else None
        self.kv_idx = torch.empty(B, H, self.nQB, self.max_sel, device=device, dtype=i32)
        self.kv_cnt = torch.empty(B, H, self.nQB, device=device, dtype=i32)


def sparstar_forward(q, k, v, text_len, image_ref_len, ref_len, cur_len, density,
                     workspace: Workspace = None, out=None, lse=None, status=None,
                     want_lse: bool = True, stream=None):
    """All four steps for one scale on one stream; returns (out, lse, workspace)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, H, Lq, D = q.shape
    ws = workspace or Workspace(B, H, D, text_len, image_ref_len, ref_len, cur_len, density,
                                q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, Lq, device=q.device, dtype=torch.float32)
    _check(lib.sparstar_forward(_ptr(q), _ptr(k), _ptr(v), _DTYPE.get(q.dtype, -1), B, H, D,
                                text_len, image_ref_len, ref_len, cur_len, density, _ptr(ws.qbar),
                                _ptr(ws.kbar), _ptr(ws.S), _ptr(ws.kv_idx), _ptr(ws.kv_cnt),
                                ws.max_sel, _ptr(out), _ptr(lse), _ptr(status), _stream(stream)),
           "sparstar_forward")
    return out, lse, ws


def sparstar_block_pool_qk(q: torch.Tensor, k: torch.Tensor, qbar: torch.Tensor = None,
                           kbar: torch.Tensor = None, stream=None):
    """Block means of q and k in one launch; returns (qbar, kbar)."""
    _dev(q, "q")
    _dev(k, "k")
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    if qbar is None:
        qbar = torch.empty(B, H, nblocks(Lq), D, device=q.device, dtype=torch.float32)
    if kbar is None:
        kbar = torch.empty(B, H, nblocks(Lk), D, device=q.device, dtype=torch.float32)
    _dev(qbar, "qbar", torch.float32)
    _dev(kbar, "kbar", torch.float32)
    dt = _DTYPE.get(q.dtype, -1) if k.dtype == q.dtype else -1
    _check(lib.sparstar_block_pool_qk(_ptr(q), _ptr(k), dt, B, H, Lq, Lk, D, _ptr(qbar),
                                      _ptr(kbar), _stream(stream)), "sparstar_block_pool_qk")
    return qbar, kbar


def sparstar_score_select_max_nkb(D: int) -> int:
    return lib.sparstar_score_select_max_nkb(D)


def sparstar_score_select(qbar: torch.Tensor, kbar: torch.Tensor, n_forced_blocks: int,
                          density: float, tau: float = None, max_sel: int = None,
                          kv_idx: torch.Tensor = None, kv_cnt: torch.Tensor = None, status=None,
                          stream=None):
    """Block scores and block Top-K in one launch (no S buffer); returns
    (kv_idx, kv_cnt)."""
    _dev(qbar, "qbar", torch.float32)
    _dev(kbar, "kbar", torch.float32)
    B, H, nQB, D = qbar.shape
    nKB = kbar.shape[2]
    if tau is None:
        tau = default_tau(D)
    if max_sel is None:
        max_sel = kv_idx.shape[-1] if kv_idx is not None else \
            sparstar_select_count(nKB, n_forced_blocks, density)
        if max_sel < 0:
            raise SparstarError(EINVAL, "sparstar_score_select")
    if kv_idx is None:
        kv_idx = torch.empty(B, H, nQB, max_sel, device=qbar.device, dtype=torch.int32)
    if kv_cnt is None:
        kv_cnt = torch.empty(B, H, nQB, device=qbar.device, dtype=torch.int32)
    _dev(kv_idx, "kv_idx", torch.int32)
    _dev(kv_cnt, "kv_cnt", torch.int32)
    _check(lib.sparstar_score_select(_ptr(qbar), _ptr(kbar), B, H, nQB, nKB, D, tau,
                                     n_forced_blocks, density, _ptr(kv_idx), _ptr(kv_cnt),
                                     max_sel, _ptr(status), _stream(stream)),
           "sparstar_score_select")
    return kv_idx, kv_cnt


def sparstar_forward_fused(q, k, v, text_len, image_ref_len, ref_len, cur_len, density,
                           workspace: Workspace = None, out=None, lse=None, status=None,
                           want_lse: bool = True, stream=None):
    """The three-launch chain (pool q and k, score + select, attention) for one
    scale on one stream; returns (out, lse, workspace).  The workspace needs
    no S buffer."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, H, Lq, D = q.shape
    ws = workspace or Workspace(B, H, D, text_len, image_ref_len, ref_len, cur_len, density,
                                q.device, scores=False)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, Lq, device=q.device, dtype=torch.float32)
    _check(lib.sparstar_forward_fused(_ptr(q), _ptr(k), _ptr(v), _DTYPE.get(q.dtype, -1), B, H,
                                      D, text_len, image_ref_len, ref_len, cur_len, density,
                                      _ptr(ws.qbar), _ptr(ws.kbar), _ptr(ws.kv_idx),
                                      _ptr(ws.kv_cnt), ws.max_sel, _ptr(out), _ptr(lse),
                                      _ptr(status), _stream(stream)), "sparstar_forward_fused")
    return out, lse, ws


def sparstar_forward_static(q, k, v, text_len, image_ref_len, ref_len, cur_len, density,
                            out=None, lse=None, status=None, want_lse: bool = True, stream=None):
    """The four steps for one scale with the intermediates in the library's
    own device arena (no workspace); returns (out, lse).  For callers that
    cannot allocate device memory; calls that overlap on the GPU race on the
    shared arena."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    B, H, Lq, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, Lq, device=q.device, dtype=torch.float32)
    _check(lib.sparstar_forward_static(_ptr(q), _ptr(k), _ptr(v), _DTYPE.get(q.dtype, -1), B, H,
                                       D, text_len, image_ref_len, ref_len, cur_len, density,
                                       _ptr(out), _ptr(lse), _ptr(status), _stream(stream)),
           "sparstar_forward_static")
    return out, lse


def sparstar_retained_mass(q, k, kv_idx, kv_cnt, n_forced_blocks: int, rows, tau: float = None,
                           scratch=None, stream=None):
    """Diagnostic: dense LSE, retained attention mass of the block lists, the
    forced-block mass and the token-wise bound at the same candidate budget,
    for the flat query rows given (int64 device tensor).  Returns a dict of
    fp64 device tensors."""
    _dev(q, "q")
    _dev(k, "k")
    _dev(kv_idx, "kv_idx", torch.int32)
    _dev(kv_cnt, "kv_cnt", torch.int32)
    _dev(rows, "rows", torch.int64)
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    n = rows.numel()
    if tau is None:
        tau = default_tau(D)
    if scratch is None:
        scratch = torch.empty(n, Lk, device=q.device, dtype=torch.float32)
    _dev(scratch, "scratch", torch.float32)
    out = {name: torch.empty(n, device=q.device, dtype=torch.float64)
           for name in ("lse_dense", "mass_block", "mass_tok", "mass_forced")}
    dt = _DTYPE.get(q.dtype, -1) if k.dtype == q.dtype else -1
    _check(lib.sparstar_retained_mass(_ptr(q), _ptr(k), dt, B, H, Lq, Lk, D, tau,
                                      n_forced_blocks, _ptr(kv_idx), _ptr(kv_cnt),
                                      kv_idx.shape[-1], _ptr(rows), n, _ptr(scratch),
                                      _ptr(out["lse_dense"]), _ptr(out["mass_block"]),
                                      _ptr(out["mass_tok"]), _ptr(out["mass_forced"]),
                                      _stream(stream)), "sparstar_retained_mass")
    return out


def _segs(src_len, dst_len):
    return ((ctypes.c_int64 * 4)(*[int(x) for x in src_len]),
            (ctypes.c_int64 * 4)(*[int(x) for x in dst_len]))


def sparstar_transfer_max_sel(src_len, dst_len, src_max_sel: int) -> int:
    """Longest row sparstar_transfer_lists can write for these layouts."""
    ls, lt = _segs(src_len, dst_len)
    return lib.sparstar_transfer_max_sel(ls, lt, src_max_sel)


def sparstar_transfer_lists(kv_idx, kv_cnt, src_len, dst_len, dst_idx=None, dst_cnt=None,
                            stream=None):
    """Diagnostic: block lists of a source scale carried by token position to
    a target scale (mask reuse).  src_len / dst_len: the four segment lengths
    (text, image_ref, ref, cur) at each scale.  Returns (dst_idx, dst_cnt);
    dst_idx's row stride is sparstar_transfer_max_sel(...) unless given."""
    _dev(kv_idx, "kv_idx", torch.int32)
    _dev(kv_cnt, "kv_cnt", torch.int32)
    B, H = kv_idx.shape[0], kv_idx.shape[1]
    ls, lt = _segs(src_len, dst_len)
    nQB_t = (int(dst_len[3]) + BLOCK - 1) // BLOCK
    if dst_idx is None:
        stride = lib.sparstar_transfer_max_sel(ls, lt, kv_idx.shape[-1])
        if stride < 0:
            raise SparstarError(EINVAL, "sparstar_transfer_lists")
        dst_idx = torch.empty(B, H, nQB_t, stride, device=kv_idx.device, dtype=torch.int32)
    if dst_cnt is None:
        dst_cnt = torch.empty(B, H, nQB_t, device=kv_idx.device, dtype=torch.int32)
    _dev(dst_idx, "dst_idx", torch.int32)
    _dev(dst_cnt, "dst_cnt", torch.int32)
    _check(lib.sparstar_transfer_lists(_ptr(kv_idx), _ptr(kv_cnt), kv_idx.shape[-1], B, H, ls, lt,
                                       _ptr(dst_idx), _ptr(dst_cnt), dst_idx.shape[-1],
                                       _stream(stream)), "sparstar_transfer_lists")
    return dst_idx, dst_cnt


def sparstar_test_attn_timeout(q, k, v, kv_idx, kv_cnt, out, status, stream=None):
    """Test hook: the attention kernel with its K/V copies withheld, so that
    its first ring wait runs out and SPARSTAR_STATUS_TIMEOUT is set in
    `status` (an int32 device tensor)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _dev(t, n)
    _dev(kv_idx, "kv_idx", torch.int32)
    _dev(kv_cnt, "kv_cnt", torch.int32)
    _dev(status, "status", torch.int32)
    B, H, Lq, D = q.shape
    _check(lib.sparstar_test_attn_timeout(_ptr(q), _ptr(k), _ptr(v), B, H, Lq, k.shape[2],
                                          _ptr(kv_idx), _ptr(kv_cnt), kv_idx.shape[-1],
                                          _ptr(out), _ptr(status), _stream(stream)),
           "sparstar_test_attn_timeout")
