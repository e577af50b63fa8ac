"""sparstar_forward_static: the allocation-free entry point for callers that
cannot allocate device memory (a host program that only hands the library
its inputs and outputs, or a plugin whose host forbids extra device
allocations).  It keeps the intermediates in the library's own device arena.

Its results must equal those of sparstar_forward, which takes caller
workspace, on two calls in a row (the second call reuses the arena the
first one left behind).  The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_18_b200 import synth
import parity

pytestmark = pytest.mark.gpu

CASES = [
    dict(H=4, D=128, dtype="bf16", text=512, image_ref=0, ref=2000, cur=1500, density=0.1875),
    dict(H=2, D=128, dtype="bf16", text=512, image_ref=3600, ref=900, cur=700, density=0.625),
    dict(H=1, D=64, dtype="f32", text=128, image_ref=0, ref=0, cur=1024, density=0.5),
]


@pytest.fixture(scope="module")
def sp():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_attention_18_b200 import build
    build.build()
    from block_sparse_attention_18_b200 import sparstar
    return sparstar


def _call_static(sp, q, k, v, w, out, lse, status):
    """Through the C ABI with raw pointers; returns the status code."""
    return sp.lib.sparstar_forward_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), 0 if w.dtype == "bf16" else 1, w.B, w.H, w.D, w.text,
        w.image_ref, w.ref, w.cur, w.density, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s_D%d_%d" % (c["dtype"], c["D"], c["cur"]))
def test_static_arena_matches_workspace_path(sp, case):
    w = synth.custom(seed=31, **case)
    q, k, v = (t.cuda() for t in synth.generate(w))
    ref_out, ref_lse, _ = sp.sparstar_forward(q, k, v, w.text, w.image_ref, w.ref, w.cur,
                                              w.density)
    torch.cuda.synchronize()
    want = ref_out.float().cpu().numpy().astype(np.float64)
    want_lse = ref_lse.cpu().numpy().astype(np.float64)
    for call in range(2):  # the second call finds the previous call's data in the arena
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _call_static(sp, q, k, v, w, out, lse, status)
        torch.cuda.synchronize()
        assert rc == sp.OK, sp.lib.sparstar_strerror(rc)
        assert int(status.item()) == 0
        got = out.float().cpu().numpy().astype(np.float64)
        parity.check_out(got.reshape(-1, w.D), want.reshape(-1, w.D), w.dtype,
                         "static call %d" % call)
        parity.check_lse(lse.cpu().numpy().astype(np.float64), want_lse, w.dtype)


def test_static_arena_rejects_oversized_calls(sp):
    # 16 heads with 1.3M keys needs far more than the arena: refused, nothing launched.
    dummy = torch.empty(16, device="cuda", dtype=torch.bfloat16)
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = sp.lib.sparstar_forward_static(p, p, p, 0, 1, 16, 128, 512, 0, 650000, 650000, 0.09375,
                                        p, None, None, None)
    assert rc == sp.ESIZE
    assert b"static arena" in sp.lib.sparstar_strerror(rc)
