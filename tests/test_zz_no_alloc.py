"""sparstar_forward_static: the allocation-free entry point for callers that
cannot allocate device memory (a host program that only hands the library
its inputs and outputs, or a plugin whose host forbids extra device
allocations).  It keeps the intermediates in the library's own device arena.

It runs the same kernels on the same inputs as sparstar_forward, which takes
caller workspace, so its outputs must be bit-identical to that path on two
calls in a row (the second call reuses the arena the first one left behind,
and the cases run in an order that leaves a larger call's data in the arena
before a smaller one).  One case is also checked against the oracle, and a
call is checked to leave the device's free memory unchanged.  The file is
named so that pytest collects it last.
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


def _static_twice(sp, w, q, k, v, like_out, like_lse):
    """Two calls in a row; returns the outputs of each."""
    res = []
    for _ in range(2):
        out = torch.full_like(like_out, float("nan"))
        lse = torch.full_like(like_lse, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _call_static(sp, q, k, v, w, out, lse, status)
        torch.cuda.synchronize()
        assert rc == sp.OK, sp.lib.sparstar_strerror(rc)
        assert int(status.item()) == 0
        res.append((out, lse))
    return res


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s_D%d_%d" % (c["dtype"], c["D"], c["cur"]))
def test_static_arena_is_bit_identical_to_workspace_path(sp, case):
    w = synth.custom(seed=31, **case)
    q, k, v = (t.cuda() for t in synth.generate(w))
    ref_out, ref_lse, _ = sp.sparstar_forward(q, k, v, w.text, w.image_ref, w.ref, w.cur,
                                              w.density)
    torch.cuda.synchronize()
    for call, (out, lse) in enumerate(_static_twice(sp, w, q, k, v, ref_out, ref_lse)):
        # Same kernels, same inputs: every output bit must agree.
        assert torch.equal(out.view(torch.int16 if out.dtype == torch.bfloat16 else torch.int32),
                           ref_out.view(torch.int16 if out.dtype == torch.bfloat16
                                        else torch.int32)), "out differs on call %d" % call
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), \
            "lse differs on call %d" % call


def test_static_arena_matches_the_oracle(sp):
    import oracle as orc
    w = synth.custom(H=2, D=128, dtype="bf16", text=512, image_ref=0, ref=1300, cur=1100,
                     density=0.25, seed=37)
    qc, kc, vc = synth.generate(w)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    like_out = torch.empty_like(q)
    like_lse = torch.empty(w.B, w.H, w.Lq, dtype=torch.float32, device="cuda")
    qn, kn, vn = (synth.as_numpy(t) for t in (qc, kc, vc))
    _, _, _, idx, cnt = orc.run_selection(qn, kn, w.text, w.image_ref, w.density)
    rows = np.arange(w.B * w.H * w.Lq, dtype=np.int64)
    want, want_lse = orc.attn_rows_f64(qn, kn, vn, idx, cnt, rows)
    for call, (out, lse) in enumerate(_static_twice(sp, w, q, k, v, like_out, like_lse)):
        parity.check_out(parity.gather_rows(out, rows), want, w.dtype, "static call %d" % call)
        parity.check_lse(parity.gather_rows(lse, rows), want_lse, w.dtype)


def test_static_call_allocates_no_device_memory(sp):
    w = synth.custom(seed=41, **CASES[0])
    q, k, v = (t.cuda() for t in synth.generate(w))
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.Lq, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _call_static(sp, q, k, v, w, out, lse, status) == sp.OK  # warm-up: modules loaded
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    torch_before = torch.cuda.memory_allocated()
    assert _call_static(sp, q, k, v, w, out, lse, status) == sp.OK
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert int(status.item()) == 0
    assert free_after == free_before
    assert torch.cuda.memory_allocated() == torch_before


def test_static_arena_rejects_oversized_calls(sp):
    # 16 heads with 1.3M keys needs far more than the arena: refused, nothing launched.
    dummy = torch.empty(16, device="cuda", dtype=torch.bfloat16)
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = sp.lib.sparstar_forward_static(p, p, p, 0, 1, 16, 128, 512, 0, 650000, 650000, 0.09375,
                                        p, None, None, None)
    assert rc == sp.ESIZE
    assert b"static arena" in sp.lib.sparstar_strerror(rc)
