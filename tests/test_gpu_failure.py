"""Failure detection on the GPU without a fault: a wait that runs out.

The tcgen05 attention kernel bounds every wait (about two seconds of
%globaltimer).  The test hook sparstar_test_attn_timeout withholds every key
and value copy, so the kernel's first wait on its K/V ring can never
complete.  The kernel must then report SPARSTAR_STATUS_TIMEOUT in the
caller's status word and leave through its abort path (copies drained, TMEM
freed), and the CUDA context must stay usable: a normal call right after
matches the oracle.  One CTA, so the test takes about two seconds.
"""
import time

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


def test_withheld_copies_time_out_and_the_context_stays_usable(sp, orc):
    w = synth.custom(H=1, D=128, dtype="bf16", text=128, ref=256, cur=256, density=1.0, seed=3)
    q, k, v = synth.generate(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    idx = torch.arange(w.nKB, dtype=torch.int32).repeat(1, 1, w.nQB, 1).contiguous().cuda()
    cnt = torch.full((1, 1, w.nQB), w.nKB, dtype=torch.int32).cuda()
    out = torch.empty_like(qd)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.monotonic()
    sp.sparstar_test_attn_timeout(qd, kd, vd, idx, cnt, out, status)
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert int(status.item()) & sp.STATUS_TIMEOUT
    assert 1.0 < elapsed < 30.0  # the bound fired; nothing hung

    # the same context runs a normal call correctly afterwards
    status.zero_()
    got, lse = sp.sparstar_attn_fwd(qd, kd, vd, idx, cnt, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    qn, kn, vn = (synth.as_numpy(t) for t in (q, k, v))
    rows = np.arange(w.Lq, dtype=np.int64)
    want, want_lse = orc.attn_rows_f64(qn, kn, vn, idx.cpu().numpy(), cnt.cpu().numpy(), rows)
    parity.check_out(parity.gather_rows(got, rows), want, "bf16")
    parity.check_lse(parity.gather_rows(lse, rows), want_lse, "bf16")
