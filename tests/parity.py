"""Shared helpers of the GPU parity tests: tolerances, comparisons and row
sampling.  Tolerances follow the stated contract: bf16 outputs within
max-abs 2e-2 and relative L2 5e-3 of the fp64 oracle, fp32 outputs within
max-abs 1e-4; LSE within 1e-2 (bf16) / 1e-4 (fp32) as a supplementary check."""
import numpy as np
import torch

BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_MAX_ABS = 1e-4
LSE_TOL = {"bf16": 1e-2, "f32": 1e-4}
NEAR_TIE_REL = 1e-6


def out_errors(got: np.ndarray, want: np.ndarray):
    got = got.astype(np.float64)
    diff = got - want
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(want))
    rel_l2 = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel_l2


def check_out(got: np.ndarray, want: np.ndarray, dtype: str, what: str = "out"):
    max_abs, rel_l2 = out_errors(got, want)
    if dtype == "bf16":
        assert max_abs <= BF16_MAX_ABS and rel_l2 <= BF16_REL_L2, \
            "%s: max_abs %.3g rel_l2 %.3g" % (what, max_abs, rel_l2)
    else:
        assert max_abs <= F32_MAX_ABS, "%s: max_abs %.3g" % (what, max_abs)
    return max_abs, rel_l2


def check_lse(got: np.ndarray, want: np.ndarray, dtype: str):
    finite = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), finite)
    if finite.any():
        err = float(np.max(np.abs(got[finite].astype(np.float64) - want[finite])))
        assert err <= LSE_TOL[dtype], "lse max err %.3g" % err
        return err
    return 0.0


def sample_rows(B, H, Lq, per_head_blocks=6, rows_per_block=16, seed=0):
    """Flat row indices (bh * Lq + r): per head the first and the last query
    block plus random blocks, and per block its first row, its last real row
    and random rows."""
    rng = np.random.default_rng(seed)
    nQB = (Lq + 127) // 128
    rows = []
    for bh in range(B * H):
        blocks = {0, nQB - 1}
        while len(blocks) < min(nQB, per_head_blocks):
            blocks.add(int(rng.integers(0, nQB)))
        for i in sorted(blocks):
            lo, hi = i * 128, min(Lq, (i + 1) * 128)
            rs = {lo, hi - 1}
            n = min(hi - lo, rows_per_block)
            while len(rs) < n:
                rs.add(int(rng.integers(lo, hi)))
            rows.extend(bh * Lq + r for r in sorted(rs))
    return np.array(rows, np.int64)


def gather_rows(t: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """Rows of a [B,H,L,D] (or [B,H,L]) device tensor at flat indices, as fp64."""
    B, H, L = t.shape[:3]
    flat = t.reshape(B * H * L, -1) if t.dim() == 4 else t.reshape(B * H * L, 1)
    idx = torch.from_numpy(rows).to(t.device)
    out = flat.index_select(0, idx).float().cpu().numpy().astype(np.float64)
    return out if t.dim() == 4 else out[:, 0]
