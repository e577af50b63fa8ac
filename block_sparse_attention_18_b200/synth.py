"""Seeded synthetic inputs shaped like SparSTAR's sparsified scales.

This module holds the workload table and the input generator that both the
CUDA path and the CPU oracle are fed from.  It contains none of the method's
arithmetic (no pooling, scoring, selection or attention): only shapes,
segment lengths, densities and random draws.

Workloads stand in for InfinityStar activations at the late refinement
scales SparSTAR sparsifies (pith.science review of SparSTAR, "What carries
the argument": 128-token blocks, the density schedule 0.625 / 0.1875 /
0.1875 / 0.09375, the 72,000-token final scale; "Assumptions & free
parameters": the sparsified scale set).  Keys are laid out as
[text | image reference (Clip 1 only) | preceding-clip reference | current
scale]; queries are the current-scale tokens.

Recipe (fixed draw order, one CPU torch.Generator seeded per workload):
  1. Q noise  [B,H,Lq,D] ~ N(0,1)
  2. K noise  [B,H,Lk,D] ~ N(0,1)
  3. V        [B,H,Lk,D] ~ N(0,1)
  4. Q offsets [B,H,nQB,D] ~ N(0, std^2), one vector per query block
  5. K offsets [B,H,nKB,D] ~ N(0, std^2), one vector per key block
Q and K are noise + the offset of the block the token falls in.  With
``share_ref_cur_offsets`` the K offset of reference block p is copied to
current block p (both grids block-aligned).  fp32 values are rounded to
bf16 (round-to-nearest-even) for bf16 workloads; the same bytes go to the
GPU and to the oracle.
"""
from dataclasses import dataclass, replace

import torch

BLOCK = 128


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    D: int
    dtype: str          # "bf16" or "f32"
    seed: int
    text: int
    image_ref: int
    ref: int
    cur: int
    density: float
    offset_std: float
    share_ref_cur_offsets: bool = False
    B: int = 1

    @property
    def Lq(self) -> int:
        return self.cur

    @property
    def Lk(self) -> int:
        return self.text + self.image_ref + self.ref + self.cur

    @property
    def nQB(self) -> int:
        return (self.Lq + BLOCK - 1) // BLOCK

    @property
    def nKB(self) -> int:
        return (self.Lk + BLOCK - 1) // BLOCK


def _sweep(clip1: bool):
    out = []
    for cur, dens in ((8000, 0.625), (18000, 0.1875), (40500, 0.1875), (72000, 0.09375)):
        tag = "clip1" if clip1 else "clip2"
        out.append(Workload(name="sweep_%s_%d" % (tag, cur), H=16, D=128, dtype="bf16", seed=4,
                            text=512, image_ref=3600 if clip1 else 0, ref=cur, cur=cur,
                            density=dens, offset_std=0.25))
    return out


WORKLOADS = {w.name: w for w in [
    Workload("tiny", H=1, D=64, dtype="f32", seed=0, text=128, image_ref=0, ref=0, cur=1024,
             density=0.5, offset_std=0.25),
    Workload("mid", H=8, D=128, dtype="bf16", seed=1, text=512, image_ref=0, ref=4096, cur=8192,
             density=0.625, offset_std=0.25, share_ref_cur_offsets=True),
    Workload("partial_tail", H=16, D=128, dtype="bf16", seed=2, text=512, image_ref=0, ref=18000,
             cur=18000, density=0.1875, offset_std=0.25),
    Workload("largest", H=16, D=128, dtype="bf16", seed=3, text=512, image_ref=0, ref=72000,
             cur=72000, density=0.09375, offset_std=0.5),
    *_sweep(clip1=False),
    *_sweep(clip1=True),
]}

# The workload the benchmark times (72,000 current-scale tokens, 16 heads,
# density 0.09375).
BENCH_WORKLOAD = "largest"


def custom(**kw) -> Workload:
    """A workload with explicit sizes (tests use these for small cases)."""
    base = dict(name="custom", H=1, D=128, dtype="bf16", seed=0, text=0, image_ref=0, ref=0,
                cur=128, density=1.0, offset_std=0.25)
    base.update(kw)
    return Workload(**base)


def with_seed(w: Workload, seed: int) -> Workload:
    return replace(w, seed=seed)


def _expand_blocks(off: torch.Tensor, L: int) -> torch.Tensor:
    # [B,H,nblk,D] -> [B,H,L,D], each token gets its block's vector
    return off.repeat_interleave(BLOCK, dim=2)[:, :, :L, :]


def generate(w: Workload):
    """Return (q, k, v) as CPU torch tensors of dtype bfloat16 or float32."""
    g = torch.Generator().manual_seed(w.seed)
    B, H, D = w.B, w.H, w.D
    q = torch.randn(B, H, w.Lq, D, generator=g, dtype=torch.float32)
    k = torch.randn(B, H, w.Lk, D, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, w.Lk, D, generator=g, dtype=torch.float32)
    qoff = torch.randn(B, H, w.nQB, D, generator=g, dtype=torch.float32) * w.offset_std
    koff = torch.randn(B, H, w.nKB, D, generator=g, dtype=torch.float32) * w.offset_std
    if w.share_ref_cur_offsets:
        prefix = w.text + w.image_ref
        if prefix % BLOCK or w.ref % BLOCK:
            raise ValueError("shared reference/current offsets need block-aligned segments")
        ref0 = prefix // BLOCK
        cur0 = (prefix + w.ref) // BLOCK
        n = min(w.ref // BLOCK, w.nKB - cur0)
        koff[:, :, cur0:cur0 + n] = koff[:, :, ref0:ref0 + n]
    q += _expand_blocks(qoff, w.Lq)
    k += _expand_blocks(koff, w.Lk)
    if w.dtype == "bf16":
        return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    if w.dtype == "f32":
        return q, k, v
    raise ValueError("unknown dtype %r" % w.dtype)


def as_numpy(t: torch.Tensor):
    """Host view for the oracle: bf16 as uint16 bit patterns, fp32 as is."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


# The scale before each scale of the sweep schedule (same clip layout), used
# by the mask-reuse diagnostic; `largest` has the Clip 2+ layout of the 72k
# scale.
PREVIOUS_SCALE = {
    "largest": "sweep_clip2_40500",
    **{"sweep_%s_%d" % (tag, b): "sweep_%s_%d" % (tag, a)
       for tag in ("clip1", "clip2")
       for a, b in ((8000, 18000), (18000, 40500), (40500, 72000))},
}


def segments(w: Workload):
    """Key segment lengths (text, image_ref, ref, cur); queries are cur."""
    return [w.text, w.image_ref, w.ref, w.cur]


def coarser_scale(q: torch.Tensor, k: torch.Tensor, seg_t, seg_s):
    """Source-scale inputs that carry the target scale's content: source
    offset p of segment g takes the target token at offset
    floor(p * len_t[g] / len_s[g]) of that segment (the same proportional
    position map as the cross-scale list transfer).  q is the cur segment.
    Works on any device; returns (q_s, k_s)."""
    dev = q.device

    def pick(len_t, len_s, start):
        p = torch.arange(len_s, device=dev, dtype=torch.int64)
        return start + (p * len_t) // len_s

    q_idx = pick(seg_t[3], seg_s[3], 0)
    k_parts, off = [], 0
    for g in range(4):
        if seg_s[g] > 0:
            if seg_t[g] == 0:
                raise ValueError("segment %d exists at the source but not at the target" % g)
            k_parts.append(pick(seg_t[g], seg_s[g], off))
        off += seg_t[g]
    k_idx = torch.cat(k_parts)
    return q.index_select(2, q_idx).contiguous(), k.index_select(2, k_idx).contiguous()
