"""Seeded synthetic inputs shaped like the pages' training crops.

This module only draws random numbers and builds masks; it holds none of the
attention arithmetic.  Both the CUDA path's tests/benchmark and the FP64
oracle consume exactly the tensors it returns (the oracle upcasts the BF16
values to FP64).

Recipe (the pages give no seeds or distributions, so this is the plain
reading of the workloads they describe -- crops of 384 / 640 / 768 tokens in
"16张H100，训练步提速1.73倍：TurboPairFormer…", section "crop size不是一个普通参数"):

* one ``torch.Generator('cpu')`` seeded with ``seed``;
* drawn in the order q, k, v, dout, bias, lengths, as FP32 standard normals
  (bias multiplied by ``bias_std``) then rounded to BF16;
* lengths ``L_b ~ U{lo..hi}`` (inclusive) via ``torch.randint``;
* key-only padding mask: ``mask[b, i, k] = -1e9`` for ``k >= L_b`` else 0, the
  same for every pair row ``i`` (query rows and pair rows past ``L_b`` are
  computed like any other).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import torch

MASK_NEG = -1.0e9


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    d: int
    bias_std: float = 1.0
    mask: str = "none"          # "none" (NULL), "zeros" (all valid), "ragged" (key padding)
    len_lo: Optional[int] = None
    len_hi: Optional[int] = None
    orientation: str = "start"  # "start" or "end"

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workload families: a tiny oracle-sized case, the three training crops,
# and the batched ragged sweep.
TINY = Workload("tiny N=32", 1, 32, 4, 32)
CROP384 = Workload("crop384", 1, 384, 4, 32, mask="ragged", len_lo=320, len_hi=384)
CROP640 = Workload("crop640", 1, 640, 4, 32, mask="ragged", len_lo=512, len_hi=640)
CROP768 = Workload("crop768", 1, 768, 4, 32, bias_std=2.0, mask="zeros")


def sweep(N: int, d: int) -> Workload:
    return Workload(f"sweep B=2 N={N} d={d}", 2, N, 4, d, mask="ragged", len_lo=N // 2, len_hi=N)


SWEEP_NS = (128, 256, 512, 768, 1024)
SWEEP_DS = (32, 64)


def make_inputs(wl: Workload, seed: int, with_dout: bool = True) -> dict:
    """Return CPU tensors: q, k, v, dout (BF16 [B,N,N,H,d] in the *storage* frame),
    bias (BF16 [B,H,N,N]), mask (FP32 [B,N,N] or None), lengths (int64 [B]).

    For ``orientation == "end"`` the pair tensors are drawn in the attention's
    frame and stored transposed (axes 1 and 2 swapped), which is how an
    ending-node caller holds them; ``to_attention_frame`` undoes it."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    shp = (wl.B, wl.N, wl.N, wl.H, wl.d)
    q = torch.randn(shp, generator=g, dtype=torch.float32)
    k = torch.randn(shp, generator=g, dtype=torch.float32)
    v = torch.randn(shp, generator=g, dtype=torch.float32)
    dout = torch.randn(shp, generator=g, dtype=torch.float32)
    bias = torch.randn((wl.B, wl.H, wl.N, wl.N), generator=g, dtype=torch.float32) * wl.bias_std
    if wl.mask == "ragged":
        lengths = torch.randint(wl.len_lo, wl.len_hi + 1, (wl.B,), generator=g)
    else:
        lengths = torch.full((wl.B,), wl.N, dtype=torch.int64)
    if wl.mask == "none":
        mask = None
    else:
        kidx = torch.arange(wl.N).view(1, 1, wl.N)
        mask = torch.where(kidx >= lengths.view(-1, 1, 1), MASK_NEG, 0.0).to(torch.float32)
        mask = mask.expand(wl.B, wl.N, wl.N).contiguous()
    out = {
        "q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16),
        "dout": dout.to(torch.bfloat16), "bias": bias.to(torch.bfloat16),
        "mask": mask, "lengths": lengths,
    }
    if not with_dout:
        out.pop("dout")
    if wl.orientation == "end":
        for key in ("q", "k", "v", "dout"):
            if key in out:
                out[key] = out[key].transpose(1, 2).contiguous()
    return out


def make_inputs_device(wl: Workload, seed: int, device) -> dict:
    """The same recipe as ``make_inputs``, drawn on ``device`` with a seeded torch
    generator there (for pair stacks whose FP32 draws would crowd the host, e.g.
    N = 4096).  Returns device tensors in the storage frame; the values differ
    from ``make_inputs``'s for the same seed (another generator), the
    distributions do not."""
    g = torch.Generator(device=device).manual_seed(int(seed))
    shp = (wl.B, wl.N, wl.N, wl.H, wl.d)
    out = {}
    for key in ("q", "k", "v", "dout"):
        out[key] = torch.randn(shp, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)
    out["bias"] = (torch.randn((wl.B, wl.H, wl.N, wl.N), generator=g, dtype=torch.float32, device=device)
                   * wl.bias_std).to(torch.bfloat16)
    if wl.mask == "ragged":
        lengths = torch.randint(wl.len_lo, wl.len_hi + 1, (wl.B,), generator=g, device=device)
    else:
        lengths = torch.full((wl.B,), wl.N, dtype=torch.int64, device=device)
    if wl.mask == "none":
        out["mask"] = None
    else:
        kidx = torch.arange(wl.N, device=device).view(1, 1, wl.N)
        mask = torch.where(kidx >= lengths.view(-1, 1, 1), MASK_NEG, 0.0).to(torch.float32)
        out["mask"] = mask.expand(wl.B, wl.N, wl.N).contiguous()
    out["lengths"] = lengths
    if wl.orientation == "end":
        for key in ("q", "k", "v", "dout"):
            out[key] = out[key].transpose(1, 2).contiguous()
    return out


def to_attention_frame(x: torch.Tensor, orientation: str) -> torch.Tensor:
    """View a stored [B,N,N,H,d] pair tensor in the attention's own frame."""
    return x.transpose(1, 2) if orientation == "end" else x


def seed_for(config_idx: int, case_idx: int) -> int:
    return 1000 * config_idx + case_idx
