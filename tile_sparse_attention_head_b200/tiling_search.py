"""Offline head-aware tiling search (section 2.2 of the Veda summary: for
every layer and head a factorisation pi = (p_t, p_h, p_w) of the tile size is
chosen offline, on a calibration set, by minimising the error between the
full-attention and the sparse-attention outputs).

``tiling_search`` composes the library's calls: for each candidate tiling it
runs the whole Veda path (TripPool, estimator + top-k, tile-skipping
attention, grid order throughout) with every head on that tiling, compares
each head's output with full attention -- the same attention kernel with
every tile kept -- through ``veda_head_error``, and keeps, per head, the
candidate with the smallest relative L2 error.  Reading: the sparse output is
the method's own output (its estimator's selection at the given keep ratio);
the error is sqrt(sum (O - O_full)^2 / sum O_full^2) per head over the batch.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch

from . import binding as B
from .pipeline import VedaAttention


def tiling_search(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid: Sequence[int], S: int, mlp_q, mlp_k,
                  keep_ratio: float, candidates: Sequence[Tuple[int, int, int]], stream=None
                  ) -> Tuple[List[Tuple[int, int, int]], torch.Tensor]:
    """q, k, v: grid-order bf16 device tensors [B, heads, N, d] of a calibration
    sample; mlp_q / mlp_k: (w1, b1, w2, b2) fp32 device tensors.

    Returns (best tiling per head, relative errors [len(candidates), heads]
    as a CPU fp32 tensor).  Ties go to the earlier candidate."""
    if not candidates:
        raise ValueError("at least one candidate tiling is required")
    Bsz, heads, _, d = q.shape
    dev = q.device

    def run(tiling, keep):
        p = B.Problem(Bsz, heads, d, S, tuple(grid), [tuple(tiling)] * heads)
        att = VedaAttention(p, mlp_q, mlp_k, keep, device=dev, layout="grid")
        return p, att(q, k, v, stream=stream)

    # full attention: every tile kept (the output does not depend on the tiling)
    p_full, o_full = run(candidates[0], 1.0)
    err = torch.empty(heads, dtype=torch.float32, device=dev)
    ref = torch.empty(heads, dtype=torch.float32, device=dev)
    ws = torch.empty(128 * heads + 64, dtype=torch.float32, device=dev)
    rel = torch.empty((len(candidates), heads), dtype=torch.float32)
    for c, tiling in enumerate(candidates):
        p, o = run(tiling, keep_ratio)
        B.veda_head_error(p, o, o_full, err, ref, ws, stream)
        B.veda_sync_status(stream)
        rel[c] = torch.sqrt(err.cpu() / ref.cpu().clamp_min(1e-30))
    best = [tuple(candidates[int(torch.argmin(rel[:, h]))]) for h in range(heads)]
    return best, rel
