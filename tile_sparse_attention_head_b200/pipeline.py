"""The whole inference path as one call sequence over the C ABI.

``VedaAttention`` owns the device buffers (torch allocations: memory
plumbing only) and enqueues, on one CUDA stream, either (layout="tile")

    veda_tile_permute_tripool(Q), (K)   (permute + TripPool in one pass)
    -> veda_tile_permute(V) -> veda_tile_score_topk -> veda_tile_sparse_attn
    -> veda_tile_unpermute

or (layout="grid", no tile-major copies: the attention kernel fetches each
tile as a box of the grid-order tensor and writes grid rows)

    veda_tripool_grid(Q), (K) -> veda_tile_score_topk -> veda_tile_sparse_attn_grid

which is the per-layer path of Veda's tile-sparse attention (technical
summary, sections 2.1-2.3).  Every step runs in the library's kernels; both
layouts give the same output.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class VedaAttention:
    def __init__(self, problem: B.Problem, mlp_q, mlp_k, keep_ratio: float, device="cuda",
                 want_probs: bool = False, want_lse: bool = False, layout: str = "grid"):
        """mlp_q / mlp_k: (w1, b1, w2, b2) fp32 tensors on ``device`` (may be the same).

        layout "tile" keeps tile-major copies of Q, K, V and O (``qp`` ...,
        ``op``; ``lse`` per tile slot); "grid" works on the grid-order tensors
        directly (``lse`` per grid row)."""
        if layout not in ("tile", "grid"):
            raise ValueError(f"layout must be 'tile' or 'grid' (got {layout!r})")
        self.layout = layout
        self.p = problem
        self.keep = float(keep_ratio)
        self.k_per_head, self.k_max = problem.keep_count(self.keep)
        self._wq = tuple(mlp_q)
        self._wk = tuple(mlp_k)
        self.mlp_q = B.make_mlp(*self._wq)
        self.mlp_k = B.make_mlp(*self._wk)
        p = problem
        ts = p.tile_shape()
        if layout == "tile":
            self.qp = torch.empty(ts, dtype=torch.bfloat16, device=device)
            self.kp = torch.empty(ts, dtype=torch.bfloat16, device=device)
            self.vp = torch.empty(ts, dtype=torch.bfloat16, device=device)
            self.op = torch.empty(ts, dtype=torch.bfloat16, device=device)
        else:
            self.qp = self.kp = self.vp = self.op = None
        self.desc_q = torch.empty((p.B, p.heads, p.nt_max, 3 * p.d), dtype=torch.float32, device=device)
        self.desc_k = torch.empty_like(self.desc_q)
        self.idx = torch.empty((p.B, p.heads, p.nt_max, self.k_max), dtype=torch.int32, device=device)
        self.probs = (torch.empty((p.B, p.heads, p.nt_max, p.nt_max), dtype=torch.float32, device=device)
                      if want_probs else None)
        lse_rows = p.nt_max * p.S if layout == "tile" else p.N
        self.lse = (torch.empty((p.B, p.heads, lse_rows), dtype=torch.float32, device=device)
                    if want_lse else None)
        ws = B.veda_score_topk_workspace(p, self.mlp_q.e)
        self.workspace = torch.empty(ws // 4 + 64, dtype=torch.float32, device=device)

    def select(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None) -> torch.Tensor:
        """Permute, pool and score; returns the selected tile indices."""
        p = self.p
        if self.layout == "tile":
            B.veda_tile_permute_tripool(p, q, self.qp, self.desc_q, stream)
            B.veda_tile_permute_tripool(p, k, self.kp, self.desc_k, stream)
            B.veda_tile_permute(p, v, self.vp, stream)
        else:
            B.veda_tripool_grid(p, q, self.desc_q, stream)
            B.veda_tripool_grid(p, k, self.desc_k, stream)
        B.veda_tile_score_topk(p, self.desc_q, self.desc_k, self.mlp_q, self.mlp_k, self.keep, self.idx, self.probs,
                               self.workspace, stream)
        return self.idx

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
        """Grid-order bf16 Q, K, V [B, heads, N, d] -> grid-order output of the same shape."""
        p = self.p
        if out is None:
            out = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device=q.device)
        self.select(q, k, v, stream)
        if self.layout == "tile":
            B.veda_tile_sparse_attn(p, self.qp, self.kp, self.vp, self.idx, self.op, self.lse, 0.0, stream)
            B.veda_tile_unpermute(p, self.op, out, stream)
        else:
            B.veda_tile_sparse_attn_grid(p, q, k, v, self.idx, out, self.lse, 0.0, stream)
        return out
