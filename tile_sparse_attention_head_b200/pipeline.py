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

``tile_sparse_attention`` is the grid-order attention as a differentiable
torch op for a given selection: its forward is veda_tile_sparse_attn_grid
(with the LSE kept for later), its backward veda_tile_sparse_attn_backward_grid.
``VedaAttention.differentiable`` selects (without gradient: top-k is
piecewise constant) and applies it.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class _TileSparseAttention(torch.autograd.Function):
    """Grid-order tile-skipping attention over a fixed selection, with the
    library's backward; torch only holds the saved tensors."""

    @staticmethod
    def forward(ctx, q, k, v, problem, idx):
        p = problem
        o = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((p.B, p.heads, p.N), dtype=torch.float32, device=q.device)
        B.veda_tile_sparse_attn_grid(p, q, k, v, idx, o, lse)
        ctx.problem = p
        ctx.save_for_backward(q, k, v, o, lse, idx)
        return o

    @staticmethod
    def backward(ctx, d_o):
        q, k, v, o, lse, idx = ctx.saved_tensors
        p = ctx.problem
        d_o = d_o.to(torch.bfloat16).contiguous()
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        ws = torch.empty(B.veda_attn_backward_workspace(p, int(idx.shape[-1])), dtype=torch.uint8, device=q.device)
        B.veda_tile_sparse_attn_backward_grid(p, q, k, v, o, lse, d_o, idx, dq, dk, dv, ws)
        return dq, dk, dv, None, None


def tile_sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, problem: B.Problem,
                          idx: torch.Tensor) -> torch.Tensor:
    """Differentiable tile-skipping attention: grid-order bf16 q, k, v
    [B, heads, N, d] attend over the K tiles listed in idx
    [B, heads, NT_max, k_max] (scale 1/sqrt(d)); gradients flow to q, k and v."""
    return _TileSparseAttention.apply(q, k, v, problem, idx)


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


    def differentiable(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        """Select tiles (no gradient), then the differentiable grid-order
        attention over that selection (layout "grid" only)."""
        if self.layout != "grid":
            raise ValueError("the differentiable path runs on grid-order tensors (layout='grid')")
        with torch.no_grad():
            idx = self.select(q.detach(), k.detach(), v.detach()).clone()
        return tile_sparse_attention(q, k, v, self.p, idx)

class VedaAttentionHost:
    """The layer on HOST buffers: pinned grid-order bf16 Q, K, V in, O out.

    Every (b, head) is independent through all steps, so the heads are cut
    into chunks and the chunks are pipelined over three CUDA streams: while
    chunk c is attended, chunk c+1's Q/K/V are copied in and chunk c-1's
    output is copied out (PCIe is full duplex, so both directions run at
    once).  ``slots`` device buffer sets rotate between the chunks.  Every
    compute step is the library's (one VedaAttention per chunk, grid-order
    layout); the copies are cudaMemcpyAsync from pinned memory.
    """

    def __init__(self, problem: B.Problem, mlp_q, mlp_k, keep_ratio: float, device="cuda", chunk_heads: int = 2,
                 slots: int = 3):
        p = problem
        self.p = p
        self.dev = torch.device(device)
        self.chunks = []                       # (b, h0, h1, slot index, VedaAttention)
        ch = max(1, int(chunk_heads))
        n = 0
        for b in range(p.B):
            for h0 in range(0, p.heads, ch):
                h1 = min(p.heads, h0 + ch)
                sub = B.Problem(1, h1 - h0, p.d, p.S, p.grid, p.tilings[h0:h1])
                mq = tuple(t[h0:h1] for t in mlp_q)
                mk = tuple(t[h0:h1] for t in mlp_k)
                self.chunks.append((b, h0, h1, n % slots, VedaAttention(sub, mq, mk, keep_ratio, device=self.dev)))
                n += 1
        self.slots = min(slots, n)
        rows = min(ch, p.heads) * p.N * p.d
        self.buf = [[torch.empty(rows, dtype=torch.bfloat16, device=self.dev) for _ in range(4)]
                    for _ in range(self.slots)]
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(device=self.dev) for _ in range(3))

    def __call__(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, out_host: torch.Tensor,
                 stream=None) -> torch.Tensor:
        """Enqueues the layer after the work already on ``stream`` (default: the
        current stream) and makes ``stream`` wait for its end; out_host is
        complete once ``stream`` reaches that point."""
        p = self.p
        shape = p.grid_shape()
        for t, n in ((q_host, "q"), (k_host, "k"), (v_host, "v"), (out_host, "out")):
            if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or t.is_cuda or not t.is_pinned():
                raise ValueError(f"{n} must be a pinned host bf16 tensor of shape {shape}")
        base = stream if stream is not None else torch.cuda.current_stream(self.dev)
        start = torch.cuda.Event()
        start.record(base)
        for s in (self.s_in, self.s_run, self.s_out):
            s.wait_event(start)
        free = [None] * self.slots             # slot reusable once its output is copied out
        last = None
        for b, h0, h1, slot, att in self.chunks:
            qb, kb, vb, ob = self.buf[slot]
            n = (h1 - h0) * p.N * p.d
            gshape = (1, h1 - h0, p.N, p.d)
            with torch.cuda.stream(self.s_in):
                if free[slot] is not None:
                    self.s_in.wait_event(free[slot])
                for dst, src in ((qb, q_host), (kb, k_host), (vb, v_host)):
                    dst[:n].view(gshape).copy_(src[b:b + 1, h0:h1], non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(self.s_in)
            self.s_run.wait_event(loaded)
            att(qb[:n].view(gshape), kb[:n].view(gshape), vb[:n].view(gshape), ob[:n].view(gshape),
                stream=self.s_run)
            done = torch.cuda.Event()
            done.record(self.s_run)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(done)
                out_host[b:b + 1, h0:h1].copy_(ob[:n].view(gshape), non_blocking=True)
                last = torch.cuda.Event()
                last.record(self.s_out)
            free[slot] = last
        base.wait_event(last)
        return out_host
