"""Seeded synthetic inputs for the head-aware tile-sparse attention path.

Both the CUDA path (tests, bench) and the fp64 oracle draw their inputs from
here.  This module holds random-number draws and input shaping only: none of
the method's arithmetic (tile layout, pooling, estimator, selection,
attention) lives here, so neither side can inherit a mistake from the other
through it.

Workload shapes follow the video-DiT settings the Veda pages evaluate on
(Wan2.1-T2V 1.3B/14B, Waver, "Experimental results" section of the Veda
summary pages); the values are synthetic stand-ins: no model weights,
prompts or datasets are used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional, Sequence, Tuple

import torch

# Factorisations of a 128-token hardware tile that per-head tilings are drawn
# from ("Head-aware tiling" section: each head gets its own (pt, ph, pw)).
TILINGS_128: Tuple[Tuple[int, int, int], ...] = ((2, 8, 8), (1, 8, 16), (8, 4, 4), (4, 4, 8))


@dataclass(frozen=True)
class Workload:
    """One synthetic problem: grid, heads, head dim, tile size, tilings, keep ratio."""

    name: str
    T: int
    H: int
    W: int
    B: int
    heads: int
    d: int
    S: int
    tilings: Tuple[Tuple[int, int, int], ...]
    keep: float
    hidden: int
    e: int
    bias: Optional[str] = None          # None | "rff" (per-head anisotropic) | "local" (isotropic)
    bias_len: float = 2.0               # length scale for "local"
    map_frac: float = 0.1               # fraction of Q tiles in the tile-map subset

    @property
    def N(self) -> int:
        return self.T * self.H * self.W


def draw_tilings(heads: int, seed: int = 3,
                 choices: Sequence[Tuple[int, int, int]] = TILINGS_128) -> Tuple[Tuple[int, int, int], ...]:
    """Per-head tilings drawn uniformly from ``choices`` with a seeded generator."""
    g = torch.Generator().manual_seed(seed)
    pick = torch.randint(0, len(choices), (heads,), generator=g).tolist()
    return tuple(tuple(choices[p]) for p in pick)


def _preset(name, T, H, W, heads, keep, bias, tilings=None, bias_len=2.0, d=128, S=128,
            hidden=256, e=64, map_frac=0.1) -> Workload:
    if tilings is None:
        tilings = draw_tilings(heads)
    return Workload(name=name, T=T, H=H, W=W, B=1, heads=heads, d=d, S=S, tilings=tuple(tilings),
                    keep=keep, hidden=hidden, e=e, bias=bias, bias_len=bias_len, map_frac=map_frac)


PRESETS = {
    # 4x8x8 grid, 2 heads, d=64, 64-token tiles; head0 (1,8,8), head1 (4,4,4);
    # estimator 192 -> 128 -> 32; keep 2 of 4 K tiles.
    "tiny": Workload(name="tiny", T=4, H=8, W=8, B=1, heads=2, d=64, S=64,
                     tilings=((1, 8, 8), (4, 4, 4)), keep=0.5, hidden=128, e=32),
    # Wan2.1-1.3B 480p shape: 21x30x52 latent grid, 12 heads, d=128, keep 10%.
    "wan1.3b": _preset("wan1.3b", 21, 30, 52, 12, 0.10, "rff"),
    # Wan2.1-14B 720p/81-frame shape: 21x45x80, 40 heads, keep 5% (and 10%, dense).
    "wan14b": _preset("wan14b", 21, 45, 80, 40, 0.05, "rff"),
    "wan14b-k10": _preset("wan14b-k10", 21, 45, 80, 40, 0.10, "rff"),
    "wan14b-dense": _preset("wan14b-dense", 21, 45, 80, 40, 1.0, "rff"),
    # Long video: 31x45x80, 24 heads, keep 5%.
    "long": _preset("long", 31, 45, 80, 24, 0.05, "rff", tilings=draw_tilings(24)),
    # Scaling sweep at ~61K / 123K / 246K tokens, uniform (2,8,8) tiles, keep 5%.
    "sweep61k": _preset("sweep61k", 15, 64, 64, 24, 0.05, "local", tilings=((2, 8, 8),) * 24),
    "sweep123k": _preset("sweep123k", 30, 64, 64, 24, 0.05, "local", tilings=((2, 8, 8),) * 24),
    "sweep246k": _preset("sweep246k", 60, 64, 64, 24, 0.05, "local", tilings=((2, 8, 8),) * 24),
}


def with_heads(w: Workload, heads: int) -> Workload:
    """Same workload restricted to its first ``heads`` heads (for bounded oracle samples)."""
    return replace(w, heads=heads, tilings=w.tilings[:heads])


def _bias_features(w: Workload, g: torch.Generator, rank: int = 16) -> torch.Tensor:
    """Per-head random-Fourier positional features, shape [heads, N, rank] fp32.

    feature_i(x) = sqrt(2/rank) * cos(<omega_i, x> + phase_i) with omega_i drawn
    from N(0, diag(1/l_t^2, 1/l_y^2, 1/l_x^2)).  Adding c*feature to the first
    ``rank`` channels of both Q and K makes Q.K carry ~c^2 * exp(-|dx|^2/2l^2),
    a smooth local-window bias whose extent differs per head.
    """
    t = torch.arange(w.T, dtype=torch.float32)
    y = torch.arange(w.H, dtype=torch.float32)
    x = torch.arange(w.W, dtype=torch.float32)
    coords = torch.stack(torch.meshgrid(t, y, x, indexing="ij"), dim=-1).reshape(-1, 3)  # [N,3]
    feats = []
    for _ in range(w.heads):
        if w.bias == "local":
            ls = torch.full((3,), float(w.bias_len))
        else:
            ls = torch.exp(torch.empty(3).uniform_(math.log(1.0), math.log(8.0), generator=g))
        omega = torch.randn(rank, 3, generator=g) / ls
        phase = torch.empty(rank).uniform_(0.0, 2 * math.pi, generator=g)
        feats.append(math.sqrt(2.0 / rank) * torch.cos(coords @ omega.T + phase))
    return torch.stack(feats)


def make_qkv(w: Workload, seed: int = 0, heads: Optional[int] = None):
    """Q, K, V as bf16 CPU tensors [B, heads, N, d] in grid order (n = (t*H + y)*W + x).

    Values are N(0,1) drawn in fp32 and rounded to bf16.  With ``w.bias`` set,
    a scaled positional feature (see ``_bias_features``) is added to channels
    0..15 of Q and K before rounding, with c^2 = 4*sqrt(d) so the bias is worth
    about 4 logits after the 1/sqrt(d) attention scale.
    ``heads`` draws only the first ``heads`` heads (same values as a full draw
    for those heads, since each head is drawn from its own sub-seed).
    """
    H_ = w.heads if heads is None else heads
    shape = (w.B, w.N, w.d)
    qs, ks, vs = [], [], []
    feats = None
    if w.bias is not None:
        feats = _bias_features(w, torch.Generator().manual_seed(seed * 7919 + 17))
    c = math.sqrt(4.0 * math.sqrt(w.d))
    for h in range(H_):
        g = torch.Generator().manual_seed(seed * 100003 + h)
        q = torch.randn(shape, generator=g)
        k = torch.randn(shape, generator=g)
        v = torch.randn(shape, generator=g)
        if feats is not None:
            r = feats.shape[-1]
            q[..., :r] += c * feats[h]
            k[..., :r] += c * feats[h]
        qs.append(q.to(torch.bfloat16))
        ks.append(k.to(torch.bfloat16))
        vs.append(v.to(torch.bfloat16))
    return (torch.stack(qs, 1).contiguous(), torch.stack(ks, 1).contiguous(),
            torch.stack(vs, 1).contiguous())


def make_qkv_on_device(w: Workload, device, seed: int = 0):
    """The recipe of ``make_qkv`` drawn on ``device`` (bf16 [B, heads, N, d]
    grid-order Q, K, V): N(0,1) values, plus the same kind of positional
    feature on channels 0..15 of Q and K when ``w.bias`` is set.  The values
    differ from ``make_qkv``'s (another generator); this is for timing runs at
    sizes whose CPU draw would take longer than the measurement itself."""
    dev = torch.device(device)
    shape = (w.B, w.N, w.d)
    feats = None
    if w.bias is not None:
        feats = _bias_features(w, torch.Generator().manual_seed(seed * 7919 + 17))
    c = math.sqrt(4.0 * math.sqrt(w.d))
    out = [torch.empty((w.B, w.heads, w.N, w.d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    for h in range(w.heads):
        g = torch.Generator(device=dev).manual_seed(seed * 100003 + h)
        for a, t in enumerate(out):
            x = torch.randn(shape, generator=g, device=dev)
            if feats is not None and a < 2:
                r = feats.shape[-1]
                x[..., :r] += c * feats[h].to(dev)
            t[:, h] = x.to(torch.bfloat16)
    return tuple(out)


def make_grad_out(w: Workload, seed: int = 4, heads: Optional[int] = None) -> torch.Tensor:
    """An upstream gradient dO for the attention backward: bf16 CPU tensor
    [B, heads, N, d] in grid order, N(0,1) drawn in fp32 per head from its own
    sub-seed and rounded to bf16."""
    H_ = w.heads if heads is None else heads
    outs = []
    for h in range(H_):
        g = torch.Generator().manual_seed(seed * 100019 + h)
        outs.append(torch.randn((w.B, w.N, w.d), generator=g).to(torch.bfloat16))
    return torch.stack(outs, 1).contiguous()


@dataclass
class MLPWeights:
    """Per-head two-layer estimator weights, fp32: W1 [heads,hid,3d], b1 [heads,hid], W2 [heads,e,hid], b2 [heads,e]."""

    w1: torch.Tensor
    b1: torch.Tensor
    w2: torch.Tensor
    b2: torch.Tensor


def make_mlp(w: Workload, seed: int = 1, heads: Optional[int] = None) -> MLPWeights:
    """Xavier-uniform weights and PyTorch-Linear-style uniform biases, per head."""
    H_ = w.heads if heads is None else heads
    fin1, fout1 = 3 * w.d, w.hidden
    fin2, fout2 = w.hidden, w.e
    a1 = math.sqrt(6.0 / (fin1 + fout1))
    a2 = math.sqrt(6.0 / (fin2 + fout2))
    w1s, b1s, w2s, b2s = [], [], [], []
    for h in range(H_):
        g = torch.Generator().manual_seed(seed * 100003 + h)
        w1s.append(torch.empty(fout1, fin1).uniform_(-a1, a1, generator=g))
        b1s.append(torch.empty(fout1).uniform_(-1 / math.sqrt(fin1), 1 / math.sqrt(fin1), generator=g))
        w2s.append(torch.empty(fout2, fin2).uniform_(-a2, a2, generator=g))
        b2s.append(torch.empty(fout2).uniform_(-1 / math.sqrt(fin2), 1 / math.sqrt(fin2), generator=g))
    return MLPWeights(torch.stack(w1s).contiguous(), torch.stack(b1s).contiguous(),
                      torch.stack(w2s).contiguous(), torch.stack(b2s).contiguous())


def make_map_rows(nt_per_head: Sequence[int], B: int, frac: float, seed: int = 2) -> torch.Tensor:
    """Random Q-tile subsets for the tile map: int32 [B*heads, R].

    Row bh holds ceil(frac*NT_h) distinct tile indices of head h drawn without
    replacement, sorted ascending, padded with -1 up to R = the largest count.
    ``nt_per_head`` (tiles per head) is supplied by the caller.
    """
    heads = len(nt_per_head)
    counts = [max(1, math.ceil(frac * nt)) for nt in nt_per_head]
    R = max(counts)
    out = torch.full((B * heads, R), -1, dtype=torch.int32)
    g = torch.Generator().manual_seed(seed)
    for b in range(B):
        for h in range(heads):
            perm = torch.randperm(nt_per_head[h], generator=g)[: counts[h]]
            out[b * heads + h, : counts[h]] = torch.sort(perm).values.to(torch.int32)
    return out
