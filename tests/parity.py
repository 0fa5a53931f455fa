"""Shared helpers for the parity tests: run the CUDA path through the C ABI and
the fp64 oracle on the same seeded inputs, and compare them element by element
with the tolerances of the tile-sparse attention contract:

* permute / unpermute / idx: bit-exact (idx up to near-ties: a selection may
  differ from the oracle's only for tiles whose exact score is within 1e-4 of
  the k-th largest score of that row);
* TripPool: max / min exact, mean relative 1e-5;
* probabilities: relative 2e-4 + absolute 1e-7.  A score error delta moves a
  softmax entry by at most 2*delta relative, and the contract already accepts
  score errors up to the 1e-4 near-tie gap;
* attention output (bf16 inputs, fp32 accumulation, bf16 output): max-abs
  1e-2 and relative L2 5e-3 against the fp64 oracle; log-sum-exp absolute 1e-3;
* tile map: relative 1e-3 on entries >= 1e-8 (absolute 1e-11 below).
"""
from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np
import torch

from oracle import veda_oracle as O
from veda_synth import PRESETS, Workload

ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 5e-3
LSE_ABS = 1e-3
MEAN_REL = 1e-5
PROBS_REL = 2e-4
PROBS_ABS = 1e-7
MAP_REL = 1e-3
NEAR_TIE = 1e-4


def wl(name, grid, B, heads, d, S, tilings, keep, hidden, e, bias=None) -> Workload:
    return Workload(name=name, T=grid[0], H=grid[1], W=grid[2], B=B, heads=heads, d=d, S=S,
                    tilings=tuple(tilings), keep=keep, hidden=hidden, e=e, bias=bias)


# Small problems the oracle finishes in seconds: several tiles per axis,
# ragged tiles on every face, both tile sizes and head dims, B = 2.
SMALL = [
    PRESETS["tiny"],
    wl("odd64", (5, 13, 19), 1, 3, 64, 64, [(1, 8, 8), (4, 4, 4), (2, 4, 8)], 0.25, 128, 32, "rff"),
    wl("odd128", (5, 19, 27), 2, 4, 128, 128, [(2, 8, 8), (1, 8, 16), (8, 4, 4), (4, 4, 8)], 0.2, 256, 64, "rff"),
    wl("d64s128", (6, 12, 20), 1, 2, 64, 128, [(2, 8, 8), (4, 4, 8)], 0.3, 128, 32),
    wl("d128s64", (4, 16, 16), 1, 2, 128, 64, [(1, 8, 8), (4, 4, 4)], 0.5, 256, 64, "local"),
]

# Ten distinct tilings of S = 64 (more than one grid-order attention launch
# covers), several with a factor larger than the grid dimension it tiles.
MANY_TILINGS = wl("many64", (5, 13, 19), 1, 10, 64, 64,
                  [(1, 8, 8), (4, 4, 4), (2, 4, 8), (8, 8, 1), (8, 1, 8), (1, 4, 16), (16, 2, 2), (2, 8, 4),
                   (4, 2, 8), (1, 2, 32)], 0.25, 128, 32, "rff")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_idx(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, nts: Sequence[int],
              ks: Sequence[int], heads: Sequence[int] = None) -> int:
    """Checks the idx contract and equality up to near-ties; returns the number of rows that differ."""
    B, H, ntmax, kmax = gpu_idx.shape
    heads = range(H) if heads is None else heads
    differ = 0
    for b in range(B):
        for hh, h in enumerate(heads):
            nt, k = nts[h], ks[h]
            for i in range(ntmax):
                g = gpu_idx[b, hh, i]
                if i >= nt:
                    assert np.all(g == -1), (b, h, i)
                    continue
                assert np.all(g[k:] == -1), (b, h, i)
                sel = g[:k]
                assert np.all(sel >= 0) and np.all(sel < nt), (b, h, i, sel)
                assert np.all(np.diff(sel) > 0), (b, h, i, sel)
                o = ora_idx[b, hh, i, :k]
                if np.array_equal(sel, o):
                    continue
                differ += 1
                s = ora_scores[b, hh, i, :nt]
                kth = np.sort(s)[::-1][k - 1]
                for j in set(sel.tolist()) ^ set(o.tolist()):
                    assert abs(s[j] - kth) < NEAR_TIE, (b, h, i, j, s[j], kth)
    return differ


def check_attn_rows(gpu_rows: np.ndarray, ora_rows: np.ndarray, what: str = "attention"):
    err = np.abs(gpu_rows - ora_rows)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(gpu_rows - ora_rows) / max(np.linalg.norm(ora_rows), 1e-30))
    assert max_abs <= ATTN_MAX_ABS, f"{what}: max abs error {max_abs:.3e} > {ATTN_MAX_ABS}"
    assert rel <= ATTN_REL_L2, f"{what}: relative L2 error {rel:.3e} > {ATTN_REL_L2}"
    return max_abs, rel


def token_rows(grid, tiling, S, i) -> np.ndarray:
    """Slots of tile i that hold a token (from the oracle's slot table)."""
    tab = O.slot_table(grid, tiling)
    return np.nonzero(tab[i * S:(i + 1) * S] >= 0)[0]


def mlp_numpy(m) -> tuple:
    return tuple(t.detach().cpu().to(torch.float64).numpy() for t in (m.w1, m.b1, m.w2, m.b2))


def mlp_device(m, device="cuda") -> tuple:
    return tuple(t.to(device).contiguous() for t in (m.w1, m.b1, m.w2, m.b2))


def keep_f32(r: float) -> float:
    """The keep ratio as the C ABI receives it (a C float), widened back to double."""
    return float(np.float32(r))


_QKV_CACHE = {}


def cached_qkv(w: Workload, seed: int = 0):
    """make_qkv(w, seed), kept for the test session: the full-size workloads
    take tens of seconds to draw on the CPU and several test files use them.
    Only the most recent workload is kept, to bound host memory."""
    key = (w, seed)
    if key not in _QKV_CACHE:
        from veda_synth import make_qkv
        _QKV_CACHE.clear()
        _QKV_CACHE[key] = make_qkv(w, seed=seed)
    return _QKV_CACHE[key]
