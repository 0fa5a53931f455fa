"""GPU checks of the offline tiling search: the per-head error reduction
against numpy on seeded bf16 tensors, and the whole search (every candidate
tiling through the Veda path, compared with full attention) against the same
search run on the fp64 oracle."""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
from veda_synth import make_mlp, make_qkv

from parity import SMALL, f64, keep_f32, mlp_device, mlp_numpy, wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def test_head_error_reduction_against_numpy(V):
    w = SMALL[2]                                      # B = 2, 4 heads, d = 128
    p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
    g = torch.Generator().manual_seed(21)
    o = torch.randn(p.grid_shape(), generator=g).to(torch.bfloat16)
    r = torch.randn(p.grid_shape(), generator=g).to(torch.bfloat16)
    err = torch.empty(w.heads, dtype=torch.float32, device="cuda")
    ref = torch.empty_like(err)
    ws = torch.empty(128 * w.heads, dtype=torch.float32, device="cuda")
    V.veda_head_error(p, o.cuda(), r.cuda(), err, ref, ws)
    V.veda_sync_status()
    od, rd = f64(o), f64(r)
    np.testing.assert_allclose(f64(err), ((od - rd) ** 2).sum(axis=(0, 2, 3)), rtol=1e-5)
    np.testing.assert_allclose(f64(ref), (rd ** 2).sum(axis=(0, 2, 3)), rtol=1e-5)


def test_tiling_search_matches_the_oracle(V):
    w = wl("search", (5, 13, 19), 1, 3, 64, 64, [(1, 8, 8)] * 3, 0.25, 128, 32, "rff")
    cands = [(1, 8, 8), (4, 4, 4), (2, 4, 8), (4, 2, 8)]
    q, k, v = make_qkv(w, seed=4)
    m = make_mlp(w, seed=1)
    md = mlp_device(m)
    best, rel = V.tiling_search(q.cuda(), k.cuda(), v.cuda(), (w.T, w.H, w.W), w.S, md, md, w.keep, cands)
    grid = (w.T, w.H, w.W)
    mn = mlp_numpy(m)
    qd, kd, vd = f64(q), f64(k), f64(v)
    full = O.forward(qd, kd, vd, grid, [cands[0]] * w.heads, w.S, mn, mn, 1.0)["o"]
    ref = np.zeros((len(cands), w.heads))
    for c, t in enumerate(cands):
        o = O.forward(qd, kd, vd, grid, [t] * w.heads, w.S, mn, mn, keep_f32(w.keep))["o"]
        ref[c] = np.sqrt(((o - full) ** 2).sum(axis=(0, 2, 3)) / (full ** 2).sum(axis=(0, 2, 3)))
    got = rel.numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 5e-3 + 2e-2 * ref), (got, ref)
    for h in range(w.heads):
        order = np.argsort(ref[:, h])
        if ref[order[1], h] - ref[order[0], h] > 1e-2 + 4e-2 * ref[order[0], h]:   # a clear winner
            assert best[h] == cands[order[0]], (h, got[:, h], ref[:, h])
