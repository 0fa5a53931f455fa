"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded inputs.

Small and odd-shaped problems are compared in full (several tiles, ragged
tiles on every face, both tile sizes and head dims, B = 2); the Wan2.1-14B
720p/81-frame shape (the benchmarked workload) is compared on sampled heads
and Q tiles in the same launch configuration the bench uses.
"""
import math

import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
from veda_synth import PRESETS, make_map_rows, make_mlp, make_qkv

from parity import (LSE_ABS, MAP_REL, MEAN_REL, PROBS_ABS, PROBS_REL, SMALL, cached_qkv, check_attn_rows, check_idx,
                    f64, keep_f32, mlp_device, mlp_numpy)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def _problem(V, w):
    return V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)


class Run:
    """Both sides of the path on one workload."""

    def __init__(self, V, w, seed=0):
        self.w = w
        self.p = _problem(V, w)
        q, k, v = make_qkv(w, seed=seed)
        m = make_mlp(w, seed=seed + 1)
        self.q, self.k, self.v = q, k, v
        self.grid = (w.T, w.H, w.W)
        dev = "cuda"
        self.att = V.VedaAttention(self.p, mlp_device(m), mlp_device(m), w.keep, want_probs=True, want_lse=True,
                                   layout="tile")
        self.out = self.att(q.to(dev), k.to(dev), v.to(dev))
        V.veda_sync_status()
        self.mlp = mlp_numpy(m)
        qd, kd, vd = (f64(t) for t in (q, k, v))
        self.ora = O.forward(qd, kd, vd, self.grid, w.tilings, w.S, self.mlp, self.mlp, keep_f32(w.keep))


@pytest.fixture(scope="module", params=SMALL, ids=[w.name for w in SMALL])
def run(V, request):
    return Run(V, request.param)


def test_permute_bit_exact(run):
    for name, dev, ref in (("qp", run.att.qp, run.ora["qp"]), ("kp", run.att.kp, run.ora["kp"]),
                           ("vp", run.att.vp, run.ora["vp"])):
        np.testing.assert_array_equal(f64(dev), ref, err_msg=name)


def test_tripool(run):
    d = run.w.d
    for dev, ref in ((run.att.desc_q, run.ora["desc_q"]), (run.att.desc_k, run.ora["desc_k"])):
        g = f64(dev)
        np.testing.assert_array_equal(g[..., d:], ref[..., d:])
        np.testing.assert_allclose(g[..., :d], ref[..., :d], rtol=MEAN_REL, atol=1e-6)


def test_tripool_standalone_matches_fused(V, run):
    """veda_tripool on the permuted tensor gives the fused permute+TripPool descriptor."""
    p, d = run.p, run.w.d
    desc = torch.full_like(run.att.desc_k, float("nan"))
    V.veda_tripool(p, run.att.kp, desc)
    V.veda_sync_status()
    g, ref = f64(desc), run.ora["desc_k"]
    np.testing.assert_array_equal(g[..., d:], ref[..., d:])
    np.testing.assert_allclose(g[..., :d], ref[..., :d], rtol=MEAN_REL, atol=1e-6)
    assert torch.equal(desc, run.att.desc_k)


def test_permute_alone_matches_fused(V, run):
    qp = torch.empty_like(run.att.qp)
    V.veda_tile_permute(run.p, run.q.cuda(), qp)
    torch.cuda.synchronize()
    assert torch.equal(qp, run.att.qp)


def test_score_topk(run):
    nts = run.p.nt_per_head
    ks, _ = run.p.keep_count(run.w.keep)
    gi = run.att.idx.cpu().numpy()
    differ = check_idx(gi, run.ora["idx"], run.ora["scores"], nts, ks)
    assert differ <= max(1, gi.shape[1] * gi.shape[2] // 50)
    np.testing.assert_allclose(f64(run.att.probs), run.ora["probs"], rtol=PROBS_REL, atol=PROBS_ABS)


def test_attention_under_oracle_idx(V, run):
    p, w = run.p, run.w
    idx = torch.from_numpy(run.ora["idx"]).to("cuda")
    op = torch.empty_like(run.att.qp)
    lse = torch.empty((p.B, p.heads, p.nt_max * p.S), dtype=torch.float32, device="cuda")
    V.veda_tile_sparse_attn(p, run.att.qp, run.att.kp, run.att.vp, idx, op, lse)
    V.veda_sync_status()
    ref_op, ref_lse = O.sparse_attention(run.ora["qp"], run.ora["kp"], run.ora["vp"], run.ora["idx"], run.grid,
                                         w.tilings, w.S)
    g, gl = f64(op), f64(lse)
    for h in range(p.heads):
        tab = O.slot_table(run.grid, w.tilings[h])
        rows = np.nonzero(tab >= 0)[0]
        check_attn_rows(g[:, h, rows], ref_op[:, h, rows], f"head {h}")
        assert np.abs(gl[:, h, rows] - ref_lse[:, h, rows]).max() <= LSE_ABS


def test_end_to_end_output(run):
    """Grid-order output; tiles whose selection differs only by a near-tie are skipped."""
    w = run.w
    g = f64(run.out)
    gi = run.att.idx.cpu().numpy()
    ref = run.ora["o"]
    for b in range(w.B):
        for h in range(w.heads):
            tab = O.slot_table(run.grid, w.tilings[h])
            nt = run.p.nt_per_head[h]
            same = [i for i in range(nt) if np.array_equal(gi[b, h, i], run.ora["idx"][b, h, i])]
            assert len(same) >= nt - max(1, nt // 50)
            n = np.concatenate([tab[i * w.S:(i + 1) * w.S] for i in same])
            n = n[n >= 0]
            check_attn_rows(g[b, h, n], ref[b, h, n], f"b{b} h{h}")


def test_unpermute_bit_exact(V, run):
    p, w = run.p, run.w
    op = run.att.op
    x = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device="cuda")
    V.veda_tile_unpermute(p, op, x)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(f64(x), O.tile_unpermute(f64(op), run.grid, w.tilings, w.S))


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_tile_map(V, w):
    p = _problem(V, w)
    q, k, _ = make_qkv(w, seed=5)
    qp = torch.empty(p.tile_shape(), dtype=torch.bfloat16, device="cuda")
    kp = torch.empty_like(qp)
    V.veda_tile_permute(p, q.cuda(), qp)
    V.veda_tile_permute(p, k.cuda(), kp)
    rows = make_map_rows(p.nt_per_head, w.B, 0.3, seed=2)
    rows[0, -1] = -1  # an unused slot
    R = rows.shape[1]
    ws = torch.empty(V.veda_tile_map_workspace(p, R) // 4 + 64, dtype=torch.float32, device="cuda")
    out = torch.full((p.B, p.heads, R, p.nt_max), float("nan"), dtype=torch.float32, device="cuda")
    V.veda_tile_map_maxpool(p, qp, kp, rows.cuda(), out, ws)
    V.veda_sync_status()
    grid = (w.T, w.H, w.W)
    ref = O.tile_map_maxpool(f64(qp), f64(kp), rows.numpy(), grid, w.tilings, w.S)
    g = f64(out)
    big = ref >= 1e-8
    assert np.all(np.abs(g[big] - ref[big]) <= MAP_REL * ref[big])
    assert np.all(np.abs(g[~big] - ref[~big]) <= 1e-11)


def test_invalid_idx_entries_end_the_list(V):
    """Entries outside [0, NT_h) terminate a selection list like -1 does."""
    w = SMALL[2]
    p = _problem(V, w)
    q, k, v = (t.cuda() for t in make_qkv(w, seed=3))
    ts = p.tile_shape()
    qp, kp, vp = (torch.empty(ts, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    for a, b in ((q, qp), (k, kp), (v, vp)):
        V.veda_tile_permute(p, a, b)
    idx = torch.full((p.B, p.heads, p.nt_max, 4), -1, dtype=torch.int32)
    idx[..., 0] = 0
    idx[..., 1] = 1
    idx2 = idx.clone()
    idx2[..., 2] = 10_000           # out of range: ends the list
    idx2[..., 3] = 2
    o1 = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    V.veda_tile_sparse_attn(p, qp, kp, vp, idx.cuda(), o1)
    V.veda_tile_sparse_attn(p, qp, kp, vp, idx2.cuda(), o2)
    V.veda_sync_status()
    for h in range(p.heads):
        tab = O.slot_table((w.T, w.H, w.W), w.tilings[h])
        rows = torch.from_numpy(np.nonzero(tab >= 0)[0]).cuda()
        assert torch.equal(o1[:, h, rows], o2[:, h, rows])


def test_timeout_is_reported_not_hung(V):
    V.veda_selftest_wait_timeout(2_000_000)   # 2 ms bounded wait that nothing satisfies
    with pytest.raises(V.VedaError) as ei:
        V.veda_sync_status()
    assert ei.value.status == 4
    V.veda_sync_status()                      # error word cleared, context usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


# ------------------------------------------------------------------ full-size sampled parity
def test_wan14b_full_size_sampled(V):
    """Wan2.1-14B 720p/81-frame shape at keep 5%, the benchmarked launch, on sampled heads and tiles."""
    w = PRESETS["wan14b"]
    p = _problem(V, w)
    q, k, v = cached_qkv(w, 0)
    m = make_mlp(w, seed=1)
    att = V.VedaAttention(p, mlp_device(m), mlp_device(m), w.keep, want_lse=True, layout="tile")
    out = att(q.cuda(), k.cuda(), v.cuda())
    V.veda_sync_status()
    heads = [0, 13, 39]
    grid = (w.T, w.H, w.W)
    ks, _ = p.keep_count(w.keep)
    mlp_all = mlp_numpy(m)
    gi = att.idx.cpu().numpy()
    rng = np.random.default_rng(0)
    checked = 0
    for h in heads:
        tl = [w.tilings[h]]
        mh = tuple(a[h:h + 1] for a in mlp_all)
        qh, kh, vh = (f64(t[:, h:h + 1]) for t in (q, k, v))
        qp, kp, vp = (O.tile_permute(a, grid, tl, w.S) for a in (qh, kh, vh))
        nt = p.nt_per_head[h]
        np.testing.assert_array_equal(f64(att.qp[:, h, :nt * w.S]), qp[:, 0])
        np.testing.assert_array_equal(f64(att.vp[:, h, :nt * w.S]), vp[:, 0])
        dq, dk = O.tripool(qp, grid, tl, w.S), O.tripool(kp, grid, tl, w.S)
        g = f64(att.desc_k[:, h, :nt])
        np.testing.assert_array_equal(g[..., w.d:], dk[:, 0, :, w.d:])
        np.testing.assert_allclose(g[..., :w.d], dk[:, 0, :, :w.d], rtol=MEAN_REL, atol=1e-6)
        idx, _, scores = O.score_topk(dq, dk, grid, tl, w.S, mh, mh, keep_f32(w.keep), want_scores=True)
        differ = check_idx(gi[:, h:h + 1, :nt], idx, scores, [nt], [ks[h]])
        assert differ <= max(1, nt // 50)
        tab = O.slot_table(grid, tl[0])
        gop = att.op
        k_h = ks[h]   # the one-head oracle pads its rows to this head's k only
        for i in rng.choice(nt, 6, replace=False):
            sel = idx[0, 0, i, :k_h]
            if not (np.array_equal(gi[0, h, i, :k_h], sel) and np.all(gi[0, h, i, k_h:] == -1)):
                continue
            checked += 1
            o_ref, lse_ref = O.attention_tile(qp[0, 0], kp[0, 0], vp[0, 0], tab, int(i), sel, w.S,
                                              1 / math.sqrt(w.d))
            rows = np.nonzero(tab[i * w.S:(i + 1) * w.S] >= 0)[0]
            og = f64(gop[0, h, i * w.S:(i + 1) * w.S])
            check_attn_rows(og[rows], o_ref[rows], f"h{h} tile {i}")
            lg = f64(att.lse[0, h, i * w.S:(i + 1) * w.S])
            assert np.abs(lg[rows] - lse_ref[rows]).max() <= LSE_ABS
            # and the grid-order output carries the same rows
            n = tab[i * w.S:(i + 1) * w.S][rows]
            np.testing.assert_array_equal(f64(out[0, h, torch.from_numpy(n).cuda()]), og[rows])
    assert checked >= 12
