"""GPU parity of kernel configurations that only large problems reach.

The launch picks kernel variants from the problem size, and the benchmark
workloads reach variants that the small parity cases do not:

* rows of more than 512 tiles score through the fp32 score matrix in the
  workspace (tensor-core GEMM, then one warp per row), including B = 2;
* top-k over rows of 257-512, 513-768 and 769-1,024 tiles: the register
  bisection with 16, 24 and 32 keys per lane (the Wan2.1-1.3B shape has up to
  336 tiles per head, the Wan2.1-14B shape 720), with every feature width the
  score kernel stages (e = 16, 32, 64, 128);
* top-k over rows of 1,025-2,048 tiles: the register bisection with 64 keys
  per lane (the 245,760-token sweep has 1,920 tiles per head);
* top-k over rows of more than 2,048 tiles: the radix select;
* the attention kernel with a 3-stage K ring and a 2-stage V ring, chosen when
  the selection list no longer leaves room for 3 + 3 stages (the dense
  keep-100% reference run at the Wan2.1-14B shape selects 720 tiles);
* the max-pooled tile map at full size (Wan2.1-14B, 10% of the Q tiles).

Each is compared with the fp64 oracle under the contract's tolerances, on the
whole problem where the oracle finishes in seconds and on sampled heads, rows
and Q tiles of the full-size launch otherwise.
"""
import math

import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
from veda_synth import PRESETS, make_map_rows, make_mlp, make_qkv

from parity import (LSE_ABS, MAP_REL, PROBS_ABS, PROBS_REL, cached_qkv, check_attn_rows, check_idx, f64, keep_f32,
                    mlp_device, mlp_numpy, wl)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def _problem(V, w):
    return V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)


def _select_on_gpu(V, w, q, k, m, want_probs):
    """TripPool (grid order) and scoring + top-k on the device; returns (idx, probs, desc_q, desc_k)."""
    p = _problem(V, w)
    md = mlp_device(m)
    att = V.VedaAttention(p, md, md, w.keep, want_probs=want_probs, layout="grid")
    att.select(q.cuda(), k.cuda(), None)
    V.veda_sync_status()
    return att


def _oracle_selection(w, q, k, m, heads):
    """The oracle's permute, TripPool and scoring + top-k for the given heads, one at a time."""
    grid = (w.T, w.H, w.W)
    mlp_all = mlp_numpy(m)
    out = []
    for h in heads:
        tl = [w.tilings[h]]
        mh = tuple(a[h:h + 1] for a in mlp_all)
        qp = O.tile_permute(f64(q[:, h:h + 1]), grid, tl, w.S)
        kp = O.tile_permute(f64(k[:, h:h + 1]), grid, tl, w.S)
        dq, dk = O.tripool(qp, grid, tl, w.S), O.tripool(kp, grid, tl, w.S)
        idx, probs, scores = O.score_topk(dq, dk, grid, tl, w.S, mh, mh, keep_f32(w.keep), want_scores=True)
        out.append((idx, probs, scores))
    return out


def _check_selection(V, w, att, ora, heads, check_probs):
    p = att.p
    ks, _ = p.keep_count(w.keep)
    gi = att.idx.cpu().numpy()
    for h, (idx, probs, scores) in zip(heads, ora):
        nt = p.nt_per_head[h]
        differ = check_idx(gi[:, h:h + 1, :nt], idx, scores, [nt], [ks[h]])
        assert differ <= max(1, nt // 50), f"head {h}: {differ} of {nt} rows differ beyond near-ties"
        if check_probs:
            g = f64(att.probs[:, h, :nt, :nt])
            np.testing.assert_allclose(g, probs[:, 0, :nt, :nt], rtol=PROBS_REL, atol=PROBS_ABS)


# ------------------------------------------------------------------ top-k variants
# Two heads of unequal tile counts each, so the launch covers rows of both
# lengths and rows past a head's own count.
TOPK_CASES = [
    # 330 and 360 tiles: 16 keys per lane, e = 16
    wl("topk360", (12, 40, 44), 1, 2, 64, 64, [(4, 4, 4), (1, 8, 8)], 0.05, 128, 16, "rff"),
    # 660 and 720 tiles: 24 keys per lane (as in the Wan2.1-14B launch), e = 32
    wl("topk720", (24, 40, 44), 1, 2, 64, 64, [(4, 4, 4), (2, 4, 8)], 0.05, 128, 32, "rff"),
    # 600 tiles, e = 128: phi_k staged partly from registers, partly directly
    wl("topk600e128", (24, 40, 40), 1, 1, 64, 64, [(4, 4, 4)], 0.05, 128, 128, "rff"),
    # 770 and 715 tiles at d = 128: 32 keys per lane, e = 64
    wl("topk770", (26, 42, 40), 1, 2, 128, 64, [(4, 4, 4), (2, 4, 8)], 0.05, 256, 64, "rff"),
    # B = 2 with rows of 660 and 720 tiles: the score-matrix path's batch and head offsets
    wl("topk720b2", (24, 40, 44), 2, 2, 64, 64, [(2, 4, 8), (4, 4, 4)], 0.05, 128, 32, "rff"),
    # 1,650 tiles: the 64-keys-per-lane register bisection
    wl("topk1650", (39, 41, 58), 1, 2, 64, 64, [(4, 4, 4), (2, 4, 8)], 0.05, 128, 32, "rff"),
    # 2,145 and 2,200 tiles: the radix select
    wl("topk2200", (50, 44, 60), 1, 2, 64, 64, [(4, 4, 4), (2, 4, 8)], 0.05, 128, 32, "rff"),
    # 2,240 tiles at d = 128, S = 128: the radix select at the benchmark's head dim
    wl("topk2240", (70, 64, 64), 1, 1, 128, 128, [(2, 8, 8)], 0.05, 256, 64, "local"),
]


@pytest.mark.parametrize("w", TOPK_CASES, ids=[w.name for w in TOPK_CASES])
def test_topk_row_lengths_against_oracle(V, w):
    p = _problem(V, w)
    assert p.nt_max > 256
    q, k, _ = make_qkv(w, seed=0)
    m = make_mlp(w, seed=1)
    att = _select_on_gpu(V, w, q, k, m, want_probs=True)
    heads = list(range(w.heads))
    _check_selection(V, w, att, _oracle_selection(w, q, k, m, heads), heads, check_probs=True)


def test_topk_sweep246k_sampled_heads(V):
    """The 245,760-token sweep workload (24 heads, 1,920 tiles each, keep 5%)
    in the launch configuration the bench times; two heads against the oracle."""
    w = PRESETS["sweep246k"]
    q, k, _ = cached_qkv(w, 0)
    m = make_mlp(w, seed=1)
    att = _select_on_gpu(V, w, q, k, m, want_probs=False)
    heads = [0, 17]
    _check_selection(V, w, att, _oracle_selection(w, q, k, m, heads), heads, check_probs=False)


# ------------------------------------------------------------------ attention ring depths
RING32 = wl("dense192", (11, 30, 64), 1, 1, 128, 128, [(2, 8, 8)], 1.0, 256, 64, "rff")


@pytest.mark.parametrize("layout", ["tile", "grid"])
def test_attention_three_k_two_v_stages_full_keep(V, layout):
    """192 tiles, all kept: the selection list is long enough that the launch
    takes 3 K stages and 2 V stages; the whole output against the oracle."""
    w = RING32
    p = _problem(V, w)
    ks, k_max = p.keep_count(w.keep)
    assert k_max == p.nt_max == 192
    kst, vst, _ = V.veda_attn_config(p, k_max)
    assert (kst, vst) == (3, 2)
    q, k, v = make_qkv(w, seed=2)
    m = make_mlp(w, seed=3)
    md = mlp_device(m)
    att = V.VedaAttention(p, md, md, w.keep, want_lse=True, layout=layout)
    out = att(q.cuda(), k.cuda(), v.cuda())
    V.veda_sync_status()
    gi = att.idx.cpu().numpy()
    assert np.array_equal(gi[0, 0], np.tile(np.arange(192, dtype=np.int32), (192, 1)))
    grid = (w.T, w.H, w.W)
    qd, kd, vd = (f64(t) for t in (q, k, v))
    perm = [O.tile_permute(a, grid, w.tilings, w.S) for a in (qd, kd, vd)]
    ref_op, ref_lse = O.sparse_attention(*perm, gi.astype(np.int64), grid, w.tilings, w.S)
    tab = O.slot_table(grid, w.tilings[0])
    rows = np.nonzero(tab >= 0)[0]
    ref_o = O.tile_unpermute(ref_op, grid, w.tilings, w.S)
    check_attn_rows(f64(out)[0, 0], ref_o[0, 0], f"{layout} layout, output")
    if layout == "tile":
        lse = f64(att.lse)[0, 0, rows]
    else:
        lse = f64(att.lse)[0, 0, tab[rows]]
    assert np.abs(lse - ref_lse[0, 0, rows]).max() <= LSE_ABS
    # keep 100% is dense attention over the head's tokens
    sdpa = torch.nn.functional.scaled_dot_product_attention(*(torch.from_numpy(a) for a in (qd, kd, vd))).numpy()
    check_attn_rows(f64(out)[0, 0], sdpa[0, 0], f"{layout} layout, against dense SDPA")


def test_attention_wan14b_dense_sampled(V):
    """The dense reference run at the Wan2.1-14B shape (keep 100%, 630-720
    tiles per head, the 3/2-stage launch), grid order as benchmarked; sampled
    Q tiles of two heads against the oracle."""
    w = PRESETS["wan14b-dense"]
    p = _problem(V, w)
    ks, k_max = p.keep_count(w.keep)
    assert V.veda_attn_config(p, k_max)[:2] == (3, 2)
    q, k, v = cached_qkv(PRESETS["wan14b"], 0)          # same tensors as the keep-5% workload
    idx = torch.full((p.B, p.heads, p.nt_max, k_max), -1, dtype=torch.int32)
    for h, nt in enumerate(p.nt_per_head):
        idx[0, h, :nt, :nt] = torch.arange(nt, dtype=torch.int32)
    out = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((p.B, p.heads, p.N), dtype=torch.float32, device="cuda")
    V.veda_tile_sparse_attn_grid(p, q.cuda(), k.cuda(), v.cuda(), idx.cuda(), out, lse)
    V.veda_sync_status()
    grid = (w.T, w.H, w.W)
    rng = np.random.default_rng(7)
    for h in (5, 31):
        tl = [w.tilings[h]]
        qp, kp, vp = (O.tile_permute(f64(t[:, h:h + 1]), grid, tl, w.S) for t in (q, k, v))
        tab = O.slot_table(grid, tl[0])
        nt = p.nt_per_head[h]
        for i in rng.choice(nt, 3, replace=False):
            o_ref, lse_ref = O.attention_tile(qp[0, 0], kp[0, 0], vp[0, 0], tab, int(i), np.arange(nt), w.S,
                                              1 / math.sqrt(w.d))
            slots = np.nonzero(tab[i * w.S:(i + 1) * w.S] >= 0)[0]
            n = torch.from_numpy(tab[i * w.S:(i + 1) * w.S][slots])
            check_attn_rows(f64(out[0, h, n.cuda()]), o_ref[slots], f"h{h} tile {i}")
            assert np.abs(f64(lse[0, h, n.cuda()]) - lse_ref[slots]).max() <= LSE_ABS


# ------------------------------------------------------------------ tile map at full size
def test_tile_map_wan14b_sampled_rows(V):
    """The max-pooled full-attention map over 10% of the Q tiles at the
    Wan2.1-14B shape (the distillation target's launch), from the permuted
    copies and from grid order (identical maps); sampled subset rows of three
    heads against the oracle's explicit softmax rows."""
    w = PRESETS["wan14b"]
    p = _problem(V, w)
    q, k, _ = cached_qkv(w, 0)
    ts = p.tile_shape()
    qp = torch.empty(ts, dtype=torch.bfloat16, device="cuda")
    kp = torch.empty_like(qp)
    V.veda_tile_permute(p, q.cuda(), qp)
    V.veda_tile_permute(p, k.cuda(), kp)
    rows = make_map_rows(p.nt_per_head, w.B, 0.1, seed=2)
    R = rows.shape[1]
    ws = torch.empty(V.veda_tile_map_workspace(p, R) // 4 + 64, dtype=torch.float32, device="cuda")
    mp = torch.full((p.B, p.heads, R, p.nt_max), float("nan"), dtype=torch.float32, device="cuda")
    V.veda_tile_map_maxpool(p, qp, kp, rows.cuda(), mp, ws)
    # the grid-order entry point on the unpermuted tensors gives the same map
    mg = torch.full_like(mp, float("nan"))
    V.veda_tile_map_maxpool_grid(p, q.cuda(), k.cuda(), rows.cuda(), mg, ws)
    V.veda_sync_status()
    assert torch.equal(mg, mp)
    del ws, mg
    grid = (w.T, w.H, w.W)
    rng = np.random.default_rng(3)
    g = f64(mp)
    scale = 1 / math.sqrt(w.d)
    for h in (2, 19, 38):
        tl = [w.tilings[h]]
        qh, kh = (O.tile_permute(f64(t[:, h:h + 1]), grid, tl, w.S) for t in (q, k))
        tab = O.slot_table(grid, tl[0])
        nt = p.nt_per_head[h]
        count = int((rows[h] >= 0).sum())
        for r in rng.choice(count, 2, replace=False):
            i = int(rows[h, r])
            ref = O.tile_map_row(qh[0, 0], kh[0, 0], tab, i, w.S, scale)
            got = g[0, h, r, :nt]
            big = ref >= 1e-8
            assert np.all(np.abs(got[big] - ref[big]) <= MAP_REL * ref[big]), (h, r)
            assert np.all(np.abs(got[~big] - ref[~big]) <= 1e-11), (h, r)
            assert np.all(g[0, h, r, nt:] == 0.0)
        # unused subset slots of this head are zero rows
        assert np.all(g[0, h, count:] == 0.0)
