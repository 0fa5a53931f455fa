"""Pins for the fp64 oracle, each tied to something other than the oracle itself.

Every check below comes from the Veda pages' description (sections 2.1-2.3 of
the technical summary) plus mathematics: hand-derived examples, closed forms,
brute force over grid coordinates, and special cases that reduce to a library
routine (dense SDPA, logsumexp, softmax).  They are chosen so that a plausible
mistake in the oracle -- a transposed tile order, a dropped bias or ReLU, a
wrong scale, an off-by-one keep count, a pad slot counted as a token -- fails
at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import veda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def box_members(grid, tiling):
    """Tokens of every tile by explicit loops over box bounds (no slot formula)."""
    T, H, W = grid
    pt, ph, pw = tiling
    nT, nH, nW = -(-T // pt), -(-H // ph), -(-W // pw)
    tiles = []
    for a in range(nT):
        for b in range(nH):
            for c in range(nW):
                mem = []
                for t in range(a * pt, min(T, (a + 1) * pt)):
                    for y in range(b * ph, min(H, (b + 1) * ph)):
                        for x in range(c * pw, min(W, (c + 1) * pw)):
                            mem.append((t * H + y) * W + x)
                tiles.append(sorted(mem))
    return tiles


def reshape_table(grid, tiling):
    """Slot table by padding, reshaping and transposing an index grid."""
    T, H, W = grid
    pt, ph, pw = tiling
    nT, nH, nW = -(-T // pt), -(-H // ph), -(-W // pw)
    g = np.full((nT * pt, nH * ph, nW * pw), -1, dtype=np.int64)
    g[:T, :H, :W] = np.arange(T * H * W).reshape(T, H, W)
    g = g.reshape(nT, pt, nH, ph, nW, pw).transpose(0, 2, 4, 1, 3, 5)
    return g.reshape(-1)


def read_golden_tables():
    cases = []
    with open(os.path.join(GOLDEN, "permutation_examples.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for hdr, body in zip(lines[0::2], lines[1::2]):
        p = hdr.split()
        grid = (int(p[1]), int(p[2]), int(p[3]))
        tiling = (int(p[5]), int(p[6]), int(p[7]))
        table = [int(v) for v in body.replace("|", " ").split()]
        cases.append((grid, tiling, np.array(table)))
    return cases


GRIDS = [((4, 8, 8), (1, 8, 8)), ((4, 8, 8), (4, 4, 4)), ((3, 5, 7), (1, 2, 4)),
         ((3, 5, 7), (2, 2, 2)), ((5, 9, 6), (2, 4, 2)), ((2, 3, 17), (1, 1, 16))]


# ---------------------------------------------------------------- step 1: tiling
def test_slot_table_hand_examples():
    cases = read_golden_tables()
    assert len(cases) == 4
    for grid, tiling, table in cases:
        np.testing.assert_array_equal(O.slot_table(grid, tiling), table)


@pytest.mark.parametrize("grid,tiling", GRIDS)
def test_slot_table_matches_reshape_construction(grid, tiling):
    np.testing.assert_array_equal(O.slot_table(grid, tiling), reshape_table(grid, tiling))


@pytest.mark.parametrize("grid,tiling", GRIDS)
def test_tile_membership_matches_box_bounds(grid, tiling):
    S = tiling[0] * tiling[1] * tiling[2]
    tab = O.slot_table(grid, tiling)
    mem = box_members(grid, tiling)
    assert tab.size == len(mem) * S
    for j, m in enumerate(mem):
        got = sorted(int(v) for v in tab[j * S:(j + 1) * S] if v >= 0)
        assert got == m


def test_frame_tiling_is_identity():
    # A (1,8,8) tile over an 8x8 frame holds exactly one frame in raster order.
    np.testing.assert_array_equal(O.slot_table((4, 8, 8), (1, 8, 8)), np.arange(256))


@pytest.mark.parametrize("grid,tiling", GRIDS)
def test_permute_unpermute_identity_and_zero_pads(grid, tiling):
    rng = np.random.default_rng(0)
    S = tiling[0] * tiling[1] * tiling[2]
    other = (tiling[2], tiling[1], tiling[0])          # second head, another tiling of the same size
    tilings = [tiling, other]
    N = grid[0] * grid[1] * grid[2]
    x = rng.standard_normal((2, 2, N, 8))
    xp = O.tile_permute(x, grid, tilings, S)
    np.testing.assert_array_equal(O.tile_unpermute(xp, grid, tilings, S), x)
    for h, tl in enumerate(tilings):
        tab = O.slot_table(grid, tl)
        full = np.full(xp.shape[2], -1)
        full[:tab.size] = tab
        assert np.all(xp[:, h, full < 0] == 0)
        # every grid token appears exactly once
        assert sorted(tab[tab >= 0].tolist()) == list(range(N))


def test_tile_counts_configs():
    # Tile counts quoted for the workloads (hand arithmetic: ceil per dim).
    assert O.num_tiles((21, 30, 52), (2, 8, 8)) == 11 * 4 * 7 == 308
    assert O.num_tiles((21, 30, 52), (1, 8, 16)) == 21 * 4 * 4 == 336
    assert O.num_tiles((21, 45, 80), (8, 4, 4)) == 3 * 12 * 20 == 720
    assert O.num_tiles((60, 64, 64), (2, 8, 8)) == 30 * 8 * 8 == 1920


# ---------------------------------------------------------------- step 2: TripPool
def test_tripool_closed_forms():
    grid, tiling, S = (1, 3, 3), (1, 2, 2), 4
    d = 3
    x = np.zeros((1, 1, 9, d))
    # channel 0: constant 2.5; channel 1: token index; channel 2: -index
    x[0, 0, :, 0] = 2.5
    x[0, 0, :, 1] = np.arange(9)
    x[0, 0, :, 2] = -np.arange(9)
    desc = O.tripool(O.tile_permute(x, grid, [tiling], S), grid, [tiling], S)[0, 0]
    # tile 0 = tokens {0,1,3,4}; tile 1 = {2,5}; tile 2 = {6,7}; tile 3 = {8}
    members = [[0, 1, 3, 4], [2, 5], [6, 7], [8]]
    for j, m in enumerate(members):
        mean, mx, mn = desc[j, :d], desc[j, d:2 * d], desc[j, 2 * d:]
        assert mean[0] == mx[0] == mn[0] == 2.5
        assert mean[1] == pytest.approx(sum(m) / len(m))
        assert mx[1] == max(m) and mn[1] == min(m)
        assert mx[2] == -min(m) and mn[2] == -max(m)


@pytest.mark.parametrize("grid,tiling", GRIDS)
def test_tripool_brute_force_over_grid(grid, tiling):
    rng = np.random.default_rng(1)
    S = tiling[0] * tiling[1] * tiling[2]
    N = grid[0] * grid[1] * grid[2]
    x = rng.standard_normal((1, 1, N, 5))
    desc = O.tripool(O.tile_permute(x, grid, [tiling], S), grid, [tiling], S)[0, 0]
    for j, m in enumerate(box_members(grid, tiling)):
        rows = torch.tensor(x[0, 0, m])
        ref = torch.cat([rows.mean(0), rows.amax(0), rows.amin(0)]).numpy()
        np.testing.assert_allclose(desc[j], ref, rtol=1e-14, atol=1e-14)
        assert np.all(desc[j, 5:10] >= desc[j, :5]) and np.all(desc[j, :5] >= desc[j, 10:])


# ---------------------------------------------------------------- step 3: estimator
def test_estimator_bias_only_closed_form():
    # W1 = 0, b1 = c > 0 -> hidden = c (ReLU passes) -> phi = c * W2 @ 1 + b2.
    rng = np.random.default_rng(2)
    desc = rng.standard_normal((4, 6))
    w1 = np.zeros((5, 6)); b1 = np.full(5, 0.7)
    w2 = rng.standard_normal((3, 5)); b2 = np.array([0.1, -0.2, 0.3])
    phi = O.estimator_head(desc, w1, b1, w2, b2)
    expect = 0.7 * w2.sum(axis=1) + b2
    for r in range(4):
        np.testing.assert_allclose(phi[r], expect, rtol=1e-14)


def test_estimator_relu_closed_form():
    # W1 = [I; -I] over the mean block: hidden = (relu(m), relu(-m)), W2 = [I, -I] -> phi = m.
    d = 4
    desc = np.array([[0.5, -1.0, 2.0, -0.25] + [9.0] * 8])
    w1 = np.zeros((2 * d, 3 * d)); w1[:d, :d] = np.eye(d); w1[d:, :d] = -np.eye(d)
    w2 = np.hstack([np.eye(d), -np.eye(d)])
    phi = O.estimator_head(desc, w1, np.zeros(2 * d), w2, np.zeros(d))
    np.testing.assert_allclose(phi[0], desc[0, :d], rtol=0, atol=0)
    # Dropping the second half of hidden (only relu(m)) must not reproduce m.
    phi_pos = O.estimator_head(desc, w1[:d], np.zeros(d), np.eye(d), np.zeros(d))
    np.testing.assert_allclose(phi_pos[0], np.maximum(desc[0, :d], 0))


def test_scores_scale_and_orientation():
    # phi_q rows = e_0 * a_i, phi_k rows = e_0 * b_j  ->  s[i,j] = a_i * b_j / sqrt(e).
    e, d3 = 16, 6
    a = np.array([1.0, 2.0, -1.0]); bvals = np.array([3.0, -0.5])
    desc_q = np.zeros((3, d3)); desc_q[:, 0] = a
    desc_k = np.zeros((2, d3)); desc_k[:, 0] = bvals
    w1 = np.zeros((2, d3)); w1[0, 0] = 1; w1[1, 0] = -1
    w2 = np.zeros((e, 2)); w2[0, 0] = 1; w2[0, 1] = -1
    wts = (w1, np.zeros(2), w2, np.zeros(e))
    s = O.tile_scores_head(desc_q, desc_k, wts, wts)
    np.testing.assert_allclose(s, np.outer(a, bvals) / 4.0, rtol=1e-15)


def test_row_softmax_matches_scipy():
    from scipy.special import softmax
    rng = np.random.default_rng(3)
    s = rng.standard_normal((7, 11)) * 5
    np.testing.assert_allclose(O.row_softmax(s), softmax(s, axis=1), rtol=1e-13)
    np.testing.assert_allclose(O.row_softmax(s).sum(1), 1.0, rtol=1e-14)


# ---------------------------------------------------------------- step 4: top-k
def test_keep_count_table():
    assert O.keep_count(4, 0.5) == 2
    assert [O.keep_count(n, 0.1) for n in (308, 336, 312)] == [31, 34, 31]
    assert [O.keep_count(n, 0.05) for n in (660, 630, 720)] == [33, 32, 36]
    assert [O.keep_count(n, 0.05) for n in (512, 960, 1920)] == [26, 48, 96]
    assert O.keep_count(10, 1e-6) == 1 and O.keep_count(10, 1.0) == 10


def test_topk_against_python_sort_with_ties():
    rng = np.random.default_rng(4)
    for trial in range(50):
        nt = int(rng.integers(1, 80))
        s = np.round(rng.standard_normal(nt), 1)         # many exact ties
        k = int(rng.integers(1, nt + 1))
        ref = sorted(sorted(range(nt), key=lambda j: (-s[j], j))[:k])
        assert O.select_topk_row(s, k).tolist() == ref
    s = rng.standard_normal(13)
    assert O.select_topk_row(s, 13).tolist() == list(range(13))


def test_score_topk_contract():
    grid, tilings, S = (3, 5, 7), [(1, 2, 4), (2, 2, 2)], 8
    rng = np.random.default_rng(5)
    nts, ntmax = O.tile_layout(grid, tilings)
    dq = rng.standard_normal((1, 2, ntmax, 12)); dk = rng.standard_normal((1, 2, ntmax, 12))
    mlp = (rng.standard_normal((2, 6, 12)), rng.standard_normal((2, 6)),
           rng.standard_normal((2, 5, 6)), rng.standard_normal((2, 5)))
    idx, probs = O.score_topk(dq, dk, grid, tilings, S, mlp, mlp, 0.3)
    for h, nt in enumerate(nts):
        k = O.keep_count(nt, 0.3)
        for i in range(ntmax):
            row = idx[0, h, i]
            if i >= nt:
                assert np.all(row == -1)
                continue
            sel = row[row >= 0]
            assert len(sel) == k and np.all(np.diff(sel) > 0) and sel.max() < nt
            assert np.all(row[k:] == -1)
            np.testing.assert_allclose(probs[0, h, i, :nt].sum(), 1.0, rtol=1e-13)


def _mlp_by_loops(x, w1, b1, w2, b2):
    """phi = W2 relu(W1 x + b1) + b2 for one descriptor row, written out as plain loops."""
    hidden = []
    for u in range(len(b1)):
        z = b1[u]
        for c in range(len(x)):
            z += w1[u][c] * x[c]
        hidden.append(z if z > 0.0 else 0.0)
    out = []
    for o in range(len(b2)):
        acc = b2[o]
        for u in range(len(hidden)):
            acc += w2[o][u] * hidden[u]
        out.append(acc)
    return out


def test_score_topk_assembly_by_explicit_loops():
    """Which side is which in the score matrix, section 2.1: row i is Q tile i
    (the Q-side MLP applied to the Q descriptor), column j is K tile j (the
    K-side MLP applied to the K descriptor).  Q and K get different weights
    and descriptors, the two heads have different tile counts, and B = 2, so
    a transposed matrix, swapped weight sets, a swapped batch or head, or a
    head read at the wrong NT all change the logits or the selection."""
    grid, tilings, S = (3, 5, 7), [(1, 2, 4), (2, 2, 2)], 8
    nts, ntmax = O.tile_layout(grid, tilings)
    assert nts[0] != nts[1]
    rng = np.random.default_rng(21)
    B, heads, d3, hid, e = 2, 2, 9, 7, 5
    dq = rng.standard_normal((B, heads, ntmax, d3))
    dk = rng.standard_normal((B, heads, ntmax, d3)) * 1.3 + 0.2
    mlp_q = (rng.standard_normal((heads, hid, d3)), rng.standard_normal((heads, hid)),
             rng.standard_normal((heads, e, hid)), rng.standard_normal((heads, e)))
    mlp_k = (rng.standard_normal((heads, hid, d3)), rng.standard_normal((heads, hid)),
             rng.standard_normal((heads, e, hid)), rng.standard_normal((heads, e)))
    keep = 0.3
    idx, probs, scores = O.score_topk(dq, dk, grid, tilings, S, mlp_q, mlp_k, keep, want_scores=True)
    for b in range(B):
        for h in range(heads):
            nt = nts[h]
            k = O.keep_count(nt, keep)
            wq = [m[h].tolist() for m in mlp_q]
            wk = [m[h].tolist() for m in mlp_k]
            phq = [_mlp_by_loops(dq[b, h, i].tolist(), *wq) for i in range(nt)]
            phk = [_mlp_by_loops(dk[b, h, j].tolist(), *wk) for j in range(nt)]
            for i in range(nt):
                s = []
                for j in range(nt):
                    dot = 0.0
                    for o in range(e):
                        dot += phq[i][o] * phk[j][o]
                    s.append(dot / math.sqrt(e))
                np.testing.assert_allclose(scores[b, h, i, :nt], s, rtol=1e-11, atol=1e-11)
                assert np.all(np.isneginf(scores[b, h, i, nt:]))
                ref = sorted(sorted(range(nt), key=lambda j: (-s[j], j))[:k])
                assert idx[b, h, i, :k].tolist() == ref, (b, h, i)
                assert np.all(idx[b, h, i, k:] == -1)
                z = [math.exp(v - max(s)) for v in s]
                np.testing.assert_allclose(probs[b, h, i, :nt], [v / sum(z) for v in z], rtol=1e-12)
            for i in range(nt, ntmax):
                assert np.all(idx[b, h, i] == -1)


# ---------------------------------------------------------------- step 5: attention
def _inputs(grid, d, heads=2, seed=6):
    rng = np.random.default_rng(seed)
    N = grid[0] * grid[1] * grid[2]
    return [rng.standard_normal((1, heads, N, d)) for _ in range(3)]


def _dense_sdpa(q, k, v):
    tq, tk, tv = (torch.tensor(a) for a in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).numpy()


@pytest.mark.parametrize("grid,tilings,S", [((4, 8, 8), [(1, 8, 8), (4, 4, 4)], 64),
                                             ((3, 5, 7), [(1, 2, 4), (2, 2, 2)], 8)])
def test_full_keep_equals_dense_sdpa(grid, tilings, S):
    q, k, v = _inputs(grid, 16)
    qp, kp, vp = (O.tile_permute(a, grid, tilings, S) for a in (q, k, v))
    nts, ntmax = O.tile_layout(grid, tilings)
    idx = np.full((1, 2, ntmax, ntmax), -1, dtype=np.int32)
    for h, nt in enumerate(nts):
        idx[0, h, :nt, :nt] = np.arange(nt)
    op, lse = O.sparse_attention(qp, kp, vp, idx, grid, tilings, S)
    o = O.tile_unpermute(op, grid, tilings, S)
    np.testing.assert_allclose(o, _dense_sdpa(q, k, v), rtol=1e-12, atol=1e-12)
    ref_lse = torch.logsumexp(torch.tensor(q) @ torch.tensor(k).transpose(-1, -2) / 4.0, dim=-1).numpy()
    lse_grid = O.tile_unpermute(lse[..., None], grid, tilings, S)[..., 0]
    np.testing.assert_allclose(lse_grid, ref_lse, rtol=1e-12, atol=1e-12)


def test_masked_attention_brute_force_in_grid_coordinates():
    grid, tilings, S = (3, 5, 7), [(1, 2, 4), (2, 2, 2)], 8
    q, k, v = _inputs(grid, 8, seed=7)
    rng = np.random.default_rng(8)
    nts, ntmax = O.tile_layout(grid, tilings)
    idx = np.full((1, 2, ntmax, 4), -1, dtype=np.int32)
    for h, nt in enumerate(nts):
        for i in range(nt):
            idx[0, h, i, :3] = np.sort(rng.choice(nt, 3, replace=False))
    qp, kp, vp = (O.tile_permute(a, grid, tilings, S) for a in (q, k, v))
    op, _ = O.sparse_attention(qp, kp, vp, idx, grid, tilings, S)
    o = O.tile_unpermute(op, grid, tilings, S)
    N = grid[0] * grid[1] * grid[2]
    for h in range(2):
        members = box_members(grid, tilings[h])
        tile_of = np.empty(N, dtype=np.int64)
        for j, m in enumerate(members):
            tile_of[m] = j
        allowed = np.zeros((N, N), dtype=bool)
        for n in range(N):
            sel = set(int(j) for j in idx[0, h, tile_of[n]] if j >= 0)
            allowed[n] = [tile_of[m] in sel for m in range(N)]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[0, h]), torch.tensor(k[0, h]), torch.tensor(v[0, h]),
            attn_mask=torch.tensor(allowed)).numpy()
        np.testing.assert_allclose(o[0, h], ref, rtol=1e-12, atol=1e-12)


def test_tiling_invariance_at_full_keep():
    grid, S = (4, 8, 8), 64
    q, k, v = _inputs(grid, 8, heads=1, seed=9)
    outs = []
    for tl in [(1, 8, 8), (4, 4, 4), (2, 4, 8), (4, 2, 8)]:
        qp, kp, vp = (O.tile_permute(a, grid, [tl], S) for a in (q, k, v))
        nt = O.num_tiles(grid, tl)
        idx = np.tile(np.arange(nt, dtype=np.int32), (1, 1, nt, 1))
        op, _ = O.sparse_attention(qp, kp, vp, idx, grid, [tl], S)
        outs.append(O.tile_unpermute(op, grid, [tl], S))
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- secondary: tile map
@pytest.mark.parametrize("grid,tiling", [((4, 8, 8), (4, 4, 4)), ((3, 5, 7), (2, 2, 2))])
def test_tile_map_equals_maxpool_of_explicit_softmax(grid, tiling):
    S = tiling[0] * tiling[1] * tiling[2]
    q, k, _ = _inputs(grid, 8, heads=1, seed=10)
    qp, kp = (O.tile_permute(a, grid, [tiling], S) for a in (q, k))
    nt = O.num_tiles(grid, tiling)
    rows = np.array([[i for i in range(nt)]], dtype=np.int32)
    M = O.tile_map_maxpool(qp, kp, rows, grid, [tiling], S)[0, 0]
    P = torch.softmax(torch.tensor(q[0, 0]) @ torch.tensor(k[0, 0]).T / math.sqrt(8), dim=-1).numpy()
    members = box_members(grid, tiling)
    N = P.shape[0]
    for i, mi in enumerate(members):
        for j, mj in enumerate(members):
            assert M[i, j] == pytest.approx(P[np.ix_(mi, mj)].max(), rel=1e-12)
        assert M[i].max() >= 1.0 / N
    assert np.all(M > 0) and np.all(M <= 1)


def test_tile_map_unused_rows_zero():
    grid, tiling, S = (3, 5, 7), (2, 2, 2), 8
    q, k, _ = _inputs(grid, 4, heads=1, seed=11)
    qp, kp = (O.tile_permute(a, grid, [tiling], S) for a in (q, k))
    rows = np.array([[2, -1, 0]], dtype=np.int32)
    M = O.tile_map_maxpool(qp, kp, rows, grid, [tiling], S)[0, 0]
    assert np.all(M[1] == 0) and np.all(M[0] > 0) and np.all(M[2] > 0)


# ---------------------------------------------------------------- whole path
def test_forward_tiny_shapes_and_full_keep_reduction():
    from veda_synth import PRESETS, make_qkv, make_mlp
    w = PRESETS["tiny"]
    q, k, v = (t.to(torch.float64).numpy() for t in make_qkv(w, seed=0))
    m = make_mlp(w, seed=1)
    mlp = tuple(t.numpy() for t in (m.w1, m.b1, m.w2, m.b2))
    grid = (w.T, w.H, w.W)
    out = O.forward(q, k, v, grid, w.tilings, w.S, mlp, mlp, 1.0)
    np.testing.assert_allclose(out["o"], _dense_sdpa(q, k, v), rtol=1e-12, atol=1e-12)
    out = O.forward(q, k, v, grid, w.tilings, w.S, mlp, mlp, w.keep)
    assert out["idx"].shape == (1, 2, 4, 2)
    assert np.all(out["idx"] >= 0)


# ---------------------------------------------------------------- distillation loss and gradients
def _distill_case(seed=0, B=1, heads=2, d=8, hidden=12, e=4, grid=(3, 4, 6), tilings=((1, 2, 4), (2, 2, 2)), S=8):
    rng = np.random.default_rng(seed)
    nts, ntmax = O.tile_layout(grid, tilings)
    dq = rng.standard_normal((B, heads, ntmax, 3 * d))
    dk = rng.standard_normal((B, heads, ntmax, 3 * d))
    mk = lambda: (rng.standard_normal((heads, hidden, 3 * d)) * 0.4, rng.standard_normal((heads, hidden)) * 0.2,
                  rng.standard_normal((heads, e, hidden)) * 0.4, rng.standard_normal((heads, e)) * 0.2)
    mlp_q, mlp_k = mk(), mk()
    R = 3
    rows = np.full((B * heads, R), -1, dtype=np.int64)
    for bh in range(B * heads):
        h = bh % heads
        rows[bh, : min(R, nts[h])] = rng.choice(nts[h], size=min(R, nts[h]), replace=False)
    rows[0, -1] = -1                                   # an unused subset slot
    tmap = np.zeros((B, heads, R, ntmax))
    for b in range(B):
        for h in range(heads):
            tmap[b, h, :, :nts[h]] = rng.uniform(0.01, 1.0, (R, nts[h]))
    return dict(desc_q=dq, desc_k=dk, grid=grid, tilings=tilings, S=S, mlp_q=mlp_q, mlp_k=mlp_k,
                tile_map=tmap, rows=rows)


def test_distill_row_loss_matches_scipy_kl():
    from scipy.special import softmax
    from scipy.stats import entropy
    rng = np.random.default_rng(4)
    for n in (1, 5, 37):
        m = rng.uniform(0.0, 1.0, n)
        m[0] = max(m[0], 1e-3)
        if n > 2:
            m[1] = 0.0                                  # a zero target entry
        s = rng.standard_normal(n) * 3
        assert O.distill_row_loss(m, s) == pytest.approx(entropy(m / m.sum(), softmax(s)), rel=1e-12, abs=1e-14)


def test_distill_gradients_match_central_differences():
    c = _distill_case()
    loss, gq, gk = O.distill_loss_grads(**c)
    assert loss > 0
    rng = np.random.default_rng(7)
    h = 1e-6
    for side, grads in (("mlp_q", gq), ("mlp_k", gk)):
        for t in range(4):
            w = c[side][t]
            for _ in range(6):
                pos = tuple(rng.integers(0, s) for s in w.shape)
                old = w[pos]
                w[pos] = old + h
                lp = O.distill_loss_grads(**c)[0]
                w[pos] = old - h
                lm = O.distill_loss_grads(**c)[0]
                w[pos] = old
                fd = (lp - lm) / (2 * h)
                assert grads[t][pos] == pytest.approx(fd, rel=1e-5, abs=1e-9), (side, t, pos)


def test_distill_gradient_of_the_k_side_output_bias_vanishes():
    """A shift of phi_k's bias adds the same amount to every score of a row, which a
    row softmax ignores, so dL/db2 of the K side is zero."""
    c = _distill_case(seed=3)
    _, gq, gk = O.distill_loss_grads(**c)
    scale = max(np.abs(g).max() for g in gk[:3])
    assert np.abs(gk[3]).max() <= 1e-12 * max(scale, 1.0)
    assert np.abs(gq[3]).max() > 1e-6                  # the Q side's is not


def test_distill_loss_and_gradients_vanish_when_the_target_is_the_prediction():
    c = _distill_case(seed=5)
    nts, _ = O.tile_layout(c["grid"], c["tilings"])
    B, heads = c["desc_q"].shape[:2]
    for b in range(B):
        for h in range(heads):
            wq = tuple(w[h] for w in c["mlp_q"])
            wk = tuple(w[h] for w in c["mlp_k"])
            s = O.tile_scores_head(c["desc_q"][b, h, :nts[h]], c["desc_k"][b, h, :nts[h]], wq, wk)
            for r in range(c["rows"].shape[1]):
                i = c["rows"][b * heads + h, r]
                if i >= 0:
                    c["tile_map"][b, h, r, :nts[h]] = 3.0 * O.row_softmax(s[i:i + 1])[0]   # any positive scale
    loss, gq, gk = O.distill_loss_grads(**c)
    assert abs(loss) < 1e-13
    for g in gq + gk:
        assert np.abs(g).max() < 1e-12


# ---------------------------------------------------------------- backward of step 5
def _bwd_case(grid=(3, 5, 7), tilings=((1, 2, 4), (2, 2, 2)), S=8, d=8, kept=3, seed=11):
    rng = np.random.default_rng(seed)
    N = grid[0] * grid[1] * grid[2]
    q, k, v, do = (rng.standard_normal((1, 2, N, d)) for _ in range(4))
    nts, ntmax = O.tile_layout(grid, tilings)
    idx = np.full((1, 2, ntmax, kept + 1), -1, dtype=np.int32)
    for h, nt in enumerate(nts):
        for i in range(nt):
            idx[0, h, i, :kept] = np.sort(rng.choice(nt, kept, replace=False))
    return grid, list(tilings), S, q, k, v, do, idx


def _bwd_grid(grid, tilings, S, q, k, v, do, idx, scale=None):
    qp, kp, vp, dop = (O.tile_permute(a, grid, tilings, S) for a in (q, k, v, do))
    return [O.tile_unpermute(g, grid, tilings, S)
            for g in O.sparse_attention_backward(qp, kp, vp, dop, idx, grid, tilings, S, scale)]


def test_attention_backward_matches_central_differences_of_the_forward():
    """dQ, dK, dV against central differences of L = <O, dO> through the
    (separately pinned) oracle forward, on every input entry."""
    grid, tilings, S, q, k, v, do, idx = _bwd_case(grid=(2, 3, 4), tilings=((1, 2, 2), (2, 1, 2)), S=4, d=3,
                                                   kept=2)
    dq, dk, dv = _bwd_grid(grid, tilings, S, q, k, v, do, idx)

    def loss(qq, kk, vv):
        qp, kp, vp = (O.tile_permute(a, grid, tilings, S) for a in (qq, kk, vv))
        op, _ = O.sparse_attention(qp, kp, vp, idx, grid, tilings, S)
        return float((O.tile_unpermute(op, grid, tilings, S) * do).sum())

    eps = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        num = np.zeros_like(grad)
        for pos in np.ndindex(grad.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][pos] += eps
            up = loss(*args)
            args[which][pos] -= 2 * eps
            num[pos] = (up - loss(*args)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


def test_attention_backward_equals_torch_autograd_of_masked_attention():
    """The same gradients from torch's fp64 autograd through a dense masked
    softmax attention (query n may see key m iff m's tile is selected by n's
    tile), built in grid coordinates without the permutation."""
    grid, tilings, S, q, k, v, do, idx = _bwd_case()
    dq, dk, dv = _bwd_grid(grid, tilings, S, q, k, v, do, idx)
    N = grid[0] * grid[1] * grid[2]
    d = q.shape[-1]
    for h in range(2):
        members = box_members(grid, tilings[h])
        tile_of = np.empty(N, dtype=np.int64)
        for j, m in enumerate(members):
            tile_of[m] = j
        allowed = np.zeros((N, N), dtype=bool)
        for n in range(N):
            sel = set(int(j) for j in idx[0, h, tile_of[n]] if j >= 0)
            allowed[n] = [tile_of[m] in sel for m in range(N)]
        tq, tk, tv = (torch.tensor(a[0, h], requires_grad=True) for a in (q, k, v))
        x = (tq @ tk.T) / math.sqrt(d)
        x = x.masked_fill(~torch.tensor(allowed), float("-inf"))
        o = torch.softmax(x, dim=-1) @ tv
        o.backward(torch.tensor(do[0, h]))
        np.testing.assert_allclose(dq[0, h], tq.grad.numpy(), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(dk[0, h], tk.grad.numpy(), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(dv[0, h], tv.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_attention_backward_at_full_keep_equals_dense_sdpa_autograd():
    grid, tilings, S = (4, 8, 8), [(1, 8, 8), (4, 4, 4)], 64
    rng = np.random.default_rng(12)
    N = 256
    q, k, v, do = (rng.standard_normal((1, 2, N, 16)) for _ in range(4))
    nts, ntmax = O.tile_layout(grid, tilings)
    idx = np.full((1, 2, ntmax, ntmax), -1, dtype=np.int32)
    for h, nt in enumerate(nts):
        idx[0, h, :nt, :nt] = np.arange(nt)
    dq, dk, dv = _bwd_grid(grid, tilings, S, q, k, v, do, idx)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).backward(torch.tensor(do))
    for g, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_backward_sum_invariants():
    """Softmax rows sum to 1 and its gradient rows to 0: summed over all keys,
    dV equals the sum of dO over the query rows that see at least one key, and
    dK sums to zero."""
    grid, tilings, S, q, k, v, do, idx = _bwd_case(seed=13)
    dq, dk, dv = _bwd_grid(grid, tilings, S, q, k, v, do, idx)
    for h in range(2):
        np.testing.assert_allclose(dv[0, h].sum(axis=0), do[0, h].sum(axis=0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dk[0, h].sum(axis=0), 0.0, atol=1e-12)
    assert np.abs(dq).max() > 1e-3 and np.abs(dk).max() > 1e-3


def test_attention_backward_scale_enters_dq_and_dk_only_through_the_logits():
    """With a custom scale c, dQ and dK carry one factor c beyond the logits:
    scaling Q by c at scale 1 must give dQ_c = c * dQ_1(cQ) and dK_c = dK_1(cQ)."""
    grid, tilings, S, q, k, v, do, idx = _bwd_case(seed=14)
    c = 0.37
    dq_c, dk_c, dv_c = _bwd_grid(grid, tilings, S, q, k, v, do, idx, scale=c)
    dq_1, dk_1, dv_1 = _bwd_grid(grid, tilings, S, c * q, k, v, do, idx, scale=1.0)
    np.testing.assert_allclose(dq_c, c * dq_1, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dk_c, dk_1, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dv_c, dv_1, rtol=1e-11, atol=1e-13)
