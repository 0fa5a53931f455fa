"""GPU parity of the grid-order path: veda_tripool_grid and
veda_tile_sparse_attn_grid, which fold the head-aware tile permutation into
the tile fetch (no tile-major copies), against the fp64 oracle and against
the tile-major path on the same inputs.

The two layouts feed the kernels identical tile contents (pad slots are zero
in both), so descriptors, selections, outputs and LSEs must agree bit for
bit; the oracle comparison uses the attention tolerances of the contract.
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
from veda_synth import PRESETS, make_mlp, make_qkv

from parity import LSE_ABS, MANY_TILINGS, MEAN_REL, SMALL, check_attn_rows, f64, keep_f32, mlp_device, mlp_numpy

pytestmark = pytest.mark.gpu

CASES = SMALL + [MANY_TILINGS]


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def _problem(V, w):
    return V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)


class GridRun:
    """The tile-major and grid-order pipelines and the oracle on one workload."""

    def __init__(self, V, w, seed=0):
        self.w = w
        self.p = _problem(V, w)
        self.grid = (w.T, w.H, w.W)
        q, k, v = make_qkv(w, seed=seed)
        m = make_mlp(w, seed=seed + 1)
        self.qd, self.kd, self.vd = (t.cuda() for t in (q, k, v))
        md = mlp_device(m)
        self.tile = V.VedaAttention(self.p, md, md, w.keep, want_lse=True, layout="tile")
        self.gridp = V.VedaAttention(self.p, md, md, w.keep, want_lse=True, layout="grid")
        self.out_t = self.tile(self.qd, self.kd, self.vd)
        self.out_g = self.gridp(self.qd, self.kd, self.vd)
        V.veda_sync_status()
        mlp = mlp_numpy(m)
        self.ora = O.forward(f64(q), f64(k), f64(v), self.grid, w.tilings, w.S, mlp, mlp, keep_f32(w.keep))


@pytest.fixture(scope="module", params=CASES, ids=[w.name for w in CASES])
def gr(V, request):
    return GridRun(V, request.param)


def test_tripool_grid(gr):
    """TripPool read from grid order: equal to the fused permute+TripPool and to the oracle."""
    d = gr.w.d
    for dev, tile, ref in ((gr.gridp.desc_q, gr.tile.desc_q, gr.ora["desc_q"]),
                           (gr.gridp.desc_k, gr.tile.desc_k, gr.ora["desc_k"])):
        assert torch.equal(dev, tile)
        g = f64(dev)
        np.testing.assert_array_equal(g[..., d:], ref[..., d:])
        np.testing.assert_allclose(g[..., :d], ref[..., :d], rtol=MEAN_REL, atol=1e-6)


def test_grid_selection_matches_tile_layout(gr):
    assert torch.equal(gr.gridp.idx, gr.tile.idx)


def test_grid_output_equals_tile_path(gr):
    """Every grid row of the grid-order output equals the unpermuted tile-major output."""
    assert torch.equal(gr.out_g, gr.out_t)


def test_grid_lse_equals_tile_path(gr):
    w = gr.w
    lt, lg = gr.tile.lse.cpu(), gr.gridp.lse.cpu()
    for h in range(w.heads):
        tab = O.slot_table(gr.grid, w.tilings[h])
        slots = np.nonzero(tab >= 0)[0]
        n = tab[slots]
        assert torch.equal(lg[:, h, torch.from_numpy(n)], lt[:, h, torch.from_numpy(slots)]), f"head {h}"


def test_grid_attention_under_oracle_idx(V, gr):
    """Grid-order attention with the oracle's selection against the oracle, every grid row."""
    p, w = gr.p, gr.w
    idx = torch.from_numpy(gr.ora["idx"]).cuda()
    o = torch.full(p.grid_shape(), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.B, p.heads, p.N), float("nan"), dtype=torch.float32, device="cuda")
    V.veda_tile_sparse_attn_grid(p, gr.qd, gr.kd, gr.vd, idx, o, lse)
    V.veda_sync_status()
    ref_o = gr.ora["o"]
    ref_lse = O.tile_unpermute(gr.ora["lse"][..., None], gr.grid, w.tilings, w.S)[..., 0]
    g, gl = f64(o), f64(lse)
    assert np.all(np.isfinite(g)) and np.all(np.isfinite(gl))   # every row and entry written
    for h in range(p.heads):
        check_attn_rows(g[:, h], ref_o[:, h], f"head {h} {w.tilings[h]}")
        assert np.abs(gl[:, h] - ref_lse[:, h]).max() <= LSE_ABS


def test_grid_attention_without_lse(V, gr):
    p = gr.p
    o = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device="cuda")
    V.veda_tile_sparse_attn_grid(p, gr.qd, gr.kd, gr.vd, gr.gridp.idx, o, None)
    V.veda_sync_status()
    assert torch.equal(o, gr.out_g)


def test_grid_tile_map_equals_tile_layout_and_oracle(V, gr):
    """veda_tile_map_maxpool_grid on the grid-order tensors gives the same map,
    bit for bit, as veda_tile_map_maxpool on the permuted copies (the tile
    boxes hold the same values), and matches the oracle; the ten-tiling case
    takes two pass-1 launches."""
    from parity import MAP_REL
    from veda_synth import make_map_rows
    w, p = gr.w, gr.p
    rows = make_map_rows(p.nt_per_head, w.B, 0.3, seed=2)
    rows[0, -1] = -1  # an unused slot
    R = rows.shape[1]
    ws = torch.empty(V.veda_tile_map_workspace(p, R) // 4 + 64, dtype=torch.float32, device="cuda")
    m_tile = torch.full((p.B, p.heads, R, p.nt_max), float("nan"), dtype=torch.float32, device="cuda")
    m_grid = torch.full_like(m_tile, float("nan"))
    V.veda_tile_map_maxpool(p, gr.tile.qp, gr.tile.kp, rows.cuda(), m_tile, ws)
    V.veda_tile_map_maxpool_grid(p, gr.qd, gr.kd, rows.cuda(), m_grid, ws)
    V.veda_sync_status()
    assert torch.equal(m_grid, m_tile)
    ref = O.tile_map_maxpool(gr.ora["qp"], gr.ora["kp"], rows.numpy(), gr.grid, w.tilings, w.S)
    g = f64(m_grid)
    big = ref >= 1e-8
    assert np.all(np.abs(g[big] - ref[big]) <= MAP_REL * ref[big])
    assert np.all(np.abs(g[~big] - ref[~big]) <= 1e-11)


def test_grid_wan14b_full_size_sampled(V):
    """The benchmarked 14B shape in the grid layout, the launch the bench times: sampled Q tiles of
    sampled heads against the oracle, and the whole output equal to the tile-major path."""
    w = PRESETS["wan14b"]
    p = _problem(V, w)
    q, k, v = make_qkv(w, seed=0)
    m = make_mlp(w, seed=1)
    md = mlp_device(m)
    att_g = V.VedaAttention(p, md, md, w.keep, want_lse=True, layout="grid")
    out_g = att_g(q.cuda(), k.cuda(), v.cuda())
    V.veda_sync_status()
    grid = (w.T, w.H, w.W)
    ks, _ = p.keep_count(w.keep)
    mlp_all = mlp_numpy(m)
    gi = att_g.idx.cpu().numpy()
    rng = np.random.default_rng(1)
    checked = 0
    for h in (2, 21, 38):
        tl = [w.tilings[h]]
        mh = tuple(a[h:h + 1] for a in mlp_all)
        qp, kp, vp = (O.tile_permute(f64(t[:, h:h + 1]), grid, tl, w.S) for t in (q, k, v))
        dq, dk = O.tripool(qp, grid, tl, w.S), O.tripool(kp, grid, tl, w.S)
        idx = O.score_topk(dq, dk, grid, tl, w.S, mh, mh, keep_f32(w.keep))[0]
        tab = O.slot_table(grid, tl[0])
        nt = p.nt_per_head[h]
        k_h = ks[h]   # the one-head oracle pads its rows to this head's k only
        for i in rng.choice(nt, 5, replace=False):
            sel = idx[0, 0, i, :k_h]
            if not (np.array_equal(gi[0, h, i, :k_h], sel) and np.all(gi[0, h, i, k_h:] == -1)):
                continue
            o_ref, lse_ref = O.attention_tile(qp[0, 0], kp[0, 0], vp[0, 0], tab, int(i), sel, w.S,
                                              1 / np.sqrt(w.d))
            slots = np.nonzero(tab[i * w.S:(i + 1) * w.S] >= 0)[0]
            n = torch.from_numpy(tab[i * w.S:(i + 1) * w.S][slots])
            check_attn_rows(f64(out_g[0, h, n.cuda()]), o_ref[slots], f"h{h} tile {i}")
            assert np.abs(f64(att_g.lse[0, h, n.cuda()]) - lse_ref[slots]).max() <= LSE_ABS
            checked += 1
    assert checked >= 10
    idx_g = att_g.idx.clone()
    del att_g
    att_t = V.VedaAttention(p, md, md, w.keep, layout="tile")
    out_t = att_t(q.cuda(), k.cuda(), v.cuda())
    V.veda_sync_status()
    assert torch.equal(idx_g, att_t.idx)
    assert torch.equal(out_g, out_t)


def test_extreme_score_in_the_last_key_slot(V):
    """One key, in the last slot of a tile, scores about 300 (log2 units) above every
    other key of a query row: the exponent reference must take it into account, or
    the exponentials of that row overflow."""
    from parity import wl
    w = wl("extreme", (4, 16, 16), 1, 1, 128, 128, [(2, 8, 8)], 1.0, 256, 64)
    p = _problem(V, w)
    q, k, v = make_qkv(w, seed=7)
    grid = (w.T, w.H, w.W)
    pt, ph, pw = w.tilings[0]
    n_last = ((pt - 1) * w.H + (ph - 1)) * w.W + (pw - 1)     # slot S-1 of tile 0
    qrow = q[0, 0, 0].float()
    k[0, 0, n_last] = (qrow * (2400.0 / float(qrow @ qrow))).to(torch.bfloat16)
    nt = p.nt_per_head[0]
    idx = torch.arange(nt, dtype=torch.int32).expand(w.B, w.heads, p.nt_max, nt).contiguous()
    o = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((p.B, p.heads, p.N), dtype=torch.float32, device="cuda")
    V.veda_tile_sparse_attn_grid(p, q.cuda(), k.cuda(), v.cuda(), idx.cuda(), o, lse)
    V.veda_sync_status()
    qp, kp, vp = (O.tile_permute(f64(t), grid, w.tilings, w.S) for t in (q, k, v))
    ref_op, ref_lse = O.sparse_attention(qp, kp, vp, idx.numpy(), grid, w.tilings, w.S)
    ref_o = O.tile_unpermute(ref_op, grid, w.tilings, w.S)
    ref_l = O.tile_unpermute(ref_lse[..., None], grid, w.tilings, w.S)[..., 0]
    g, gl = f64(o), f64(lse)
    assert np.all(np.isfinite(g)) and np.all(np.isfinite(gl))
    assert ref_l[0, 0, 0] > 150.0                               # the extreme row really is extreme
    check_attn_rows(g[0, 0], ref_o[0, 0])
    assert np.abs(gl[0, 0] - ref_l[0, 0]).max() <= LSE_ABS


def test_host_buffer_pipeline_equals_the_device_path(V):
    """VedaAttentionHost (head chunks pipelined over three streams, pinned host
    buffers) gives exactly the device-resident layer's output, B = 2 included."""
    w = SMALL[2]                                      # odd128: B = 2, 4 heads
    p = _problem(V, w)
    q, k, v = make_qkv(w, seed=3)
    md = mlp_device(make_mlp(w, seed=1))
    ref = V.VedaAttention(p, md, md, w.keep, layout="grid")(q.cuda(), k.cuda(), v.cuda())
    host = V.VedaAttentionHost(p, md, md, w.keep, chunk_heads=3, slots=2)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.full(p.grid_shape(), float("nan"), dtype=torch.bfloat16).pin_memory()
    for _ in range(2):                                # slot reuse across calls
        host(qh, kh, vh, oh)
        torch.cuda.synchronize()
        V.veda_sync_status()
        assert torch.equal(oh, ref.cpu())
