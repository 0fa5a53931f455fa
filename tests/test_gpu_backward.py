"""GPU parity of the attention backward (veda_tile_sparse_attn_backward_grid)
against the fp64 oracle's chain rule, on the oracle's own tile selection.

The GPU forward runs with the oracle's idx to produce o and lse; the backward
takes them, as a training step would.  The oracle recomputes the gradients
from q, k, v, dO and the same idx in fp64.

Tolerance (bf16 inputs, fp32 accumulation, bf16 outputs): P and dS are
rounded to bf16 as product operands and the outputs are rounded to bf16, each
a relative perturbation of at most 2^-9 per element; the rounding errors are
independent, so the norm-wise error of each gradient stays a small multiple
of 2^-9.  dQ and dK are sums of dX = P (dP - D) terms whose rows sum to zero,
so they cancel more than dV does and get twice the margin:
    dV: relative L2 <= 1e-2;  dQ, dK: relative L2 <= 2e-2;
    every gradient: max-abs error <= 2e-2 * max |oracle| of its head.
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
from veda_synth import PRESETS, make_grad_out, make_mlp, make_qkv

from parity import MANY_TILINGS, SMALL, f64, keep_f32, mlp_numpy, wl

pytestmark = pytest.mark.gpu

REL_L2 = {"dq": 2e-2, "dk": 2e-2, "dv": 1e-2}
MAX_ABS_FRAC = 2e-2


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def _problem(V, w):
    return V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)


def gpu_backward(V, p, qd, kd, vd, dod, idx, scale=0.0):
    """GPU forward (o, lse) then backward with the given selection."""
    o = torch.empty(p.grid_shape(), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((p.B, p.heads, p.N), dtype=torch.float32, device="cuda")
    V.veda_tile_sparse_attn_grid(p, qd, kd, vd, idx, o, lse, scale)
    grads = [torch.full(p.grid_shape(), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    ws = torch.empty(V.veda_attn_backward_workspace(p, int(idx.shape[-1])), dtype=torch.uint8, device="cuda")
    V.veda_tile_sparse_attn_backward_grid(p, qd, kd, vd, o, lse, dod, idx, *grads, ws, scale)
    V.veda_sync_status()
    return grads


def check_grad(name, g, ref, what):
    assert np.all(np.isfinite(g)), f"{what} {name}: non-finite entries"
    rel = float(np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.abs(g - ref).max())
    lim = MAX_ABS_FRAC * float(np.abs(ref).max())
    assert rel <= REL_L2[name], f"{what} {name}: relative L2 {rel:.3e} > {REL_L2[name]}"
    assert mx <= lim, f"{what} {name}: max abs error {mx:.3e} > {lim:.3e}"
    return rel, mx


def run_case(V, w, seed=0, scale=None):
    p = _problem(V, w)
    grid = (w.T, w.H, w.W)
    q, k, v = make_qkv(w, seed=seed)
    do = make_grad_out(w, seed=seed + 4)
    mlp = mlp_numpy(make_mlp(w, seed=seed + 1))
    ora = O.forward(f64(q), f64(k), f64(v), grid, w.tilings, w.S, mlp, mlp, keep_f32(w.keep))
    idx = ora["idx"]
    qp, kp, vp, dop = (O.tile_permute(f64(t), grid, w.tilings, w.S) for t in (q, k, v, do))
    refs = [O.tile_unpermute(g, grid, w.tilings, w.S)
            for g in O.sparse_attention_backward(qp, kp, vp, dop, idx, grid, w.tilings, w.S, scale)]
    grads = gpu_backward(V, p, q.cuda(), k.cuda(), v.cuda(), do.cuda(), torch.from_numpy(idx).cuda(),
                         0.0 if scale is None else scale)
    return p, grads, refs


@pytest.mark.parametrize("w", SMALL + [MANY_TILINGS], ids=[w.name for w in SMALL + [MANY_TILINGS]])
def test_backward_matches_oracle(V, w):
    p, grads, refs = run_case(V, w)
    for b in range(w.B):
        for h in range(w.heads):
            for name, g, ref in zip(("dq", "dk", "dv"), grads, refs):
                check_grad(name, f64(g[b, h]), ref[b, h], f"{w.name} b{b} h{h}")


def test_backward_custom_scale(V):
    w = SMALL[1]
    p, grads, refs = run_case(V, w, seed=5, scale=0.2)
    for name, g, ref in zip(("dq", "dk", "dv"), grads, refs):
        for h in range(w.heads):
            check_grad(name, f64(g[0, h]), ref[0, h], f"scale 0.2 h{h}")


def test_backward_unselected_keys_get_zero_and_is_deterministic(V):
    """Every Q tile selects only tile 0: keys outside tile 0 get dK = dV = 0;
    a second run gives identical bits."""
    w = wl("one_tile", (4, 16, 16), 1, 2, 128, 128, [(2, 8, 8), (4, 4, 8)], 1.0, 256, 64)
    p = _problem(V, w)
    q, k, v = make_qkv(w, seed=9)
    do = make_grad_out(w, seed=10)
    idx = torch.full((1, 2, p.nt_max, 3), -1, dtype=torch.int32)
    idx[..., 0] = 0
    args = [t.cuda() for t in (q, k, v, do)] + [idx.cuda()]
    g1 = gpu_backward(V, p, *args)
    g2 = gpu_backward(V, p, *args)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    grid = (w.T, w.H, w.W)
    for h in range(2):
        tab = O.slot_table(grid, w.tilings[h])
        in0 = np.zeros(p.N, dtype=bool)
        in0[tab[:w.S][tab[:w.S] >= 0]] = True
        assert torch.count_nonzero(g1[1][0, h][torch.from_numpy(~in0).cuda()]) == 0
        assert torch.count_nonzero(g1[2][0, h][torch.from_numpy(~in0).cuda()]) == 0
        assert torch.count_nonzero(g1[2][0, h][torch.from_numpy(in0).cuda()]) > 0
    qp, kp, vp, dop = (O.tile_permute(f64(t), grid, w.tilings, w.S) for t in (q, k, v, do))
    refs = [O.tile_unpermute(g, grid, w.tilings, w.S)
            for g in O.sparse_attention_backward(qp, kp, vp, dop, idx.numpy(), grid, w.tilings, w.S)]
    for name, g, ref in zip(("dq", "dk", "dv"), g1, refs):
        for h in range(2):
            check_grad(name, f64(g[0, h]), ref[0, h], f"one tile h{h}")


def _oracle_dkdv_tile(qp, kp, vp, dop, tab, idx_rows, j, S, scale):
    """dK, dV rows (slot order) of K tile j of one head: the sum over every Q
    tile whose selection holds j of its contribution to j's keys."""
    d = qp.shape[1]
    dk, dv = np.zeros((S, d)), np.zeros((S, d))
    for i, row in enumerate(idx_rows):
        sel = row[row >= 0]
        if j not in sel:
            continue
        _, kr, dki, dvi = O.attention_tile_backward(qp, kp, vp, dop, tab, i, sel, S, scale)
        m = (kr // S) == j
        dk[kr[m] % S] += dki[m]
        dv[kr[m] % S] += dvi[m]
    return dk, dv


def test_backward_wan14b_full_size_sampled(V):
    """The benchmarked 14B shape (40 heads, grid order, the launch the bench
    times): dQ of sampled Q tiles and dK, dV of sampled K tiles (the most
    selected one and random ones) of two heads against the oracle, with the
    oracle's selection for those heads."""
    w = PRESETS["wan14b"]
    p = _problem(V, w)
    grid = (w.T, w.H, w.W)
    q, k, v = make_qkv(w, seed=0)
    do = make_grad_out(w, seed=4)
    m = make_mlp(w, seed=1)
    md = tuple(t.cuda() for t in (m.w1, m.b1, m.w2, m.b2))
    att = V.VedaAttention(p, md, md, w.keep, layout="grid")
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    att(qd, kd, vd)
    V.veda_sync_status()
    idx = att.idx.clone()
    k_max = idx.shape[-1]
    mlp_all = mlp_numpy(m)
    heads = (5, 30)
    ora = {}
    for h in heads:
        tl = [w.tilings[h]]
        mh = tuple(a[h:h + 1] for a in mlp_all)
        qp, kp, vp, dop = (O.tile_permute(f64(t[:, h:h + 1]), grid, tl, w.S) for t in (q, k, v, do))
        dq_, dk_ = O.tripool(qp, grid, tl, w.S), O.tripool(kp, grid, tl, w.S)
        oi = O.score_topk(dq_, dk_, grid, tl, w.S, mh, mh, keep_f32(w.keep))[0][0, 0]
        nt = p.nt_per_head[h]
        row = np.full((p.nt_max, k_max), -1, dtype=np.int32)
        row[:nt, :oi.shape[1]] = oi[:nt]
        idx[0, h] = torch.from_numpy(row).cuda()
        ora[h] = (qp[0, 0], kp[0, 0], vp[0, 0], dop[0, 0], row[:nt])
    grads = gpu_backward(V, p, qd, kd, vd, dod, idx)
    rng = np.random.default_rng(3)
    scale = 1 / np.sqrt(w.d)
    checked = 0
    for h in heads:
        qp, kp, vp, dop, rows = ora[h]
        tab = O.slot_table(grid, w.tilings[h])
        nt = rows.shape[0]
        for i in rng.choice(nt, 3, replace=False):
            dq_ref, _, _, _ = O.attention_tile_backward(qp, kp, vp, dop, tab, int(i), rows[i][rows[i] >= 0], w.S, scale)
            slots = np.nonzero(tab[i * w.S:(i + 1) * w.S] >= 0)[0]
            n = torch.from_numpy(tab[i * w.S:(i + 1) * w.S][slots]).cuda()
            check_grad("dq", f64(grads[0][0, h, n]), dq_ref[slots], f"h{h} Q tile {i}")
            checked += 1
        counts = np.bincount(rows[rows >= 0], minlength=nt)
        for j in [int(np.argmax(counts))] + [int(x) for x in rng.choice(nt, 2, replace=False)]:
            dk_ref, dv_ref = _oracle_dkdv_tile(qp, kp, vp, dop, tab, rows, j, w.S, scale)
            slots = np.nonzero(tab[j * w.S:(j + 1) * w.S] >= 0)[0]
            n = torch.from_numpy(tab[j * w.S:(j + 1) * w.S][slots]).cuda()
            if counts[j] == 0:
                assert torch.count_nonzero(grads[1][0, h, n]) == 0 and torch.count_nonzero(grads[2][0, h, n]) == 0
                continue
            check_grad("dk", f64(grads[1][0, h, n]), dk_ref[slots], f"h{h} K tile {j} ({counts[j]} selections)")
            check_grad("dv", f64(grads[2][0, h, n]), dv_ref[slots], f"h{h} K tile {j}")
            checked += 1
    assert checked >= 10
    for g in grads:
        assert bool(torch.isfinite(g.float()).all())


def test_autograd_op_equals_the_c_abi_calls(V):
    """tile_sparse_attention (torch autograd) gives exactly the output and the
    gradients of the direct calls; VedaAttention.differentiable selects first."""
    w = SMALL[2]                                       # odd128: B = 2, 4 heads, ragged tiles
    p = _problem(V, w)
    q, k, v = (t.cuda() for t in make_qkv(w, seed=6))
    do = make_grad_out(w, seed=7).cuda()
    md = tuple(t.cuda() for t in (lambda m: (m.w1, m.b1, m.w2, m.b2))(make_mlp(w, seed=1)))
    att = V.VedaAttention(p, md, md, w.keep, layout="grid")
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = att.differentiable(qa, ka, va)
    o.backward(do)
    V.veda_sync_status()
    ref = gpu_backward(V, p, q, k, v, do, att.idx)
    o_ref = att(q, k, v)
    assert torch.equal(o.detach(), o_ref)
    for t, r in zip((qa, ka, va), ref):
        assert torch.equal(t.grad, r)


def test_backward_invalid_idx_entries_end_the_list(V):
    """An entry outside [0, NT_h) ends a selection list like -1 does, for the
    dQ side (the row's prefix) and the dK/dV side (the inverse lists) alike."""
    w = SMALL[2]
    p = _problem(V, w)
    q, k, v = (t.cuda() for t in make_qkv(w, seed=3))
    do = make_grad_out(w, seed=8).cuda()
    idx = torch.full((p.B, p.heads, p.nt_max, 4), -1, dtype=torch.int32)
    idx[..., 0] = 0
    idx[..., 1] = 1
    idx2 = idx.clone()
    idx2[..., 2] = 10_000           # out of range: ends the list
    idx2[..., 3] = 2
    g1 = gpu_backward(V, p, q, k, v, do, idx.cuda())
    g2 = gpu_backward(V, p, q, k, v, do, idx2.cuda())
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
