"""GPU parity of the estimator's distillation step (veda_distill_loss_grad)
against the fp64 oracle: the row-wise KL loss and the gradients of both
estimators, on seeded synthetic descriptors, weights, tile maps and subset
rows (several heads and tilings, B = 2, unused subset slots, ragged tiles).

Tolerances: the forward estimator runs at fp32 accuracy on the tensor cores
and the backward in fp32, so the loss is compared to 1e-5 relative and each
gradient tensor to 1e-4 relative L2 (max-abs 1e-4 of the largest entry of
that side's gradients, which also covers the K side's output-bias gradient,
zero in exact arithmetic).
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O
from veda_synth import make_map_rows, make_mlp

from parity import SMALL, f64, mlp_device, mlp_numpy

pytestmark = pytest.mark.gpu

LOSS_REL = 1e-5
GRAD_REL_L2 = 1e-4
GRAD_MAX_ABS = 1e-4


@pytest.fixture(scope="module")
def V():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import tile_sparse_attention_head_b200 as V
    return V


def _inputs(w, seed):
    g = torch.Generator().manual_seed(seed)
    nts, ntmax = O.tile_layout((w.T, w.H, w.W), w.tilings)
    desc_q = torch.randn((w.B, w.heads, ntmax, 3 * w.d), generator=g)
    desc_k = torch.randn((w.B, w.heads, ntmax, 3 * w.d), generator=g)
    rows = make_map_rows(nts, w.B, 0.3, seed=seed)
    rows[0, -1] = -1
    R = rows.shape[1]
    tmap = torch.rand((w.B, w.heads, R, ntmax), generator=g) + 0.01
    for h in range(w.heads):
        tmap[:, h, :, nts[h]:] = 0.0
    return desc_q, desc_k, rows, tmap


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_distill_loss_and_gradients(V, w):
    p = V.Problem(w.B, w.heads, w.d, w.S, (w.T, w.H, w.W), w.tilings)
    desc_q, desc_k, rows, tmap = _inputs(w, seed=11)
    mq, mk = make_mlp(w, seed=1), make_mlp(w, seed=2)
    dq, dk = mlp_device(mq), mlp_device(mk)
    grads = [tuple(torch.full_like(t, float("nan")) for t in m) for m in (dq, dk)]
    loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(V.veda_distill_workspace(p, w.hidden, w.e, rows.shape[1]) // 4 + 64, dtype=torch.float32,
                     device="cuda")
    V.veda_distill_loss_grad(p, desc_q.cuda(), desc_k.cuda(), V.make_mlp(*dq), V.make_mlp(*dk), tmap.cuda(),
                             rows.cuda(), loss, V.make_mlp_grad(*grads[0]), V.make_mlp_grad(*grads[1]), ws)
    V.veda_sync_status()
    ref_loss, ref_gq, ref_gk = O.distill_loss_grads(f64(desc_q), f64(desc_k), (w.T, w.H, w.W), w.tilings, w.S,
                                                    mlp_numpy(mq), mlp_numpy(mk), f64(tmap), rows.numpy())
    assert float(loss) == pytest.approx(ref_loss, rel=LOSS_REL, abs=1e-7)
    for side, (got, ref) in enumerate(((grads[0], ref_gq), (grads[1], ref_gk))):
        scale = max(float(np.abs(r).max()) for r in ref)
        for name, g, r in zip(("w1", "b1", "w2", "b2"), got, ref):
            g = f64(g)
            assert np.all(np.isfinite(g)), (side, name)
            assert np.abs(g - r).max() <= GRAD_MAX_ABS * scale, (side, name, np.abs(g - r).max(), scale)
            if np.linalg.norm(r) > 1e-3 * scale * np.sqrt(r.size):
                rel = np.linalg.norm(g - r) / np.linalg.norm(r)
                assert rel <= GRAD_REL_L2, (side, name, rel)
