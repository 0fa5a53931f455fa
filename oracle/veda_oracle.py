"""Plain fp64 CPU oracle for Veda's head-aware tile-sparse attention path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run this module; the product
path (the C-ABI library and its Python binding) never does, and this module
imports nothing from it.  It is slow on purpose: every step is written out in
the order the Veda pages describe, with no blocking, fusion or reordering, so
a reader can check it against the pages by eye.

Source: "Veda: Scalable Video Diffusion via Distilled Sparse Attention"
(technical summary pages, gist.science, zh/fr/es), sections
  2.1 "Distilled tile scoring" (max-pooled full-attention target, TripPool
      mean||max||min descriptor, head-specific MLP projections, row-wise
      distribution over tiles),
  2.2 "Head-aware tiling" (per layer and head a factorisation
      pi = (p_t, p_h, p_w) of the hardware tile size),
  2.3 "Hardware-efficient implementation" (tile-skipping sparse attention over
      only the selected K/V tiles; two-pass heat-map kernel over a random
      subset of Q tiles),
and the aikraft.ru news page ("95% sparsity", "tile skipping").

The pages describe the method in prose only (no formulas, dimensions or code);
where they are silent this module takes the plainest reading, stated at each
function:
  * grid flattening n = (t*H + y)*W + x;
  * tiles and tokens inside a tile are ordered row-major over (t, y, x);
  * a dimension that its factor does not divide is padded up to a multiple of
    it; pad slots hold no token, are excluded from pooling and masked as keys;
  * estimator: phi = W2 relu(W1 desc + b1) + b2 per head; tile score
    s[i, j] = <phi_q(i), phi_k(j)> / sqrt(e);
  * keep count k = max(1, min(NT, floor(r*NT + 1/2))); the k largest scores
    are kept, ties going to the smaller tile index, returned ascending;
  * attention scale 1/sqrt(d); the tile map holds post-softmax probabilities
    of full attention (softmax over every valid key), max-pooled over each
    (Q tile, K tile) block.
Parity of the estimator on *trained* weights is unpinned (the pages print no
values); every function here is pinned by the checks in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

Tiling = Tuple[int, int, int]
Grid = Tuple[int, int, int]


# --------------------------------------------------------------------------
# Step 1 -- head-aware 3D tiling (section 2.2, pi_{l,h} = (p_t, p_h, p_w)).
# --------------------------------------------------------------------------
def tile_counts(grid: Grid, tiling: Tiling) -> Tuple[int, int, int]:
    """Tiles along t, y, x after padding each dimension up to its factor."""
    T, H, W = grid
    pt, ph, pw = tiling
    return -(-T // pt), -(-H // ph), -(-W // pw)


def num_tiles(grid: Grid, tiling: Tiling) -> int:
    nT, nH, nW = tile_counts(grid, tiling)
    return nT * nH * nW


def tile_layout(grid: Grid, tilings: Sequence[Tiling]) -> Tuple[List[int], int]:
    """Tiles per head and the largest of them (the per-head row stride in tiles)."""
    nts = [num_tiles(grid, tl) for tl in tilings]
    return nts, max(nts)


def slot_table(grid: Grid, tiling: Tiling) -> np.ndarray:
    """For one head: table[j*S + l] = grid index n of the token at slot l of
    tile j, or -1 for a pad slot.  S = pt*ph*pw.

    Token (t, y, x) goes to tile j = ((t//pt)*nH + y//ph)*nW + x//pw at local
    slot l = ((t%pt)*ph + y%ph)*pw + x%pw.
    """
    T, H, W = grid
    pt, ph, pw = tiling
    S = pt * ph * pw
    nT, nH, nW = tile_counts(grid, tiling)
    table = np.full(nT * nH * nW * S, -1, dtype=np.int64)
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    n = (t * H + y) * W + x
    j = ((t // pt) * nH + y // ph) * nW + x // pw
    l = ((t % pt) * ph + y % ph) * pw + x % pw
    table[(j * S + l).ravel()] = n.ravel()
    return table


def tile_permute(x: np.ndarray, grid: Grid, tilings: Sequence[Tiling], S: int) -> np.ndarray:
    """Grid order [B, heads, N, d] -> per-head tile-major [B, heads, NT_max*S, d].

    Row j*S + l of head h holds the token at slot l of tile j under that
    head's tiling; pad slots and tiles j >= NT_h are zero.
    """
    B, heads, N, d = x.shape
    _, ntmax = tile_layout(grid, tilings)
    out = np.zeros((B, heads, ntmax * S, d), dtype=np.float64)
    for h in range(heads):
        tab = slot_table(grid, tilings[h])
        assert tab.size % S == 0 and tab.size // S == num_tiles(grid, tilings[h])
        valid = tab >= 0
        rows = np.nonzero(valid)[0]
        out[:, h, rows, :] = x[:, h, tab[valid], :]
    return out


def tile_unpermute(xp: np.ndarray, grid: Grid, tilings: Sequence[Tiling], S: int) -> np.ndarray:
    """Inverse of ``tile_permute`` on valid rows: [B, heads, NT_max*S, d] -> [B, heads, N, d]."""
    B, heads, _, d = xp.shape
    T, H, W = grid
    out = np.zeros((B, heads, T * H * W, d), dtype=np.float64)
    for h in range(heads):
        tab = slot_table(grid, tilings[h])
        valid = tab >= 0
        out[:, h, tab[valid], :] = xp[:, h, np.nonzero(valid)[0], :]
    return out


# --------------------------------------------------------------------------
# Step 2 -- TripPool descriptor (section 2.1: concatenated mean, max, min).
# --------------------------------------------------------------------------
def tripool_head(xp_h: np.ndarray, table: np.ndarray, S: int) -> np.ndarray:
    """One head: desc[j] = [mean_c || max_c || min_c] over the tokens of tile j.

    ``xp_h`` is [NT_max*S, d] tile-major; only slots that hold a token count.
    """
    nt = table.size // S
    d = xp_h.shape[1]
    desc = np.zeros((nt, 3 * d), dtype=np.float64)
    for j in range(nt):
        slots = np.nonzero(table[j * S:(j + 1) * S] >= 0)[0]
        rows = xp_h[j * S + slots]                      # tokens of tile j
        desc[j, :d] = rows.sum(axis=0) / len(slots)
        desc[j, d:2 * d] = rows.max(axis=0)
        desc[j, 2 * d:] = rows.min(axis=0)
    return desc


def tripool(xp: np.ndarray, grid: Grid, tilings: Sequence[Tiling], S: int) -> np.ndarray:
    """[B, heads, NT_max*S, d] -> [B, heads, NT_max, 3d]; rows j >= NT_h are zero."""
    B, heads, _, d = xp.shape
    _, ntmax = tile_layout(grid, tilings)
    out = np.zeros((B, heads, ntmax, 3 * d), dtype=np.float64)
    for h in range(heads):
        tab = slot_table(grid, tilings[h])
        nt = tab.size // S
        for b in range(B):
            out[b, h, :nt] = tripool_head(xp[b, h], tab, S)
    return out


# --------------------------------------------------------------------------
# Step 3 -- head-specific MLP estimator and tile scores (section 2.1).
# --------------------------------------------------------------------------
def estimator_head(desc: np.ndarray, w1, b1, w2, b2) -> np.ndarray:
    """phi = W2 relu(W1 desc + b1) + b2 applied to every row of desc [NT, 3d]."""
    hidden = desc @ np.asarray(w1, np.float64).T + np.asarray(b1, np.float64)
    hidden = np.maximum(hidden, 0.0)
    return hidden @ np.asarray(w2, np.float64).T + np.asarray(b2, np.float64)


def tile_scores_head(desc_q: np.ndarray, desc_k: np.ndarray, wq, wk) -> np.ndarray:
    """s[i, j] = <phi_q(desc_q[i]), phi_k(desc_k[j])> / sqrt(e), shape [NT, NT]."""
    phi_q = estimator_head(desc_q, *wq)
    phi_k = estimator_head(desc_k, *wk)
    e = phi_q.shape[1]
    return (phi_q @ phi_k.T) / math.sqrt(e)


def row_softmax(s: np.ndarray) -> np.ndarray:
    """Row-wise softmax (the pages' per-row distribution over K tiles)."""
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return p / p.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------
# Step 4 -- top-k tile selection ("keep ~5-10% of tiles", 95% sparsity).
# --------------------------------------------------------------------------
def keep_count(nt: int, keep_ratio: float) -> int:
    """k = max(1, min(NT, floor(r*NT + 1/2)))."""
    return max(1, min(nt, int(math.floor(keep_ratio * nt + 0.5))))


def select_topk_row(s_row: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries, ties to the smaller index, ascending."""
    nt = s_row.shape[0]
    order = np.lexsort((np.arange(nt), -s_row))        # by score desc, then index asc
    return np.sort(order[:k])


def score_topk(desc_q, desc_k, grid, tilings, S, mlp_q, mlp_k, keep_ratio, want_scores=False):
    """Estimator + row softmax + top-k for all heads.

    ``mlp_q`` / ``mlp_k`` are (W1 [heads,hid,3d], b1, W2 [heads,e,hid], b2).
    Returns idx int32 [B, heads, NT_max, k_max] (ascending, -1 padded; rows
    i >= NT_h all -1), probs fp64 [B, heads, NT_max, NT_max] (zero outside the
    valid block) and, if asked, the logits (-inf outside the valid block).
    """
    B, heads = desc_q.shape[:2]
    nts, ntmax = tile_layout(grid, tilings)
    ks = [keep_count(nt, keep_ratio) for nt in nts]
    kmax = max(ks)
    idx = np.full((B, heads, ntmax, kmax), -1, dtype=np.int32)
    probs = np.zeros((B, heads, ntmax, ntmax), dtype=np.float64)
    scores = np.full((B, heads, ntmax, ntmax), -np.inf, dtype=np.float64)
    for b in range(B):
        for h in range(heads):
            nt = nts[h]
            wq = tuple(np.asarray(m[h], np.float64) for m in mlp_q)
            wk = tuple(np.asarray(m[h], np.float64) for m in mlp_k)
            s = tile_scores_head(desc_q[b, h, :nt], desc_k[b, h, :nt], wq, wk)
            scores[b, h, :nt, :nt] = s
            probs[b, h, :nt, :nt] = row_softmax(s)
            for i in range(nt):
                idx[b, h, i, :ks[h]] = select_topk_row(s[i], ks[h])
    if want_scores:
        return idx, probs, scores
    return idx, probs


# --------------------------------------------------------------------------
# Step 5 -- tile-skipping attention (section 2.3) and unpermute.
# --------------------------------------------------------------------------
def attention_tile(qp_h, kp_h, vp_h, table, i, sel, S, scale):
    """Output rows of Q tile i of one head, attending only to the K/V tiles in ``sel``.

    For each query slot of tile i: o = softmax(scale * q K^T) V over every
    valid key slot of the selected tiles; lse = log sum exp(scale * q K^T).
    Pad query slots are returned as zero rows with lse 0.
    """
    sel = [int(j) for j in sel if j >= 0]
    key_rows = np.concatenate([j * S + np.nonzero(table[j * S:(j + 1) * S] >= 0)[0] for j in sel])
    K = kp_h[key_rows]
    V = vp_h[key_rows]
    d = qp_h.shape[1]
    o = np.zeros((S, d), dtype=np.float64)
    lse = np.zeros(S, dtype=np.float64)
    qslots = np.nonzero(table[i * S:(i + 1) * S] >= 0)[0]
    Q = qp_h[i * S + qslots]
    logits = scale * (Q @ K.T)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    denom = p.sum(axis=1, keepdims=True)
    o[qslots] = (p / denom) @ V
    lse[qslots] = (m + np.log(denom))[:, 0]
    return o, lse


def sparse_attention(qp, kp, vp, idx, grid, tilings, S, scale=None):
    """All heads and Q tiles: Op [B, heads, NT_max*S, d] (pad rows zero) and lse [B, heads, NT_max*S]."""
    B, heads, rows, d = qp.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    op = np.zeros_like(qp, dtype=np.float64)
    lse = np.zeros((B, heads, rows), dtype=np.float64)
    for h in range(heads):
        tab = slot_table(grid, tilings[h])
        nt = tab.size // S
        for b in range(B):
            for i in range(nt):
                o_i, l_i = attention_tile(qp[b, h], kp[b, h], vp[b, h], tab, i, idx[b, h, i], S, scale)
                op[b, h, i * S:(i + 1) * S] = o_i
                lse[b, h, i * S:(i + 1) * S] = l_i
    return op, lse


# --------------------------------------------------------------------------
# Backward of step 5 -- gradients of the tile-skipping attention with respect
# to Q, K and V, over the selected tiles only.  The pages train only the
# estimator (section 2.1, "Optimization"); this is the chain rule through the
# forward defined above, for callers that fine-tune the backbone with the
# sparse pattern fixed.
# --------------------------------------------------------------------------
def attention_tile_backward(qp_h, kp_h, vp_h, dop_h, table, i, sel, S, scale):
    """Gradient contributions of Q tile i of one head.

    With X = scale * Q K^T over every valid key slot of the selected tiles
    (the rows of attention_tile), P = softmax over each row of X and O = P V,
    an upstream gradient dO gives
        dV = P^T dO,   dP = dO V^T,   dX = P * (dP - rowsum(P * dP)),
        dQ = scale * dX K,   dK = scale * dX^T Q.
    Returns (dq [S, d] with pad query slots zero, key_rows, dk, dv), where
    key_rows are the permuted rows of the keys used and dk, dv the
    contributions to those rows.
    """
    sel = [int(j) for j in sel if j >= 0]
    key_rows = np.concatenate([j * S + np.nonzero(table[j * S:(j + 1) * S] >= 0)[0] for j in sel])
    K = kp_h[key_rows]
    V = vp_h[key_rows]
    d = qp_h.shape[1]
    qslots = np.nonzero(table[i * S:(i + 1) * S] >= 0)[0]
    Q = qp_h[i * S + qslots]
    dO = dop_h[i * S + qslots]
    x = scale * (Q @ K.T)
    p = np.exp(x - x.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dv = p.T @ dO
    dp = dO @ V.T
    dx = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    dq = np.zeros((S, d), dtype=np.float64)
    dq[qslots] = scale * (dx @ K)
    dk = scale * (dx.T @ Q)
    return dq, key_rows, dk, dv


def sparse_attention_backward(qp, kp, vp, dop, idx, grid, tilings, S, scale=None):
    """dQp, dKp, dVp [B, heads, NT_max*S, d] (tile-major, pad rows zero) of the
    tile-skipping attention for the upstream gradient dOp (same layout).
    A key row's dK and dV sum the contributions of every Q tile that
    selected its tile."""
    B, heads, rows, d = qp.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dqp = np.zeros((B, heads, rows, d), dtype=np.float64)
    dkp = np.zeros_like(dqp)
    dvp = np.zeros_like(dqp)
    for h in range(heads):
        tab = slot_table(grid, tilings[h])
        nt = tab.size // S
        for b in range(B):
            for i in range(nt):
                dq, kr, dk, dv = attention_tile_backward(qp[b, h], kp[b, h], vp[b, h], dop[b, h], tab, i,
                                                         idx[b, h, i], S, scale)
                dqp[b, h, i * S:(i + 1) * S] = dq
                dkp[b, h, kr] += dk
                dvp[b, h, kr] += dv
    return dqp, dkp, dvp


# --------------------------------------------------------------------------
# Secondary path -- max-pooled full-attention tile map (sections 2.1, 2.3).
# --------------------------------------------------------------------------
def tile_map_row(qp_h, kp_h, table, i, S, scale):
    """M[j] = max over query slots of tile i and key slots of tile j of the
    full-attention probability P[q, key] (softmax over every valid key)."""
    nt = table.size // S
    valid = table >= 0
    key_rows = np.nonzero(valid)[0]
    qslots = np.nonzero(valid[i * S:(i + 1) * S])[0]
    Q = qp_h[i * S + qslots]
    logits = scale * (Q @ kp_h[key_rows].T)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    P = p / p.sum(axis=1, keepdims=True)               # [q, valid keys]
    key_tile = key_rows // S
    out = np.zeros(nt, dtype=np.float64)
    for j in range(nt):
        out[j] = P[:, key_tile == j].max()
    return out


def tile_map_maxpool(qp, kp, rows, grid, tilings, S, scale=None):
    """rows int [B*heads, R] (-1 = unused) -> map [B, heads, R, NT_max] (zero where unused)."""
    B, heads, _, d = qp.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nts, ntmax = tile_layout(grid, tilings)
    R = rows.shape[1]
    out = np.zeros((B, heads, R, ntmax), dtype=np.float64)
    for h in range(heads):
        tab = slot_table(grid, tilings[h])
        for b in range(B):
            for r in range(R):
                i = int(rows[b * heads + h, r])
                if i >= 0:
                    out[b, h, r, :nts[h]] = tile_map_row(qp[b, h], kp[b, h], tab, i, S, scale)
    return out


# --------------------------------------------------------------------------
# Whole inference path.
# --------------------------------------------------------------------------
def forward(q, k, v, grid, tilings, S, mlp_q, mlp_k, keep_ratio, scale=None):
    """permute -> TripPool -> estimator + top-k -> sparse attention -> unpermute.

    q, k, v: grid-order [B, heads, N, d] (any float dtype; used as fp64).
    Returns a dict of every intermediate.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    qp = tile_permute(q, grid, tilings, S)
    kp = tile_permute(k, grid, tilings, S)
    vp = tile_permute(v, grid, tilings, S)
    dq = tripool(qp, grid, tilings, S)
    dk = tripool(kp, grid, tilings, S)
    idx, probs, scores = score_topk(dq, dk, grid, tilings, S, mlp_q, mlp_k, keep_ratio, want_scores=True)
    op, lse = sparse_attention(qp, kp, vp, idx, grid, tilings, S, scale)
    o = tile_unpermute(op, grid, tilings, S)
    return dict(qp=qp, kp=kp, vp=vp, desc_q=dq, desc_k=dk, idx=idx, probs=probs, scores=scores,
                op=op, lse=lse, o=o)


# --------------------------------------------------------------------------
# Training the estimator -- row-wise KL distillation (section 2.1,
# "Optimization": the predicted distribution of tile scores is aligned with
# the full-attention reference row by row with a KL divergence; gradients do
# not flow into the backbone features that feed the estimator).
# --------------------------------------------------------------------------
def distill_row_loss(m_row: np.ndarray, s_row: np.ndarray) -> float:
    """KL(T || P) for one row, over the entries given (the head's valid K tiles):
    T = m_row / sum(m_row), the max-pooled full-attention row as a distribution;
    P = softmax(s_row), the estimator's row distribution.  Terms with T = 0
    contribute 0."""
    t = np.asarray(m_row, np.float64) / float(np.sum(m_row))
    s = np.asarray(s_row, np.float64)
    log_p = s - s.max() - math.log(float(np.exp(s - s.max()).sum()))
    nz = t > 0
    return float(np.sum(t[nz] * (np.log(t[nz]) - log_p[nz])))


def _estimator_with_hidden(desc, w1, b1, w2, b2):
    """Forward pass of estimator_head keeping the pre-activation z and the hidden a."""
    z = desc @ np.asarray(w1, np.float64).T + np.asarray(b1, np.float64)
    a = np.maximum(z, 0.0)
    return z, a, a @ np.asarray(w2, np.float64).T + np.asarray(b2, np.float64)


def distill_loss_grads(desc_q, desc_k, grid, tilings, S, mlp_q, mlp_k, tile_map, rows):
    """L = mean over the subset rows (b, h, r) with rows[b*heads+h, r] >= 0 of
    KL(T || P), with T the map row tile_map[b, h, r, :NT_h] normalised to sum 1
    and P = softmax_j s[i, j] over j < NT_h, i = rows[b*heads+h, r]
    (s = <phi_q(i), phi_k(j)> / sqrt(e) as in tile_scores_head).

    Returns (L, grads_q, grads_k); each grads tuple matches (W1, b1, W2, b2)
    of its estimator.  The descriptors are inputs only (the stop-gradient on
    the backbone features).  Reading: the direction KL(target || predicted)
    and the mean over rows are the plainest reading of "row-wise KL
    distillation objective"; the derivative of ReLU at 0 is taken as 0.
    """
    desc_q = np.asarray(desc_q, np.float64)
    desc_k = np.asarray(desc_k, np.float64)
    tile_map = np.asarray(tile_map, np.float64)
    rows = np.asarray(rows)
    B, heads = desc_q.shape[:2]
    nts, _ = tile_layout(grid, tilings)
    valid = [(b, h, r) for b in range(B) for h in range(heads) for r in range(rows.shape[1])
             if 0 <= rows[b * heads + h, r] < nts[h]]
    n_rows = len(valid)
    gq = [np.zeros(np.shape(w), np.float64) for w in mlp_q]
    gk = [np.zeros(np.shape(w), np.float64) for w in mlp_k]
    loss = 0.0
    for b in range(B):
        for h in range(heads):
            nt = nts[h]
            wq = tuple(np.asarray(w, np.float64)[h] for w in mlp_q)
            wk = tuple(np.asarray(w, np.float64)[h] for w in mlp_k)
            zq, aq, phq = _estimator_with_hidden(desc_q[b, h, :nt], *wq)
            zk, ak, phk = _estimator_with_hidden(desc_k[b, h, :nt], *wk)
            e = phq.shape[1]
            dphq = np.zeros_like(phq)
            dphk = np.zeros_like(phk)
            for r in range(rows.shape[1]):
                i = int(rows[b * heads + h, r])
                if not 0 <= i < nt:
                    continue
                s = phq[i] @ phk.T / math.sqrt(e)
                m = tile_map[b, h, r, :nt]
                loss += distill_row_loss(m, s)
                p = np.exp(s - s.max())
                p /= p.sum()
                g = (p - m / m.sum()) / n_rows          # dL/ds[i, :]
                dphq[i] += g @ phk / math.sqrt(e)
                dphk += np.outer(g, phq[i]) / math.sqrt(e)
            # back through phi = W2 a + b2, a = relu(z), z = W1 desc + b1
            for dph, z, a, desc, w, grad in ((dphq, zq, aq, desc_q[b, h, :nt], wq, gq),
                                             (dphk, zk, ak, desc_k[b, h, :nt], wk, gk)):
                grad[2][h] += dph.T @ a
                grad[3][h] += dph.sum(axis=0)
                dz = (dph @ w[2]) * (z > 0)
                grad[0][h] += dz.T @ desc
                grad[1][h] += dz.sum(axis=0)
    return loss / max(n_rows, 1), tuple(gq), tuple(gk)
