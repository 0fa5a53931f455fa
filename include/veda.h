/*
 * veda.h -- C ABI of the B200 (sm_100a) tile-sparse attention library.
 *
 * The method is Veda's head-aware tile-sparse self-attention over a T x H x W
 * video token grid ("Veda: Scalable Video Diffusion via Distilled Sparse
 * Attention", technical summary, sections 2.1-2.3).  The inference path is
 *
 *   veda_tile_permute (Q, K, V)  ->  veda_tripool (Q, K)  ->  veda_tile_score_topk
 *   ->  veda_tile_sparse_attn  ->  veda_tile_unpermute
 *
 * or, with the permutation folded into the attention kernel's tile fetch and
 * no tile-major copies at all,
 *
 *   veda_tripool_grid (Q, K)  ->  veda_tile_score_topk  ->  veda_tile_sparse_attn_grid
 *
 * and the distillation target is built by veda_tile_map_maxpool.  Training
 * calls: veda_distill_loss_grad (the estimator's row-wise KL loss and MLP
 * gradients) and veda_tile_sparse_attn_backward_grid (dQ, dK, dV of the
 * grid-order attention over the same selected tiles).
 *
 * Conventions shared by every call
 * --------------------------------
 * Layout.  Grid-order tensors are [B, heads, N, d] row-major bf16 with
 *   N = T*H*W and grid index n = (t*H + y)*W + x.  Tile-major ("permuted")
 *   tensors are [B, heads, NT_max*S, d] bf16: head h's tile j occupies rows
 *   j*S .. j*S+S-1, S = pt*ph*pw, and NT_max is the largest tile count over
 *   heads (veda_tile_layout).  Inside a tile, slots are row-major over
 *   (t, y, x) offsets; tiles are row-major over tile coordinates; a grid
 *   dimension that its factor does not divide is padded up to a multiple of
 *   it.  Pad slots hold no token.
 * Memory.  Every tensor pointer is caller-owned DEVICE memory, 16-byte
 *   aligned, and must not alias another argument of the same call unless the
 *   call says so.  The library allocates no device memory; calls that need
 *   scratch take a caller-provided workspace whose size a *_workspace query
 *   returns.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call only enqueues work and returns; nothing synchronises.
 *   Faults and kernel time-outs surface through veda_sync_status().
 * Errors.  Every call validates its arguments on the host first and returns
 *   VEDA_ERR_INVALID_ARG / VEDA_ERR_UNSUPPORTED without launching anything;
 *   veda_last_error() returns a thread-local description of the last failure.
 * Sizes.  d in {64, 128}; S in {64, 128} with pt*ph*pw == S for every head;
 *   1 <= heads <= VEDA_MAX_HEADS; B >= 1; every grid dimension >= 1.
 */
#ifndef VEDA_H_
#define VEDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VEDA_MAX_HEADS 128

typedef enum {
  VEDA_OK = 0,
  VEDA_ERR_INVALID_ARG = 1,   /* bad pointer, size, ratio or tiling */
  VEDA_ERR_UNSUPPORTED = 2,   /* valid request outside the built shapes (d, S) */
  VEDA_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed */
  VEDA_ERR_TIMEOUT = 4,       /* a kernel gave up on a bounded wait (device error word set) */
  VEDA_ERR_BOUNDS = 5         /* debug builds only: a kernel's index check failed and the access was skipped */
} veda_status;

/* Video token grid: frames T, height H, width W (latent tokens). */
typedef struct { int32_t T, H, W; } veda_grid;

/* One head's tile factorisation pi = (p_t, p_h, p_w) of the tile size S
 * ("Head-aware tiling", section 2.2: each layer and head factorises the
 * hardware tile size in its own way). */
typedef struct { int32_t pt, ph, pw; } veda_tiling;

/* Problem statement shared by all calls.  `tilings` is a HOST array of
 * `heads` entries, read during the call only. */
typedef struct {
  int32_t B, heads, d, S;
  veda_grid grid;
  const veda_tiling* tilings;
} veda_problem;

/* Per-head two-layer estimator (section 2.1, "head-specific MLP
 * projections"): phi = W2 relu(W1 desc + b1) + b2.  DEVICE fp32 pointers:
 * w1 [heads, hidden, 3d], b1 [heads, hidden], w2 [heads, e, hidden],
 * b2 [heads, e], all row-major.  hidden a multiple of 4 in [4, 512];
 * e in {16, 32, 64, 128}. */
typedef struct {
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
  int32_t hidden, e;
} veda_mlp;

/* Gradient outputs for one estimator, DEVICE fp32, shaped like its weights:
 * w1 [heads, hidden, 3d], b1 [heads, hidden], w2 [heads, e, hidden],
 * b2 [heads, e]; 16-byte aligned; written in full by the call. */
typedef struct {
  float* w1;
  float* b1;
  float* w2;
  float* b2;
} veda_mlp_grad;

/* ---------------------------------------------------------------- host helpers */

/* Tiles per head after padding, NT_h = ceil(T/pt)*ceil(H/ph)*ceil(W/pw), and
 * their maximum.  `nt_per_head` is a HOST array of `heads` entries (may be
 * NULL); `nt_max` a host scalar (may be NULL).  Pure host arithmetic. */
veda_status veda_tile_layout(const veda_problem* p, int32_t* nt_per_head, int32_t* nt_max);

/* Kept K tiles per Q tile for keep ratio r in (0, 1]:
 * k_h = max(1, min(NT_h, floor(r*NT_h + 1/2))) (the pages fix only "keep
 * about 5-10% of tiles"; this rounding is this library's reading).  Host
 * arrays as in veda_tile_layout. */
veda_status veda_keep_count(const veda_problem* p, float keep_ratio, int32_t* k_per_head,
                            int32_t* k_max);

/* ---------------------------------------------------------------- step 1: tiling */

/* Per-head token permutation, grid order -> tile-major (section 2.2).
 * x  [B, heads, N, d] bf16 (read), xp [B, heads, NT_max*S, d] bf16 (written
 * in full: pad slots and rows of tiles j >= NT_h are written as zeros).
 * x and xp must not overlap. */
veda_status veda_tile_permute(const veda_problem* p, const void* x, void* xp, void* stream);

/* Inverse of veda_tile_permute on token rows ("output scattered back to grid
 * order"): xp [B, heads, NT_max*S, d] bf16 (read), x [B, heads, N, d] bf16
 * (every row written).  Pad rows of xp are ignored. */
veda_status veda_tile_unpermute(const veda_problem* p, const void* xp, void* x, void* stream);

/* ---------------------------------------------------------------- step 2: TripPool */

/* TripPool descriptor per tile (section 2.1, "statistics-aware estimator":
 * channel-wise mean, max and min concatenated).  xp [B, heads, NT_max*S, d]
 * bf16 tile-major (read); desc [B, heads, NT_max, 3d] fp32 (written in full):
 * desc[.., j, 0:d] = mean, [d:2d] = max, [2d:3d] = min over the token slots of
 * tile j (pad slots excluded); rows j >= NT_h are zero. */
veda_status veda_tripool(const veda_problem* p, const void* xp, float* desc, void* stream);

/* veda_tile_permute and veda_tripool in one pass over x (the pages' future
 * work names "tighter kernel fusion", section 5): xp as veda_tile_permute
 * writes it and desc as veda_tripool would compute it from xp, with x read
 * from HBM once.  Arguments as in the two calls; x, xp and desc must not
 * overlap. */
veda_status veda_tile_permute_tripool(const veda_problem* p, const void* x, void* xp, float* desc,
                                      void* stream);

/* TripPool straight from a grid-order tensor: x [B, heads, N, d] bf16 (read),
 * desc [B, heads, NT_max, 3d] fp32 (written in full), equal to veda_tripool
 * of veda_tile_permute(x); no permuted copy is made.  x and desc must not
 * overlap. */
veda_status veda_tripool_grid(const veda_problem* p, const void* x, float* desc, void* stream);

/* ---------------------------------------------------------------- steps 3-4: estimator + top-k */

/* Bytes of workspace veda_tile_score_topk needs for estimator width e: the
 * estimator features (2*B*heads*NT_max*e fp32) and, for e <= 64, the fp32
 * score matrix [B, heads, NT_max, NT_max rounded up to a multiple of 4]
 * (83 MB at the Wan2.1-14B 720p shape), each rounded up to 256 bytes. */
veda_status veda_score_topk_workspace(const veda_problem* p, int32_t e, size_t* bytes);

/* Distilled tile scoring and selection (section 2.1 "distilled tile scoring",
 * "row-wise distribution over tiles"; news page "95% sparsity").
 * desc_q, desc_k [B, heads, NT_max, 3d] fp32 (read).  mlp_q / mlp_k: HOST
 * structs holding device weight pointers; they may describe the same
 * weights.  For each head and valid Q tile i:
 *   s[i, j] = <phi_q(desc_q[i]), phi_k(desc_k[j])> / sqrt(e),  j < NT_h,
 *   probs[i, :] = softmax_j s[i, :]                (optional),
 *   idx[i, :] = the k_h indices j of largest s[i, j], ties to the smaller j,
 *               ascending, then -1 up to k_max.
 * idx [B, heads, NT_max, k_max] int32 (written in full; rows i >= NT_h are -1);
 * k_max >= max_h k_h (veda_keep_count).  probs [B, heads, NT_max, NT_max]
 * fp32 or NULL (written in full, zero outside the valid block).
 * workspace: device scratch of >= veda_score_topk_workspace() bytes, 256-byte
 * aligned, owned by the caller, not read before it is written. */
veda_status veda_tile_score_topk(const veda_problem* p, const float* desc_q, const float* desc_k,
                                 const veda_mlp* mlp_q, const veda_mlp* mlp_k, float keep_ratio,
                                 int32_t* idx, int32_t k_max, float* probs, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* veda_tile_score_topk for callers that cannot provide device scratch memory
 * -- a plugin whose host framework owns all device memory and gives it no
 * workspace, or a latency-critical loop that must not call cudaMalloc (which
 * can stall the whole device).  The paper has no counterpart; it is a
 * deployment convenience.  Arguments, results and errors are those of
 * veda_tile_score_topk, without the workspace: the estimator features live
 * in a 16 MiB device array inside the library (2*B*heads*NT_max*e floats
 * must fit; larger problems get VEDA_ERR_UNSUPPORTED and should use
 * veda_tile_score_topk).  This call allocates nothing.  Every GPU that loads
 * the library holds the array until the process exits.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) for that
 * device; make that first call before any stream capture.  The address is
 * kept per device and per context: after cudaDeviceReset the next call looks
 * it up again (so, again, not inside a capture).  All calls share
 * the one array, so calls that may overlap on the GPU (different streams,
 * or different host threads on one device) race: serialise them.  Nothing
 * needs clearing between calls -- every value read is written earlier in the
 * same call. */
veda_status veda_tile_score_topk_noalloc(const veda_problem* p, const float* desc_q, const float* desc_k,
                                         const veda_mlp* mlp_q, const veda_mlp* mlp_k, float keep_ratio,
                                         int32_t* idx, int32_t k_max, float* probs, void* stream);

/* ---------------------------------------------------------------- step 5: tile-skipping attention */

/* Block-sparse attention over only the selected K/V tiles (section 2.3,
 * "tile-skipping sparse attention kernel"; news page "tile skipping").
 * qp, kp, vp [B, heads, NT_max*S, d] bf16 tile-major (read).
 * idx [B, heads, NT_max, k_max] int32: per Q tile the selected K tiles, each
 * in [0, NT_h), distinct, terminated by -1 or by k_max entries; at least one
 * entry per valid Q tile.  For every token slot q of Q tile i:
 *   op[q] = sum_key softmax(scale * <Q_q, K_key>) V_key over the token slots of
 *   the selected tiles (pad key slots masked),
 *   lse[q] = ln sum_key exp(scale * <Q_q, K_key>).
 * scale <= 0 selects 1/sqrt(d).  op [B, heads, NT_max*S, d] bf16: token rows
 * written, pad rows and rows of tiles i >= NT_h left unspecified.  lse
 * [B, heads, NT_max*S] fp32 or NULL, same row rule.  Runs on the tcgen05
 * tensor cores; fp32 accumulation. */
veda_status veda_tile_sparse_attn(const veda_problem* p, const void* qp, const void* kp,
                                  const void* vp, const int32_t* idx, int32_t k_max, float scale,
                                  void* op, float* lse, void* stream);

/* The same attention on grid-order tensors (section 2.2's head-aware tiling
 * applied inside the kernel; the output goes straight back to grid order).
 * q, k, v [B, heads, N, d] bf16 (read); idx, k_max and scale as in
 * veda_tile_sparse_attn.  Each selected tile is fetched as one pt x ph x pw
 * box of the grid, so the result equals veda_tile_unpermute of
 * veda_tile_sparse_attn on the permuted tensors: o [B, heads, N, d] bf16,
 * every row written; lse [B, heads, N] fp32 or NULL, every entry written.
 * o must not overlap q, k or v.  Heads are grouped by tiling; one launch
 * covers up to 8 distinct tilings, so more tilings take several launches. */
veda_status veda_tile_sparse_attn_grid(const veda_problem* p, const void* q, const void* k,
                                       const void* v, const int32_t* idx, int32_t k_max, float scale,
                                       void* o, float* lse, void* stream);

/* Launch configuration the two attention calls use for this problem and
 * k_max (host-side query, no device work): the depths of the K and V tile
 * rings in shared memory and the dynamic shared memory per CTA.  Deeper
 * rings are chosen whenever they fit; the bookkeeping (selection list) grows
 * with k_max.  Returns VEDA_ERR_UNSUPPORTED when no configuration fits. */
veda_status veda_attn_config(const veda_problem* p, int32_t k_max, int32_t* k_stages, int32_t* v_stages,
                             size_t* smem_bytes);

/* ---------------------------------------------------------------- secondary: tile map */

/* Bytes of workspace veda_tile_map_maxpool needs for R subset rows. */
veda_status veda_tile_map_workspace(const veda_problem* p, int32_t R, size_t* bytes);

/* Max-pooled full-attention tile map, the distillation target (section 2.1
 * "target construction": max-pool the full attention matrix over Q-tile x
 * K-tile regions; section 2.3: built in two passes over a random subset of Q
 * tiles).  qp, kp [B, heads, NT_max*S, d] bf16 tile-major (read).
 * rows [B*heads, R] int32: Q tiles of the subset per (b, h), each in
 * [0, NT_h) or -1 (unused).  With P the softmax of scale * Q K^T over every
 * valid key of the head:
 *   map[b, h, r, j] = max_{q in tile rows[r], key in tile j} P[q, key]
 * for j < NT_h; entries j >= NT_h and unused rows are 0.  map
 * [B, heads, R, NT_max] fp32 (written in full).  scale <= 0 selects
 * 1/sqrt(d).  workspace: >= veda_tile_map_workspace() bytes of device
 * scratch, 256-byte aligned. */
veda_status veda_tile_map_maxpool(const veda_problem* p, const void* qp, const void* kp,
                                  const int32_t* rows, int32_t R, float scale, float* map,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* veda_tile_map_maxpool on grid-order tensors: q, k [B, heads, N, d] bf16
 * (read), no tile-major copies needed.  Each tile is fetched as one 5D box of
 * the grid-order tensor, which holds the same values as the permuted tile
 * (zeros in pad slots), so the map is identical to veda_tile_map_maxpool's on
 * the permuted tensors.  Other arguments, workspace (veda_tile_map_workspace)
 * and errors as for veda_tile_map_maxpool. */
veda_status veda_tile_map_maxpool_grid(const veda_problem* p, const void* q, const void* k,
                                       const int32_t* rows, int32_t R, float scale, float* map,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- training the estimator */

/* Bytes of workspace veda_distill_loss_grad needs. */
veda_status veda_distill_workspace(const veda_problem* p, int32_t hidden, int32_t e, int32_t R, size_t* bytes);

/* The estimator's distillation objective and its gradients (section 2.1,
 * "Optimization": a row-wise KL divergence aligns the predicted tile-score
 * distribution with the full-attention reference; the backbone features fed
 * to the estimator are stop-gradient).  With the subset rows and tile map of
 * veda_tile_map_maxpool (map [B, heads, R, NT_max] fp32, rows [B*heads, R]
 * int32, -1 = unused) and s[i, j] = <phi_q(i), phi_k(j)> / sqrt(e):
 *   loss = mean over valid subset rows (b, h, r), i = rows[b*heads+h, r], of
 *          KL(T || P),  T = map[b, h, r, :NT_h] / sum_j map[b, h, r, j],
 *                       P = softmax_j s[i, j], j < NT_h;
 *   grad_q / grad_k = d loss / d (W1, b1, W2, b2) of the Q-side and K-side
 *          estimators; the descriptors get no gradient.
 * loss: one DEVICE fp32.  When mlp_q and mlp_k are the same weights, their
 * gradient is grad_q + grad_k.  desc_q, desc_k as for veda_tile_score_topk.
 * Map rows must have a positive sum.  workspace: >= veda_distill_workspace()
 * bytes of device scratch, 256-byte aligned.  The forward estimator runs on
 * the tensor cores as in veda_tile_score_topk; the backward runs in fp32. */
veda_status veda_distill_loss_grad(const veda_problem* p, const float* desc_q, const float* desc_k,
                                   const veda_mlp* mlp_q, const veda_mlp* mlp_k, const float* map,
                                   const int32_t* rows, int32_t R, float* loss, const veda_mlp_grad* grad_q,
                                   const veda_mlp_grad* grad_k, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* ---------------------------------------------------------------- offline tiling search */

/* Per-head error between two grid-order outputs, for the offline choice of
 * each head's tiling (section 2.2: the tiling is selected on a calibration
 * set by minimising the error between full- and sparse-attention outputs).
 * o, o_ref [B, heads, N, d] bf16 (read).  err[h] = sum over b, n, channels
 * of (o - o_ref)^2 and ref_sq[h] = sum of o_ref^2; both DEVICE fp32 [heads],
 * written in full, summed in a fixed order.  workspace: >= 512 * heads bytes
 * of device scratch, 16-byte aligned. */
veda_status veda_head_error(const veda_problem* p, const void* o, const void* o_ref, float* err, float* ref_sq,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- backward of step 5 */

/* Workspace bytes veda_tile_sparse_attn_backward_grid needs for a problem and
 * k_max: the row sums D, the inverse selection lists and their offsets. */
veda_status veda_attn_backward_workspace(const veda_problem* p, int32_t k_max, size_t* bytes);

/* Gradients of veda_tile_sparse_attn_grid with respect to q, k and v over
 * the same selected tiles (section 2.3 defines the forward; this is its chain
 * rule, for fine-tuning the backbone with the sparse pattern fixed).  With
 * P = softmax(scale Q K^T) over the selected tiles' token slots:
 *   dV = P^T dO,  dP = dO V^T,  dX = P (dP - rowsum(dO * O)),
 *   dQ = scale dX K,  dK = scale dX^T Q,
 * where a key row's dK and dV sum over every Q tile that selected its tile.
 * q, k, v, o, d_o [B, heads, N, d] bf16 grid order (read): the forward's
 * inputs, its output o and the upstream gradient.  lse [B, heads, N] fp32
 * (read): the forward's LSE (required).  idx, k_max and scale as given to the
 * forward (rows read up to their first entry outside [0, NT_h); entries
 * distinct).  dq, dk, dv [B, heads, N, d] bf16 (written, every row; rows of
 * keys that no Q tile selected get zero).  They must not overlap the inputs.
 * workspace: device memory of veda_attn_backward_workspace bytes, 256-byte
 * aligned, owned by the caller; its contents need no initialisation.  Runs on
 * the tcgen05 tensor cores with fp32 accumulation; P and dS are rounded to
 * bf16 as product operands, as in the forward.  Deterministic: no atomics on
 * the gradients.  Errors: VEDA_ERR_INVALID_ARG for NULL or misaligned
 * tensors or a short workspace; VEDA_ERR_UNSUPPORTED for NT_max > 32767. */
veda_status veda_tile_sparse_attn_backward_grid(const veda_problem* p, const void* q, const void* k, const void* v,
                                                const void* o, const float* lse, const void* d_o,
                                                const int32_t* idx, int32_t k_max, float scale, void* dq,
                                                void* dk, void* dv, void* workspace, size_t workspace_bytes,
                                                void* stream);

/* ---------------------------------------------------------------- status */

/* Synchronises `stream`, then reads and clears the library's device error
 * word (set by a kernel that gave up on a bounded wait).  Returns VEDA_OK,
 * VEDA_ERR_TIMEOUT or VEDA_ERR_CUDA.  The error word is one per device and
 * process, shared by every stream and thread: a status read through stream A
 * can report (and clears) a fault raised by a kernel on stream B.  Callers
 * that need per-stream attribution synchronise the other streams first. */
veda_status veda_sync_status(void* stream);

/* Limit of every bounded wait inside the library's kernels, in nanoseconds
 * (default 2 s; accepted range [1 us, 60 s]).  Process-wide, read at launch
 * time.  A kernel that runs a wait out sets the device error word, drains
 * its in-flight copies, frees its tensor memory and returns. */
veda_status veda_set_wait_timeout_ns(uint64_t ns);

/* Failure-detection self-test (no counterpart on the pages): launches one
 * tiny kernel that waits on an mbarrier nothing ever arrives on, for at most
 * `timeout_ns` ([1 us, 10 s]).  The following veda_sync_status(stream)
 * must report VEDA_ERR_TIMEOUT; the context stays usable. */
veda_status veda_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* 1 for a debug build (compiled with -DVEDA_DEBUG_BOUNDS: every index a
 * kernel computes -- tile ids, tensor rows, selection entries -- is checked
 * before use; a failed check skips the access, sets the device error word and
 * veda_sync_status returns VEDA_ERR_BOUNDS naming the source line), 0 for a
 * release build, where the checks compile away. */
int32_t veda_bounds_checked(void);

/* Bounds-check self-test (no counterpart on the pages; debug builds only):
 * launches one tiny kernel whose last thread fails a bounds check and touches
 * no memory.  The following veda_sync_status(stream) must return
 * VEDA_ERR_BOUNDS.  A release build returns VEDA_ERR_UNSUPPORTED and launches
 * nothing. */
veda_status veda_selftest_bounds(void* stream);

/* Thread-local text of the last failure ("" if none).  Valid until the next
 * call on this thread. */
const char* veda_last_error(void);

/* Library version, "major.minor.patch". */
const char* veda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VEDA_H_ */
