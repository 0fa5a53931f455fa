// C ABI of the library (declared in include/veda.h): host-side validation,
// geometry set-up, TMA descriptor encoding and kernel launches.  Built as one
// translation unit together with the kernel sources so the device error word
// needs no separate device link.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "veda_common.cuh"
#include "kernels.h"

#include "permute_tripool.cu"
#include "score_topk.cu"
#include "sparse_attn.cu"
#include "tile_map.cu"
#include "distill.cu"
#include "attn_bwd.cu"

namespace veda {
namespace {

thread_local char g_last_error[512] = "";
uint64_t g_timeout_ns = 2000000000ull;  // bounded-wait limit for every kernel (2 s)

veda_status fail(veda_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

veda_status ok() {
  g_last_error[0] = '\0';
  return VEDA_OK;
}

veda_status cuda_fail(cudaError_t e, const char* where) {
  return fail(VEDA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Validates the problem statement and fills the kernels' geometry block.
veda_status make_geometry(const veda_problem* p, Geometry* G) {
  if (p == nullptr) return fail(VEDA_ERR_INVALID_ARG, "problem is NULL");
  if (p->B < 1) return fail(VEDA_ERR_INVALID_ARG, "B must be >= 1 (got %d)", p->B);
  if (p->heads < 1 || p->heads > VEDA_MAX_HEADS)
    return fail(VEDA_ERR_INVALID_ARG, "heads must be in [1, %d] (got %d)", VEDA_MAX_HEADS, p->heads);
  if (p->grid.T < 1 || p->grid.H < 1 || p->grid.W < 1)
    return fail(VEDA_ERR_INVALID_ARG, "grid dimensions must be >= 1 (got %d x %d x %d)", p->grid.T,
                p->grid.H, p->grid.W);
  if (p->d != 64 && p->d != 128) return fail(VEDA_ERR_UNSUPPORTED, "head dim d must be 64 or 128 (got %d)", p->d);
  if (p->S != 64 && p->S != 128) return fail(VEDA_ERR_UNSUPPORTED, "tile size S must be 64 or 128 (got %d)", p->S);
  if (p->tilings == nullptr) return fail(VEDA_ERR_INVALID_ARG, "tilings is NULL");
  const long long N = (long long)p->grid.T * p->grid.H * p->grid.W;
  if (N > (1LL << 30)) return fail(VEDA_ERR_INVALID_ARG, "grid has too many tokens (%lld)", N);
  std::memset(G, 0, sizeof(*G));
  G->B = p->B;
  G->heads = p->heads;
  G->d = p->d;
  G->S = p->S;
  G->T = p->grid.T;
  G->H = p->grid.H;
  G->W = p->grid.W;
  G->N = (int)N;
  int ntmax = 0;
  for (int h = 0; h < p->heads; ++h) {
    const veda_tiling t = p->tilings[h];
    if (t.pt < 1 || t.ph < 1 || t.pw < 1 || t.pt > 4096 || t.ph > 4096 || t.pw > 4096)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: tiling factors must be >= 1", h);
    if ((long long)t.pt * t.ph * t.pw != p->S)
      return fail(VEDA_ERR_INVALID_ARG, "head %d: pt*ph*pw = %d*%d*%d must equal S = %d", h, t.pt, t.ph,
                  t.pw, p->S);
    HeadGeom& g = G->g[h];
    g.pt = (int16_t)t.pt;
    g.ph = (int16_t)t.ph;
    g.pw = (int16_t)t.pw;
    const int a = ceil_div(p->grid.T, t.pt), b = ceil_div(p->grid.H, t.ph), c = ceil_div(p->grid.W, t.pw);
    if (a > 32767 || b > 32767 || c > 32767) return fail(VEDA_ERR_INVALID_ARG, "head %d: too many tiles", h);
    g.nTt = (int16_t)a;
    g.nTh = (int16_t)b;
    g.nTw = (int16_t)c;
    g.nt = a * b * c;
    if (g.nt > ntmax) ntmax = g.nt;
  }
  G->ntmax = ntmax;
  const long long rows = (long long)p->B * p->heads * ntmax * p->S;
  if (rows >= (1LL << 31)) return fail(VEDA_ERR_INVALID_ARG, "B*heads*NT_max*S = %lld rows exceeds 2^31", rows);
  if ((long long)p->B * p->heads * N >= (1LL << 31))
    return fail(VEDA_ERR_INVALID_ARG, "B*heads*N exceeds 2^31 rows");
  if ((long long)p->B * p->heads > 65535) return fail(VEDA_ERR_INVALID_ARG, "B*heads exceeds 65535");
  return VEDA_OK;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D view [rows, d] of a tile-major bf16 tensor, boxes of 64 channels x S rows,
// 128-byte swizzle (the layout the tcgen05 descriptors expect).
veda_status encode_tile_major(const Geometry& G, const void* ptr, CUtensorMap* out) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)G.d, (cuuint64_t)G.B * G.heads * G.ntmax * G.S};
  const cuuint64_t strides[1] = {(cuuint64_t)G.d * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)G.S};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return VEDA_OK;
}

// 5D view [B*heads, T, H, W, d] of a grid-order bf16 tensor [B, heads, N, d]
// with boxes of 64 channels x pw x ph x pt tokens x 1: one box is one 3D tile
// of a head with tiling (pt, ph, pw), in within-tile slot order.  Boxes that
// reach past the grid are zero-filled.  128-byte swizzle as above.
veda_status encode_grid_tiles(const Geometry& G, const void* ptr, const HeadGeom& hg, CUtensorMap* out) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t row = (cuuint64_t)G.d * 2;
  const cuuint64_t dims[5] = {(cuuint64_t)G.d, (cuuint64_t)G.W, (cuuint64_t)G.H, (cuuint64_t)G.T,
                              (cuuint64_t)G.B * G.heads};
  const cuuint64_t strides[4] = {row, row * G.W, row * G.W * G.H, row * (cuuint64_t)G.N};
  const cuuint32_t box[5] = {64u, (cuuint32_t)hg.pw, (cuuint32_t)hg.ph, (cuuint32_t)hg.pt, 1u};
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  const CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled (grid tiles %dx%dx%d) failed (CUresult %d)", hg.pt, hg.ph,
                hg.pw, (int)r);
  return VEDA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// The estimator features: 2*B*heads*NT_max*e floats.
size_t phi_ws_bytes(const Geometry& G, int e) {
  return round256(sizeof(float) * 2 * (size_t)G.B * G.heads * G.ntmax * e);
}

// veda_tile_score_topk's workspace: the features, then the score matrix.
size_t score_ws_bytes(const Geometry& G, int e) { return phi_ws_bytes(G, e) + round256(score_matrix_bytes(G, e)); }

size_t map_rowmax_bytes(const Geometry& G, int R) {
  return round256(sizeof(float) * (size_t)G.B * G.heads * R * G.ntmax * G.S);
}

size_t map_ws_bytes(const Geometry& G, int R) {
  return map_rowmax_bytes(G, R) + round256(sizeof(float) * (size_t)G.B * G.heads * R * G.S);
}

veda_status keep_counts(const Geometry& G, float r, int32_t* k, int32_t* kmax) {
  if (!(r > 0.f && r <= 1.f)) return fail(VEDA_ERR_INVALID_ARG, "keep_ratio must be in (0, 1] (got %g)", (double)r);
  int m = 0;
  for (int h = 0; h < G.heads; ++h) {
    const int nt = G.g[h].nt;
    long long kk = (long long)std::floor((double)r * nt + 0.5);
    if (kk > nt) kk = nt;
    if (kk < 1) kk = 1;
    if (k) k[h] = (int32_t)kk;
    if (kk > m) m = (int)kk;
  }
  if (kmax) *kmax = m;
  return VEDA_OK;
}

}  // namespace
}  // namespace veda

using namespace veda;

extern "C" {

const char* veda_last_error(void) { return g_last_error; }

const char* veda_version(void) { return "0.1.0"; }

veda_status veda_tile_layout(const veda_problem* p, int32_t* nt_per_head, int32_t* nt_max) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (nt_per_head)
    for (int h = 0; h < G.heads; ++h) nt_per_head[h] = G.g[h].nt;
  if (nt_max) *nt_max = G.ntmax;
  return ok();
}

veda_status veda_keep_count(const veda_problem* p, float keep_ratio, int32_t* k_per_head, int32_t* k_max) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if ((s = keep_counts(G, keep_ratio, k_per_head, k_max)) != VEDA_OK) return s;
  return ok();
}

veda_status veda_tile_permute(const veda_problem* p, const void* x, void* xp, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!x || !xp) return fail(VEDA_ERR_INVALID_ARG, "x and xp must be non-NULL");
  if (!aligned16(x) || !aligned16(xp)) return fail(VEDA_ERR_INVALID_ARG, "x and xp must be 16-byte aligned");
  cudaError_t e = launch_permute(G, x, xp, (cudaStream_t)stream, sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_permute");
  return ok();
}

veda_status veda_tile_permute_tripool(const veda_problem* p, const void* x, void* xp, float* desc, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!x || !xp || !desc) return fail(VEDA_ERR_INVALID_ARG, "x, xp and desc must be non-NULL");
  if (!aligned16(x) || !aligned16(xp) || !aligned16(desc))
    return fail(VEDA_ERR_INVALID_ARG, "x, xp and desc must be 16-byte aligned");
  cudaError_t e = launch_permute_tripool(G, x, xp, desc, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_permute_tripool");
  return ok();
}

veda_status veda_tile_unpermute(const veda_problem* p, const void* xp, void* x, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!x || !xp) return fail(VEDA_ERR_INVALID_ARG, "x and xp must be non-NULL");
  if (!aligned16(x) || !aligned16(xp)) return fail(VEDA_ERR_INVALID_ARG, "x and xp must be 16-byte aligned");
  cudaError_t e = launch_unpermute(G, xp, x, (cudaStream_t)stream, sm_count());
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_unpermute");
  return ok();
}

veda_status veda_tripool(const veda_problem* p, const void* xp, float* desc, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!xp || !desc) return fail(VEDA_ERR_INVALID_ARG, "xp and desc must be non-NULL");
  if (!aligned16(xp) || !aligned16(desc)) return fail(VEDA_ERR_INVALID_ARG, "xp and desc must be 16-byte aligned");
  cudaError_t e = launch_tripool(G, xp, desc, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tripool");
  return ok();
}

veda_status veda_tripool_grid(const veda_problem* p, const void* x, float* desc, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!x || !desc) return fail(VEDA_ERR_INVALID_ARG, "x and desc must be non-NULL");
  if (!aligned16(x) || !aligned16(desc)) return fail(VEDA_ERR_INVALID_ARG, "x and desc must be 16-byte aligned");
  cudaError_t e = launch_tripool_grid(G, x, desc, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tripool_grid");
  return ok();
}

veda_status veda_score_topk_workspace(const veda_problem* p, int32_t e, size_t* bytes) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (e != 16 && e != 32 && e != 64 && e != 128) return fail(VEDA_ERR_INVALID_ARG, "e must be 16, 32, 64 or 128 (got %d)", e);
  if (!bytes) return fail(VEDA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = score_ws_bytes(G, e);
  return ok();
}

static veda_status check_mlp(const veda_mlp* m, const char* which) {
  if (!m) return fail(VEDA_ERR_INVALID_ARG, "%s estimator is NULL", which);
  if (!m->w1 || !m->b1 || !m->w2 || !m->b2) return fail(VEDA_ERR_INVALID_ARG, "%s estimator has a NULL weight", which);
  if (m->hidden < 4 || m->hidden > 512 || m->hidden % 4)
    return fail(VEDA_ERR_INVALID_ARG, "hidden must be a multiple of 4 in [4, 512] (got %d)", m->hidden);
  if (m->e != 16 && m->e != 32 && m->e != 64 && m->e != 128)
    return fail(VEDA_ERR_INVALID_ARG, "e must be 16, 32, 64 or 128 (got %d)", m->e);
  return VEDA_OK;
}

veda_status veda_tile_score_topk(const veda_problem* p, const float* desc_q, const float* desc_k,
                                 const veda_mlp* mlp_q, const veda_mlp* mlp_k, float keep_ratio, int32_t* idx,
                                 int32_t k_max, float* probs, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if ((s = check_mlp(mlp_q, "q")) != VEDA_OK || (s = check_mlp(mlp_k, "k")) != VEDA_OK) return s;
  if (mlp_q->hidden != mlp_k->hidden || mlp_q->e != mlp_k->e)
    return fail(VEDA_ERR_INVALID_ARG, "q and k estimators must have the same hidden and e");
  if (!desc_q || !desc_k || !idx || !workspace) return fail(VEDA_ERR_INVALID_ARG, "NULL tensor argument");
  if (!aligned16(desc_q) || !aligned16(desc_k) || !aligned16(idx) || (probs && !aligned16(probs)))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(VEDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const int e = mlp_q->e, hidden = mlp_q->hidden;
  if (workspace_bytes < score_ws_bytes(G, e))
    return fail(VEDA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, score_ws_bytes(G, e));
  TopkArgs args;
  std::memset(&args, 0, sizeof(args));
  int32_t kmax_needed = 0;
  if ((s = keep_counts(G, keep_ratio, args.k_per_head, &kmax_needed)) != VEDA_OK) return s;
  if (k_max < kmax_needed) return fail(VEDA_ERR_INVALID_ARG, "k_max = %d is below the largest keep count %d", k_max, kmax_needed);
  int qb, ntpad;
  size_t smem;
  score_topk_config(G.ntmax, e, &qb, &ntpad, &smem);
  if (smem > 227 * 1024 || estimator_smem_bytes(G.d, hidden, e) > 227 * 1024)
    return fail(VEDA_ERR_UNSUPPORTED, "NT_max = %d / hidden = %d exceed the shared-memory budget", G.ntmax, hidden);
  args.idx = idx;
  args.probs = probs;
  args.k_max = k_max;
  args.timeout_ns = g_timeout_ns;
  EstimatorWeights wq{mlp_q->w1, mlp_q->b1, mlp_q->w2, mlp_q->b2};
  EstimatorWeights wk{mlp_k->w1, mlp_k->b1, mlp_k->w2, mlp_k->b2};
  float* phi = static_cast<float*>(workspace);
  float* scores = score_matrix_bytes(G, e) > 0
                      ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + phi_ws_bytes(G, e))
                      : nullptr;
  cudaError_t ce = launch_score_topk(G, desc_q, desc_k, wq, wk, hidden, e, phi, scores, args, (cudaStream_t)stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "veda_tile_score_topk");
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Scoring without a caller-provided workspace.
//
// Some callers cannot hand the library scratch memory: a plugin whose host
// framework owns every byte of device memory and offers no workspace hook,
// or a latency-critical loop that must not call cudaMalloc (it can stall the
// whole device).  For them the estimator's per-tile features go to this
// file-scope device array instead, sized for the largest workloads this
// library is built for (16 MiB: the Wan2.1-14B 720p shape needs 14.1 MiB).
// Every GPU that loads the library holds it until the process exits.
// ---------------------------------------------------------------------------
namespace veda {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Unique id of the calling thread's current CUDA context, or 0 when none is
// current (or the driver predates cuCtxGetId).  Ids are never reused within a
// process, so a context torn down by cudaDeviceReset and created again gets a
// new one.
unsigned long long current_context_id() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device.  It is looked
// up once per device and context (the host-side symbol is only a stand-in,
// never a device pointer) and looked up again when the device's context has
// changed since, e.g. after cudaDeviceReset.
veda_status noalloc_scratch(float** out) {
  constexpr int kMaxDevices = 64;
  static float* ptrs[kMaxDevices] = {};
  static unsigned long long ctx_ids[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_score_topk_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(VEDA_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices - 1);
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_context_id();
  if (ptrs[dev] == nullptr || id == 0 || id != ctx_ids[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // also makes the device's primary context current
    if (e != cudaSuccess) return cuda_fail(e, "veda_tile_score_topk_noalloc: cudaGetSymbolAddress");
    ptrs[dev] = static_cast<float*>(p);
    ctx_ids[dev] = current_context_id();
  }
  *out = ptrs[dev];
  return VEDA_OK;
}
}  // namespace
}  // namespace veda

extern "C" {

veda_status veda_tile_score_topk_noalloc(const veda_problem* p, const float* desc_q, const float* desc_k,
                                         const veda_mlp* mlp_q, const veda_mlp* mlp_k, float keep_ratio,
                                         int32_t* idx, int32_t k_max, float* probs, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if ((s = check_mlp(mlp_q, "q")) != VEDA_OK || (s = check_mlp(mlp_k, "k")) != VEDA_OK) return s;
  if (mlp_q->hidden != mlp_k->hidden || mlp_q->e != mlp_k->e)
    return fail(VEDA_ERR_INVALID_ARG, "q and k estimators must have the same hidden and e");
  if (!desc_q || !desc_k || !idx) return fail(VEDA_ERR_INVALID_ARG, "NULL tensor argument");
  if (!aligned16(desc_q) || !aligned16(desc_k) || !aligned16(idx) || (probs && !aligned16(probs)))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  const int e = mlp_q->e, hidden = mlp_q->hidden;
  const size_t need = phi_ws_bytes(G, e);
  if (need > kNoAllocScratchBytes)
    return fail(VEDA_ERR_UNSUPPORTED,
                "estimator scratch of %zu bytes exceeds the built-in %zu bytes (2*B*heads*NT_max*e floats); "
                "use veda_tile_score_topk with a workspace",
                need, kNoAllocScratchBytes);
  TopkArgs args;
  std::memset(&args, 0, sizeof(args));
  int32_t kmax_needed = 0;
  if ((s = keep_counts(G, keep_ratio, args.k_per_head, &kmax_needed)) != VEDA_OK) return s;
  if (k_max < kmax_needed) return fail(VEDA_ERR_INVALID_ARG, "k_max = %d is below the largest keep count %d", k_max, kmax_needed);
  int qb, ntpad;
  size_t smem;
  score_topk_config(G.ntmax, e, &qb, &ntpad, &smem);
  if (smem > 227 * 1024 || estimator_smem_bytes(G.d, hidden, e) > 227 * 1024)
    return fail(VEDA_ERR_UNSUPPORTED, "NT_max = %d / hidden = %d exceed the shared-memory budget", G.ntmax, hidden);
  float* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != VEDA_OK) return s;
  args.idx = idx;
  args.probs = probs;
  args.k_max = k_max;
  args.timeout_ns = g_timeout_ns;
  EstimatorWeights wq{mlp_q->w1, mlp_q->b1, mlp_q->w2, mlp_q->b2};
  EstimatorWeights wk{mlp_k->w1, mlp_k->b1, mlp_k->w2, mlp_k->b2};
  cudaError_t ce = launch_score_topk(G, desc_q, desc_k, wq, wk, hidden, e, scratch, nullptr, args, (cudaStream_t)stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "veda_tile_score_topk_noalloc");
  return ok();
}

veda_status veda_tile_sparse_attn(const veda_problem* p, const void* qp, const void* kp, const void* vp,
                                  const int32_t* idx, int32_t k_max, float scale, void* op, float* lse,
                                  void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!qp || !kp || !vp || !idx || !op) return fail(VEDA_ERR_INVALID_ARG, "NULL tensor argument");
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(vp) || !aligned16(op) || !aligned16(idx) ||
      (lse && !aligned16(lse)))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if (k_max < 1) return fail(VEDA_ERR_INVALID_ARG, "k_max must be >= 1 (got %d)", k_max);
  if (!(std::isfinite(scale))) return fail(VEDA_ERR_INVALID_ARG, "scale must be finite");
  if (sparse_attn_smem_bytes(G.d, G.S, k_max) > 227 * 1024)
    return fail(VEDA_ERR_UNSUPPORTED, "k_max = %d exceeds the shared-memory budget", k_max);
  if (G.ntmax > 32767) return fail(VEDA_ERR_UNSUPPORTED, "NT_max = %d exceeds 32767 tiles per head", G.ntmax);
  CUtensorMap tq, tk, tv;
  if ((s = encode_tile_major(G, qp, &tq)) != VEDA_OK || (s = encode_tile_major(G, kp, &tk)) != VEDA_OK ||
      (s = encode_tile_major(G, vp, &tv)) != VEDA_OK)
    return s;
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.idx = idx;
  a.k_max = k_max;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)G.d);
  a.scale_log2 = sc * 1.4426950408889634f;
  a.op = op;
  a.lse = lse;
  a.timeout_ns = g_timeout_ns;
  cudaError_t e = launch_sparse_attn(G, tq, tk, tv, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_sparse_attn");
  return ok();
}

veda_status veda_tile_sparse_attn_grid(const veda_problem* p, const void* q, const void* k, const void* v,
                                       const int32_t* idx, int32_t k_max, float scale, void* o, float* lse,
                                       void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!q || !k || !v || !idx || !o) return fail(VEDA_ERR_INVALID_ARG, "NULL tensor argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(idx) ||
      (lse && !aligned16(lse)))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if (k_max < 1) return fail(VEDA_ERR_INVALID_ARG, "k_max must be >= 1 (got %d)", k_max);
  if (!(std::isfinite(scale))) return fail(VEDA_ERR_INVALID_ARG, "scale must be finite");
  if (sparse_attn_smem_bytes(G.d, G.S, k_max) > 227 * 1024)
    return fail(VEDA_ERR_UNSUPPORTED, "k_max = %d exceeds the shared-memory budget", k_max);
  if (G.ntmax > 32767) return fail(VEDA_ERR_UNSUPPORTED, "NT_max = %d exceeds 32767 tiles per head", G.ntmax);
  // Distinct tilings in order of first appearance; a launch covers up to
  // kMaxGridMaps of them (one set of tensor maps each).
  int tiling_of_head[VEDA_MAX_HEADS];
  int distinct[VEDA_MAX_HEADS];
  int n_distinct = 0;
  for (int h = 0; h < G.heads; ++h) {
    int u = 0;
    while (u < n_distinct && !(G.g[distinct[u]].pt == G.g[h].pt && G.g[distinct[u]].ph == G.g[h].ph &&
                               G.g[distinct[u]].pw == G.g[h].pw))
      ++u;
    if (u == n_distinct) distinct[n_distinct++] = h;
    tiling_of_head[h] = u;
  }
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.idx = idx;
  a.k_max = k_max;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)G.d);
  a.scale_log2 = sc * 1.4426950408889634f;
  a.op = o;
  a.lse = lse;
  a.timeout_ns = g_timeout_ns;
  AttnMaps<kMaxGridMaps> maps;  // copied into the kernel parameters at launch
  std::memset(&maps, 0, sizeof(maps));
  for (int u0 = 0; u0 < n_distinct; u0 += kMaxGridMaps) {
    const int nu = std::min(kMaxGridMaps, n_distinct - u0);
    for (int u = 0; u < nu; ++u) {
      const HeadGeom& hg = G.g[distinct[u0 + u]];
      if ((s = encode_grid_tiles(G, q, hg, &maps.q[u])) != VEDA_OK ||
          (s = encode_grid_tiles(G, k, hg, &maps.k[u])) != VEDA_OK ||
          (s = encode_grid_tiles(G, v, hg, &maps.v[u])) != VEDA_OK)
        return s;
    }
    a.n_group = 0;
    for (int h = 0; h < G.heads; ++h) {
      const int u = tiling_of_head[h] - u0;
      if (u < 0 || u >= nu) continue;
      a.head_list[a.n_group++] = (int16_t)h;
      a.map_of_head[h] = (int8_t)u;
    }
    cudaError_t e = launch_sparse_attn_grid(G, maps, a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "veda_tile_sparse_attn_grid");
  }
  return ok();
}

veda_status veda_attn_config(const veda_problem* p, int32_t k_max, int32_t* k_stages, int32_t* v_stages,
                             size_t* smem_bytes) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (k_max < 1) return fail(VEDA_ERR_INVALID_ARG, "k_max must be >= 1 (got %d)", k_max);
  if (!k_stages || !v_stages || !smem_bytes) return fail(VEDA_ERR_INVALID_ARG, "NULL output argument");
  if (sparse_attn_smem_bytes(G.d, G.S, k_max) > 227 * 1024)
    return fail(VEDA_ERR_UNSUPPORTED, "k_max = %d exceeds the shared-memory budget", k_max);
  int ks = 0, vs = 0;
  size_t bytes = 0;
  sparse_attn_config(G.d, G.S, k_max, &ks, &vs, &bytes);
  *k_stages = ks;
  *v_stages = vs;
  *smem_bytes = bytes;
  return ok();
}

veda_status veda_tile_map_workspace(const veda_problem* p, int32_t R, size_t* bytes) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (R < 1) return fail(VEDA_ERR_INVALID_ARG, "R must be >= 1 (got %d)", R);
  if (!bytes) return fail(VEDA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = map_ws_bytes(G, R);
  return ok();
}

veda_status veda_tile_map_maxpool(const veda_problem* p, const void* qp, const void* kp, const int32_t* rows,
                                  int32_t R, float scale, float* map, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (R < 1) return fail(VEDA_ERR_INVALID_ARG, "R must be >= 1 (got %d)", R);
  if (!qp || !kp || !rows || !map || !workspace) return fail(VEDA_ERR_INVALID_ARG, "NULL tensor argument");
  if (!aligned16(qp) || !aligned16(kp) || !aligned16(map) || !aligned16(rows))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(VEDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < map_ws_bytes(G, R))
    return fail(VEDA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, map_ws_bytes(G, R));
  if ((long long)G.B * G.heads * R >= (1LL << 31)) return fail(VEDA_ERR_INVALID_ARG, "B*heads*R too large");
  if (!(std::isfinite(scale))) return fail(VEDA_ERR_INVALID_ARG, "scale must be finite");
  CUtensorMap tq, tk;
  if ((s = encode_tile_major(G, qp, &tq)) != VEDA_OK || (s = encode_tile_major(G, kp, &tk)) != VEDA_OK) return s;
  MapArgs a;
  std::memset(&a, 0, sizeof(a));
  a.rows = rows;
  a.R = R;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)G.d);
  a.scale_log2 = sc * 1.4426950408889634f;
  a.rowmax = static_cast<float*>(workspace);
  a.lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + map_rowmax_bytes(G, R));
  a.map = map;
  a.timeout_ns = g_timeout_ns;
  cudaError_t e = launch_tile_map(G, tq, tk, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_map_maxpool");
  return ok();
}

veda_status veda_tile_map_maxpool_grid(const veda_problem* p, const void* q, const void* k, const int32_t* rows,
                                       int32_t R, float scale, float* map, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (R < 1) return fail(VEDA_ERR_INVALID_ARG, "R must be >= 1 (got %d)", R);
  if (!q || !k || !rows || !map || !workspace) return fail(VEDA_ERR_INVALID_ARG, "NULL tensor argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(map) || !aligned16(rows))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(VEDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < map_ws_bytes(G, R))
    return fail(VEDA_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, map_ws_bytes(G, R));
  if ((long long)G.B * G.heads * R >= (1LL << 31)) return fail(VEDA_ERR_INVALID_ARG, "B*heads*R too large");
  if (!(std::isfinite(scale))) return fail(VEDA_ERR_INVALID_ARG, "scale must be finite");
  // Distinct tilings in order of first appearance; one pass-1 launch covers up
  // to kMaxGridMaps of them (one set of tensor maps each).
  int tiling_of_head[VEDA_MAX_HEADS];
  int distinct[VEDA_MAX_HEADS];
  int n_distinct = 0;
  for (int h = 0; h < G.heads; ++h) {
    int u = 0;
    while (u < n_distinct && !(G.g[distinct[u]].pt == G.g[h].pt && G.g[distinct[u]].ph == G.g[h].ph &&
                               G.g[distinct[u]].pw == G.g[h].pw))
      ++u;
    if (u == n_distinct) distinct[n_distinct++] = h;
    tiling_of_head[h] = u;
  }
  MapArgs a;
  std::memset(&a, 0, sizeof(a));
  a.rows = rows;
  a.R = R;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)G.d);
  a.scale_log2 = sc * 1.4426950408889634f;
  a.rowmax = static_cast<float*>(workspace);
  a.lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + map_rowmax_bytes(G, R));
  a.map = map;
  a.timeout_ns = g_timeout_ns;
  AttnMaps<kMaxGridMaps> maps;  // copied into the kernel parameters at launch
  std::memset(&maps, 0, sizeof(maps));
  for (int u0 = 0; u0 < n_distinct; u0 += kMaxGridMaps) {
    const int nu = std::min(kMaxGridMaps, n_distinct - u0);
    for (int u = 0; u < nu; ++u) {
      const HeadGeom& hg = G.g[distinct[u0 + u]];
      if ((s = encode_grid_tiles(G, q, hg, &maps.q[u])) != VEDA_OK ||
          (s = encode_grid_tiles(G, k, hg, &maps.k[u])) != VEDA_OK)
        return s;
      maps.v[u] = maps.k[u];   // unused by the map
    }
    a.n_group = 0;
    for (int h = 0; h < G.heads; ++h) {
      const int u = tiling_of_head[h] - u0;
      if (u < 0 || u >= nu) continue;
      a.head_list[a.n_group++] = (int16_t)h;
      a.map_of_head[h] = (int8_t)u;
    }
    cudaError_t e = launch_tile_map_pass1_grid(G, maps, a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "veda_tile_map_maxpool_grid (pass 1)");
  }
  cudaError_t e = launch_tile_map_pass2(G, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_tile_map_maxpool_grid (pass 2)");
  return ok();
}

veda_status veda_distill_workspace(const veda_problem* p, int32_t hidden, int32_t e, int32_t R, size_t* bytes) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (hidden < 4 || hidden > 512 || hidden % 4) return fail(VEDA_ERR_INVALID_ARG, "hidden must be a multiple of 4 in [4, 512]");
  if (e != 16 && e != 32 && e != 64 && e != 128) return fail(VEDA_ERR_INVALID_ARG, "e must be 16, 32, 64 or 128 (got %d)", e);
  if (R < 1) return fail(VEDA_ERR_INVALID_ARG, "R must be >= 1 (got %d)", R);
  if (!bytes) return fail(VEDA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = distill_ws_bytes(G, hidden, e, R);
  return ok();
}

veda_status veda_distill_loss_grad(const veda_problem* p, const float* desc_q, const float* desc_k,
                                   const veda_mlp* mlp_q, const veda_mlp* mlp_k, const float* map,
                                   const int32_t* rows, int32_t R, float* loss, const veda_mlp_grad* grad_q,
                                   const veda_mlp_grad* grad_k, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if ((s = check_mlp(mlp_q, "q")) != VEDA_OK || (s = check_mlp(mlp_k, "k")) != VEDA_OK) return s;
  if (mlp_q->hidden != mlp_k->hidden || mlp_q->e != mlp_k->e)
    return fail(VEDA_ERR_INVALID_ARG, "q and k estimators must have the same hidden and e");
  if (R < 1) return fail(VEDA_ERR_INVALID_ARG, "R must be >= 1 (got %d)", R);
  if (!desc_q || !desc_k || !map || !rows || !loss || !grad_q || !grad_k || !workspace)
    return fail(VEDA_ERR_INVALID_ARG, "NULL argument");
  const veda_mlp_grad* gs[2] = {grad_q, grad_k};
  for (const veda_mlp_grad* g : gs) {
    if (!g->w1 || !g->b1 || !g->w2 || !g->b2) return fail(VEDA_ERR_INVALID_ARG, "NULL gradient pointer");
    if (!aligned16(g->w1) || !aligned16(g->b1) || !aligned16(g->w2) || !aligned16(g->b2))
      return fail(VEDA_ERR_INVALID_ARG, "gradient pointers must be 16-byte aligned");
  }
  if (!aligned16(desc_q) || !aligned16(desc_k) || !aligned16(map) || !aligned16(rows) || !aligned16(loss))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VEDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const int e = mlp_q->e, hidden = mlp_q->hidden;
  if (workspace_bytes < distill_ws_bytes(G, hidden, e, R))
    return fail(VEDA_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu required", workspace_bytes,
                distill_ws_bytes(G, hidden, e, R));
  EstimatorWeights wq{mlp_q->w1, mlp_q->b1, mlp_q->w2, mlp_q->b2};
  EstimatorWeights wk{mlp_k->w1, mlp_k->b1, mlp_k->w2, mlp_k->b2};
  EstimatorWeights gq{grad_q->w1, grad_q->b1, grad_q->w2, grad_q->b2};
  EstimatorWeights gk{grad_k->w1, grad_k->b1, grad_k->w2, grad_k->b2};
  cudaError_t ce = launch_distill(G, desc_q, desc_k, wq, wk, hidden, e, map, rows, R, loss, gq, gk, workspace,
                                  g_timeout_ns, (cudaStream_t)stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "veda_distill_loss_grad");
  return ok();
}

veda_status veda_head_error(const veda_problem* p, const void* o, const void* o_ref, float* err, float* ref_sq,
                            void* workspace, size_t workspace_bytes, void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!o || !o_ref || !err || !ref_sq || !workspace) return fail(VEDA_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(o) || !aligned16(o_ref) || !aligned16(workspace))
    return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  const size_t need = sizeof(float) * 2 * (size_t)kHeadErrBlocks * G.heads;
  if (workspace_bytes < need) return fail(VEDA_ERR_INVALID_ARG, "workspace needs %zu bytes", need);
  cudaError_t ce = launch_head_error(G, o, o_ref, err, ref_sq, static_cast<float*>(workspace), (cudaStream_t)stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "veda_head_error");
  return ok();
}

veda_status veda_attn_backward_workspace(const veda_problem* p, int32_t k_max, size_t* bytes) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (k_max < 1) return fail(VEDA_ERR_INVALID_ARG, "k_max must be >= 1 (got %d)", k_max);
  if (!bytes) return fail(VEDA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = attn_bwd_ws_bytes(G, k_max);
  return ok();
}

veda_status veda_tile_sparse_attn_backward_grid(const veda_problem* p, const void* q, const void* k, const void* v,
                                                const void* o, const float* lse, const void* d_o,
                                                const int32_t* idx, int32_t k_max, float scale, void* dq,
                                                void* dk, void* dv, void* workspace, size_t workspace_bytes,
                                                void* stream) {
  Geometry G;
  veda_status s = make_geometry(p, &G);
  if (s != VEDA_OK) return s;
  if (!q || !k || !v || !o || !lse || !d_o || !idx || !dq || !dk || !dv || !workspace)
    return fail(VEDA_ERR_INVALID_ARG, "NULL argument");
  const void* ptrs[] = {q, k, v, o, lse, d_o, idx, dq, dk, dv};
  for (const void* x : ptrs)
    if (!aligned16(x)) return fail(VEDA_ERR_INVALID_ARG, "tensor arguments must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VEDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (k_max < 1) return fail(VEDA_ERR_INVALID_ARG, "k_max must be >= 1 (got %d)", k_max);
  if (!(std::isfinite(scale))) return fail(VEDA_ERR_INVALID_ARG, "scale must be finite");
  if (G.ntmax > 32767) return fail(VEDA_ERR_UNSUPPORTED, "NT_max = %d exceeds 32767 tiles per head", G.ntmax);
  if (workspace_bytes < attn_bwd_ws_bytes(G, k_max))
    return fail(VEDA_ERR_INVALID_ARG, "workspace of %zu bytes is below the %zu required", workspace_bytes,
                attn_bwd_ws_bytes(G, k_max));
  const cudaStream_t st = (cudaStream_t)stream;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  cudaError_t ce = launch_attn_bwd_prep(G, o, d_o, lse, idx, k_max, workspace, &a, st);
  if (ce != cudaSuccess) return cuda_fail(ce, "veda_tile_sparse_attn_backward_grid (prep)");
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)G.d);
  a.scale = sc;
  a.scale_log2 = sc * 1.4426950408889634f;
  a.timeout_ns = g_timeout_ns;
  // Distinct tilings in order of first appearance, up to kMaxGridMaps per launch.
  int tiling_of_head[VEDA_MAX_HEADS];
  int distinct[VEDA_MAX_HEADS];
  int n_distinct = 0;
  for (int h = 0; h < G.heads; ++h) {
    int u = 0;
    while (u < n_distinct && !(G.g[distinct[u]].pt == G.g[h].pt && G.g[distinct[u]].ph == G.g[h].ph &&
                               G.g[distinct[u]].pw == G.g[h].pw))
      ++u;
    if (u == n_distinct) distinct[n_distinct++] = h;
    tiling_of_head[h] = u;
  }
  BwdMaps<kMaxGridMaps> mq, mkv;   // copied into the kernel parameters at launch
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mkv, 0, sizeof(mkv));
  for (int u0 = 0; u0 < n_distinct; u0 += kMaxGridMaps) {
    const int nu = std::min(kMaxGridMaps, n_distinct - u0);
    for (int u = 0; u < nu; ++u) {
      const HeadGeom& hg = G.g[distinct[u0 + u]];
      if ((s = encode_grid_tiles(G, q, hg, &mq.a0[u])) != VEDA_OK ||
          (s = encode_grid_tiles(G, d_o, hg, &mq.a1[u])) != VEDA_OK ||
          (s = encode_grid_tiles(G, k, hg, &mq.b0[u])) != VEDA_OK ||
          (s = encode_grid_tiles(G, v, hg, &mq.b1[u])) != VEDA_OK)
        return s;
      mkv.a0[u] = mq.b0[u];   // K
      mkv.a1[u] = mq.b1[u];   // V
      mkv.b0[u] = mq.a0[u];   // Q
      mkv.b1[u] = mq.a1[u];   // dO
    }
    a.n_group = 0;
    for (int h = 0; h < G.heads; ++h) {
      const int u = tiling_of_head[h] - u0;
      if (u < 0 || u >= nu) continue;
      a.head_list[a.n_group++] = (int16_t)h;
      a.map_of_head[h] = (int8_t)u;
    }
    a.dx = dq;
    a.dv = nullptr;
    if ((ce = launch_attn_bwd_dq(G, mq, a, st)) != cudaSuccess)
      return cuda_fail(ce, "veda_tile_sparse_attn_backward_grid (dQ)");
    a.dx = dk;
    a.dv = dv;
    if ((ce = launch_attn_bwd_dkdv(G, mkv, a, st)) != cudaSuccess)
      return cuda_fail(ce, "veda_tile_sparse_attn_backward_grid (dK, dV)");
  }
  return ok();
}

veda_status veda_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_sync_status: stream synchronize");
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "veda_sync_status: read device error word");
  if (word != kErrNone) {
    int site = 0;
    if (word == kErrBounds) cudaMemcpyFromSymbol(&site, g_bounds_site, sizeof(int));
    const int zero = 0;
    cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    cudaMemcpyToSymbol(g_bounds_site, &zero, sizeof(int));
    if (word == kErrSmemAlign)
      return fail(VEDA_ERR_CUDA, "a kernel found its dynamic shared memory base not 1024-byte aligned");
    if (word == kErrBounds) {
      static const char* const files[] = {"?", "permute_tripool.cu", "score_topk.cu", "estimator.cu",
                                          "sparse_attn.cu", "tile_map.cu", "attn_bwd.cu", "distill.cu"};
      const int f = site / 10000;
      return fail(VEDA_ERR_BOUNDS, "debug bounds check failed at %s:%d; the access was skipped",
                  files[(f >= 0 && f < 8) ? f : 0], site % 10000);
    }
    return fail(VEDA_ERR_TIMEOUT, "a kernel gave up on a bounded wait (device error word %d)", word);
  }
  return ok();
}

veda_status veda_set_wait_timeout_ns(uint64_t ns) {
  if (ns < 1000ull || ns > 60000000000ull) return fail(VEDA_ERR_INVALID_ARG, "timeout must be in [1 us, 60 s]");
  g_timeout_ns = ns;
  return ok();
}

veda_status veda_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull)
    return fail(VEDA_ERR_INVALID_ARG, "timeout must be in [1 us, 10 s]");
  cudaError_t e = launch_timeout_selftest(timeout_ns, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_selftest_wait_timeout");
  return ok();
}

int32_t veda_bounds_checked(void) {
#ifdef VEDA_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

veda_status veda_selftest_bounds(void* stream) {
#ifdef VEDA_DEBUG_BOUNDS
  cudaError_t e = launch_bounds_selftest((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "veda_selftest_bounds");
  return ok();
#else
  (void)stream;
  return fail(VEDA_ERR_UNSUPPORTED, "veda_selftest_bounds: this library is a release build without bounds checks");
#endif
}

}  // extern "C"
