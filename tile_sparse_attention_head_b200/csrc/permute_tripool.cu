// HBM-bound stages: the per-head tile permutation and its inverse ("head-aware
// tiling", section 2.2 of the Veda summary) and the TripPool descriptor
// (section 2.1: channel-wise mean, max and min of each tile, concatenated).
//
// Layout of the work: one CTA per (b, h, tile) for the permutation, one per
// (b, h, 128 grid rows) for the inverse.  The index arithmetic (divisions by
// the tiling factors) is done once per row by one thread into shared memory;
// the copy phase then moves 16-byte vectors (8 bf16 channels) with every
// thread keeping several independent loads in flight, so whole 128-byte lines
// move per warp.  The permutation can also produce the TripPool descriptor
// of the tile it is writing (fused: the tile is read from HBM once).
#include "veda_common.cuh"
#include "kernels.h"

namespace veda {

constexpr int kPermThreads = 256;

// Per-thread running statistics of 8 channels.
struct Stats8 {
  float sum[8], mx[8], mn[8];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      sum[k] = 0.f;
      mx[k] = -INFINITY;
      mn[k] = INFINITY;
    }
  }
  __device__ __forceinline__ void add(const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(p[k]);
      sum[2 * k] += f.x;
      sum[2 * k + 1] += f.y;
      mx[2 * k] = fmaxf(mx[2 * k], f.x);
      mx[2 * k + 1] = fmaxf(mx[2 * k + 1], f.y);
      mn[2 * k] = fminf(mn[2 * k], f.x);
      mn[2 * k + 1] = fminf(mn[2 * k + 1], f.y);
    }
  }
};

// Combines the per-thread statistics of all threads that own the same
// 16-byte chunk of a row (threads tid, tid + CPR, ...) and writes
// desc = [mean || max || min] for the tile.  `red` holds 3 * 256 * 8 floats.
template <int D>
__device__ __forceinline__ void tripool_reduce_store(const Stats8& st, float* red, int count, float* out) {
  constexpr int CPR = D / 8;
  constexpr int GROUPS = kPermThreads / CPR;
  const int tid = threadIdx.x;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    red[(0 * kPermThreads + tid) * 8 + k] = st.sum[k];
    red[(1 * kPermThreads + tid) * 8 + k] = st.mx[k];
    red[(2 * kPermThreads + tid) * 8 + k] = st.mn[k];
  }
  __syncthreads();
  // Thread c (< D) finishes channel c: chunk c/8, lane-in-chunk c%8.
  for (int c = tid; c < D; c += kPermThreads) {
    const int chunk = c >> 3, k = c & 7;
    float s = 0.f, mx = -INFINITY, mn = INFINITY;
#pragma unroll 4
    for (int g = 0; g < GROUPS; ++g) {
      const int t = g * CPR + chunk;
      s += red[(0 * kPermThreads + t) * 8 + k];
      mx = fmaxf(mx, red[(1 * kPermThreads + t) * 8 + k]);
      mn = fminf(mn, red[(2 * kPermThreads + t) * 8 + k]);
    }
    out[c] = s / (float)count;
    out[D + c] = mx;
    out[2 * D + c] = mn;
  }
}

// grid: (NT_max, B*heads).  Gathers tile j of head h from the grid-order
// tensor.  With WRITE, writes all S rows of it (zeros for pad slots and tiles
// j >= NT_h); with POOL, also desc[b, h, j, :].  POOL without WRITE is the
// TripPool of a grid-order tensor (no permuted copy is made).
template <int D, int S, bool POOL, bool WRITE = true>
__global__ void __launch_bounds__(kPermThreads) permute_kernel(const __grid_constant__ Geometry G,
                                                               const uint4* __restrict__ x,
                                                               uint4* __restrict__ xp,
                                                               float* __restrict__ desc) {
  constexpr int CPR = D / 8;                        // 16-byte chunks per row
  constexpr int RPP = kPermThreads / CPR;           // rows per pass
  constexpr int PASSES = S / RPP;
  __shared__ int s_src[S];
  __shared__ float s_red[POOL ? 3 * kPermThreads * 8 : 1];
  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const HeadGeom& hg = G.g[h];
  const int tid = threadIdx.x;
  const bool live = j < hg.nt;
  if (tid < S) s_src[tid] = live ? slot_to_grid(G, hg, j, tid) : -1;
  __syncthreads();

  const uint4* xb = x + (size_t)bh * G.N * CPR;
  const int chunk = tid % CPR, r0 = tid / CPR;
  uint4 v[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int n = s_src[r0 + p * RPP];
    v[p] = (n >= 0) ? __ldg(xb + (size_t)n * CPR + chunk) : make_uint4(0u, 0u, 0u, 0u);
  }
  if constexpr (WRITE) {
    uint4* xo = xp + ((size_t)bh * G.ntmax + j) * (size_t)S * CPR;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) xo[(size_t)(r0 + p * RPP) * CPR + chunk] = v[p];
  }

  if constexpr (POOL) {
    float* out = desc + ((size_t)bh * G.ntmax + j) * 3 * D;
    if (!live) {
      for (int c = tid; c < 3 * D; c += kPermThreads) out[c] = 0.f;
      return;
    }
    Stats8 st;
    st.init();
#pragma unroll
    for (int p = 0; p < PASSES; ++p)
      if (s_src[r0 + p * RPP] >= 0) st.add(v[p]);
    tripool_reduce_store<D>(st, s_red, tile_token_count(G, hg, j), out);
  }
}

// TripPool alone, from an already permuted tensor.  grid: (NT_max, B*heads).
template <int D, int S>
__global__ void __launch_bounds__(kPermThreads) tripool_kernel(const __grid_constant__ Geometry G,
                                                               const uint4* __restrict__ xp,
                                                               float* __restrict__ desc) {
  constexpr int CPR = D / 8;
  constexpr int RPP = kPermThreads / CPR;
  constexpr int PASSES = S / RPP;
  __shared__ unsigned char s_valid[S];
  __shared__ float s_red[3 * kPermThreads * 8];
  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const HeadGeom& hg = G.g[h];
  const int tid = threadIdx.x;
  float* out = desc + ((size_t)bh * G.ntmax + j) * 3 * D;
  if (j >= hg.nt) {
    for (int c = tid; c < 3 * D; c += kPermThreads) out[c] = 0.f;
    return;
  }
  if (tid < S) s_valid[tid] = slot_to_grid(G, hg, j, tid) >= 0;
  __syncthreads();
  const uint4* xi = xp + ((size_t)bh * G.ntmax + j) * (size_t)S * CPR;
  const int chunk = tid % CPR, r0 = tid / CPR;
  uint4 v[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) v[p] = __ldg(xi + (size_t)(r0 + p * RPP) * CPR + chunk);
  Stats8 st;
  st.init();
#pragma unroll
  for (int p = 0; p < PASSES; ++p)
    if (s_valid[r0 + p * RPP]) st.add(v[p]);
  tripool_reduce_store<D>(st, s_red, tile_token_count(G, hg, j), out);
}

// X[b,h, n, :] = Xp[b,h, pos_h(n), :].  grid: (ceil(N / 128), B*heads).
template <int D>
__global__ void __launch_bounds__(kPermThreads) unpermute_kernel(const __grid_constant__ Geometry G,
                                                                 const uint4* __restrict__ xp,
                                                                 uint4* __restrict__ x) {
  constexpr int CPR = D / 8;
  constexpr int ROWS = 128;
  constexpr int RPP = kPermThreads / CPR;
  constexpr int PASSES = ROWS / RPP;
  __shared__ int s_pos[ROWS];
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const int n0 = blockIdx.x * ROWS;
  const int tid = threadIdx.x;
  if (tid < ROWS) s_pos[tid] = (n0 + tid < G.N) ? grid_to_slot(G, G.g[h], n0 + tid) : -1;
  __syncthreads();
  const uint4* xi = xp + (size_t)bh * G.ntmax * G.S * CPR;
  uint4* xo = x + ((size_t)bh * G.N + n0) * CPR;
  const int chunk = tid % CPR, r0 = tid / CPR;
  uint4 v[PASSES];
#pragma unroll
  for (int p = 0; p < PASSES; ++p) {
    const int pos = s_pos[r0 + p * RPP];
    if (pos >= 0) v[p] = __ldg(xi + (size_t)pos * CPR + chunk);
  }
#pragma unroll
  for (int p = 0; p < PASSES; ++p)
    if (s_pos[r0 + p * RPP] >= 0) xo[(size_t)(r0 + p * RPP) * CPR + chunk] = v[p];
}

template <bool POOL>
static cudaError_t launch_permute_t(const Geometry& G, const void* x, void* xp, float* desc, cudaStream_t s) {
  dim3 grid(G.ntmax, G.B * G.heads);
  const uint4* xi = (const uint4*)x;
  uint4* xo = (uint4*)xp;
  if (G.d == 128 && G.S == 128) permute_kernel<128, 128, POOL><<<grid, kPermThreads, 0, s>>>(G, xi, xo, desc);
  else if (G.d == 128) permute_kernel<128, 64, POOL><<<grid, kPermThreads, 0, s>>>(G, xi, xo, desc);
  else if (G.S == 128) permute_kernel<64, 128, POOL><<<grid, kPermThreads, 0, s>>>(G, xi, xo, desc);
  else permute_kernel<64, 64, POOL><<<grid, kPermThreads, 0, s>>>(G, xi, xo, desc);
  return cudaGetLastError();
}

cudaError_t launch_permute(const Geometry& G, const void* x, void* xp, cudaStream_t s, int sms) {
  (void)sms;
  return launch_permute_t<false>(G, x, xp, nullptr, s);
}

cudaError_t launch_permute_tripool(const Geometry& G, const void* x, void* xp, float* desc, cudaStream_t s) {
  return launch_permute_t<true>(G, x, xp, desc, s);
}

cudaError_t launch_unpermute(const Geometry& G, const void* xp, void* x, cudaStream_t s, int sms) {
  (void)sms;
  dim3 grid((G.N + 127) / 128, G.B * G.heads);
  if (G.d == 128) unpermute_kernel<128><<<grid, kPermThreads, 0, s>>>(G, (const uint4*)xp, (uint4*)x);
  else unpermute_kernel<64><<<grid, kPermThreads, 0, s>>>(G, (const uint4*)xp, (uint4*)x);
  return cudaGetLastError();
}

cudaError_t launch_tripool_grid(const Geometry& G, const void* x, float* desc, cudaStream_t s) {
  dim3 grid(G.ntmax, G.B * G.heads);
  const uint4* xi = (const uint4*)x;
  if (G.d == 128 && G.S == 128) permute_kernel<128, 128, true, false><<<grid, kPermThreads, 0, s>>>(G, xi, nullptr, desc);
  else if (G.d == 128) permute_kernel<128, 64, true, false><<<grid, kPermThreads, 0, s>>>(G, xi, nullptr, desc);
  else if (G.S == 128) permute_kernel<64, 128, true, false><<<grid, kPermThreads, 0, s>>>(G, xi, nullptr, desc);
  else permute_kernel<64, 64, true, false><<<grid, kPermThreads, 0, s>>>(G, xi, nullptr, desc);
  return cudaGetLastError();
}

cudaError_t launch_tripool(const Geometry& G, const void* xp, float* desc, cudaStream_t s) {
  dim3 grid(G.ntmax, G.B * G.heads);
  const uint4* xi = (const uint4*)xp;
  if (G.d == 128 && G.S == 128) tripool_kernel<128, 128><<<grid, kPermThreads, 0, s>>>(G, xi, desc);
  else if (G.d == 128) tripool_kernel<128, 64><<<grid, kPermThreads, 0, s>>>(G, xi, desc);
  else if (G.S == 128) tripool_kernel<64, 128><<<grid, kPermThreads, 0, s>>>(G, xi, desc);
  else tripool_kernel<64, 64><<<grid, kPermThreads, 0, s>>>(G, xi, desc);
  return cudaGetLastError();
}

}  // namespace veda
