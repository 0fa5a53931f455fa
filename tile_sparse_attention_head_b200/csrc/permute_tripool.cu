// HBM-bound stages: the per-head tile permutation and its inverse ("head-aware
// tiling", section 2.2 of the Veda summary) and the TripPool descriptor
// (section 2.1: channel-wise mean, max and min of each tile, concatenated).
//
// Gather kernels (permutation, TripPool, both fused): one warp per
// (b, h, tile), eight per CTA, no shared memory and no CTA barrier, so an SM
// keeps dozens of tiles in flight.  A row of the tile is d channels = d/8
// 16-byte chunks; lane l owns chunk l % (d/8) of every (32 / (d/8))-th row,
// keeps 4 row loads in flight, and the lanes that share a chunk combine
// their statistics with shuffles at the end.  Slot coordinates come from
// shifts: every tiling factor is a power of two, since pt*ph*pw = S is.  All
// three TripPool entry points accumulate in exactly this order, so the
// descriptor of a tile is bit-identical whichever layout it is read from.
// Sums run in fp32; the maximum and minimum of bf16 values are exact in bf16
// and run on packed pairs.
//
// The inverse permutation: one CTA per (b, h, 128 grid rows); the slot of
// each row is computed once into shared memory, then 16-byte vectors move
// with several loads in flight per thread.
#include "veda_common.cuh"
#include "kernels.h"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 1   // bounds-check site id of this file (debug builds)

namespace veda {

constexpr int kPermThreads = 256;
constexpr int kGatherWarps = 8;     // warps (tiles) per gather CTA
// Row loads in flight per lane, and gather CTAs per SM.  Four loads per lane
// at four CTAs (32 warps) per SM keep more bytes in flight than sixteen loads
// at the two CTAs that their registers allow: TripPool from grid order at the
// Wan2.1-14B shape takes 0.283 ms for Q and K (5.5 TB/s) against 0.313 ms.
constexpr int kGatherUnroll = 4;
constexpr int kGatherMinBlocks = 4;

// Running TripPool statistics of one 16-byte chunk (8 channels).
struct Pool8 {
  float sum[8];
  __nv_bfloat162 mx[4], mn[4];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int k = 0; k < 8; ++k) sum[k] = 0.f;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(-INFINITY, -INFINITY);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(INFINITY, INFINITY);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mx[k] = lo;
      mn[k] = hi;
    }
  }
  __device__ __forceinline__ void add(const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(p[k]);
      sum[2 * k] += f.x;
      sum[2 * k + 1] += f.y;
      mx[k] = __hmax2(mx[k], p[k]);
      mn[k] = __hmin2(mn[k], p[k]);
    }
  }
  // combine with the lane `off` away (lanes that own the same chunk)
  __device__ __forceinline__ void combine_xor(int off) {
#pragma unroll
    for (int k = 0; k < 8; ++k) sum[k] += __shfl_xor_sync(0xffffffffu, sum[k], off);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t a = *reinterpret_cast<uint32_t*>(&mx[k]), b = *reinterpret_cast<uint32_t*>(&mn[k]);
      a = __shfl_xor_sync(0xffffffffu, a, off);
      b = __shfl_xor_sync(0xffffffffu, b, off);
      mx[k] = __hmax2(mx[k], *reinterpret_cast<__nv_bfloat162*>(&a));
      mn[k] = __hmin2(mn[k], *reinterpret_cast<__nv_bfloat162*>(&b));
    }
  }
  // desc[0:d] = mean, [d:2d] = max, [2d:3d] = min for this lane's 8 channels
  template <int D>
  __device__ __forceinline__ void store(float* out, int chunk, float inv_count) const {
    float4* m = reinterpret_cast<float4*>(out + 8 * chunk);
    m[0] = make_float4(sum[0] * inv_count, sum[1] * inv_count, sum[2] * inv_count, sum[3] * inv_count);
    m[1] = make_float4(sum[4] * inv_count, sum[5] * inv_count, sum[6] * inv_count, sum[7] * inv_count);
    float4* a = reinterpret_cast<float4*>(out + D + 8 * chunk);
    float4* b = reinterpret_cast<float4*>(out + 2 * D + 8 * chunk);
    const float2 x0 = __bfloat1622float2(mx[0]), x1 = __bfloat1622float2(mx[1]);
    const float2 x2 = __bfloat1622float2(mx[2]), x3 = __bfloat1622float2(mx[3]);
    a[0] = make_float4(x0.x, x0.y, x1.x, x1.y);
    a[1] = make_float4(x2.x, x2.y, x3.x, x3.y);
    const float2 n0 = __bfloat1622float2(mn[0]), n1 = __bfloat1622float2(mn[1]);
    const float2 n2 = __bfloat1622float2(mn[2]), n3 = __bfloat1622float2(mn[3]);
    b[0] = make_float4(n0.x, n0.y, n1.x, n1.y);
    b[1] = make_float4(n2.x, n2.y, n3.x, n3.y);
  }
};

// One warp per (b, h, tile j).  SRC_GRID: the rows are read from the
// grid-order tensor x [B, heads, N, d] (pad slots read nothing); otherwise
// from the tile-major tensor [B, heads, NT_max*S, d].  WRITE: the tile's S
// rows are written tile-major to xp (zeros for pad slots and for tiles
// j >= NT_h).  POOL: desc[b, h, j, :] = [mean || max || min] over the token
// slots of the tile (zeros for tiles j >= NT_h).
template <int D, int S, bool SRC_GRID, bool WRITE, bool POOL>
__global__ void __launch_bounds__(kGatherWarps * 32, kGatherMinBlocks) gather_kernel(const __grid_constant__ Geometry G,
                                                                   const uint4* __restrict__ src,
                                                                   uint4* __restrict__ xp,
                                                                   float* __restrict__ desc) {
  constexpr int CPR = D / 8;       // 16-byte chunks per row
  constexpr int RPI = 32 / CPR;    // rows per warp step
  constexpr int STEPS = S / RPI;
  constexpr int UNR = STEPS < kGatherUnroll ? STEPS : kGatherUnroll;
  static_assert(STEPS % UNR == 0, "");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kGatherWarps + warp;
  if (gw >= (long long)G.B * G.heads * G.ntmax) return;   // warp-uniform
  const int bh = (int)(gw / G.ntmax), j = (int)(gw % G.ntmax);
  const HeadGeom hg = G.g[bh % G.heads];
  const int chunk = lane % CPR, r0 = lane / CPR;
  uint4* xo = WRITE ? xp + (size_t)gw * S * CPR + chunk : nullptr;
  if (j >= hg.nt) {
    if constexpr (WRITE) {
#pragma unroll 4
      for (int st = 0; st < STEPS; ++st) xo[(size_t)(st * RPI + r0) * CPR] = make_uint4(0u, 0u, 0u, 0u);
    }
    if constexpr (POOL) {
      float4* out = reinterpret_cast<float4*>(desc + gw * 3 * D);
      for (int c = lane; c < 3 * D / 4; c += 32) out[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  const int jw = j % hg.nTw, jh = (j / hg.nTw) % hg.nTh, jt = j / (hg.nTw * hg.nTh);
  const int t0 = jt * hg.pt, y0 = jh * hg.ph, x0 = jw * hg.pw;
  const int ct = min((int)hg.pt, G.T - t0), ch = min((int)hg.ph, G.H - y0), cw = min((int)hg.pw, G.W - x0);
  const int sw = __ffs(hg.pw) - 1, sh = __ffs(hg.ph) - 1;   // log2 of the factors
  const uint4* sb = SRC_GRID ? src + (size_t)bh * G.N * CPR + chunk : src + (size_t)gw * S * CPR + chunk;
  Pool8 st8;
  if constexpr (POOL) st8.init();
#pragma unroll 1
  for (int s0 = 0; s0 < STEPS; s0 += UNR) {
    uint4 v[UNR];
    bool ok[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int l = (s0 + u) * RPI + r0;   // slot of this row
      const int ow = l & (hg.pw - 1), oh = (l >> sw) & (hg.ph - 1), ot = l >> (sw + sh);
      ok[u] = ot < ct && oh < ch && ow < cw;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (ok[u]) {
        const size_t row = SRC_GRID ? ((size_t)(t0 + ot) * G.H + (y0 + oh)) * G.W + (x0 + ow) : (size_t)l;
        if (VEDA_IN_BOUNDS(row < (SRC_GRID ? (size_t)G.N : (size_t)S))) v[u] = __ldg(sb + row * CPR);
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      if constexpr (WRITE) {
        if (VEDA_IN_BOUNDS((s0 + u) * RPI + r0 < S)) xo[(size_t)((s0 + u) * RPI + r0) * CPR] = v[u];
      }
      if constexpr (POOL) {
        if (ok[u]) st8.add(v[u]);
      }
    }
  }
  if constexpr (POOL) {
#pragma unroll
    for (int off = CPR; off < 32; off <<= 1) st8.combine_xor(off);
    if (lane < CPR) st8.store<D>(desc + gw * 3 * D, chunk, 1.0f / (float)(ct * ch * cw));
  }
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
    if (pos >= 0 && VEDA_IN_BOUNDS(pos < G.ntmax * G.S)) v[p] = __ldg(xi + (size_t)pos * CPR + chunk);
  }
#pragma unroll
  for (int p = 0; p < PASSES; ++p)
    if (s_pos[r0 + p * RPP] >= 0 && VEDA_IN_BOUNDS(n0 + r0 + p * RPP < G.N))
      xo[(size_t)(r0 + p * RPP) * CPR + chunk] = v[p];
}

template <bool SRC_GRID, bool WRITE, bool POOL>
static cudaError_t launch_gather_t(const Geometry& G, const void* src, void* xp, float* desc, cudaStream_t s) {
  const long long tiles = (long long)G.B * G.heads * G.ntmax;
  const unsigned blocks = (unsigned)((tiles + kGatherWarps - 1) / kGatherWarps);
  const uint4* in = (const uint4*)src;
  uint4* out = (uint4*)xp;
  constexpr int T = kGatherWarps * 32;
  if (G.d == 128 && G.S == 128) gather_kernel<128, 128, SRC_GRID, WRITE, POOL><<<blocks, T, 0, s>>>(G, in, out, desc);
  else if (G.d == 128) gather_kernel<128, 64, SRC_GRID, WRITE, POOL><<<blocks, T, 0, s>>>(G, in, out, desc);
  else if (G.S == 128) gather_kernel<64, 128, SRC_GRID, WRITE, POOL><<<blocks, T, 0, s>>>(G, in, out, desc);
  else gather_kernel<64, 64, SRC_GRID, WRITE, POOL><<<blocks, T, 0, s>>>(G, in, out, desc);
  return cudaGetLastError();
}

cudaError_t launch_permute(const Geometry& G, const void* x, void* xp, cudaStream_t s, int sms) {
  (void)sms;
  return launch_gather_t<true, true, false>(G, x, xp, nullptr, s);
}

cudaError_t launch_permute_tripool(const Geometry& G, const void* x, void* xp, float* desc, cudaStream_t s) {
  return launch_gather_t<true, true, true>(G, x, xp, desc, s);
}

cudaError_t launch_tripool_grid(const Geometry& G, const void* x, float* desc, cudaStream_t s) {
  return launch_gather_t<true, false, true>(G, x, nullptr, desc, s);
}

cudaError_t launch_tripool(const Geometry& G, const void* xp, float* desc, cudaStream_t s) {
  return launch_gather_t<false, false, true>(G, xp, nullptr, desc, s);
}

cudaError_t launch_unpermute(const Geometry& G, const void* xp, void* x, cudaStream_t s, int sms) {
  (void)sms;
  dim3 grid((G.N + 127) / 128, G.B * G.heads);
  if (G.d == 128) unpermute_kernel<128><<<grid, kPermThreads, 0, s>>>(G, (const uint4*)xp, (uint4*)x);
  else unpermute_kernel<64><<<grid, kPermThreads, 0, s>>>(G, (const uint4*)xp, (uint4*)x);
  return cudaGetLastError();
}

}  // namespace veda
