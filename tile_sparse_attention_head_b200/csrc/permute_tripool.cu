// HBM-bound stages: the per-head tile permutation and its inverse ("head-aware
// tiling", section 2.2 of the Veda summary) and the TripPool descriptor
// (section 2.1: channel-wise mean, max and min of each tile, concatenated).
//
// All three move 16-byte vectors (8 bf16 channels) per thread so every warp
// touches whole 128-byte lines; the permutations are output-driven so each
// output row is written exactly once (pad slots as zeros).
#include "veda_common.cuh"
#include "kernels.h"

namespace veda {

// Xp[b,h, j*S + l, :] = X[b,h, n(j,l), :], zeros for pad slots and j >= NT_h.
// One thread per 16-byte chunk of an output row; grid-stride.
__global__ void __launch_bounds__(256) permute_kernel(const __grid_constant__ Geometry G,
                                                      const uint4* __restrict__ x,
                                                      uint4* __restrict__ xp) {
  const int cpr = G.d >> 3;  // 16-byte chunks per row
  const long long rows_per_head = (long long)G.ntmax * G.S;
  const long long total = (long long)G.B * G.heads * rows_per_head * cpr;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < total;
       c += (long long)gridDim.x * blockDim.x) {
    const int chunk = (int)(c % cpr);
    const long long row = c / cpr;
    const int r = (int)(row % rows_per_head);
    const long long bh = row / rows_per_head;
    const int h = (int)(bh % G.heads);
    const HeadGeom& hg = G.g[h];
    const int j = r / G.S, l = r % G.S;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < hg.nt) {
      const int n = slot_to_grid(G, hg, j, l);
      if (n >= 0) v = __ldg(x + ((bh * G.N + n) * cpr + chunk));
    }
    xp[c] = v;
  }
}

// X[b,h, n, :] = Xp[b,h, pos_h(n), :].  One thread per 16-byte chunk of a grid row.
__global__ void __launch_bounds__(256) unpermute_kernel(const __grid_constant__ Geometry G,
                                                        const uint4* __restrict__ xp,
                                                        uint4* __restrict__ x) {
  const int cpr = G.d >> 3;
  const long long rows_per_head_p = (long long)G.ntmax * G.S;
  const long long total = (long long)G.B * G.heads * G.N * cpr;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < total;
       c += (long long)gridDim.x * blockDim.x) {
    const int chunk = (int)(c % cpr);
    const long long row = c / cpr;
    const int n = (int)(row % G.N);
    const long long bh = row / G.N;
    const int h = (int)(bh % G.heads);
    const int pos = grid_to_slot(G, G.g[h], n);
    x[c] = __ldg(xp + ((bh * rows_per_head_p + pos) * cpr + chunk));
  }
}

// TripPool: one warp per (b, h, tile).  Lanes split a tile row into 16-byte
// chunks (8 channels); with d = 128 a warp covers 2 rows per step, with
// d = 64 four.  Each lane keeps fp32 sum / max / min of its 8 channels over
// the token slots it visits; lanes sharing a chunk are then combined by
// shuffles.  desc = [mean || max || min], fp32.
template <int D>
__global__ void __launch_bounds__(256) tripool_kernel(const __grid_constant__ Geometry G,
                                                      const uint4* __restrict__ xp,
                                                      float* __restrict__ desc) {
  constexpr int CPR = D / 8;          // chunks per row
  constexpr int RPS = 32 / CPR;       // rows per warp step
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long ntiles = (long long)G.B * G.heads * G.ntmax;
  if (warp >= ntiles) return;
  const int j = (int)(warp % G.ntmax);
  const long long bh = warp / G.ntmax;
  const int h = (int)(bh % G.heads);
  const HeadGeom& hg = G.g[h];
  float* out = desc + (long long)warp * 3 * D;
  const int chunk = lane % CPR;
  if (j >= hg.nt) {
    for (int c = lane; c < 3 * D; c += 32) out[c] = 0.f;
    return;
  }
  float sum[8], mx[8], mn[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    sum[k] = 0.f;
    mx[k] = -INFINITY;
    mn[k] = INFINITY;
  }
  const uint4* base = xp + ((bh * G.ntmax + j) * (long long)G.S) * CPR;
  const int full = (tile_token_count(G, hg, j) == G.S);
  for (int r0 = 0; r0 < G.S; r0 += RPS) {
    const int l = r0 + lane / CPR;
    if (!full && slot_to_grid(G, hg, j, l) < 0) continue;
    const uint4 v = __ldg(base + (long long)l * CPR + chunk);
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
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      sum[k] += __shfl_xor_sync(0xffffffffu, sum[k], off);
      mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], off));
      mn[k] = fminf(mn[k], __shfl_xor_sync(0xffffffffu, mn[k], off));
    }
  }
  if (lane < CPR) {
    const float inv = 1.0f / (float)tile_token_count(G, hg, j);
    float4* o_mean = reinterpret_cast<float4*>(out + chunk * 8);
    float4* o_max = reinterpret_cast<float4*>(out + D + chunk * 8);
    float4* o_min = reinterpret_cast<float4*>(out + 2 * D + chunk * 8);
    o_mean[0] = make_float4(sum[0] * inv, sum[1] * inv, sum[2] * inv, sum[3] * inv);
    o_mean[1] = make_float4(sum[4] * inv, sum[5] * inv, sum[6] * inv, sum[7] * inv);
    o_max[0] = make_float4(mx[0], mx[1], mx[2], mx[3]);
    o_max[1] = make_float4(mx[4], mx[5], mx[6], mx[7]);
    o_min[0] = make_float4(mn[0], mn[1], mn[2], mn[3]);
    o_min[1] = make_float4(mn[4], mn[5], mn[6], mn[7]);
  }
}

static int grid_for(long long work, int threads, int sms) {
  long long blocks = (work + threads - 1) / threads;
  const long long cap = (long long)sms * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

cudaError_t launch_permute(const Geometry& G, const void* x, void* xp, cudaStream_t s, int sms) {
  const long long work = (long long)G.B * G.heads * G.ntmax * G.S * (G.d / 8);
  permute_kernel<<<grid_for(work, 256, sms), 256, 0, s>>>(G, (const uint4*)x, (uint4*)xp);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const Geometry& G, const void* xp, void* x, cudaStream_t s, int sms) {
  const long long work = (long long)G.B * G.heads * G.N * (G.d / 8);
  unpermute_kernel<<<grid_for(work, 256, sms), 256, 0, s>>>(G, (const uint4*)xp, (uint4*)x);
  return cudaGetLastError();
}

cudaError_t launch_tripool(const Geometry& G, const void* xp, float* desc, cudaStream_t s) {
  const long long warps = (long long)G.B * G.heads * G.ntmax;
  const int blocks = (int)((warps * 32 + 255) / 256);
  if (G.d == 128)
    tripool_kernel<128><<<blocks, 256, 0, s>>>(G, (const uint4*)xp, desc);
  else
    tripool_kernel<64><<<blocks, 256, 0, s>>>(G, (const uint4*)xp, desc);
  return cudaGetLastError();
}

}  // namespace veda
