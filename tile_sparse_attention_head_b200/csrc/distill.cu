// Training the estimator: the row-wise KL distillation loss and its gradients
// (section 2.1 of the Veda summary, "Optimization": the predicted
// distribution of tile scores is aligned row by row with the full-attention
// reference -- the max-pooled tile map -- by a KL divergence; the backbone
// features feeding the estimator are stop-gradient).
//
// For every subset row (b, h, r) with Q tile i = rows[b*heads+h, r]:
//   T = map[b, h, r, :NT_h] / sum,  P = softmax_j s[i, j],
//   s[i, j] = <phi_q(i), phi_k(j)> / sqrt(e),
//   L = mean over valid rows of KL(T || P),  dL/ds[i, :] = (P - T) / n_rows.
// Then back through s to phi_q(i) and phi_k(j), and through each MLP
// phi = W2 relu(z) + b2, z = W1 desc + b1, to (W1, b1, W2, b2) of both sides.
// The descriptors get no gradient.
//
// Kernels, in launch order (the estimator forward runs first, keeping its
// hidden activations a = relu(z)):
//   distill_count_kernel   number of valid subset rows;
//   distill_rows_kernel    one CTA per subset row: scores against every K tile
//                          of the head, row softmax, normalised target, the
//                          row's KL, dL/ds, and dphi_q of that row;
//   distill_dphik_kernel   dphi_k(j) = sum_r dL/ds[r, j] phi_q(rows[r]) / sqrt(e);
//   distill_loss_kernel    the mean of the row losses, summed in a fixed order;
//   grad_reduce_kernel     dW = sum over (b, tile) of X^T Y: dW2 from (dphi, a),
//                          dW1 from (dz, desc); bias_reduce_kernel sums dphi
//                          and dz into db2 and db1;
//   dz_kernel              dz = (dphi W2) * [a > 0], written over a.
// All fp32 on the CUDA cores: these are small reductions next to the layer.
#pragma once
#include "veda_common.cuh"
#include "kernels.h"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 7   // bounds-check site id of this file (debug builds)

namespace veda {

constexpr int kDistillThreads = 256;

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];   // same order in every thread
  return t;
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = fmaxf(t, red[w]);
  return t;
}

__global__ void distill_count_kernel(const __grid_constant__ Geometry G, const int32_t* __restrict__ rows, int R,
                                     int* __restrict__ count) {
  __shared__ float red[32];
  float c = 0.f;
  const int total = G.B * G.heads * R;
  for (int x = threadIdx.x; x < total; x += blockDim.x) {
    const int bh = x / R;
    const int i = rows[x];
    c += (i >= 0 && i < G.g[bh % G.heads].nt) ? 1.f : 0.f;
  }
  c = block_reduce_sum(c, red);
  if (threadIdx.x == 0) *count = (int)c;
}

__global__ void fill_zero_kernel(float4* __restrict__ p, long long n4) {
  for (long long x = blockIdx.x * (long long)blockDim.x + threadIdx.x; x < n4; x += (long long)gridDim.x * blockDim.x)
    p[x] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// grid (R, B*heads).  g [B*heads, R, NT_max] (zero outside valid rows and
// columns), row_loss [B*heads, R], dphi_q rows of the subset.
template <int E>
__global__ void __launch_bounds__(kDistillThreads)
    distill_rows_kernel(const __grid_constant__ Geometry G, const float* __restrict__ phi,
                        const float* __restrict__ map, const int32_t* __restrict__ rows, int R,
                        const int* __restrict__ n_valid, float* __restrict__ g, float* __restrict__ row_loss,
                        float* __restrict__ dphi) {
  __shared__ __align__(16) float s_phq[E];
  __shared__ float red[32];
  __shared__ float s_part[kDistillThreads];
  const int r = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int nt = G.g[bh % G.heads].nt;
  const long long row_id = (long long)bh * R + r;
  float* grow = g + row_id * G.ntmax;
  const int i = rows[row_id];
  if (i < 0 || i >= nt) {
    for (int j = tid; j < G.ntmax; j += kDistillThreads) grow[j] = 0.f;
    if (tid == 0) row_loss[row_id] = 0.f;
    return;
  }
  const long long BH = (long long)G.B * G.heads;
  const float inv_n = 1.0f / (float)max(*n_valid, 1);
  const float inv_sqrt_e = 1.0f / sqrtf((float)E);
  const float* phq = phi + ((long long)bh * G.ntmax + i) * E;
  const float* phk = phi + ((BH + bh) * G.ntmax) * E;
  const float* mrow = map + row_id * G.ntmax;
  if (tid < E) s_phq[tid] = phq[tid];
  __syncthreads();

  // scores and the target's normaliser
  float lmax = -INFINITY, lmsum = 0.f;
  for (int j = tid; j < nt; j += kDistillThreads) {
    const float4* kr = reinterpret_cast<const float4*>(phk + (long long)j * E);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < E / 4; ++c) {
      const float4 kv = __ldg(kr + c);
      const float4 qv = reinterpret_cast<const float4*>(s_phq)[c];
      acc = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, acc))));
    }
    const float s = acc * inv_sqrt_e;
    grow[j] = s;
    lmax = fmaxf(lmax, s);
    lmsum += mrow[j];
  }
  const float M = block_reduce_max(lmax, red);
  const float msum = block_reduce_sum(lmsum, red);
  float lz = 0.f;
  for (int j = tid; j < nt; j += kDistillThreads) lz += expf(grow[j] - M);
  const float logZ = M + logf(block_reduce_sum(lz, red));
  const float inv_msum = 1.0f / msum;
  float lloss = 0.f;
  for (int j = tid; j < nt; j += kDistillThreads) {
    const float t = mrow[j] * inv_msum;
    const float lp = grow[j] - logZ;
    if (t > 0.f) lloss += t * (logf(t) - lp);
    grow[j] = (expf(lp) - t) * inv_n;
  }
  for (int j = nt + tid; j < G.ntmax; j += kDistillThreads) grow[j] = 0.f;
  const float loss = block_reduce_sum(lloss, red);
  if (tid == 0) row_loss[row_id] = loss;

  // dphi_q(i) = sum_j dL/ds[i, j] phi_k(j) / sqrt(e); thread (o, jg)
  __syncthreads();   // every g of the row is written
  constexpr int GR = kDistillThreads / E;
  const int o = tid % E, jg = tid / E;
  float acc = 0.f;
  for (int j = jg; j < nt; j += GR) acc = fmaf(grow[j], __ldg(phk + (long long)j * E + o), acc);
  s_part[tid] = acc;
  __syncthreads();
  if (jg == 0) {
    float t = 0.f;
    for (int q = 0; q < GR; ++q) t += s_part[q * E + o];
    dphi[((long long)bh * G.ntmax + i) * E + o] = t * inv_sqrt_e;
  }
}

// grid (ceil(NT_max / 32), B*heads).  dphi_k(j) for 32 K tiles per CTA.
template <int E>
__global__ void __launch_bounds__(kDistillThreads)
    distill_dphik_kernel(const __grid_constant__ Geometry G, const float* __restrict__ phi,
                         const int32_t* __restrict__ rows, int R, const float* __restrict__ g,
                         float* __restrict__ dphi) {
  const int bh = blockIdx.y, j0 = blockIdx.x * 32, tid = threadIdx.x;
  const int nt = G.g[bh % G.heads].nt;
  const long long BH = (long long)G.B * G.heads;
  const float inv_sqrt_e = 1.0f / sqrtf((float)E);
  float* out = dphi + ((BH + bh) * G.ntmax) * E;
  for (int x = tid; x < 32 * E; x += kDistillThreads) {
    const int jj = x / E, o = x % E, j = j0 + jj;
    if (j >= G.ntmax) continue;
    float acc = 0.f;
    if (j < nt) {
      for (int r = 0; r < R; ++r) {
        const int i = rows[(long long)bh * R + r];
        if (i < 0 || i >= nt) continue;
        acc = fmaf(g[((long long)bh * R + r) * G.ntmax + j], phi[((long long)bh * G.ntmax + i) * E + o], acc);
      }
    }
    out[(long long)j * E + o] = acc * inv_sqrt_e;
  }
}

__global__ void distill_loss_kernel(const float* __restrict__ row_loss, int n, const int* __restrict__ n_valid,
                                    float* __restrict__ loss) {
  __shared__ float red[32];
  float t = 0.f;
  for (int x = threadIdx.x; x < n; x += blockDim.x) t += row_loss[x];
  t = block_reduce_sum(t, red);
  if (threadIdx.x == 0) *loss = t / (float)max(*n_valid, 1);
}

// dW[h][m][n] = sum_{b, t < NT_h} X[b, h, t, m] Y[b, h, t, n]; X [B, heads,
// NT_max, M], Y [B, heads, NT_max, N], dW [heads, M, N].  grid
// (ceil(M/64) * ceil(N/64), heads); 64 x 64 tile, k chunks of 16, 4 x 4 per
// thread.  M and N are multiples of 4.
__global__ void __launch_bounds__(256)
    grad_reduce_kernel(const __grid_constant__ Geometry G, const float* __restrict__ X, int M,
                       const float* __restrict__ Y, int N, float* __restrict__ dW) {
  __shared__ __align__(16) float xs[16][64];
  __shared__ __align__(16) float ys[16][64];
  const int h = blockIdx.y;
  const int tiles_n = (N + 63) / 64;
  const int m0 = (blockIdx.x / tiles_n) * 64, n0 = (blockIdx.x % tiles_n) * 64;
  const int nt = G.g[h].nt;
  const int K = G.B * nt;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    __syncthreads();
    {
      const int kk = tid >> 4, c4 = (tid & 15) * 4;   // 16 rows x 16 float4
      const int k = k0 + kk;
      float4 xv = make_float4(0.f, 0.f, 0.f, 0.f), yv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < K) {
        const int b = k / nt, t = k % nt;
        const long long rowi = ((long long)(b * G.heads + h) * G.ntmax + t);
        if (m0 + c4 < M) xv = __ldg(reinterpret_cast<const float4*>(X + rowi * M + m0 + c4));
        if (n0 + c4 < N) yv = __ldg(reinterpret_cast<const float4*>(Y + rowi * N + n0 + c4));
      }
      *reinterpret_cast<float4*>(&xs[kk][c4]) = xv;
      *reinterpret_cast<float4*>(&ys[kk][c4]) = yv;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&ys[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(av[p], bw[q], acc[p][q]);
    }
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int m = m0 + ty * 4 + p;
    if (m >= M) continue;
    if (n0 + tx * 4 < N)
      *reinterpret_cast<float4*>(dW + ((long long)h * M + m) * N + n0 + tx * 4) =
          make_float4(acc[p][0], acc[p][1], acc[p][2], acc[p][3]);
  }
}

// db[h][m] = sum_{b, t < NT_h} X[b, h, t, m].  grid (heads), one thread per m.
__global__ void bias_reduce_kernel(const __grid_constant__ Geometry G, const float* __restrict__ X, int M,
                                   float* __restrict__ db) {
  const int h = blockIdx.x;
  const int nt = G.g[h].nt;
  for (int m = threadIdx.x; m < M; m += blockDim.x) {
    float t = 0.f;
    for (int b = 0; b < G.B; ++b)
      for (int j = 0; j < nt; ++j) t += X[((long long)(b * G.heads + h) * G.ntmax + j) * M + m];
    db[(long long)h * M + m] = t;
  }
}

// dz[b, h, t, u] = (sum_o dphi[b, h, t, o] W2[h][o][u]) * [a[b, h, t, u] > 0],
// written over a.  grid (ceil(NT_max/64) * ceil(hidden/64), B*heads); the
// e outputs are taken 32 at a time.
template <int E>
__global__ void __launch_bounds__(256)
    dz_kernel(const __grid_constant__ Geometry G, const float* __restrict__ dphi, const float* __restrict__ W2,
              int hidden, float* __restrict__ a) {
  constexpr int OC = E < 32 ? E : 32;
  __shared__ __align__(16) float ps[OC][64];   // dphi rows, k-major
  __shared__ __align__(16) float ws[OC][64];   // W2 columns u0..u0+63
  const int bh = blockIdx.y, h = bh % G.heads;
  const int tiles_u = (hidden + 63) / 64;
  const int t0 = (blockIdx.x / tiles_u) * 64, u0 = (blockIdx.x % tiles_u) * 64;
  const int nt = G.g[h].nt;
  if (t0 >= nt) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  for (int o0 = 0; o0 < E; o0 += OC) {
    __syncthreads();
    for (int x = tid; x < 64 * OC; x += 256) {
      const int tt = x / OC, o = x % OC;
      ps[o][tt] = (t0 + tt < nt) ? dphi[((long long)bh * G.ntmax + t0 + tt) * E + o0 + o] : 0.f;
      const int uu = x % 64, o2 = x / 64;
      ws[o2][uu] = (u0 + uu < hidden) ? W2[((long long)h * E + o0 + o2) * hidden + u0 + uu] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int o = 0; o < OC; ++o) {
      const float4 p = *reinterpret_cast<const float4*>(&ps[o][ty * 4]);
      const float4 w = *reinterpret_cast<const float4*>(&ws[o][tx * 4]);
      const float pv[4] = {p.x, p.y, p.z, p.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(pv[i], wv[q], acc[i][q]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= nt || u0 + tx * 4 >= hidden) continue;
    float4* ap = reinterpret_cast<float4*>(a + ((long long)bh * G.ntmax + t) * hidden + u0 + tx * 4);
    const float4 av = *ap;
    *ap = make_float4(av.x > 0.f ? acc[i][0] : 0.f, av.y > 0.f ? acc[i][1] : 0.f, av.z > 0.f ? acc[i][2] : 0.f,
                      av.w > 0.f ? acc[i][3] : 0.f);
  }
}

// Per-head output error for the offline tiling search (section 2.2: a head's
// tiling is chosen to minimise the error between full and sparse attention
// outputs): err[h] = sum_{b, n, c} (o - o_ref)^2 and ref[h] = sum o_ref^2 over
// grid-order bf16 tensors [B, heads, N, d].  grid (blocks_per_head, heads);
// each CTA writes one partial pair, summed in a fixed order by
// head_error_finish_kernel.
__global__ void __launch_bounds__(256) head_error_kernel(const __grid_constant__ Geometry G,
                                                         const uint4* __restrict__ o, const uint4* __restrict__ o_ref,
                                                         float* __restrict__ part) {
  __shared__ float red[32];
  const int h = blockIdx.y;
  const long long per_bh = (long long)G.N * G.d / 8;   // 16-byte chunks per (b, h)
  float se = 0.f, sr = 0.f;
  for (int b = 0; b < G.B; ++b) {
    const uint4* x = o + ((long long)b * G.heads + h) * per_bh;
    const uint4* y = o_ref + ((long long)b * G.heads + h) * per_bh;
    for (long long c = blockIdx.x * 256LL + threadIdx.x; c < per_bh; c += (long long)gridDim.x * 256) {
      const uint4 u = __ldg(x + c), v = __ldg(y + c);
      const __nv_bfloat162* pu = reinterpret_cast<const __nv_bfloat162*>(&u);
      const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 a = __bfloat1622float2(pu[k]), r = __bfloat1622float2(pv[k]);
        se = fmaf(a.x - r.x, a.x - r.x, fmaf(a.y - r.y, a.y - r.y, se));
        sr = fmaf(r.x, r.x, fmaf(r.y, r.y, sr));
      }
    }
  }
  se = block_reduce_sum(se, red);
  sr = block_reduce_sum(sr, red);
  if (threadIdx.x == 0) {
    part[((long long)h * gridDim.x + blockIdx.x) * 2 + 0] = se;
    part[((long long)h * gridDim.x + blockIdx.x) * 2 + 1] = sr;
  }
}

__global__ void head_error_finish_kernel(const float* __restrict__ part, int nblk, int heads, float* __restrict__ err,
                                         float* __restrict__ ref) {
  for (int h = threadIdx.x; h < heads; h += blockDim.x) {
    float se = 0.f, sr = 0.f;
    for (int k = 0; k < nblk; ++k) {
      se += part[((long long)h * nblk + k) * 2 + 0];
      sr += part[((long long)h * nblk + k) * 2 + 1];
    }
    err[h] = se;
    ref[h] = sr;
  }
}

constexpr int kHeadErrBlocks = 64;   // partial sums per head

cudaError_t launch_head_error(const Geometry& G, const void* o, const void* o_ref, float* err, float* ref,
                              float* part, cudaStream_t s) {
  head_error_kernel<<<dim3(kHeadErrBlocks, G.heads), 256, 0, s>>>(G, (const uint4*)o, (const uint4*)o_ref, part);
  head_error_finish_kernel<<<1, 128, 0, s>>>(part, kHeadErrBlocks, G.heads, err, ref);
  return cudaGetLastError();
}

size_t distill_ws_bytes(const Geometry& G, int hidden, int e, int R) {
  const size_t BH = (size_t)G.B * G.heads, nt = (size_t)G.ntmax;
  auto r256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  return r256(4 * 2 * BH * nt * e)            // phi
         + r256(4 * 2 * BH * nt * hidden)     // hidden activations, then dz
         + r256(4 * BH * R * nt)              // dL/ds
         + r256(4 * BH * R)                   // row losses
         + r256(4 * 2 * BH * nt * e)          // dphi
         + 256;                               // valid-row count
}

template <int E>
static cudaError_t launch_distill_t(const Geometry& G, const float* desc_q, const float* desc_k,
                                    const EstimatorWeights& wq, const EstimatorWeights& wk, int hidden,
                                    const float* map, const int32_t* rows, int R, float* loss,
                                    const EstimatorWeights& gq, const EstimatorWeights& gk, void* ws,
                                    uint64_t timeout_ns, cudaStream_t s) {
  const size_t BH = (size_t)G.B * G.heads, nt = (size_t)G.ntmax;
  auto r256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* phi = reinterpret_cast<float*>(base);
  base += r256(4 * 2 * BH * nt * E);
  float* hid = reinterpret_cast<float*>(base);
  base += r256(4 * 2 * BH * nt * hidden);
  float* g = reinterpret_cast<float*>(base);
  base += r256(4 * BH * R * nt);
  float* row_loss = reinterpret_cast<float*>(base);
  base += r256(4 * BH * R);
  float* dphi = reinterpret_cast<float*>(base);
  base += r256(4 * 2 * BH * nt * E);
  int* count = reinterpret_cast<int*>(base);

  cudaError_t err = launch_estimator(G, desc_q, desc_k, wq, wk, hidden, E, phi, hid, timeout_ns, s);
  if (err != cudaSuccess) return err;
  distill_count_kernel<<<1, 256, 0, s>>>(G, rows, R, count);
  const long long nq4 = (long long)(BH * nt * E) / 4;
  fill_zero_kernel<<<(unsigned)std::min<long long>((nq4 + 255) / 256, 148 * 8), 256, 0, s>>>(
      reinterpret_cast<float4*>(dphi), nq4);
  distill_rows_kernel<E><<<dim3(R, (unsigned)BH), kDistillThreads, 0, s>>>(G, phi, map, rows, R, count, g, row_loss,
                                                                           dphi);
  distill_dphik_kernel<E><<<dim3((unsigned)((nt + 31) / 32), (unsigned)BH), kDistillThreads, 0, s>>>(G, phi, rows, R,
                                                                                                     g, dphi);
  distill_loss_kernel<<<1, 256, 0, s>>>(row_loss, (int)(BH * R), count, loss);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int d3 = 3 * G.d;
  for (int side = 0; side < 2; ++side) {
    const float* dph = dphi + (size_t)side * BH * nt * E;
    float* a = hid + (size_t)side * BH * nt * hidden;
    const float* desc = side ? desc_k : desc_q;
    const EstimatorWeights& w = side ? wk : wq;
    const EstimatorWeights& gr = side ? gk : gq;
    grad_reduce_kernel<<<dim3((unsigned)(((E + 63) / 64) * ((hidden + 63) / 64)), (unsigned)G.heads), 256, 0, s>>>(
        G, dph, E, a, hidden, const_cast<float*>(gr.w2));
    bias_reduce_kernel<<<G.heads, 128, 0, s>>>(G, dph, E, const_cast<float*>(gr.b2));
    dz_kernel<E><<<dim3((unsigned)(((nt + 63) / 64) * ((hidden + 63) / 64)), (unsigned)BH), 256, 0, s>>>(
        G, dph, w.w2, hidden, a);
    grad_reduce_kernel<<<dim3((unsigned)(((hidden + 63) / 64) * ((d3 + 63) / 64)), (unsigned)G.heads), 256, 0, s>>>(
        G, a, hidden, desc, d3, const_cast<float*>(gr.w1));
    bias_reduce_kernel<<<G.heads, 256, 0, s>>>(G, a, hidden, const_cast<float*>(gr.b1));
  }
  return cudaGetLastError();
}

cudaError_t launch_distill(const Geometry& G, const float* desc_q, const float* desc_k, const EstimatorWeights& wq,
                           const EstimatorWeights& wk, int hidden, int e, const float* map, const int32_t* rows,
                           int R, float* loss, const EstimatorWeights& gq, const EstimatorWeights& gk, void* ws,
                           uint64_t timeout_ns, cudaStream_t s) {
  switch (e) {
    case 16: return launch_distill_t<16>(G, desc_q, desc_k, wq, wk, hidden, map, rows, R, loss, gq, gk, ws, timeout_ns, s);
    case 32: return launch_distill_t<32>(G, desc_q, desc_k, wq, wk, hidden, map, rows, R, loss, gq, gk, ws, timeout_ns, s);
    case 64: return launch_distill_t<64>(G, desc_q, desc_k, wq, wk, hidden, map, rows, R, loss, gq, gk, ws, timeout_ns, s);
    case 128: return launch_distill_t<128>(G, desc_q, desc_k, wq, wk, hidden, map, rows, R, loss, gq, gk, ws, timeout_ns, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace veda
