// Head-specific MLP estimator (section 2.1 of the Veda summary: a separate
// MLP projection per attention head maps each tile's TripPool descriptor
// into the space where tile scores are formed):
//     phi = W2 relu(W1 desc + b1) + b2,   fp32.
//
// Per (head, Q-or-K side) this is two small GEMMs, [NT x 3d] x [3d x hidden]
// and [NT x hidden] x [hidden x e].  They stay in fp32 on the CUDA cores
// (tile selection is decided on these values, so they must not be rounded to
// a tensor-core input type): one CTA takes 64 tiles, stages 32-wide k panels
// of both operands k-major in shared memory, and every thread accumulates a
// 4 x 4 register block, so each pair of 16-byte shared loads feeds 16 FMAs.
// The hidden activations stay in shared memory for the second GEMM.
#pragma once
#include "veda_common.cuh"
#include "kernels.h"

namespace veda {

constexpr int kEstRows = 64;     // tiles per CTA
constexpr int kEstK = 32;        // k panel width
constexpr int kEstLd = 68;       // shared row stride (floats) of 64-wide k-major panels

__host__ __device__ inline int est_ws_ld(int e) { return (e + 4) > kEstLd ? (e + 4) : kEstLd; }

size_t estimator_smem_bytes(int d, int hidden, int e) {
  (void)d;
  const int hid_pad = (hidden + 63) / 64 * 64;
  return sizeof(float) * ((size_t)kEstK * kEstLd + (size_t)kEstK * est_ws_ld(e) + (size_t)hid_pad * kEstLd);
}

// grid: (ceil(NT_max / 64), B*heads, 2); z = 0 -> Q descriptors, z = 1 -> K.
// CW = e / 16 output columns per thread in the second GEMM.
template <int CW>
__global__ void __launch_bounds__(256)
    estimator_kernel(const __grid_constant__ Geometry G, const float* __restrict__ desc_q,
                     const float* __restrict__ desc_k, EstimatorWeights wq, EstimatorWeights wk, int hidden,
                     float* __restrict__ phi) {
  constexpr int E = 16 * CW;
  extern __shared__ float sm[];
  const int ws_ld = est_ws_ld(E);
  float* xs = sm;                       // [32][68]     descriptor panel, k-major
  float* ws = xs + kEstK * kEstLd;      // [32][ws_ld]  W1 panel (64 units) / W2 panel (e outputs)
  float* hs = ws + kEstK * ws_ld;       // [hid][68]    relu(hidden), k-major

  const int which = blockIdx.z;
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const int nt = G.g[h].nt;
  const int j0 = blockIdx.x * kEstRows;
  if (j0 >= nt) return;
  const int nrows = min(kEstRows, nt - j0);
  const int in_dim = 3 * G.d;
  const EstimatorWeights& w = which ? wk : wq;
  const float* X = (which ? desc_k : desc_q) + ((long long)bh * G.ntmax + j0) * in_dim;
  const float* W1 = w.w1 + (long long)h * hidden * in_dim;
  const float* B1 = w.b1 + (long long)h * hidden;
  const float* W2 = w.w2 + (long long)h * E * hidden;
  const float* B2 = w.b2 + (long long)h * E;

  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int lr = tid & 63, lk = (tid >> 6) * 4;   // loader: row / unit, k offset (plus 16 on the second half)

  // ---- layer 1: hidden = relu(X W1^T + b1), 64 units at a time
  for (int nb = 0; nb < hidden; nb += 64) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < in_dim; k0 += kEstK) {
      __syncthreads();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int kq = lk + half * 16;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f), u = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lr < nrows) v = *reinterpret_cast<const float4*>(X + (long long)lr * in_dim + k0 + kq);
        if (nb + lr < hidden) u = *reinterpret_cast<const float4*>(W1 + (long long)(nb + lr) * in_dim + k0 + kq);
        xs[(kq + 0) * kEstLd + lr] = v.x;
        xs[(kq + 1) * kEstLd + lr] = v.y;
        xs[(kq + 2) * kEstLd + lr] = v.z;
        xs[(kq + 3) * kEstLd + lr] = v.w;
        ws[(kq + 0) * ws_ld + lr] = u.x;
        ws[(kq + 1) * ws_ld + lr] = u.y;
        ws[(kq + 2) * ws_ld + lr] = u.z;
        ws[(kq + 3) * ws_ld + lr] = u.w;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kEstK; ++kk) {
        const float4 a = *reinterpret_cast<const float4*>(xs + kk * kEstLd + ty * 4);
        const float4 b = *reinterpret_cast<const float4*>(ws + kk * ws_ld + tx * 4);
        const float av[4] = {a.x, a.y, a.z, a.w};
        const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int unit = nb + tx * 4 + j;
      if (unit < hidden) {
        const float bias = B1[unit];
#pragma unroll
        for (int i = 0; i < 4; ++i) hs[unit * kEstLd + ty * 4 + i] = fmaxf(acc[i][j] + bias, 0.f);
      }
    }
  }

  // ---- layer 2: phi = hidden W2^T + b2
  float acc2[4][CW];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < CW; ++c) acc2[i][c] = 0.f;
  for (int k0 = 0; k0 < hidden; k0 += kEstK) {
    __syncthreads();
    for (int t = tid; t < E * (kEstK / 4); t += 256) {
      const int o = t % E, kq = (t / E) * 4;
      float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k0 + kq < hidden) u = *reinterpret_cast<const float4*>(W2 + (long long)o * hidden + k0 + kq);
      ws[(kq + 0) * ws_ld + o] = u.x;
      ws[(kq + 1) * ws_ld + o] = u.y;
      ws[(kq + 2) * ws_ld + o] = u.z;
      ws[(kq + 3) * ws_ld + o] = u.w;
    }
    __syncthreads();
    const int kn = min(kEstK, hidden - k0);
    for (int kk = 0; kk < kn; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(hs + (k0 + kk) * kEstLd + ty * 4);
      const float av[4] = {a.x, a.y, a.z, a.w};
      float bv[CW];
#pragma unroll
      for (int c = 0; c < CW; ++c) bv[c] = ws[kk * ws_ld + tx * CW + c];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < CW; ++c) acc2[i][c] = fmaf(av[i], bv[c], acc2[i][c]);
    }
  }
  float* out = phi + (((long long)which * G.B * G.heads + bh) * G.ntmax + j0) * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r < nrows) {
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        const int o = tx * CW + c;
        out[(long long)r * E + o] = acc2[i][c] + B2[o];
      }
    }
  }
}

template <int CW>
static cudaError_t launch_est_t(const Geometry& G, const float* dq, const float* dk, const EstimatorWeights& wq,
                                const EstimatorWeights& wk, int hidden, float* phi, cudaStream_t s) {
  const size_t smem = estimator_smem_bytes(G.d, hidden, 16 * CW);
  cudaError_t err = cudaFuncSetAttribute(estimator_kernel<CW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((G.ntmax + kEstRows - 1) / kEstRows, G.B * G.heads, 2);
  estimator_kernel<CW><<<grid, 256, smem, s>>>(G, dq, dk, wq, wk, hidden, phi);
  return cudaGetLastError();
}

cudaError_t launch_estimator(const Geometry& G, const float* dq, const float* dk, const EstimatorWeights& wq,
                             const EstimatorWeights& wk, int hidden, int e, float* phi, cudaStream_t s) {
  switch (e) {
    case 16: return launch_est_t<1>(G, dq, dk, wq, wk, hidden, phi, s);
    case 32: return launch_est_t<2>(G, dq, dk, wq, wk, hidden, phi, s);
    case 64: return launch_est_t<4>(G, dq, dk, wq, wk, hidden, phi, s);
    case 128: return launch_est_t<8>(G, dq, dk, wq, wk, hidden, phi, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace veda
