// Head-specific MLP estimator (section 2.1 of the Veda summary: a separate
// MLP projection per attention head maps each tile's TripPool descriptor
// into the space where tile scores are formed):
//     phi = W2 relu(W1 desc + b1) + b2,   fp32 in, fp32 out.
//
// Per (head, Q-or-K side) this is two dense contractions,
// [NT x 3d] x [3d x hidden] and [NT x hidden] x [hidden x e], so it runs on
// the sm_100a tensor cores (tcgen05, kind::tf32, accumulators in TMEM).
// Tile selection is decided on these values, so they keep fp32 accuracy:
// every operand is split as x = hi + lo (hi the nearest tf32 value, lo the
// exact fp32 remainder) and each product is formed as hi*hi + hi*lo + lo*hi,
// which carries it to about 2^-21 relative (the dropped lo*lo term is below
// that).
//
// One CTA takes 128 tiles (the MMA's M) of one (b, h, side).  The hidden
// layer is produced in passes of up to 256 units (the MMA's N):
//   layer 1: 32-wide k panels of the descriptor and of W1 are loaded by all
//     256 threads, split, and written 128-byte-swizzled (K-major) into one
//     of two shared-memory stages while the MMAs of the previous panel run;
//     one thread issues 4 k-steps x 3 products per panel into TMEM.
//   layer 2: for every 32 hidden units, warps 0-3 read the layer-1
//     accumulator from TMEM (one tile row per thread), add b1, apply ReLU and
//     split; warps 4-7 stage the matching 32 columns of W2; the products
//     accumulate phi in a second TMEM region across all passes.
// Finally warps 0-3 add b2 and store phi.  Waits are bounded; the whole CTA
// agrees on an abort at every barrier (a predicate-reducing __syncthreads),
// so no thread is left behind at a barrier, and all MMAs are drained before
// TMEM is freed.
#pragma once
#include "veda_common.cuh"
#include "kernels.h"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 3   // bounds-check site id of this file (debug builds)

namespace veda {

constexpr int kEstRows = 128;                       // tiles per CTA (MMA M)
constexpr int kEstThreads = 256;
constexpr int kEstN1 = 256;                         // hidden units per layer-1 pass (MMA N)
constexpr int kEstPanelA = 128 * 128;               // 128 rows x 32 fp32
constexpr int kEstPanelB = 256 * 128;               // up to 256 rows x 32 fp32
constexpr int kEstStage = 2 * kEstPanelA + 2 * kEstPanelB;   // A hi/lo, B hi/lo: 96 KB
constexpr uint32_t kEstTmemCols = 512;
constexpr uint32_t kEstAcc1 = 0;                    // layer-1 accumulator, up to 256 columns
constexpr uint32_t kEstAcc2 = 256;                  // phi accumulator, e <= 128 columns

size_t estimator_smem_bytes(int d, int hidden, int e) {
  (void)d;
  (void)hidden;
  (void)e;
  return 1024 + 2 * (size_t)kEstStage + 4 * 8 + 16;
}

// Address of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled, K-major
// panel whose base is 1024-byte aligned.
__device__ __forceinline__ uint8_t* sw128_chunk(uint8_t* panel, int r, int c) {
  return panel + r * 128 + ((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ void store_split4(uint8_t* hi_panel, uint8_t* lo_panel, int r, int c, float4 v) {
  float4 h, l;
  split_tf32(v.x, h.x, l.x);
  split_tf32(v.y, h.y, l.y);
  split_tf32(v.z, h.z, l.z);
  split_tf32(v.w, h.w, l.w);
  *reinterpret_cast<float4*>(sw128_chunk(hi_panel, r, c)) = h;
  *reinterpret_cast<float4*>(sw128_chunk(lo_panel, r, c)) = l;
}

// grid: (ceil(NT_max / 128), B*heads, 2); z = 0 -> Q descriptors, z = 1 -> K.
template <int E>
__global__ void __launch_bounds__(kEstThreads, 1)
    estimator_kernel(const __grid_constant__ Geometry G, const float* __restrict__ desc_q,
                     const float* __restrict__ desc_k, EstimatorWeights wq, EstimatorWeights wk, int hidden,
                     float* __restrict__ phi, float* __restrict__ hid_out, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kEstStage);   // [0,1] stage free, [2] layer done, [3] drain
  int* misc = reinterpret_cast<int*>(bars + 4);                          // [0] TMEM base, [1] abort

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int which = blockIdx.z;
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const int nt = G.g[h].nt;
  const int j0 = blockIdx.x * kEstRows;
  if (j0 >= nt) return;   // CTA-uniform, before any barrier or TMEM use
  const int nrows = min(kEstRows, nt - j0);
  const int K1 = 3 * G.d;
  const EstimatorWeights& w = which ? wk : wq;
  const float* X = (which ? desc_k : desc_q) + ((long long)bh * G.ntmax + j0) * K1;
  const float* W1 = w.w1 + (long long)h * hidden * K1;
  const float* B1 = w.b1 + (long long)h * hidden;
  const float* W2 = w.w2 + (long long)h * E * hidden;
  const float* B2 = w.b2 + (long long)h * E;

  if (tid == 0) {
    for (int b = 0; b < 4; ++b) mbar_init(smem_u32(&bars[b]), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&misc[0]), kEstTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  volatile int* abort = misc + 1;

  int use = 0;     // shared-memory stage uses so far; use u takes stage u & 1
  int done_phase = 0;
  bool acc2_started = false;
  bool ok = true;
  // Stage (u & 1) is free once the MMAs of use u - 2 have completed.
  auto wait_stage = [&](int u) -> bool {
    if (u < 2) return true;
    return mbar_wait(smem_u32(&bars[u & 1]), ((u - 2) >> 1) & 1, abort, timeout_ns);
  };
  auto stage = [&](int u) { return smem + (u & 1) * kEstStage; };

  for (int n0 = 0; ok && n0 < hidden; n0 += kEstN1) {
    const int n1 = min(kEstN1, hidden - n0);
    const int n1p = (n1 + 15) & ~15;
    // ------------------------------------------------------------ layer 1
    // A panel: 128 descriptor rows x 32 features; B panel: up to 256 W1 rows
    // (hidden units n0 ..) x 32 features.  16-byte piece t of a panel is row
    // t / 8, chunk t % 8, and thread tid takes pieces tid + 256 q, so a warp
    // reads four whole 128-byte row segments per load.  Panel kc + 1 is
    // loaded into registers as soon as panel kc is stored, so its load
    // latency overlaps the barrier and the products of panel kc.
    const int pr = tid >> 3, pc = tid & 7;   // row and chunk of piece tid
    float4 xv[4], wv[8];
    auto load_panel = [&](int kc) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = pr + 32 * q;
        xv[q] = (r < nrows) ? __ldg(reinterpret_cast<const float4*>(X + (long long)r * K1 + kc * 32) + pc)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int r = pr + 32 * q;
        wv[q] = (r < n1) ? __ldg(reinterpret_cast<const float4*>(W1 + (long long)(n0 + r) * K1 + kc * 32) + pc)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    load_panel(0);
    for (int kc = 0; kc < K1 / 32; ++kc) {
      ok = wait_stage(use) && ok;
      uint8_t* st = stage(use);
      uint8_t *ahi = st, *alo = st + kEstPanelA, *bhi = st + 2 * kEstPanelA, *blo = bhi + kEstPanelB;
#pragma unroll
      for (int q = 0; q < 4; ++q) store_split4(ahi, alo, pr + 32 * q, pc, xv[q]);
#pragma unroll
      for (int q = 0; q < 8; ++q) store_split4(bhi, blo, pr + 32 * q, pc, wv[q]);
      if (kc + 1 < K1 / 32) load_panel(kc + 1);
      fence_proxy_async_smem();
      tc_fence_before();
      ok = __syncthreads_and(ok);
      if (!ok) break;
      if (tid == 0) {
        tc_fence_after();
        const uint32_t idesc = make_idesc_tf32(128, n1p);
        const uint64_t dah = make_sdesc_sw128(smem_u32(ahi), 16, 1024), dal = make_sdesc_sw128(smem_u32(alo), 16, 1024);
        const uint64_t dbh = make_sdesc_sw128(smem_u32(bhi), 16, 1024), dbl = make_sdesc_sw128(smem_u32(blo), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = (uint64_t)((kk * 32) >> 4);
          umma_tf32_ss(tmem + kEstAcc1, dah + off, dbh + off, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          umma_tf32_ss(tmem + kEstAcc1, dah + off, dbl + off, idesc, 1u);
          umma_tf32_ss(tmem + kEstAcc1, dal + off, dbh + off, idesc, 1u);
        }
        umma_commit(smem_u32(&bars[use & 1]));
      }
      ++use;
    }
    if (!ok) break;
    // every layer-1 product of this pass has completed
    if (tid == 0) umma_commit(smem_u32(&bars[2]));
    ok = mbar_wait(smem_u32(&bars[2]), done_phase & 1, abort, timeout_ns);
    ++done_phase;
    tc_fence_after();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    // ------------------------------------------------------------ layer 2
    // W2[o, u0 .. u0+31] for every output o, staged by warps 4-7: thread
    // t = tid - 128 takes 16-byte chunks t, t + 128, ... (E * 8 of them); the
    // next panel's chunks are loaded while the current one is multiplied.
    constexpr int kW2Per = (E * 8 + 127) / 128;
    float4 w2v[kW2Per];
    auto load_w2 = [&](int u0) {
#pragma unroll
      for (int q = 0; q < kW2Per; ++q) {
        const int t = tid - 128 + q * 128;
        const int o = t >> 3, unit = u0 + (t & 7) * 4;
        w2v[q] = (t < E * 8 && unit < hidden) ? __ldg(reinterpret_cast<const float4*>(W2 + (long long)o * hidden + unit))
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    if (warp >= 4) load_w2(n0);
    for (int pi = 0; pi < (n1 + 31) / 32; ++pi) {
      const int u0 = n0 + pi * 32;   // first hidden unit of this panel
      ok = wait_stage(use) && ok;
      uint8_t* st = stage(use);
      uint8_t *ahi = st, *alo = st + kEstPanelA, *bhi = st + 2 * kEstPanelA, *blo = bhi + kEstPanelB;
      if (warp < 4) {
        // relu(acc1 + b1) for this thread's tile row and the panel's 32 units
        const int r = warp * 32 + lane;
        float v[32];
        tmem_ld32(tmem + kEstAcc1 + ((uint32_t)(warp * 32) << 16) + (uint32_t)(pi * 32), v);
        tmem_ld_wait();
        // optional copy of the hidden activations [2, B*heads, NT_max, hidden]
        float* hrow = (hid_out != nullptr && r < nrows)
                          ? hid_out + (((long long)which * G.B * G.heads + bh) * G.ntmax + j0 + r) * hidden
                          : nullptr;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float4 hv;
          float* hp = reinterpret_cast<float*>(&hv);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int unit = u0 + c * 4 + q;
            hp[q] = (unit < hidden) ? fmaxf(v[c * 4 + q] + __ldg(B1 + unit), 0.f) : 0.f;
          }
          if (hrow != nullptr && u0 + c * 4 < hidden) *reinterpret_cast<float4*>(hrow + u0 + c * 4) = hv;
          store_split4(ahi, alo, r, c, hv);
        }
      } else {
#pragma unroll
        for (int q = 0; q < kW2Per; ++q) {
          const int t = tid - 128 + q * 128;
          if (t < E * 8) store_split4(bhi, blo, t >> 3, t & 7, w2v[q]);
        }
        if (pi + 1 < (n1 + 31) / 32) load_w2(u0 + 32);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      ok = __syncthreads_and(ok);
      if (!ok) break;
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t idesc = make_idesc_tf32(128, E);
        const uint64_t dah = make_sdesc_sw128(smem_u32(ahi), 16, 1024), dal = make_sdesc_sw128(smem_u32(alo), 16, 1024);
        const uint64_t dbh = make_sdesc_sw128(smem_u32(bhi), 16, 1024), dbl = make_sdesc_sw128(smem_u32(blo), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = (uint64_t)((kk * 32) >> 4);
          umma_tf32_ss(tmem + kEstAcc2, dah + off, dbh + off, idesc, (acc2_started || kk > 0) ? 1u : 0u);
          umma_tf32_ss(tmem + kEstAcc2, dah + off, dbl + off, idesc, 1u);
          umma_tf32_ss(tmem + kEstAcc2, dal + off, dbh + off, idesc, 1u);
        }
        umma_commit(smem_u32(&bars[use & 1]));
      }
      acc2_started = true;
      ++use;
    }
  }
  // ------------------------------------------------------------ phi = acc2 + b2
  if (ok) {
    if (tid == 0) umma_commit(smem_u32(&bars[2]));
    ok = mbar_wait(smem_u32(&bars[2]), done_phase & 1, abort, timeout_ns);
    tc_fence_after();
  }
  ok = __syncthreads_and(ok);
  if (ok && warp < 4) {
    const int r = warp * 32 + lane;
    float* out = phi + (((long long)which * G.B * G.heads + bh) * G.ntmax + j0 + r) * E;
#pragma unroll
    for (int c0 = 0; c0 < E; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + kEstAcc2 + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
      tmem_ld_wait();
      if (r < nrows && VEDA_IN_BOUNDS(j0 + r < G.ntmax)) {
#pragma unroll
        for (int q = 0; q < 32 && c0 + q < E; q += 4) {
          float4 o4 = make_float4(v[q] + __ldg(B2 + c0 + q), v[q + 1] + __ldg(B2 + c0 + q + 1),
                                  v[q + 2] + __ldg(B2 + c0 + q + 2), v[q + 3] + __ldg(B2 + c0 + q + 3));
          *reinterpret_cast<float4*>(out + c0 + q) = o4;
        }
      }
    }
  }
  // Every MMA issued above completes before TMEM is released.
  if (tid == 0) {
    umma_commit(smem_u32(&bars[3]));
    int dummy = 0;
    mbar_wait(smem_u32(&bars[3]), 0, &dummy, timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kEstTmemCols);
  }
}

template <int E>
static cudaError_t launch_est_t(const Geometry& G, const float* dq, const float* dk, const EstimatorWeights& wq,
                                const EstimatorWeights& wk, int hidden, float* phi, float* hid, uint64_t timeout_ns,
                                cudaStream_t s) {
  const size_t smem = estimator_smem_bytes(G.d, hidden, E);
  cudaError_t err = cudaFuncSetAttribute(estimator_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((G.ntmax + kEstRows - 1) / kEstRows, G.B * G.heads, 2);
  estimator_kernel<E><<<grid, kEstThreads, smem, s>>>(G, dq, dk, wq, wk, hidden, phi, hid, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_estimator(const Geometry& G, const float* dq, const float* dk, const EstimatorWeights& wq,
                             const EstimatorWeights& wk, int hidden, int e, float* phi, float* hid,
                             uint64_t timeout_ns, cudaStream_t s) {
  switch (e) {
    case 16: return launch_est_t<16>(G, dq, dk, wq, wk, hidden, phi, hid, timeout_ns, s);
    case 32: return launch_est_t<32>(G, dq, dk, wq, wk, hidden, phi, hid, timeout_ns, s);
    case 64: return launch_est_t<64>(G, dq, dk, wq, wk, hidden, phi, hid, timeout_ns, s);
    case 128: return launch_est_t<128>(G, dq, dk, wq, wk, hidden, phi, hid, timeout_ns, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace veda
