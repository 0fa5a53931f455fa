// Max-pooled full-attention tile map, the distillation target of the
// estimator (section 2.1 "target construction": max-pool the full attention
// matrix over query-tile x key-tile regions, max rather than mean to keep
// salient peaks; section 2.3: built in two passes over a random subset of Q
// tiles).
//
// With P = softmax(scale * Q K^T) over every valid key,
//   M[i, j] = max_{q in tile i, key in tile j} P[q, key]
//           = max_q 2^( rowmax_j(q) - lse2(q) ),
// where rowmax_j(q) is the largest scaled logit (log2 units) of row q over
// tile j and lse2(q) the row's log2-sum-exp2.  So:
//   pass 1 (tcgen05): one CTA per subset Q tile streams every K tile of the
//           head through the tensor cores (S = Q K^T in TMEM), and the
//           softmax warps record rowmax_j(q) for every (q, j) in the
//           workspace while accumulating the online log-sum-exp;
//   pass 2: a warp per (Q tile, K tile) reads the 128 recorded maxima and
//           the row lse2 values and takes the max of 2^(rowmax - lse2) over
//           the token rows of the Q tile.
// This replaces a second Q K^T sweep (the pages' second pass) by one write
// and one read of the per-row maxima, which costs far less HBM time on B200
// than re-running the tensor-core sweep.
#include "veda_common.cuh"
#include "kernels.h"

namespace veda {

// Pass 1 is exponential-bound (Q K^T only); one exponential in
// kMapPolyEvery runs on the FMA pipe (exp2_fma), the rest on the
// special-function unit.
constexpr int kMapPolyEvery = 3;

template <int D, int BN>
struct MapCfg {
  static constexpr int BM = 128;
  static constexpr int kThreads = 192;
  static constexpr int kStages = 4;
  static constexpr int kChunk = 128 * 128;
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffK + kStages * kKBytes;
  static constexpr int kOffMisc = kOffBar + 16 * 8;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr size_t kSmem = 1024 + kOffMisc + 64;
};

enum {
  MBAR_Q = 0,
  MBAR_KFULL = 1,   // +stage (4)
  MBAR_KEMPTY = 5,  // +stage (4)
  MBAR_SFULL = 9,   // +buffer (2)
  MBAR_SFREE = 11,  // +buffer (2)
  MBAR_DRAIN = 13
};

__device__ __forceinline__ bool map_warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                              uint64_t timeout_ns) {
  const bool ok = mbar_wait(bar, parity, abort, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

template <int D, int BN>
__global__ void __launch_bounds__(192, 1)
    tile_map_pass1_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ Geometry G, const __grid_constant__ MapArgs A) {
  using C = MapCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x % A.R;
  const int bh = blockIdx.x / A.R;
  const int h = bh % G.heads;
  const HeadGeom hg = G.g[h];
  const int i = A.rows[(long long)bh * A.R + r];
  if (i < 0 || i >= hg.nt) return;  // CTA-uniform
  const int S = G.S;
  const int nt = hg.nt;

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  auto bar = [&](int b) { return bar0 + 8u * (uint32_t)b; };
  int* misc = reinterpret_cast<int*>(smem + C::kOffMisc);
  volatile int* abort = misc + 1;

  if (tid == 0) {
    misc[1] = 0;
    mbar_init(bar(MBAR_Q), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(MBAR_KFULL + s), 1);
      mbar_init(bar(MBAR_KEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(MBAR_SFULL + s), 1);
      mbar_init(bar(MBAR_SFREE + s), 4);
    }
    mbar_init(bar(MBAR_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc[0]), C::kTmemCols);
    tmem_relinquish();
  }
  if (BN < 128 && warp >= 2) {
    for (int c = 0; c < D / 64; ++c) {
      uint4* p = reinterpret_cast<uint4*>(smem + C::kOffQ + c * C::kChunk + 64 * 128);
      for (int e = tid - 64; e < 64 * 128 / 16; e += 128) p[e] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const uint64_t tmo = A.timeout_ns;

  if (warp == 0) {
    int issued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(bar(MBAR_Q), (uint32_t)(S * D * 2));
      for (int c = 0; c < D / 64; ++c)
        tma_load_2d(sQ + c * C::kChunk, &tmQ, bar(MBAR_Q), 64 * c, (bh * G.ntmax + i) * S);
    }
    for (int t = 0; t < nt; ++t) {
      const int st = t % C::kStages;
      const int fill = t / C::kStages;
      if (fill >= 1 && !map_warp_wait(bar(MBAR_KEMPTY + st), (fill - 1) & 1, abort, tmo)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(MBAR_KFULL + st), (uint32_t)C::kKBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(sK + st * C::kKBytes + c * BN * 128, &tmK, bar(MBAR_KFULL + st), 64 * c,
                      (bh * G.ntmax + t) * S);
      }
      __syncwarp();
      issued = t + 1;
    }
    if (*abort) {
      int dummy = 0;
      mbar_wait(bar(MBAR_Q), 0, &dummy, tmo);
      for (int t = issued > C::kStages ? issued - C::kStages : 0; t < issued; ++t)
        mbar_wait(bar(MBAR_KFULL + t % C::kStages), (t / C::kStages) & 1, &dummy, tmo);
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc = make_idesc_bf16(128, BN, false);
    // Descriptors built once; per MMA only compile-time offsets are added.
    const uint64_t dq0 = make_sdesc_sw128(sQ, 16, 1024);
    const uint64_t dk0 = make_sdesc_sw128(sK, 16, 1024);
    bool ok = map_warp_wait(bar(MBAR_Q), 0, abort, tmo);
    for (int t = 0; ok && t < nt; ++t) {
      const int st = t % C::kStages, sb = t & 1;
      if (!(ok = map_warp_wait(bar(MBAR_KFULL + st), (t / C::kStages) & 1, abort, tmo))) break;
      if (t >= 2 && !(ok = map_warp_wait(bar(MBAR_SFREE + sb), ((t >> 1) - 1) & 1, abort, tmo))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint64_t dk = dk0 + (uint64_t)((st * C::kKBytes) >> 4);
        const uint32_t dS = tmem + sb * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t da = dq0 + (uint64_t)(((kk >> 2) * C::kChunk + (kk & 3) * 32) >> 4);
          const uint64_t db = dk + (uint64_t)(((kk >> 2) * BN * 128 + (kk & 3) * 32) >> 4);
          umma_ss(dS, da, db, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(MBAR_KEMPTY + st));
        umma_commit(bar(MBAR_SFULL + sb));
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(bar(MBAR_DRAIN));
    __syncwarp();
    int dummy = 0;
    mbar_wait(bar(MBAR_DRAIN), 0, &dummy, tmo);
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = A.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    float* rm = A.rowmax + (((long long)bh * A.R + r) * G.ntmax) * S + row;
    for (int t = 0; t < nt; ++t) {
      const int sb = t & 1;
      if (!(ok = map_warp_wait(bar(MBAR_SFULL + sb), (t >> 1) & 1, abort, tmo))) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_lane + sb * 128 + c * 32, &s[c * 32]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(MBAR_SFREE + sb));

      const int jw = t % hg.nTw, jh = (t / hg.nTw) % hg.nTh, jt = t / (hg.nTw * hg.nTh);
      const int ct = min((int)hg.pt, G.T - jt * hg.pt);
      const int ch = min((int)hg.ph, G.H - jh * hg.ph);
      const int cw = min((int)hg.pw, G.W - jw * hg.pw);
      if (ct * ch * cw != S) {
        uint32_t mw[BN / 32];
#pragma unroll
        for (int w = 0; w < BN / 32; ++w) {
          const int c = w * 32 + lane;
          const int lw = c % hg.pw, lh = (c / hg.pw) % hg.ph, lt = c / (hg.pw * hg.ph);
          mw[w] = __ballot_sync(0xffffffffu, lt < ct && lh < ch && lw < cw);
        }
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (!((mw[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
      }
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = s[q];
#pragma unroll
      for (int c = 8; c < BN; c += 8)
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = fmaxf(m8[q], s[c + q]);
      float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      mt *= sl2;
      if (row < S) rm[(long long)t * S] = mt;
      const float m_new = fmaxf(m_run, mt);
      float r8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) r8[q] = 0.f;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const float x = fmaf(s[c], sl2, -m_new);
        r8[c & 7] += (c % kMapPolyEvery == kMapPolyEvery - 1) ? exp2_fma(x) : fast_exp2(x);
      }
      const float rs = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      l_run = l_run * fast_exp2(m_run - m_new) + rs;
      m_run = m_new;
    }
    if (ok && row < S) A.lse2[((long long)bh * A.R + r) * S + row] = m_run + log2f(l_run);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Pass 2: map[bh, r, j] = max over token rows q of tile rows[bh, r] of
// 2^(rowmax[bh, r, j, q] - lse2[bh, r, q]).  One warp per (bh, r, j).
__global__ void __launch_bounds__(256) tile_map_pass2_kernel(const __grid_constant__ Geometry G,
                                                             const __grid_constant__ MapArgs A) {
  const long long total = (long long)G.B * G.heads * A.R * G.ntmax;
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; w < total; w += warps) {
    const int j = (int)(w % G.ntmax);
    const long long br = w / G.ntmax;  // bh * R + r
    const int bh = (int)(br / A.R);
    const int h = bh % G.heads;
    const HeadGeom& hg = G.g[h];
    const int i = A.rows[br];
    float best = 0.f;
    if (i >= 0 && i < hg.nt && j < hg.nt) {
      const float* rm = A.rowmax + (br * G.ntmax + j) * G.S;
      const float* ls = A.lse2 + br * G.S;
      float m = -INFINITY;
      for (int q = lane; q < G.S; q += 32) {
        if (slot_to_grid(G, hg, i, q) >= 0) m = fmaxf(m, rm[q] - ls[q]);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      best = exp2f(m);
    }
    if (lane == 0) A.map[w] = best;
  }
}

template <int D, int BN>
static cudaError_t launch_map_t(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                                const MapArgs& a, cudaStream_t s) {
  using C = MapCfg<D, BN>;
  cudaError_t err = cudaFuncSetAttribute(tile_map_pass1_kernel<D, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (err != cudaSuccess) return err;
  const unsigned blocks = (unsigned)(G.B * G.heads * a.R);
  tile_map_pass1_kernel<D, BN><<<blocks, C::kThreads, C::kSmem, s>>>(tq, tk, G, a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  return cudaSuccess;
}

cudaError_t launch_tile_map(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                            const MapArgs& a, cudaStream_t s) {
  cudaError_t err;
  if (G.d == 128 && G.S == 128) err = launch_map_t<128, 128>(G, tq, tk, a, s);
  else if (G.d == 128 && G.S == 64) err = launch_map_t<128, 64>(G, tq, tk, a, s);
  else if (G.d == 64 && G.S == 128) err = launch_map_t<64, 128>(G, tq, tk, a, s);
  else err = launch_map_t<64, 64>(G, tq, tk, a, s);
  if (err != cudaSuccess) return err;
  const long long total_threads = (long long)G.B * G.heads * a.R * G.ntmax * 32;
  long long blocks = (total_threads + 255) / 256;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
  tile_map_pass2_kernel<<<(unsigned)blocks, 256, 0, s>>>(G, a);
  return cudaGetLastError();
}

// A kernel whose only job is to run one bounded wait out: it waits on an
// mbarrier that nothing ever arrives on, gives up after `timeout_ns`, sets
// the device error word and returns.  Used to test time-out reporting
// without hanging anything.
__global__ void timeout_selftest_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t b;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&b), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&b), 0, &abort_flag, timeout_ns);
}

cudaError_t launch_timeout_selftest(uint64_t timeout_ns, cudaStream_t s) {
  timeout_selftest_kernel<<<1, 32, 0, s>>>(timeout_ns);
  return cudaGetLastError();
}

}  // namespace veda
