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
//           head through the tensor cores (S = Q K^T into one of two TMEM
//           buffers), and two softmax streams -- even and odd K tiles, one
//           S buffer each, so two softmax warps share every scheduler --
//           record rowmax_j(q) for every (q, j) in the workspace while
//           accumulating an online log-sum-exp; the two partial sums are
//           merged exactly at the end;
//   pass 2: a warp per (Q tile, K tile) reads the 128 recorded maxima and
//           the row lse2 values and takes the max of 2^(rowmax - lse2) over
//           the token rows of the Q tile.
// This replaces a second Q K^T sweep (the pages' second pass) by one write
// and one read of the per-row maxima, which costs far less HBM time on B200
// than re-running the tensor-core sweep.
#include "veda_common.cuh"
#include "kernels.h"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 5   // bounds-check site id of this file (debug builds)

namespace veda {

// Pass 1 is exponential-bound (Q K^T only): one pair of exponentials in
// eight runs on the FMA pipe (exp2_fma_x2), the rest on the special-function
// unit.  At the board's power cap this split measured fastest (10.1 ms at
// the 14B shape against 10.4 with none and 10.9 with 3/8 on the FMA pipe).
__host__ __device__ constexpr bool map_poly_pair(int pair) { return pair % 8 == 7; }

template <int D, int BN>
struct MapCfg {
  static constexpr int BM = 128;
  static constexpr int kThreads = 320;   // producer, MMA issuer, two softmax warpgroups
  static constexpr int kStages = 4;
  static constexpr int kChunk = 128 * 128;
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffK + kStages * kKBytes;
  static constexpr int kOffMisc = kOffBar + 16 * 8;
  static constexpr int kOffRed = kOffMisc + 64;   // float [2: m, l][128 rows] of stream B
  static constexpr uint32_t kTmemCols = 256;
  static constexpr size_t kSmem = 1024 + kOffRed + 2 * 128 * 4;
};

enum {
  MBAR_Q = 0,
  MBAR_KFULL = 1,   // +stage (4)
  MBAR_KEMPTY = 5,  // +stage (4)
  MBAR_SFULL = 9,   // +buffer (2)
  MBAR_SFREE = 11,  // +buffer (2)
  MBAR_DRAIN = 13,
  MBAR_XFIN = 14    // stream B's final (m, l) are in shared memory (128 arrivals)
};

__device__ __forceinline__ bool map_warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                              uint64_t timeout_ns) {
  const bool ok = mbar_wait(bar, parity, abort, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// GRID = false: Q and K are tile-major [B, heads, NT_max*S, d], a tile is a 2D
// box of S rows.  GRID = true: Q and K stay in grid order [B, heads, N, d]; a
// tile is the 5D box of its pt x ph x pw tokens, which lands in shared memory
// in slot order with zeros for the parts outside the grid -- the same tile
// contents the permutation writes -- so both layouts give identical maps.  A
// grid-order launch covers the heads A.head_list[0 .. A.n_group), head h
// using tensor maps number A.map_of_head[h].
template <int D, int BN, bool GRID>
__global__ void __launch_bounds__(320, 1)
    tile_map_pass1_kernel(const __grid_constant__ AttnMaps<GRID ? kMaxGridMaps : 1> M,
                          const __grid_constant__ Geometry G, const __grid_constant__ MapArgs A) {
  using C = MapCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x % A.R;
  int bh, h, mi = 0;
  if constexpr (GRID) {
    const int hb = blockIdx.x / A.R;        // b * n_group + position in the head list
    h = A.head_list[hb % A.n_group];
    bh = (hb / A.n_group) * G.heads + h;
    mi = A.map_of_head[h];
  } else {
    bh = blockIdx.x / A.R;
    h = bh % G.heads;
  }
  const HeadGeom hg = G.g[h];
  const CUtensorMap* tmQ = &M.q[mi];
  const CUtensorMap* tmK = &M.k[mi];
  // Channel chunk c (64 channels) of tile j of this head into shared memory.
  auto load_tile = [&](uint32_t dst, const CUtensorMap* map, uint32_t b, int c, int j) {
    if constexpr (GRID) {
      const int jw = j % hg.nTw, jh = (j / hg.nTw) % hg.nTh, jt = j / (hg.nTw * hg.nTh);
      tma_load_5d(dst, map, b, 64 * c, jw * hg.pw, jh * hg.ph, jt * hg.pt, bh);
    } else {
      tma_load_2d(dst, map, b, 64 * c, (bh * G.ntmax + j) * G.S);
    }
  };
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
    mbar_init(bar(MBAR_XFIN), 128);
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
      tma_prefetch_desc(tmQ);
      tma_prefetch_desc(tmK);
      mbar_arrive_expect_tx(bar(MBAR_Q), (uint32_t)(S * D * 2));
      for (int c = 0; c < D / 64; ++c)
        load_tile(sQ + c * C::kChunk, tmQ, bar(MBAR_Q), c, i);
    }
    for (int t = 0; t < nt; ++t) {
      const int st = t % C::kStages;
      const int fill = t / C::kStages;
      if (fill >= 1 && !map_warp_wait(bar(MBAR_KEMPTY + st), (fill - 1) & 1, abort, tmo)) break;
      if (lane == 0 && VEDA_IN_BOUNDS(t < hg.nt && (long long)(bh * G.ntmax + t) * S < (long long)G.B * G.heads * G.ntmax * S)) {
        mbar_arrive_expect_tx(bar(MBAR_KFULL + st), (uint32_t)C::kKBytes);
        for (int c = 0; c < D / 64; ++c)
          load_tile(sK + st * C::kKBytes + c * BN * 128, tmK, bar(MBAR_KFULL + st), c, t);
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
    // ------------------------------------------------------------ softmax streams
    const int sb = (warp - 2) >> 2;        // stream: K tiles t with t % 2 == sb, S buffer sb
    const int quarter = warp & 3;          // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(sb * 128);
    const float sl2 = A.scale_log2;
    const uint64_t scl2 = f2(sl2, sl2);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    float* rm = A.rowmax + (((long long)bh * A.R + r) * G.ntmax) * S + row;
    // Slot offsets (t, y, x) of this lane's key columns c = 32 w + lane.
    int8_t kt[BN / 32], ky[BN / 32], kx[BN / 32];
#pragma unroll
    for (int w = 0; w < BN / 32; ++w) {
      const int c = w * 32 + lane;
      kx[w] = (int8_t)(c % hg.pw);
      ky[w] = (int8_t)((c / hg.pw) % hg.ph);
      kt[w] = (int8_t)(c / (hg.pw * hg.ph));
    }
    // Tile coordinates of t = sb, advanced by 2 tiles per step without division.
    int jw = sb % hg.nTw, jh = (sb / hg.nTw) % hg.nTh, jt = sb / (hg.nTw * hg.nTh);
    for (int t = sb; t < nt; t += 2) {
      const int k = t >> 1;
      if (!(ok = map_warp_wait(bar(MBAR_SFULL + sb), k & 1, abort, tmo))) break;
      tc_fence_after();
      float sc[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_lane + c * 32, &sc[c * 32]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(MBAR_SFREE + sb));

      const int ct = min((int)hg.pt, G.T - jt * hg.pt);
      const int ch = min((int)hg.ph, G.H - jh * hg.ph);
      const int cw = min((int)hg.pw, G.W - jw * hg.pw);
      if (ct * ch * cw != S) {
        uint32_t mw[BN / 32];
#pragma unroll
        for (int w = 0; w < BN / 32; ++w) mw[w] = __ballot_sync(0xffffffffu, kt[w] < ct && ky[w] < ch && kx[w] < cw);
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (!((mw[c >> 5] >> (c & 31)) & 1u)) sc[c] = -INFINITY;
      }
      jw += 2;
      while (jw >= hg.nTw) {
        jw -= hg.nTw;
        if (++jh == hg.nTh) {
          jh = 0;
          ++jt;
        }
      }
      // Row maximum of the tile: three-input max over 8 chains.
      float m8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) m8[q] = sc[q];
#pragma unroll
      for (int c = 8; c + 16 <= BN; c += 16)
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = fmax3(m8[q], sc[c + q], sc[c + 8 + q]);
      if constexpr ((BN - 8) % 16 == 8) {   // the last 8 columns
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = fmaxf(m8[q], sc[BN - 8 + q]);
      }
      const float mt = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * sl2;
      if (row < S && VEDA_IN_BOUNDS(t < nt)) rm[(long long)t * S] = mt;
      const float m_new = fmaxf(m_run, mt);
      const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t nref2 = f2(-m_ref, -m_ref);
      uint64_t r4[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        float x0, x1, p0, p1;
        f2_split(f2_fma(f2(sc[c], sc[c + 1]), scl2, nref2), x0, x1);
        if (map_poly_pair(c >> 1)) {
          exp2_fma_x2(x0, x1, p0, p1);
        } else {
          p0 = fast_exp2(x0);
          p1 = fast_exp2(x1);
        }
        r4[(c >> 1) & 3] = f2_add(r4[(c >> 1) & 3], f2(p0, p1));
      }
      float ra, rb, rc, rd;
      f2_split(f2_add(r4[0], r4[1]), ra, rb);
      f2_split(f2_add(r4[2], r4[3]), rc, rd);
      const float rs = (ra + rb) + (rc + rd);
      l_run = (m_run == -INFINITY ? 0.f : l_run * fast_exp2(m_run - m_ref)) + rs;
      m_run = m_new;
    }
    // Merge the streams: stream B hands its (m, l) to stream A.
    float* red = reinterpret_cast<float*>(smem + C::kOffRed);
    if (sb == 1) {
      red[row] = m_run;
      red[128 + row] = l_run;
      mbar_arrive(bar(MBAR_XFIN));
    } else {
      if (ok) ok = map_warp_wait(bar(MBAR_XFIN), 0, abort, tmo);
      if (ok && row < S) {
        const float mB = red[row], lB = red[128 + row];
        const float m = fmaxf(m_run, mB);
        const float l = (m_run == -INFINITY ? 0.f : l_run * fast_exp2(m_run - m)) +
                        (mB == -INFINITY ? 0.f : lB * fast_exp2(mB - m));
        A.lse2[((long long)bh * A.R + r) * S + row] = m + log2f(l);
      }
    }
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
    if (lane == 0 && VEDA_IN_BOUNDS(w < total)) A.map[w] = best;
  }
}

template <int D, int BN, bool GRID>
static cudaError_t launch_map_t(const Geometry& G, const AttnMaps<GRID ? kMaxGridMaps : 1>& m, const MapArgs& a,
                                cudaStream_t s) {
  using C = MapCfg<D, BN>;
  cudaError_t err = cudaFuncSetAttribute(tile_map_pass1_kernel<D, BN, GRID>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (err != cudaSuccess) return err;
  const unsigned blocks = (unsigned)(G.B * (GRID ? a.n_group : G.heads) * a.R);
  tile_map_pass1_kernel<D, BN, GRID><<<blocks, C::kThreads, C::kSmem, s>>>(m, G, a);
  return cudaGetLastError();
}

template <bool GRID>
static cudaError_t launch_pass1(const Geometry& G, const AttnMaps<GRID ? kMaxGridMaps : 1>& m, const MapArgs& a,
                                cudaStream_t s) {
  if (G.d == 128 && G.S == 128) return launch_map_t<128, 128, GRID>(G, m, a, s);
  if (G.d == 128 && G.S == 64) return launch_map_t<128, 64, GRID>(G, m, a, s);
  if (G.d == 64 && G.S == 128) return launch_map_t<64, 128, GRID>(G, m, a, s);
  return launch_map_t<64, 64, GRID>(G, m, a, s);
}

cudaError_t launch_tile_map_pass1_grid(const Geometry& G, const AttnMaps<kMaxGridMaps>& m, const MapArgs& a,
                                       cudaStream_t s) {
  return launch_pass1<true>(G, m, a, s);
}

cudaError_t launch_tile_map_pass2(const Geometry& G, const MapArgs& a, cudaStream_t s) {
  const long long total_threads = (long long)G.B * G.heads * a.R * G.ntmax * 32;
  long long blocks = (total_threads + 255) / 256;
  if (blocks > 148LL * 32) blocks = 148LL * 32;
  tile_map_pass2_kernel<<<(unsigned)blocks, 256, 0, s>>>(G, a);
  return cudaGetLastError();
}

cudaError_t launch_tile_map(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                            const MapArgs& a, cudaStream_t s) {
  AttnMaps<1> m;
  m.q[0] = tq;
  m.k[0] = tk;
  m.v[0] = tk;   // unused
  cudaError_t err = launch_pass1<false>(G, m, a, s);
  if (err != cudaSuccess) return err;
  return launch_tile_map_pass2(G, a, s);
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

// Bounds-check self-test (debug builds): thread t checks t < limit, the way
// the kernels check a computed index, and touches no memory.
__global__ void bounds_selftest_kernel(int limit) { (void)VEDA_IN_BOUNDS((int)threadIdx.x < limit); }

cudaError_t launch_bounds_selftest(cudaStream_t s) {
  bounds_selftest_kernel<<<1, 32, 0, s>>>(31);
  return cudaGetLastError();
}

}  // namespace veda
