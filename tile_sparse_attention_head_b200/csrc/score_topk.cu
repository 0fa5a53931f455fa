// Distilled tile scoring and top-k selection (section 2.1 of the Veda summary:
// a head-specific MLP maps each tile's TripPool descriptor to a feature;
// tile scores form a row-wise distribution over K tiles; section 4 / news
// page: keep the top ~5-10% of tiles).
//
// Two launches:
//   estimator_kernel  phi = W2 relu(W1 desc + b1) + b2 for every Q and K tile,
//                     on the tensor cores at fp32 accuracy (estimator.cu),
//                     written to the workspace;
//   score_topk_kernel (score_topk_tc_kernel for rows of more than 1,024
//                     tiles, scores on the tensor cores)
//                     per block of Q-tile rows: s = phi_q phi_k^T / sqrt(e)
//                     into shared memory, optional row softmax, then the
//                     exact k-th largest score per row and an ascending
//                     compaction of the winners.  Rows of up to 2048 tiles
//                     find the k-th largest by bisection over order-preserving
//                     32-bit keys held in registers (one warp per row, a
//                     compare-and-count per step, no shared-memory traffic);
//                     longer rows use a 4-pass radix select over shared
//                     histograms.
// Scores stay fp32 end to end so that selections only differ from an exact
// evaluation on genuine near-ties.
#include "veda_common.cuh"
#include "kernels.h"
#include "estimator.cu"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 2   // bounds-check site id of this file (debug builds)

namespace veda {

// Order-preserving map fp32 -> uint32 (larger float <-> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0: equal scores get equal keys
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// k-th largest key of a row by bisection: each lane holds keys of columns
// lane, lane + 32, ... (KPL of them, 0 past the row end; every real key is
// above 0).  Returns the key value t and, in *gt, the number of keys above t.
// Invariant: count(key >= lo) >= k > count(key >= hi); a midpoint with exactly
// k keys at or above it ends the search early.
template <int KPL>
__device__ __forceinline__ uint32_t kth_key_bisect(const uint32_t (&key)[KPL], int nt, int k, int lane, int* gt) {
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < KPL; ++i)
    if (i * 32 + lane < nt) {
      kmin = min(kmin, key[i]);
      kmax = max(kmax, key[i]);
    }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  auto count_ge = [&](uint32_t t) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += key[i] >= t ? 1 : 0;
    return (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
  };
  uint64_t lo = kmin, hi = (uint64_t)kmax + 1;
  uint32_t t = 0;
  bool found = false;
  while (hi - lo > 1) {
    const uint64_t mid = lo + ((hi - lo) >> 1);
    const int c = count_ge((uint32_t)mid);
    if (c == k) {   // exactly the k largest are >= mid: t is the smallest of them
      uint32_t m = 0xffffffffu;
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (key[i] >= (uint32_t)mid) m = min(m, key[i]);
      t = __reduce_min_sync(0xffffffffu, m);
      found = true;
      break;
    }
    if (c > k) lo = mid;
    else hi = mid;
  }
  if (!found) t = (uint32_t)lo;
  int c = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) c += key[i] > t ? 1 : 0;
  *gt = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
  return t;
}

constexpr int kScoreThreads = 256;
constexpr int kKChunk = 128;       // K tiles staged per step
constexpr int kQRows = 16;         // most Q-tile rows per CTA (the score tile is 16 x 128)

// Optional row softmax and the exact top-k of a block of Q-tile rows whose
// scores s_scores [qb][ntpad] are in shared memory (rows i0 .. i0+qb-1 of
// head row bh; nrows of them exist).  One warp per row.
template <int KPL>
__device__ __forceinline__ void select_rows(const Geometry& G, const TopkArgs& args, const float* s_scores,
                                            uint32_t* s_hist, int qb, int ntpad, int nrows, int nt, int k, int i0,
                                            int32_t* idx_base, float* probs_base, int warp, int lane) {
  uint32_t* hist = s_hist + warp * 256;
  for (int r = warp; r < qb; r += kScoreThreads / 32) {
    const int i = i0 + r;
    if (i >= G.ntmax) break;
    int32_t* irow = idx_base + (long long)i * args.k_max;
    if (r >= nrows) {
      for (int c = lane; c < args.k_max; c += 32) irow[c] = -1;
      if (probs_base)
        for (int c = lane; c < G.ntmax; c += 32) probs_base[(long long)i * G.ntmax + c] = 0.f;
      continue;
    }
    const float* srow = s_scores + r * ntpad;

    // Optional row softmax.
    if (probs_base) {
      float m = -INFINITY;
      for (int c = lane; c < nt; c += 32) m = fmaxf(m, srow[c]);
#pragma unroll
      for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float sum = 0.f;
      for (int c = lane; c < nt; c += 32) sum += expf(srow[c] - m);
#pragma unroll
      for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      const float inv = 1.0f / sum;
      float* prow = probs_base + (long long)i * G.ntmax;
      for (int c = lane; c < G.ntmax; c += 32) prow[c] = (c < nt) ? expf(srow[c] - m) * inv : 0.f;
    }

    uint32_t prefix = 0;
    int remaining = k;
    if (KPL > 0 && nt <= 32 * KPL) {
      // Bisection over the keys, held in registers.
      uint32_t key[KPL > 0 ? KPL : 1];
#pragma unroll
      for (int i = 0; i < (KPL > 0 ? KPL : 1); ++i) {
        const int c = i * 32 + lane;
        key[i] = c < nt ? float_key(srow[c]) : 0u;
      }
      int gt = 0;
      prefix = kth_key_bisect(key, nt, k, lane, &gt);
      remaining = k - gt;
    } else {
    // Radix select: find the k-th largest key, 8 bits per pass from the top.
    uint32_t pmask = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = lane; b < 256; b += 32) hist[b] = 0;
      __syncwarp();
      for (int c = lane; c < nt; c += 32) {
        const uint32_t key = float_key(srow[c]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncwarp();
      // Lane L owns bins 255-8L .. 248-8L (descending); scan counts from the top.
      uint32_t cnt[8];
      uint32_t local = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = hist[255 - (lane * 8 + q)];
        local += cnt[q];
      }
      uint32_t incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const uint32_t excl = incl - local;
      // The bin holding the remaining-th largest key: excl + partial < remaining <= excl + partial + cnt.
      int found_bin = -1;
      uint32_t above = 0;
      if ((uint32_t)remaining > excl && (uint32_t)remaining <= incl) {
        uint32_t run = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (found_bin < 0 && (uint32_t)remaining <= run + cnt[q]) {
            found_bin = 255 - (lane * 8 + q);
            above = run;
          }
          run += cnt[q];
        }
      }
      const unsigned who = __ballot_sync(0xffffffffu, found_bin >= 0);
      const int src = __ffs(who) - 1;
      found_bin = __shfl_sync(0xffffffffu, found_bin, src);
      above = __shfl_sync(0xffffffffu, above, src);
      remaining -= (int)above;
      prefix |= (uint32_t)found_bin << shift;
      pmask |= 255u << shift;
      __syncwarp();
    }
    }
    // prefix = k-th largest key; take every key above it and the first
    // `remaining` keys equal to it (smallest tile indices), in ascending order.
    int out = 0, eq_taken = 0;
    for (int c0 = 0; c0 < nt; c0 += 32) {
      const int c = c0 + lane;
      uint32_t key = 0;
      const bool in = c < nt;
      if (in) key = float_key(srow[c]);
      const bool gt = in && key > prefix;
      const bool eq = in && key == prefix;
      const unsigned eqmask = __ballot_sync(0xffffffffu, eq);
      const int eq_before = __popc(eqmask & ((1u << lane) - 1u));
      const bool take = gt || (eq && eq_taken + eq_before < remaining);
      const unsigned tmask = __ballot_sync(0xffffffffu, take);
      const int pos = out + __popc(tmask & ((1u << lane) - 1u));
      if (take && pos < k && VEDA_IN_BOUNDS(c < nt && pos < args.k_max)) irow[pos] = c;
      out += __popc(tmask);
      eq_taken += __popc(eqmask);
    }
    for (int c = k + lane; c < args.k_max; c += 32) irow[c] = -1;
  }
}

// grid: (ceil(NT_max / qb), B*heads), qb <= 16.  Shared memory: scores
// [qb][ntmax_pad], phi_q^T [e][16], phi_k chunk^T [e][128] (both k-major, so
// a score step is one float2 and one float4 load feeding 8 FMAs: thread t
// forms rows 2(t/32), 2(t/32)+1 x columns 4(t%32)..+3 of the 16 x 128 tile),
// radix histograms [8][256].
template <int KPL>
__global__ void __launch_bounds__(kScoreThreads)
    score_topk_kernel(const __grid_constant__ Geometry G, const float* __restrict__ phi, int e,
                      int qb, int ntpad, const __grid_constant__ TopkArgs args) {
  extern __shared__ float sm[];
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const int nt = G.g[h].nt;
  const int i0 = blockIdx.x * qb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = args.k_per_head[h];
  int32_t* idx_base = args.idx + ((long long)bh * G.ntmax) * args.k_max;
  float* probs_base = args.probs ? args.probs + ((long long)bh * G.ntmax) * G.ntmax : nullptr;

  if (i0 >= nt) {
    // Rows of tiles that do not exist in this head: idx -1, probs 0.
    for (int r = 0; r < qb; ++r) {
      const int i = i0 + r;
      if (i >= G.ntmax) break;
      for (int c = tid; c < args.k_max; c += kScoreThreads) idx_base[(long long)i * args.k_max + c] = -1;
      if (probs_base)
        for (int c = tid; c < G.ntmax; c += kScoreThreads) probs_base[(long long)i * G.ntmax + c] = 0.f;
    }
    return;
  }
  const int nrows = min(qb, nt - i0);
  float* s_scores = sm;                            // [qb][ntpad]
  float* s_phiq = s_scores + qb * ntpad;           // [e][16]
  float* s_phik = s_phiq + e * kQRows;             // [e][128]
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_phik + e * kKChunk);  // [8][256]

  const float* phq = phi + ((long long)bh * G.ntmax + i0) * e;
  const float* phk = phi + (((long long)G.B * G.heads + bh) * G.ntmax) * e;
  for (int t = tid; t < kQRows * e; t += kScoreThreads) {
    const int r = t % kQRows, cc = t / kQRows;
    s_phiq[cc * kQRows + r] = (r < nrows) ? phq[(long long)r * e + cc] : 0.f;
  }
  const float inv_sqrt_e = rsqrtf((float)e);

  // Scores, one 16 x 128 tile per chunk of K tiles.
  const int cg = tid & 31, rp = tid >> 5;
  for (int jc = 0; jc < nt; jc += kKChunk) {
    __syncthreads();
    const int ncols = min(kKChunk, nt - jc);
    // phi_k rows jc .. jc+127, transposed; consecutive threads take
    // consecutive rows, so the transposed stores do not conflict.
    for (int t = tid; t < kKChunk * (e / 4); t += kScoreThreads) {
      const int jj = t % kKChunk, q4 = t / kKChunk;
      const float4 v = (jj < ncols) ? __ldg(reinterpret_cast<const float4*>(phk + (long long)(jc + jj) * e) + q4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      s_phik[(4 * q4 + 0) * kKChunk + jj] = v.x;
      s_phik[(4 * q4 + 1) * kKChunk + jj] = v.y;
      s_phik[(4 * q4 + 2) * kKChunk + jj] = v.z;
      s_phik[(4 * q4 + 3) * kKChunk + jj] = v.w;
    }
    __syncthreads();
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
    for (int cc = 0; cc < e; ++cc) {
      const float2 a = *reinterpret_cast<const float2*>(s_phiq + cc * kQRows + 2 * rp);
      const float4 b = *reinterpret_cast<const float4*>(s_phik + cc * kKChunk + 4 * cg);
      acc[0][0] = fmaf(a.x, b.x, acc[0][0]);
      acc[0][1] = fmaf(a.x, b.y, acc[0][1]);
      acc[0][2] = fmaf(a.x, b.z, acc[0][2]);
      acc[0][3] = fmaf(a.x, b.w, acc[0][3]);
      acc[1][0] = fmaf(a.y, b.x, acc[1][0]);
      acc[1][1] = fmaf(a.y, b.y, acc[1][1]);
      acc[1][2] = fmaf(a.y, b.z, acc[1][2]);
      acc[1][3] = fmaf(a.y, b.w, acc[1][3]);
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int r = 2 * rp + q;
      if (r < nrows) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (4 * cg + c < ncols && VEDA_IN_BOUNDS(jc + 4 * cg + c < ntpad))
            s_scores[r * ntpad + jc + 4 * cg + c] = acc[q][c] * inv_sqrt_e;
      }
    }
  }
  __syncthreads();

  select_rows<KPL>(G, args, s_scores, s_hist, qb, ntpad, nrows, nt, k, i0, idx_base, probs_base, warp, lane);
}

// ---------------------------------------------------------------------------
// Scores on the tensor cores.  Per chunk of 128 K tiles (the MMA's M) and the
// CTA's block of up to 16 Q rows (N = 16): S^T = phi_k phi_q^T with
// tcgen05.mma kind::tf32 at fp32 accuracy -- each operand split as x = hi + lo
// (hi the nearest tf32 value) and each product formed as hi*hi + hi*lo +
// lo*hi, about 2^-21 relative, the same split the estimator uses.  The
// accumulator lands in TMEM with one K tile per lane; warps 0-3 scale it and
// write the chunk's column of the shared score block, from which the same
// row softmax and top-k as above select the tiles.  phi_k is staged split into
// 128-byte-swizzled K-major panels; the next chunk's rows are loaded into
// registers while the current chunk's products run.  Feature widths e up to
// 64 (panels of 32 features; e = 16 is zero-padded to 32).
// ---------------------------------------------------------------------------
constexpr int kTcRows = 16;     // Q rows per CTA: the MMA's N
constexpr int kTcCols = 128;    // K tiles per chunk: the MMA's M

template <int KP>
struct ScoreTcCfg {
  static constexpr int kPanels = KP / 32;
  static constexpr int kAPanel = kTcCols * 128;   // 128 K-tile rows x 32 fp32
  static constexpr int kBPanel = kTcRows * 128;   // 16 Q rows x 32 fp32
  static constexpr int kOffAhi = 0;
  static constexpr int kOffAlo = kPanels * kAPanel;
  static constexpr int kOffBhi = 2 * kPanels * kAPanel;
  static constexpr int kOffBlo = kOffBhi + kPanels * kBPanel;
  static constexpr int kOffBar = kOffBlo + kPanels * kBPanel;   // [0] products done, [1] drain; misc after
  static constexpr int kOffScores = kOffBar + 64;
  static size_t smem_bytes(int qb, int ntpad, bool radix) {
    return 1024 + kOffScores + sizeof(float) * (size_t)qb * ntpad + (radix ? sizeof(uint32_t) * 8 * 256 : 0);
  }
};

template <int KPL, int KP>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_topk_tc_kernel(const __grid_constant__ Geometry G, const float* __restrict__ phi, int e, int qb,
                         int ntpad, const __grid_constant__ TopkArgs args) {
  using C = ScoreTcCfg<KP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const int nt = G.g[h].nt;
  const int i0 = blockIdx.x * qb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = args.k_per_head[h];
  int32_t* idx_base = args.idx + ((long long)bh * G.ntmax) * args.k_max;
  float* probs_base = args.probs ? args.probs + ((long long)bh * G.ntmax) * G.ntmax : nullptr;

  if (i0 >= nt) {
    // Rows of tiles that do not exist in this head: idx -1, probs 0.
    for (int r = 0; r < qb; ++r) {
      const int i = i0 + r;
      if (i >= G.ntmax) break;
      for (int c = tid; c < args.k_max; c += kScoreThreads) idx_base[(long long)i * args.k_max + c] = -1;
      if (probs_base)
        for (int c = tid; c < G.ntmax; c += kScoreThreads) probs_base[(long long)i * G.ntmax + c] = 0.f;
    }
    return;   // CTA-uniform, before any barrier or TMEM use
  }
  const int nrows = min(qb, nt - i0);
  uint8_t *ahi = smem + C::kOffAhi, *alo = smem + C::kOffAlo, *bhi = smem + C::kOffBhi, *blo = smem + C::kOffBlo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  int* misc = reinterpret_cast<int*>(bars + 2);   // [0] TMEM base, [1] abort
  float* s_scores = reinterpret_cast<float*>(smem + C::kOffScores);
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_scores + (size_t)qb * ntpad);
  volatile int* abort = misc + 1;

  const float* phq = phi + ((long long)bh * G.ntmax + i0) * e;
  const float* phk = phi + (((long long)G.B * G.heads + bh) * G.ntmax) * e;
  if (tid == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&misc[0]), 32);
    tmem_relinquish();
  }
  // phi_q of the CTA's rows, split, as the B operand (rows past nrows and
  // features past e are zero): one 16-byte chunk per thread and pass.
  for (int t = tid; t < kTcRows * (KP / 4); t += kScoreThreads) {
    const int r = t / (KP / 4), c = t % (KP / 4);
    const float4 v = (r < nrows && 4 * c < e) ? __ldg(reinterpret_cast<const float4*>(phq + (long long)r * e) + c)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
    store_split4(bhi + (c >> 3) * C::kBPanel, blo + (c >> 3) * C::kBPanel, r, c & 7, v);
  }
  // The chunk's phi_k rows: thread -> row tid/2, KP/8 consecutive 16-byte chunks.
  const int lr = tid >> 1, lc0 = (tid & 1) * (KP / 8);
  float4 xv[KP / 8];
  auto load_chunk = [&](int jc) {
#pragma unroll
    for (int q = 0; q < KP / 8; ++q) {
      const int c = lc0 + q;
      xv[q] = (jc + lr < nt && 4 * c < e)
                  ? __ldg(reinterpret_cast<const float4*>(phk + (long long)(jc + lr) * e) + c)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load_chunk(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const float inv_sqrt_e = rsqrtf((float)e);
  const uint64_t timeout_ns = args.timeout_ns;
  bool ok = true;
  int phase = 0;
  for (int jc = 0; jc < nt; jc += kTcCols) {
#pragma unroll
    for (int q = 0; q < KP / 8; ++q) {
      const int c = lc0 + q;
      store_split4(ahi + (c >> 3) * C::kAPanel, alo + (c >> 3) * C::kAPanel, lr, c & 7, xv[q]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc_tf32(kTcCols, kTcRows);
      const uint64_t dah = make_sdesc_sw128(smem_u32(ahi), 16, 1024), dal = make_sdesc_sw128(smem_u32(alo), 16, 1024);
      const uint64_t dbh = make_sdesc_sw128(smem_u32(bhi), 16, 1024), dbl = make_sdesc_sw128(smem_u32(blo), 16, 1024);
#pragma unroll
      for (int p = 0; p < KP / 32; ++p) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t oa = (uint64_t)((p * C::kAPanel + kk * 32) >> 4);
          const uint64_t ob = (uint64_t)((p * C::kBPanel + kk * 32) >> 4);
          umma_tf32_ss(tmem, dah + oa, dbh + ob, idesc, (p > 0 || kk > 0) ? 1u : 0u);
          umma_tf32_ss(tmem, dah + oa, dbl + ob, idesc, 1u);
          umma_tf32_ss(tmem, dal + oa, dbh + ob, idesc, 1u);
        }
      }
      umma_commit(smem_u32(&bars[0]));
    }
    if (jc + kTcCols < nt) load_chunk(jc + kTcCols);   // overlaps the products
    ok = mbar_wait(smem_u32(&bars[0]), phase & 1, abort, timeout_ns) && ok;
    ++phase;
    tc_fence_after();
    if (ok && warp < 4) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), v);
      tmem_ld_wait();
      const int j = jc + warp * 32 + lane;
      if (j < nt && VEDA_IN_BOUNDS(j < ntpad)) {
#pragma unroll
        for (int r = 0; r < kTcRows; ++r)
          if (r < nrows) s_scores[r * ntpad + j] = v[r] * inv_sqrt_e;
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);   // the A panels and TMEM are free for the next chunk
    if (!ok) break;
  }
  // Every MMA issued above completes before TMEM is released.
  if (tid == 0) {
    umma_commit(smem_u32(&bars[1]));
    int dummy = 0;
    mbar_wait(smem_u32(&bars[1]), 0, &dummy, timeout_ns);
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
  if (!ok) return;   // a wait ran out: the device error word reports it
  select_rows<KPL>(G, args, s_scores, s_hist, qb, ntpad, nrows, nt, k, i0, idx_base, probs_base, warp, lane);
}

// Which scoring kernel runs.  The tensor-core one for rows longer than 1,024
// tiles (e <= 64): there the score product dominates and it is about 11%
// faster end to end (245,760 tokens: 1.47 against 1.65 ms for estimator plus
// selection).  Shorter rows keep the fp32 SIMT kernel, which needs fewer
// registers and fits two CTAs per SM (Wan2.1-14B: 0.46 against 0.53 ms).
static bool score_on_tensor_cores(int ntmax, int e) { return e <= 64 && ntmax > 1024; }

cudaError_t launch_score_topk(const Geometry& G, const float* desc_q, const float* desc_k,
                              const EstimatorWeights& wq, const EstimatorWeights& wk, int hidden,
                              int e, float* phi, const TopkArgs& args, cudaStream_t s) {
  cudaError_t err = launch_estimator(G, desc_q, desc_k, wq, wk, hidden, e, phi, nullptr, args.timeout_ns, s);
  if (err != cudaSuccess) return err;

  int qb, ntpad;
  size_t smem;
  score_topk_config(G.ntmax, e, &qb, &ntpad, &smem);
  dim3 g2((G.ntmax + qb - 1) / qb, G.B * G.heads);
  // keys per lane of the register bisection: the row length it covers is 32 x KPL
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    kernel<<<g2, kScoreThreads, smem, s>>>(G, phi, e, qb, ntpad, args);
    return cudaGetLastError();
  };
  if (score_on_tensor_cores(G.ntmax, e)) {
    if (e <= 32) {
      if (G.ntmax <= 32 * 64) return go(score_topk_tc_kernel<64, 32>);
      return go(score_topk_tc_kernel<0, 32>);
    }
    if (G.ntmax <= 32 * 64) return go(score_topk_tc_kernel<64, 64>);
    return go(score_topk_tc_kernel<0, 64>);
  }
  if (G.ntmax <= 32 * 32) return go(score_topk_kernel<32>);
  if (G.ntmax <= 32 * 64) return go(score_topk_kernel<64>);
  return go(score_topk_kernel<0>);
}

// Rows per CTA so that the score block fits beside the staging buffers in
// the 227 KB of shared memory a CTA may use.
void score_topk_config(int ntmax, int e, int* qb, int* ntpad, size_t* smem) {
  const int pad = (ntmax + 3) & ~3;
  const bool radix = ntmax > 32 * 64;
  int rows;
  if (score_on_tensor_cores(ntmax, e)) {
    const size_t fixed = e <= 32 ? ScoreTcCfg<32>::smem_bytes(0, pad, radix) : ScoreTcCfg<64>::smem_bytes(0, pad, radix);
    rows = (int)(((size_t)227 * 1024 - fixed) / (4 * (size_t)pad));
    if (rows > kTcRows) rows = kTcRows;
  } else {
    rows = (int)((140 * 1024) / (4 * (size_t)pad));
    if (rows > kQRows) rows = kQRows;
  }
  if (rows < 1) rows = 1;
  *qb = rows;
  *ntpad = pad;
  if (score_on_tensor_cores(ntmax, e))
    *smem = e <= 32 ? ScoreTcCfg<32>::smem_bytes(rows, pad, radix) : ScoreTcCfg<64>::smem_bytes(rows, pad, radix);
  else
    *smem = sizeof(float) * ((size_t)rows * pad + (size_t)e * kQRows + (size_t)e * kKChunk) +
            sizeof(uint32_t) * 8 * 256;
}

}  // namespace veda
