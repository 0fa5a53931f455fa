// Distilled tile scoring and top-k selection (section 2.1 of the Veda summary:
// a head-specific MLP maps each tile's TripPool descriptor to a feature;
// tile scores form a row-wise distribution over K tiles; section 4 / news
// page: keep the top ~5-10% of tiles).
//
// The estimator, then one of two selection paths:
//   estimator_kernel  phi = W2 relu(W1 desc + b1) + b2 for every Q and K tile,
//                     on the tensor cores at fp32 accuracy (estimator.cu),
//                     written to the workspace;
//   rows of more than 512 tiles, e <= 64, with the score matrix in the
//   workspace:
//     score_gemm_kernel  s = phi_q phi_k^T / sqrt(e) for a head's whole
//                        [NT, NT] block, on the tensor cores, into the
//                        workspace;
//     topk_rows_kernel   one warp per row: optional row softmax, the exact
//                        k-th largest score and an ascending compaction of
//                        the winners;
//   otherwise (shorter rows, e = 128, or no room for the matrix):
//     score_topk_tc_kernel (scores on the tensor cores; e up to 64) or
//                        score_topk_kernel (fp32 SIMT scores, e = 128) per
//                        block of Q-tile rows, the scores kept in shared
//                        memory, then the same select.
// Rows of up to 2048 tiles find the k-th largest by bisection over
// order-preserving 32-bit keys held in registers (one warp per row, a
// compare-and-count per step); longer rows use a 4-pass radix select over
// shared histograms.
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
// above 0).  Invariant: count(key >= lo) = c_lo >= k > count(key >= hi) =
// c_hi; a midpoint with exactly k keys at or above it ends the search early.
// Returns the k-th largest key t.  *exact is set when exactly k keys are at
// or above t (then those are the selection); otherwise *gt is the number of
// keys above t, and the selection takes the first k - *gt keys equal to t.
// With a candidate buffer (`cand`, 64 entries owned by the warp), once at
// most 64 keys lie in [lo, hi) they are gathered there and the search goes on
// over those two per lane instead of all KPL keys per lane; the result is
// the same.
template <int KPL>
__device__ __forceinline__ uint32_t kth_key_bisect(const uint32_t (&key)[KPL], int nt, int k, int lane, int* gt,
                                                   bool* exact, uint32_t* cand) {
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < KPL; ++i)
    if (i * 32 + lane < nt) {
      kmin = min(kmin, key[i]);
      kmax = max(kmax, key[i]);
    }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  uint64_t lo = kmin, hi = (uint64_t)kmax + 1;
  int c_lo = nt, c_hi = 0;
  *exact = false;
  // Phase 1: all keys.
  while (hi - lo > 1 && (cand == nullptr || c_lo - c_hi > 64)) {
    const uint32_t mid = (uint32_t)(lo + ((hi - lo) >> 1));
    int c = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) c += key[i] >= mid ? 1 : 0;
    c = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
    if (c == k) {   // exactly the k largest are >= mid: t is the smallest of them
      uint32_t m = 0xffffffffu;
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (key[i] >= mid) m = min(m, key[i]);
      *exact = true;
      return __reduce_min_sync(0xffffffffu, m);
    }
    if (c > k) {
      lo = mid;
      c_lo = c;
    } else {
      hi = mid;
      c_hi = c;
    }
  }
  if (hi - lo > 1) {
    // Phase 2: the c_lo - c_hi <= 64 keys in [lo, hi), gathered in order of
    // appearance; every key outside is either counted in c_hi or below lo.
    int base = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      if (i * 32 >= nt) break;   // warp-uniform
      const bool in = i * 32 + lane < nt && key[i] >= lo && key[i] < hi;
      const unsigned m = __ballot_sync(0xffffffffu, in);
      if (in) cand[base + __popc(m & ((1u << lane) - 1u))] = key[i];
      base += __popc(m);
    }
    __syncwarp();
    const uint32_t k0 = lane < base ? cand[lane] : 0u, k1 = lane + 32 < base ? cand[lane + 32] : 0u;
    __syncwarp();   // the buffer is free for the warp's next row
    const int above = c_hi;   // keys at or above the bracket, none of them gathered
    while (hi - lo > 1) {
      const uint32_t mid = (uint32_t)(lo + ((hi - lo) >> 1));
      const int c = above + (int)__reduce_add_sync(0xffffffffu, (unsigned)((k0 >= mid) + (k1 >= mid)));
      if (c == k) {
        uint32_t m = 0xffffffffu;
        if (k0 >= mid) m = k0;
        if (k1 >= mid) m = min(m, k1);
        *exact = true;
        return __reduce_min_sync(0xffffffffu, m);
      }
      if (c > k) {
        lo = mid;
        c_lo = c;
      } else {
        hi = mid;
        c_hi = c;
      }
    }
  }
  // hi = lo + 1: t = lo, count(key >= t) = c_lo, count(key > t) = c_hi.
  *exact = c_lo == k;
  *gt = c_hi;
  return (uint32_t)lo;
}

constexpr int kScoreThreads = 256;
constexpr int kKChunk = 128;       // K tiles staged per step
constexpr int kQRows = 16;         // most Q-tile rows per CTA (the score tile is 16 x 128)

// Optional row softmax and the exact top-k of a block of Q-tile rows whose
// scores s_scores [qb][ntpad] are in shared memory (rows i0 .. i0+qb-1 of
// head row bh; nrows of them exist).  One warp per row.
template <int KPL, int NWARPS>
__device__ __forceinline__ void select_rows(const Geometry& G, const TopkArgs& args, const float* s_scores,
                                            uint32_t* s_hist, int qb, int ntpad, int nrows, int nt, int k, int i0,
                                            int32_t* idx_base, float* probs_base, int warp, int lane,
                                            uint32_t* cand = nullptr) {
  uint32_t* hist = s_hist + warp * 256;
  for (int r = warp; r < qb; r += NWARPS) {
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
      bool exact = false;
      prefix = kth_key_bisect(key, nt, k, lane, &gt, &exact, cand);
      remaining = k - gt;
      int out = 0, eq_taken = 0;
      if (exact) {
        // Exactly k keys are >= the k-th largest: take them all, in ascending
        // column order (column i * 32 + lane is key[i] of this lane).
#pragma unroll
        for (int i = 0; i < (KPL > 0 ? KPL : 1); ++i) {
          if (i * 32 >= nt) break;   // warp-uniform
          const int c = i * 32 + lane;
          const bool take = c < nt && key[i] >= prefix;
          const unsigned tmask = __ballot_sync(0xffffffffu, take);
          const int pos = out + __popc(tmask & ((1u << lane) - 1u));
          if (take && pos < k && VEDA_IN_BOUNDS(c < nt && pos < args.k_max)) irow[pos] = c;
          out += __popc(tmask);
        }
        for (int c = k + lane; c < args.k_max; c += 32) irow[c] = -1;
        continue;
      }
      // Every key above the k-th largest and the first `remaining` keys equal
      // to it (smallest tile indices), in ascending column order.
#pragma unroll
      for (int i = 0; i < (KPL > 0 ? KPL : 1); ++i) {
        if (i * 32 >= nt) break;   // warp-uniform
        const int c = i * 32 + lane;
        const bool in = c < nt;
        const bool gt_ = in && key[i] > prefix;
        const bool eq = in && key[i] == prefix;
        const unsigned eqmask = __ballot_sync(0xffffffffu, eq);
        const int eq_before = __popc(eqmask & ((1u << lane) - 1u));
        const bool take = gt_ || (eq && eq_taken + eq_before < remaining);
        const unsigned tmask = __ballot_sync(0xffffffffu, take);
        const int pos = out + __popc(tmask & ((1u << lane) - 1u));
        if (take && pos < k && VEDA_IN_BOUNDS(c < nt && pos < args.k_max)) irow[pos] = c;
        out += __popc(tmask);
        eq_taken += __popc(eqmask);
      }
      for (int c = k + lane; c < args.k_max; c += 32) irow[c] = -1;
      continue;
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

  // Scores, one 16 x 128 tile per chunk of K tiles.  phi_k rows jc .. jc+127
  // are staged transposed; 16-byte piece t of the chunk is row t % 128,
  // features 4 (t / 128) .. +3, so consecutive threads take consecutive rows
  // and the transposed stores do not conflict.  The first kPf pieces of each
  // thread (all of them for e <= 64) are loaded into registers while the
  // previous chunk's scores are formed.
  constexpr int kPf = kKChunk * 16 / kScoreThreads;
  const int npiece = kKChunk * (e / 4);
  float4 pf[kPf];
  auto load_pf = [&](int jc) {
    const int ncols = min(kKChunk, nt - jc);
#pragma unroll
    for (int q = 0; q < kPf; ++q) {
      const int t = tid + q * kScoreThreads;
      const int jj = t % kKChunk, q4 = t / kKChunk;
      pf[q] = (t < npiece && jj < ncols) ? __ldg(reinterpret_cast<const float4*>(phk + (long long)(jc + jj) * e) + q4)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto put = [&](int t, float4 v) {
    const int jj = t % kKChunk, q4 = t / kKChunk;
    s_phik[(4 * q4 + 0) * kKChunk + jj] = v.x;
    s_phik[(4 * q4 + 1) * kKChunk + jj] = v.y;
    s_phik[(4 * q4 + 2) * kKChunk + jj] = v.z;
    s_phik[(4 * q4 + 3) * kKChunk + jj] = v.w;
  };
  load_pf(0);
  const int cg = tid & 31, rp = tid >> 5;
  for (int jc = 0; jc < nt; jc += kKChunk) {
    __syncthreads();
    const int ncols = min(kKChunk, nt - jc);
#pragma unroll
    for (int q = 0; q < kPf; ++q) {
      const int t = tid + q * kScoreThreads;
      if (t < npiece) put(t, pf[q]);
    }
    for (int t = tid + kPf * kScoreThreads; t < npiece; t += kScoreThreads) {   // e > 64 only
      const int jj = t % kKChunk, q4 = t / kKChunk;
      put(t, (jj < ncols) ? __ldg(reinterpret_cast<const float4*>(phk + (long long)(jc + jj) * e) + q4)
                          : make_float4(0.f, 0.f, 0.f, 0.f));
    }
    __syncthreads();
    if (jc + kKChunk < nt) load_pf(jc + kKChunk);
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

  select_rows<KPL, kScoreThreads / 32>(G, args, s_scores, s_hist, qb, ntpad, nrows, nt, k, i0, idx_base, probs_base,
                                       warp, lane);
}

// ---------------------------------------------------------------------------
// Scores on the tensor cores.  A CTA takes a block of up to 32 Q-tile rows of
// one head (the MMA's N, 16 or 32) and walks the head's K tiles in chunks of
// 128 (the MMA's M): S^T = phi_k phi_q^T with tcgen05.mma kind::tf32 at fp32
// accuracy -- each operand split as x = hi + lo (hi the nearest tf32 value)
// and each product formed as hi*hi + hi*lo + lo*hi, about 2^-21 relative,
// the same split the estimator uses.
//
//   A operand: a 3-stage ring, one stage per 32-feature panel of a chunk
//     (hi and lo, 128-byte-swizzled K-major).  Every thread stages 16-byte
//     pieces of the panel (a warp reads four whole 128-byte row segments per
//     load); the pieces of the next stage are loaded into registers while
//     the current stage is stored and multiplied.
//   B operand: the block's phi_q rows, split once.
//   Accumulators: four 32-column TMEM buffers, chunk c in buffer c % 4.  The
//     chunk's products are read back two chunks later by warps 0-7 (one K tile
//     per lane, 16 Q rows per warp), so the products never wait for the read
//     and the read never waits for the products.  The scores land in a shared
//     block [rows][ntpad], from which the row softmax and top-k of the SIMT
//     kernel select the tiles, one warp per row.
// Waits are bounded; the whole CTA agrees on an abort at every barrier, and
// every MMA completes before TMEM is released.
// ---------------------------------------------------------------------------
constexpr int kTcCols = 128;     // K tiles per chunk: the MMA's M
constexpr int kTcMaxRows = 32;   // Q rows per CTA at most: the MMA's N
constexpr int kTcStages = 3;     // A-operand ring depth (one 32-feature panel pair per stage)
constexpr int kTcAcc = 4;        // TMEM accumulator buffers of 32 columns

template <int KP>
struct ScoreTcCfg {
  static constexpr int kPanels = KP / 32;
  static constexpr int kAPanel = kTcCols * 128;      // 128 K-tile rows x 32 fp32
  static constexpr int kStage = 2 * kAPanel;         // hi, lo
  static constexpr int kBPanel = kTcMaxRows * 128;   // 32 Q rows x 32 fp32
  static constexpr int kOffA = 0;
  static constexpr int kOffBhi = kTcStages * kStage;
  static constexpr int kOffBlo = kOffBhi + kPanels * kBPanel;
  static constexpr int kOffBar = kOffBlo + kPanels * kBPanel;   // stage free [3], accumulator full [4], drain; misc
  static constexpr int kOffScores = kOffBar + 128;
  static size_t smem_bytes(int qb, int ntpad, bool radix, int nthreads) {
    return 1024 + kOffScores + sizeof(float) * (size_t)qb * ntpad +
           (radix ? sizeof(uint32_t) * (nthreads / 32) * 256 : 0);
  }
};

template <int KPL, int KP, int NTHR>
__global__ void __launch_bounds__(NTHR, 1)
    score_topk_tc_kernel(const __grid_constant__ Geometry G, const float* __restrict__ phi, int e, int qb,
                         int ntpad, const __grid_constant__ TopkArgs args) {
  using C = ScoreTcCfg<KP>;
  constexpr int kP = C::kPanels;
  constexpr int kPieces = kTcCols * 8 / NTHR;   // 16-byte pieces of an A panel per thread
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
      for (int c = tid; c < args.k_max; c += NTHR) idx_base[(long long)i * args.k_max + c] = -1;
      if (probs_base)
        for (int c = tid; c < G.ntmax; c += NTHR) probs_base[(long long)i * G.ntmax + c] = 0.f;
    }
    return;   // CTA-uniform, before any barrier or TMEM use
  }
  const int nrows = min(qb, nt - i0);
  const int nq = qb > 16 ? 32 : 16;   // the MMA's N
  uint8_t* bhi = smem + C::kOffBhi;
  uint8_t* blo = smem + C::kOffBlo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);   // [0,3) stage free, [3,7) acc full, [7] drain
  int* misc = reinterpret_cast<int*>(bars + 8);                         // [0] TMEM base, [1] abort
  float* s_scores = reinterpret_cast<float*>(smem + C::kOffScores);
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_scores + (size_t)qb * ntpad);
  volatile int* abort = misc + 1;

  const float* phq = phi + ((long long)bh * G.ntmax + i0) * e;
  const float* phk = phi + (((long long)G.B * G.heads + bh) * G.ntmax) * e;
  if (tid == 0) {
    for (int b = 0; b < 8; ++b) mbar_init(smem_u32(&bars[b]), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&misc[0]), kTcAcc * 32);
    tmem_relinquish();
  }
  // phi_q of the block's rows, split, as the B operand (rows past nrows and
  // features past e are zero).
  for (int t = tid; t < kTcMaxRows * (KP / 4); t += NTHR) {
    const int r = t / (KP / 4), c = t % (KP / 4);
    const float4 v = (r < nrows && 4 * c < e) ? __ldg(reinterpret_cast<const float4*>(phq + (long long)r * e) + c)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
    store_split4(bhi + (c >> 3) * C::kBPanel, blo + (c >> 3) * C::kBPanel, r, c & 7, v);
  }
  // Stage u is chunk u / kP, panel u % kP.  Piece tid + NTHR q of a panel is
  // K-tile row (tid + NTHR q) / 8, 16-byte chunk tid % 8.
  const int nch = (nt + kTcCols - 1) / kTcCols;
  const int nst = nch * kP;
  const int pc = tid & 7;
  float4 xv[kPieces];
  auto load_stage = [&](int u) {
    const int jc = (u / kP) * kTcCols, f0 = (u % kP) * 32 + 4 * pc;
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
      const int r = (tid + NTHR * q) >> 3;
      xv[q] = (jc + r < nt && f0 < e) ? __ldg(reinterpret_cast<const float4*>(phk + (long long)(jc + r) * e + f0))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  const float inv_sqrt_e = rsqrtf((float)e);
  const uint64_t timeout_ns = args.timeout_ns;
  bool ok = true;
  uint32_t tmem = 0;
  // Chunk c's scores from TMEM buffer c % kTcAcc into the shared block:
  // warp w < 8 reads lanes 32 (w % 4) .. +31 (K tiles) and columns
  // 16 (w / 4) .. +15 (Q rows) of the buffer.
  auto read_chunk = [&](int c) {
    if (warp >= 8 || 16 * (warp >> 2) >= nq) return;
    ok = mbar_wait(smem_u32(&bars[3 + c % kTcAcc]), (c / kTcAcc) & 1, abort, timeout_ns) && ok;
    tc_fence_after();
    if (!ok) return;
    float v[16];
    tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((c % kTcAcc) * 32 + 16 * (warp >> 2)), v);
    tmem_ld_wait();
    const int j = c * kTcCols + (warp & 3) * 32 + lane;
    if (j < nt && VEDA_IN_BOUNDS(j < ntpad)) {
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int q = 16 * (warp >> 2) + r;
        if (q < nrows) s_scores[q * ntpad + j] = v[r] * inv_sqrt_e;
      }
    }
  };

  load_stage(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tmem = static_cast<uint32_t>(misc[0]);
  for (int u = 0; u < nst; ++u) {
    const int c = u / kP, p = u % kP;
    if (p == 0 && c >= 2) read_chunk(c - 2);
    // stage u % 3 is free once the products of stage u - 3 have completed
    if (u >= kTcStages) ok = mbar_wait(smem_u32(&bars[u % kTcStages]), ((u - kTcStages) / kTcStages) & 1, abort,
                                       timeout_ns) && ok;
    uint8_t* ahi = smem + C::kOffA + (u % kTcStages) * C::kStage;
    uint8_t* alo = ahi + C::kAPanel;
#pragma unroll
    for (int q = 0; q < kPieces; ++q) store_split4(ahi, alo, (tid + NTHR * q) >> 3, pc, xv[q]);
    if (u + 1 < nst) load_stage(u + 1);   // overlaps the barrier and the products
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = make_idesc_tf32(kTcCols, nq);
      const uint64_t dah = make_sdesc_sw128(smem_u32(ahi), 16, 1024), dal = make_sdesc_sw128(smem_u32(alo), 16, 1024);
      const uint64_t dbh = make_sdesc_sw128(smem_u32(bhi + p * C::kBPanel), 16, 1024);
      const uint64_t dbl = make_sdesc_sw128(smem_u32(blo + p * C::kBPanel), 16, 1024);
      const uint32_t acc = tmem + (uint32_t)((c % kTcAcc) * 32);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t off = (uint64_t)((kk * 32) >> 4);
        umma_tf32_ss(acc, dah + off, dbh + off, idesc, (p > 0 || kk > 0) ? 1u : 0u);
        umma_tf32_ss(acc, dah + off, dbl + off, idesc, 1u);
        umma_tf32_ss(acc, dal + off, dbh + off, idesc, 1u);
      }
      umma_commit(smem_u32(&bars[u % kTcStages]));
      if (p == kP - 1) umma_commit(smem_u32(&bars[3 + c % kTcAcc]));
    }
  }
  if (ok)
    for (int c = max(0, nch - 2); c < nch; ++c) read_chunk(c);
  // Every MMA issued above completes before TMEM is released.
  if (tid == 0) {
    umma_commit(smem_u32(&bars[7]));
    int dummy = 0;
    mbar_wait(smem_u32(&bars[7]), 0, &dummy, timeout_ns);
  }
  tc_fence_before();
  ok = __syncthreads_and(ok);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcAcc * 32);
  }
  if (!ok) return;   // a wait ran out: the device error word reports it
  select_rows<KPL, NTHR / 32>(G, args, s_scores, s_hist, qb, ntpad, nrows, nt, k, i0, idx_base, probs_base, warp,
                              lane);
}

// ---------------------------------------------------------------------------
// Score matrix on the tensor cores, for callers whose workspace holds it:
// S[b, h, i, j] = <phi_q[i], phi_k[j]> / sqrt(e) for i, j < NT_h, fp32
// [B*heads][NT_max][ntpad].  A CTA takes 128 Q rows of one head (the MMA's N)
// and walks the head's K tiles in chunks of 128 (the MMA's M) with the same
// tcgen05 kind::tf32 split and the same product order as the kernel above
// (S^T = phi_k phi_q^T, hi*hi, hi*lo, lo*hi per 8-feature step), so the two
// give the same scores.  The next chunk's phi_k rows are loaded into
// registers (a warp reads two whole rows per load) while the current chunk is
// multiplied; two A stages and two TMEM accumulators let chunk c's products
// run while chunk c - 1 is read back and stored.  Warp w reads K tiles
// 32 (w % 4) .. +31 and Q rows 64 (w / 4) .. +63 of the accumulator and
// stores 32 consecutive scores of one row per instruction.
// ---------------------------------------------------------------------------
constexpr int kSgRows = 128;      // Q rows per CTA: the MMA's N
constexpr int kSgThreads = 256;

template <int KP>
struct ScoreGemmCfg {
  static constexpr int kPanels = KP / 32;
  static constexpr int kAPanel = kTcCols * 128;          // 128 K-tile rows x 32 fp32
  static constexpr int kBPanel = kSgRows * 128;          // 128 Q rows x 32 fp32
  static constexpr int kStage = 2 * kPanels * kAPanel;   // hi panels, then lo panels, of one chunk
  static constexpr int kOffA = 0;                        // two stages
  static constexpr int kOffBhi = 2 * kStage;
  static constexpr int kOffBlo = kOffBhi + kPanels * kBPanel;
  static constexpr int kOffBar = kOffBlo + kPanels * kBPanel;   // A stage free [2], accumulator full [2], drain; misc
  static constexpr size_t kSmem = 1024 + kOffBar + 64;
};

template <int KP>
__global__ void __launch_bounds__(kSgThreads, 1)
    score_gemm_kernel(const __grid_constant__ Geometry G, const float* __restrict__ phi, int e, int ntpad,
                      float* __restrict__ S, uint64_t timeout_ns) {
  using C = ScoreGemmCfg<KP>;
  constexpr int kP = C::kPanels;
  constexpr int kRowPieces = KP / 4;                             // 16-byte pieces of a phi row
  constexpr int kPieces = kTcCols * kRowPieces / kSgThreads;     // of a chunk, per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bh = blockIdx.y;
  const int nt = G.g[bh % G.heads].nt;
  const int i0 = blockIdx.x * kSgRows;
  if (i0 >= nt) return;   // CTA-uniform, before any barrier or TMEM use
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nrows = min(kSgRows, nt - i0);
  uint8_t* bhi = smem + C::kOffBhi;
  uint8_t* blo = smem + C::kOffBlo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);   // [0,2) A free, [2,4) acc full, [4] drain
  int* misc = reinterpret_cast<int*>(bars + 5);                        // [0] TMEM base, [1] abort
  volatile int* abort = misc + 1;
  const float* phq = phi + ((long long)bh * G.ntmax + i0) * e;
  const float* phk = phi + (((long long)G.B * G.heads + bh) * G.ntmax) * e;
  if (tid == 0) {
    for (int b = 0; b < 5; ++b) mbar_init(smem_u32(&bars[b]), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&misc[0]), 256);
    tmem_relinquish();
  }
  // B: the block's phi_q rows, split (rows past nrows and features past e are zero)
  for (int t = tid; t < kSgRows * kRowPieces; t += kSgThreads) {
    const int r = t / kRowPieces, c4 = t % kRowPieces;
    const float4 v = (r < nrows && 4 * c4 < e) ? __ldg(reinterpret_cast<const float4*>(phq + (long long)r * e) + c4)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
    store_split4(bhi + (c4 >> 3) * C::kBPanel, blo + (c4 >> 3) * C::kBPanel, r, c4 & 7, v);
  }
  // A: piece tid + 256 q of a chunk is K-tile row (tid + 256 q) / (KP / 4),
  // 16-byte piece (tid % (KP / 4)) of that row.
  float4 xv[kPieces];
  auto load_chunk = [&](int jc) {
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
      const int t = tid + kSgThreads * q, r = t / kRowPieces, c4 = t % kRowPieces;
      xv[q] = (jc + r < nt && 4 * c4 < e) ? __ldg(reinterpret_cast<const float4*>(phk + (long long)(jc + r) * e) + c4)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  const int nch = (nt + kTcCols - 1) / kTcCols;
  load_chunk(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const float inv_sqrt_e = rsqrtf((float)e);
  bool ok = true;
  auto store_chunk = [&](int c) {
    ok = mbar_wait(smem_u32(&bars[2 + (c & 1)]), (c >> 1) & 1, abort, timeout_ns) && ok;
    tc_fence_after();
    if (!ok) return;
    const int j = c * kTcCols + (warp & 3) * 32 + lane;
    float* row0 = S + ((long long)bh * G.ntmax + i0) * ntpad + j;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      const int q0 = (warp >> 2) * 64 + cb * 32;
      float v[32];
      tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((c & 1) * kSgRows + q0), v);
      tmem_ld_wait();
      if (j < nt && VEDA_IN_BOUNDS(j < ntpad)) {
#pragma unroll
        for (int r = 0; r < 32; ++r)
          if (q0 + r < nrows) row0[(long long)(q0 + r) * ntpad] = v[r] * inv_sqrt_e;
      }
    }
  };
  for (int c = 0; c < nch; ++c) {
    const int st = c & 1;
    // A stage st is free once the products of chunk c - 2 have completed
    if (c >= 2) ok = mbar_wait(smem_u32(&bars[st]), ((c - 2) >> 1) & 1, abort, timeout_ns) && ok;
    uint8_t* ahi = smem + C::kOffA + st * C::kStage;
    uint8_t* alo = ahi + kP * C::kAPanel;
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
      const int t = tid + kSgThreads * q, r = t / kRowPieces, c4 = t % kRowPieces;
      store_split4(ahi + (c4 >> 3) * C::kAPanel, alo + (c4 >> 3) * C::kAPanel, r, c4 & 7, xv[q]);
    }
    if (c + 1 < nch) load_chunk((c + 1) * kTcCols);   // overlaps the products
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc_tf32(kTcCols, kSgRows);
      const uint32_t acc = tmem + (uint32_t)(st * kSgRows);
#pragma unroll
      for (int p = 0; p < kP; ++p) {
        const uint64_t dah = make_sdesc_sw128(smem_u32(ahi + p * C::kAPanel), 16, 1024);
        const uint64_t dal = make_sdesc_sw128(smem_u32(alo + p * C::kAPanel), 16, 1024);
        const uint64_t dbh = make_sdesc_sw128(smem_u32(bhi + p * C::kBPanel), 16, 1024);
        const uint64_t dbl = make_sdesc_sw128(smem_u32(blo + p * C::kBPanel), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = (uint64_t)((kk * 32) >> 4);
          umma_tf32_ss(acc, dah + off, dbh + off, idesc, (p > 0 || kk > 0) ? 1u : 0u);
          umma_tf32_ss(acc, dah + off, dbl + off, idesc, 1u);
          umma_tf32_ss(acc, dal + off, dbh + off, idesc, 1u);
        }
      }
      umma_commit(smem_u32(&bars[st]));
      umma_commit(smem_u32(&bars[2 + st]));
    }
    if (c >= 1) store_chunk(c - 1);   // runs while chunk c is multiplied
  }
  if (ok) store_chunk(nch - 1);
  // Every MMA issued above completes before TMEM is released.
  if (tid == 0) {
    umma_commit(smem_u32(&bars[4]));
    int dummy = 0;
    mbar_wait(smem_u32(&bars[4]), 0, &dummy, timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Row softmax and top-k from the score matrix in the workspace: one warp per
// Q-tile row, eight rows per CTA; the select is the one above, reading the
// row's scores from global memory (a warp loads 32 consecutive scores).
constexpr int kTrWarps = 8;

template <int KPL>
__global__ void __launch_bounds__(kTrWarps * 32)
    topk_rows_kernel(const __grid_constant__ Geometry G, const float* __restrict__ S, int ntpad,
                     const __grid_constant__ TopkArgs args) {
  extern __shared__ uint32_t s_hist_rows[];   // radix select only: [8][256]
  __shared__ uint32_t s_cand[kTrWarps][64];   // the bisection's candidate buffers
  const int bh = blockIdx.y;
  const int h = bh % G.heads;
  const int nt = G.g[h].nt;
  const int i0 = blockIdx.x * kTrWarps;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t* idx_base = args.idx + ((long long)bh * G.ntmax) * args.k_max;
  float* probs_base = args.probs ? args.probs + ((long long)bh * G.ntmax) * G.ntmax : nullptr;
  const int nrows = max(0, min(kTrWarps, nt - i0));
  select_rows<KPL, kTrWarps>(G, args, S + ((long long)bh * G.ntmax + i0) * ntpad, s_hist_rows, kTrWarps, ntpad, nrows,
                             nt, args.k_per_head[h], i0, idx_base, probs_base, warp, lane, s_cand[warp]);
}

// Bytes of the score matrix in the workspace, 0 when the fused kernels score:
// for e = 128, and for rows of up to 512 tiles, where the fused kernel is
// faster.  Estimator plus selection, fused kernel against score matrix:
// Wan2.1-1.3B (336 tiles) 0.062 against 0.073 ms, Wan2.1-14B (720 tiles)
// 0.314 against 0.265 ms.
size_t score_matrix_bytes(const Geometry& G, int e) {
  if (e > 64 || G.ntmax <= 512) return 0;
  return sizeof(float) * (size_t)G.B * G.heads * G.ntmax * (size_t)((G.ntmax + 3) & ~3);
}

static cudaError_t launch_score_matrix_topk(const Geometry& G, int e, const float* phi, float* S,
                                            const TopkArgs& args, cudaStream_t s) {
  const int ntpad = (G.ntmax + 3) & ~3;
  const dim3 g1((G.ntmax + kSgRows - 1) / kSgRows, G.B * G.heads);
  auto gemm = [&](auto kernel, size_t smem) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    kernel<<<g1, kSgThreads, smem, s>>>(G, phi, e, ntpad, S, args.timeout_ns);
    return cudaGetLastError();
  };
  cudaError_t err = e <= 32 ? gemm(score_gemm_kernel<32>, ScoreGemmCfg<32>::kSmem)
                            : gemm(score_gemm_kernel<64>, ScoreGemmCfg<64>::kSmem);
  if (err != cudaSuccess) return err;
  const dim3 g2((G.ntmax + kTrWarps - 1) / kTrWarps, G.B * G.heads);
  const int n = G.ntmax;
  auto rows = [&](auto kernel, size_t smem) -> cudaError_t {
    kernel<<<g2, kTrWarps * 32, smem, s>>>(G, S, ntpad, args);
    return cudaGetLastError();
  };
  if (n <= 32 * 8) return rows(topk_rows_kernel<8>, 0);
  if (n <= 32 * 16) return rows(topk_rows_kernel<16>, 0);
  if (n <= 32 * 24) return rows(topk_rows_kernel<24>, 0);
  if (n <= 32 * 32) return rows(topk_rows_kernel<32>, 0);
  if (n <= 32 * 64) return rows(topk_rows_kernel<64>, 0);
  return rows(topk_rows_kernel<0>, sizeof(uint32_t) * kTrWarps * 256);
}

// Which scoring kernel runs: the tensor-core one for feature widths up to 64
// (every row length), the fp32 SIMT one for e = 128.
static bool score_on_tensor_cores(int e) { return e <= 64; }

// Threads of the tensor-core kernel: 16 warps for rows of up to 1,024 tiles
// (at most 32 keys per lane in registers), 8 for longer rows.
static int score_tc_threads(int ntmax) { return ntmax <= 1024 ? 512 : 256; }

cudaError_t launch_score_topk(const Geometry& G, const float* desc_q, const float* desc_k,
                              const EstimatorWeights& wq, const EstimatorWeights& wk, int hidden,
                              int e, float* phi, float* scores, const TopkArgs& args, cudaStream_t s) {
  cudaError_t err = launch_estimator(G, desc_q, desc_k, wq, wk, hidden, e, phi, nullptr, args.timeout_ns, s);
  if (err != cudaSuccess) return err;
  if (scores != nullptr && score_matrix_bytes(G, e) > 0) return launch_score_matrix_topk(G, e, phi, scores, args, s);

  int qb, ntpad;
  size_t smem;
  score_topk_config(G.ntmax, e, &qb, &ntpad, &smem);
  dim3 g2((G.ntmax + qb - 1) / qb, G.B * G.heads);
  auto go = [&](auto kernel, int threads) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    kernel<<<g2, threads, smem, s>>>(G, phi, e, qb, ntpad, args);
    return cudaGetLastError();
  };
  // keys per lane of the register bisection: the row length it covers is 32 x KPL
  if (score_on_tensor_cores(e)) {
    const int n = G.ntmax;
    if (e <= 32) {
      if (n <= 32 * 8) return go(score_topk_tc_kernel<8, 32, 512>, 512);
      if (n <= 32 * 16) return go(score_topk_tc_kernel<16, 32, 512>, 512);
      if (n <= 32 * 24) return go(score_topk_tc_kernel<24, 32, 512>, 512);
      if (n <= 32 * 32) return go(score_topk_tc_kernel<32, 32, 512>, 512);
      if (n <= 32 * 64) return go(score_topk_tc_kernel<64, 32, 256>, 256);
      return go(score_topk_tc_kernel<0, 32, 256>, 256);
    }
    if (n <= 32 * 8) return go(score_topk_tc_kernel<8, 64, 512>, 512);
    if (n <= 32 * 16) return go(score_topk_tc_kernel<16, 64, 512>, 512);
    if (n <= 32 * 24) return go(score_topk_tc_kernel<24, 64, 512>, 512);
    if (n <= 32 * 32) return go(score_topk_tc_kernel<32, 64, 512>, 512);
    if (n <= 32 * 64) return go(score_topk_tc_kernel<64, 64, 256>, 256);
    return go(score_topk_tc_kernel<0, 64, 256>, 256);
  }
  if (G.ntmax <= 32 * 8) return go(score_topk_kernel<8>, kScoreThreads);
  if (G.ntmax <= 32 * 16) return go(score_topk_kernel<16>, kScoreThreads);
  if (G.ntmax <= 32 * 24) return go(score_topk_kernel<24>, kScoreThreads);
  if (G.ntmax <= 32 * 32) return go(score_topk_kernel<32>, kScoreThreads);
  if (G.ntmax <= 32 * 64) return go(score_topk_kernel<64>, kScoreThreads);
  return go(score_topk_kernel<0>, kScoreThreads);
}

// Rows per CTA so that the score block fits beside the staging buffers in
// the 227 KB of shared memory a CTA may use.
void score_topk_config(int ntmax, int e, int* qb, int* ntpad, size_t* smem) {
  const int pad = (ntmax + 3) & ~3;
  const bool radix = ntmax > 32 * 64;
  const bool tc = score_on_tensor_cores(e);
  const int nthr = score_tc_threads(ntmax);
  auto tc_bytes = [&](int rows) {
    return e <= 32 ? ScoreTcCfg<32>::smem_bytes(rows, pad, radix, nthr) : ScoreTcCfg<64>::smem_bytes(rows, pad, radix, nthr);
  };
  int rows;
  if (tc) {
    rows = (int)(((size_t)227 * 1024 - tc_bytes(0)) / (4 * (size_t)pad));
    if (rows > kTcMaxRows) rows = kTcMaxRows;
  } else {
    rows = (int)((140 * 1024) / (4 * (size_t)pad));
    if (rows > kQRows) rows = kQRows;
  }
  if (rows < 1) rows = 1;
  *qb = rows;
  *ntpad = pad;
  if (tc)
    *smem = tc_bytes(rows);
  else
    *smem = sizeof(float) * ((size_t)rows * pad + (size_t)e * kQRows + (size_t)e * kKChunk) +
            sizeof(uint32_t) * 8 * 256;
}

}  // namespace veda
