// Distilled tile scoring and top-k selection (section 2.1 of the Veda summary:
// a head-specific MLP maps each tile's TripPool descriptor to a feature;
// tile scores form a row-wise distribution over K tiles; section 4 / news
// page: keep the top ~5-10% of tiles).
//
// Two kernels:
//   estimator_kernel  phi = W2 relu(W1 desc + b1) + b2 for every Q and K tile,
//                     on the tensor cores at fp32 accuracy (estimator.cu),
//                     written to the workspace;
//   score_topk_kernel per block of Q-tile rows: s = phi_q phi_k^T / sqrt(e)
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
  if (G.ntmax <= 32 * 32) return go(score_topk_kernel<32>);
  if (G.ntmax <= 32 * 64) return go(score_topk_kernel<64>);
  return go(score_topk_kernel<0>);
}

// Rows per CTA so that the score block fits in ~160 KB of shared memory.
void score_topk_config(int ntmax, int e, int* qb, int* ntpad, size_t* smem) {
  const int pad = (ntmax + 3) & ~3;
  int rows = (int)((140 * 1024) / (4 * (size_t)pad));
  if (rows > kQRows) rows = kQRows;
  if (rows < 1) rows = 1;
  *qb = rows;
  *ntpad = pad;
  *smem = sizeof(float) * ((size_t)rows * pad + (size_t)e * kQRows + (size_t)e * kKChunk) +
          sizeof(uint32_t) * 8 * 256;
}

}  // namespace veda
