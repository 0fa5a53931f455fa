// Tile-skipping sparse attention on the sm_100a tensor cores (section 2.3 of
// the Veda summary: a block-sparse attention kernel that fetches only the
// selected, non-contiguous K/V tiles and hides the data movement behind the
// matrix math with warp-specialised producer/consumer roles).
//
// Blackwell design, one CTA per (b, h, Q tile), 6 warps:
//   warp 0      TMA producer: the Q tile once, then K_j and V_j of every
//               selected tile j into an NST-stage shared-memory ring (a
//               permuted tile is S contiguous rows, so each fetch is a plain
//               2D box; panels are 128-byte swizzled for the tensor cores);
//   warp 1      tcgen05 issuer: S_t = Q K_t^T into one of three TMEM S/P
//               buffers, then O += P_t V_t with P_t read straight from TMEM
//               (the A operand of the "TS" form), O accumulating in TMEM;
//               completions are signalled with tcgen05.commit on mbarriers.
//               S_{t+1} is issued before P_t is ready so the tensor cores
//               compute the next scores while the softmax runs;
//   warps 2-5   softmax: one thread per query row loads its S row from TMEM,
//               masks the pad keys of edge tiles, runs the online softmax in
//               the log2 domain (a share of the exponentials on the FMA pipe),
//               rescales its O row in TMEM only when the running maximum grows
//               by more than 2^8, writes P as packed bf16 over its S row, and
//               finally normalises O and stores it with the log-sum-exp.
// TMEM: three S/P buffers (3 x 128 columns) + O (d columns) = 512 columns.
// Shared memory: Q (S x d) + NST x (K + V) tiles; NST = 3 when it fits.
// Every wait is bounded (veda_common.cuh); on a time-out every role leaves
// its loop, in-flight copies and MMAs are drained and TMEM is freed.
#include "veda_common.cuh"
#include "kernels.h"

namespace veda {

// One exponential in kPolyEvery is evaluated with exp2_fma (FMA pipe), the
// others with ex2.approx (special-function unit), balancing the two pipes.
constexpr int kPolyEvery = 4;
constexpr int kSmemLimit = 232448;   // dynamic shared memory per CTA on sm_100

template <int D, int BN, int NST>
struct AttnCfg {
  static constexpr int BM = 128;                 // MMA rows (query slots; S = 64 tiles use half)
  static constexpr int kThreads = 192;
  static constexpr int kChunk = 128 * 128;       // one [128 rows x 128 B] swizzle panel
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + NST * kKVBytes;
  static constexpr int kOffBar = kOffV + NST * kKVBytes;
  static constexpr int kNumBars = 24;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffIdx = kOffMisc + 64;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemO = 384;        // O accumulator column; S/P buffers at 0, 128, 256
  static size_t smem_bytes(int k_max) { return 1024 + kOffIdx + 2 * (size_t)((k_max + 7) & ~7); }
};

// mbarrier slots
enum {
  BAR_Q = 0,
  BAR_KFULL = 1,    // +stage (<= 3)
  BAR_VFULL = 4,    // +stage
  BAR_KVEMPTY = 7,  // +stage
  BAR_SFULL = 10,   // +S/P buffer (3)
  BAR_PVDONE = 13,  // +S/P buffer (3): PV of the tile in that buffer completed
  BAR_PFULL = 16,
  BAR_DRAIN = 17
};

// Warp-uniform bounded wait: every lane polls, the warp agrees on the result.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint64_t timeout_ns) {
  const bool ok = mbar_wait(bar, parity, abort, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

// Wait used only while shutting down after an abort: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy, timeout_ns);
}

template <int D, int BN, int NST>
__global__ void __launch_bounds__(192, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Geometry G,
                       const __grid_constant__ AttnArgs A) {
  using C = AttnCfg<D, BN, NST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = blockIdx.x % G.ntmax;
  const int bh = blockIdx.x / G.ntmax;
  const int h = bh % G.heads;
  const HeadGeom hg = G.g[h];
  if (i >= hg.nt) return;  // CTA-uniform, before any barrier or TMEM use
  const int S = G.S;

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  auto bar = [&](int b) { return bar0 + 8u * (uint32_t)b; };
  int* misc = reinterpret_cast<int*>(smem + C::kOffMisc);  // [0] tmem base, [1] abort, [2] n_sel
  int16_t* s_idx = reinterpret_cast<int16_t*>(smem + C::kOffIdx);
  volatile int* abort = misc + 1;

  if (tid == 0) {
    misc[1] = 0;
    misc[2] = A.k_max;
  }
  __syncthreads();
  const int32_t* irow = A.idx + ((long long)bh * G.ntmax + i) * A.k_max;
  for (int c = tid; c < A.k_max; c += C::kThreads) {
    const int v = irow[c];
    s_idx[c] = (int16_t)v;
    if (v < 0 || v >= hg.nt) atomicMin(&misc[2], c);  // the list ends at the first invalid entry
  }
  if (tid == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_KVEMPTY + s), 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(bar(BAR_SFULL + b), 1);
      mbar_init(bar(BAR_PVDONE + b), 1);
    }
    mbar_init(bar(BAR_PFULL), 4);
    mbar_init(bar(BAR_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc[0]), C::kTmemCols);
    tmem_relinquish();
  }
  if (BN < 128 && warp >= 2) {
    // S = 64: the MMA always runs 128 rows; rows 64..127 of the Q panels are zero.
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
  const int n_sel = misc[2];
  const uint64_t tmo = A.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0;
    bool q_issued = false;
    if (n_sel > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(bar(BAR_Q), (uint32_t)(S * D * 2));
        for (int c = 0; c < D / 64; ++c)
          tma_load_2d(sQ + c * C::kChunk, &tmQ, bar(BAR_Q), 64 * c, (bh * G.ntmax + i) * S);
      }
      q_issued = true;
      for (int t = 0; t < n_sel; ++t) {
        const int st = t % NST, fill = t / NST;
        if (fill >= 1 && !warp_wait(bar(BAR_KVEMPTY + st), (fill - 1) & 1, abort, tmo)) break;
        if (lane == 0) {
          const int y = (bh * G.ntmax + s_idx[t]) * S;
          mbar_arrive_expect_tx(bar(BAR_KFULL + st), (uint32_t)C::kKVBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(sK + st * C::kKVBytes + c * BN * 128, &tmK, bar(BAR_KFULL + st), 64 * c, y);
          mbar_arrive_expect_tx(bar(BAR_VFULL + st), (uint32_t)C::kKVBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(sV + st * C::kKVBytes + c * BN * 128, &tmV, bar(BAR_VFULL + st), 64 * c, y);
        }
        __syncwarp();
        issued = t + 1;
      }
    }
    if (*abort) {
      // Let every copy still in flight land before the CTA can exit.
      if (q_issued) drain_wait(bar(BAR_Q), 0, tmo);
      for (int t = issued > NST ? issued - NST : 0; t < issued; ++t) {
        drain_wait(bar(BAR_KFULL + t % NST), (t / NST) & 1, tmo);
        drain_wait(bar(BAR_VFULL + t % NST), (t / NST) & 1, tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (n_sel > 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, BN, false);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D, true);
      auto issue_s = [&](int t) -> bool {
        const int st = t % NST, b = t % 3;
        if (!warp_wait(bar(BAR_KFULL + st), (t / NST) & 1, abort, tmo)) return false;
        // The S/P buffer is free once the PV product of its previous tile is done.
        if (t >= 3 && !warp_wait(bar(BAR_PVDONE + b), ((t / 3) - 1) & 1, abort, tmo)) return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kbase = sK + st * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t da = make_sdesc_sw128(sQ + (kk >> 2) * C::kChunk + (kk & 3) * 32, 16, 1024);
            const uint64_t db = make_sdesc_sw128(kbase + (kk >> 2) * BN * 128 + (kk & 3) * 32, 16, 1024);
            umma_ss(tmem + b * 128, da, db, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(BAR_SFULL + b));
        }
        __syncwarp();
        return true;
      };
      bool ok = warp_wait(bar(BAR_Q), 0, abort, tmo) && issue_s(0);
      for (int t = 0; ok && t < n_sel; ++t) {
        if (t + 1 < n_sel && !(ok = issue_s(t + 1))) break;
        if (!(ok = warp_wait(bar(BAR_PFULL), t & 1, abort, tmo))) break;
        if (!(ok = warp_wait(bar(BAR_VFULL + t % NST), (t / NST) & 1, abort, tmo))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vbase = sV + (t % NST) * C::kKVBytes;
          const uint32_t pbase = tmem + (t % 3) * 128;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t db = make_sdesc_sw128(vbase + kk * 16 * 128, BN * 128, 1024);
            umma_ts(tmem + C::kTmemO, pbase + kk * 8, db, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar(BAR_KVEMPTY + t % NST));
          umma_commit(bar(BAR_PVDONE + t % 3));
        }
        __syncwarp();
      }
      // Every MMA issued above completes before TMEM is released.
      if (lane == 0) umma_commit(bar(BAR_DRAIN));
      __syncwarp();
      drain_wait(bar(BAR_DRAIN), 0, tmo);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = A.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < n_sel; ++t) {
      const int b = t % 3;
      if (!(ok = warp_wait(bar(BAR_SFULL + b), (t / 3) & 1, abort, tmo))) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_lane + b * 128 + c * 32, &s[c * 32]);
      tmem_ld_wait();

      // Pad keys of an edge tile are masked out.
      const int j = s_idx[t];
      const int jw = j % hg.nTw, jh = (j / hg.nTw) % hg.nTh, jt = j / (hg.nTw * hg.nTh);
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
      // Row maximum over 8 independent chains.
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
      // Lazy rescaling: keep the old reference maximum unless the new one is
      // more than 8 (log2 units) above it.
      float m_use;
      bool rescale = false;
      if (t == 0) {
        m_use = mt;
      } else if (mt > m_run + 8.0f) {
        m_use = mt;
        rescale = true;
      } else {
        m_use = m_run;
      }
      const float m_ref = (m_use == -INFINITY) ? 0.f : m_use;
      float r8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) r8[q] = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float x0 = fmaf(s[c], sl2, -m_ref);
        const float x1 = fmaf(s[c + 1], sl2, -m_ref);
        const float p0 = (c % kPolyEvery == kPolyEvery - 1) ? exp2_fma(x0) : fast_exp2(x0);
        const float p1 = ((c + 1) % kPolyEvery == kPolyEvery - 1) ? exp2_fma(x1) : fast_exp2(x1);
        r8[c & 7] += p0;
        r8[(c + 1) & 7] += p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      const float rs = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      const float alpha = rescale ? fast_exp2(m_run - m_ref) : 1.f;
      l_run = l_run * alpha + rs;
      m_run = m_use;

      // P_t (bf16 pairs) over the S_t row in TMEM: the A operand of PV_t.
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) tmem_st32u(t_lane + b * 128 + c * 32, &pk[c * 32]);

      // PV of the previous tile must be done before O is rescaled.
      if (t >= 1) {
        if (!(ok = warp_wait(bar(BAR_PVDONE + (t - 1) % 3), ((t - 1) / 3) & 1, abort, tmo))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(t_lane + C::kTmemO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] *= alpha;
            tmem_st32(t_lane + C::kTmemO + c * 32, o);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_PFULL));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n_sel > 0) ok = warp_wait(bar(BAR_PVDONE + (n_sel - 1) % 3), ((n_sel - 1) / 3) & 1, abort, tmo);
    if (ok) {
      tc_fence_after();
      const long long grow = ((long long)bh * G.ntmax + i) * S + row;
      const float inv_l = (l_run > 0.f) ? 1.0f / l_run : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(A.op) + grow * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (n_sel > 0) {
          tmem_ld32(t_lane + C::kTmemO + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] = 0.f;
        }
        if (row < S) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(o[q * 8 + 0] * inv_l, o[q * 8 + 1] * inv_l);
            v.y = pack_bf16x2(o[q * 8 + 2] * inv_l, o[q * 8 + 3] * inv_l);
            v.z = pack_bf16x2(o[q * 8 + 4] * inv_l, o[q * 8 + 5] * inv_l);
            v.w = pack_bf16x2(o[q * 8 + 6] * inv_l, o[q * 8 + 7] * inv_l);
            orow[c * 4 + q] = v;
          }
        }
      }
      if (A.lse != nullptr && row < S)
        A.lse[grow] = (n_sel > 0) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, int BN, int NST>
static cudaError_t launch_attn_t(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
  using C = AttnCfg<D, BN, NST>;
  const size_t smem = C::smem_bytes(a.k_max);
  cudaError_t err = cudaFuncSetAttribute(sparse_attn_kernel<D, BN, NST>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const unsigned blocks = (unsigned)(G.B * G.heads * G.ntmax);
  sparse_attn_kernel<D, BN, NST><<<blocks, C::kThreads, smem, s>>>(tq, tk, tv, G, a);
  return cudaGetLastError();
}

template <int D, int BN>
static cudaError_t launch_attn_d(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
  if (AttnCfg<D, BN, 3>::smem_bytes(a.k_max) <= (size_t)kSmemLimit) return launch_attn_t<D, BN, 3>(G, tq, tk, tv, a, s);
  return launch_attn_t<D, BN, 2>(G, tq, tk, tv, a, s);
}

size_t sparse_attn_smem_bytes(int d, int S, int k_max) {
  // the smallest configuration that can run (two stages)
  if (d == 128 && S == 128) return AttnCfg<128, 128, 2>::smem_bytes(k_max);
  if (d == 128 && S == 64) return AttnCfg<128, 64, 2>::smem_bytes(k_max);
  if (d == 64 && S == 128) return AttnCfg<64, 128, 2>::smem_bytes(k_max);
  return AttnCfg<64, 64, 2>::smem_bytes(k_max);
}

cudaError_t launch_sparse_attn(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
  if (G.d == 128 && G.S == 128) return launch_attn_d<128, 128>(G, tq, tk, tv, a, s);
  if (G.d == 128 && G.S == 64) return launch_attn_d<128, 64>(G, tq, tk, tv, a, s);
  if (G.d == 64 && G.S == 128) return launch_attn_d<64, 128>(G, tq, tk, tv, a, s);
  return launch_attn_d<64, 64>(G, tq, tk, tv, a, s);
}

}  // namespace veda
