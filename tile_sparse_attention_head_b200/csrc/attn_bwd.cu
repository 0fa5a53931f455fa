// Backward of the tile-skipping attention.  Section 2.3 of the Veda summary
// defines the forward (each Q tile attends to the keys of its selected K/V
// tiles only); the gradients are the chain rule through it, over the same
// selected tiles and nothing else:
//   P = softmax(scale Q K^T),  dV = P^T dO,  dP = dO V^T,
//   dX = P * (dP - D) with D = rowsum(dO * O) (= rowsum(P * dP)),
//   dQ = scale dX K,  dK = scale dX^T Q.
// All tensors are in grid order [B, heads, T*H*W, d]; the LSE is the one the
// forward wrote (natural log of the softmax denominator, scale included).
//
// Steps, all on the caller's stream:
//   attn_bwd_prep_kernel     per tile slot (L, D) = (lse log2 e, <dO, O>) in
//                            tile order, (+inf, 0) on pad slots (HBM-bound)
//   inv_scatter_kernel       bit (j, i) set when Q tile i selects K tile j
//   inv_build_kernel         per (b, h): for every K tile j the ascending list
//                            of the Q tiles that select it (count, scan, fill)
//   attn_bwd_kernel<KV = false>  one CTA per (b, h, Q tile i): dQ_i, streaming
//                            the selected K/V tiles
//   attn_bwd_kernel<KV = true>   one CTA per (b, h, K tile j): dK_j and dV_j,
//                            streaming Q/dO of every Q tile that selected j
// No atomics touch the gradients: each output row is written by one CTA, in a
// fixed order, so results are deterministic.
//
// The two tcgen05 kernels share one body.  A CTA holds a "stationary" pair of
// tiles (Q_i, dO_i or K_j, V_j, 128 TMEM lanes = its rows) and streams
// "moving" pairs (K_n, V_n or Q_n, dO_n):
//   T0 = A0 B0^T   (S, or S^T on the K side)
//   T1 = A1 B1^T   (dP, or dP^T)
//   softmax warps: P = 2^(T0 scale log2e - L), dS = P (T1 - D); once a warp
//   has read its part of T1 it writes dS (and on the K side P) back into it
//   as packed bf16, the "TS" operand form of the next products;
//   acc0 += dS B0  (dQ += dS K_n, or dK += dS^T Q_n)
//   acc1 += P B1   (dV += P^T dO_n, K side only)
// Two issuer warps keep the tensor pipe fed: one issues T0 and T1 of each
// moving tile as soon as their TMEM buffers are free, the other the
// accumulating products as soon as dS is packed.  T0 is released once the
// softmax warps have read it; T1 holds the packed operands until the
// accumulating products have read them.  The Q side has TMEM to spare and
// double-buffers T1; on the K side the two accumulators fill TMEM.  Columns:
//   Q side: T0 at 0, T1 buffer 0 at 128, dQ at 256, T1 buffer 1 at 384;
//   K side: T0 at 0, T1 at 128, dK at 256, dV at 384.
// Moving tiles: on the Q side K and V have rings of their own, and a V stage
// is released right after its T1 product, so the deeper K ring (3 stages at
// d = S = 128) refills one tile ahead of use; on the K side a stage holds Q,
// dO and the tile's (L, D) and is released after the accumulating products.
// The selection list (or inverse list) is staged in shared memory.
// Every wait is bounded; on a time-out each role leaves its loop, in-flight
// copies and products are drained and TMEM is freed.
#include "veda_common.cuh"
#include "kernels.h"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 6   // bounds-check site id of this file (debug builds)

namespace veda {

constexpr int kBwdSmemLimit = 232448;   // dynamic shared memory per CTA on sm_100
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int BN, bool KV>
struct BwdCfg {
  static constexpr int BM = 128;                     // MMA rows = stationary tile slots (S = 64 uses half)
  static constexpr int kThreads = 384;
  static constexpr int kChunk = 128 * 128;           // stationary panel: 128 rows x 128 B (64 channels)
  static constexpr int kStatBytes = BM * D * 2;
  static constexpr int kTileBytes = BN * D * 2;      // one moving tile
  static constexpr int kMaxStages = 4;
  static constexpr int kOffBar = 0;
  static constexpr int kNumBars = 32;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;    // [0] TMEM base, [1] abort, [2] list length
  static constexpr int kOffLD = kOffMisc + 64;               // K side: float2 (L, D) [stage][BN]
  static constexpr int kLDBytes = KV ? kMaxStages * BN * 8 : 0;
  static constexpr int kOffList = kOffLD + kLDBytes;         // int16 moving-tile list (first kListCap entries)
  static constexpr int kListCap = KV ? 4096 : 1024;
  static constexpr int kBookBytes = (kOffList + 2 * kListCap + 1023) & ~1023;
  static constexpr int kRingBytes = kBwdSmemLimit - kBookBytes - 2 * kStatBytes;
  // Q side: K ring (ST0) and V ring (ST1), one tile per stage, ST0 >= ST1.
  // K side: one ring (ST0 = ST1) of Q + dO stages.
  static constexpr int kPerPair = kRingBytes / (2 * kTileBytes);   // stages of both rings that fit
  static constexpr int kOdd = (kRingBytes - kPerPair * 2 * kTileBytes) >= kTileBytes ? 1 : 0;
  static constexpr int ST1 = kPerPair < kMaxStages ? kPerPair : kMaxStages;
  static constexpr int ST0 = KV ? ST1 : (ST1 + kOdd < kMaxStages ? ST1 + kOdd : kMaxStages);
  static_assert(ST1 >= 2, "the moving-tile rings need two stages");
  // operand region (1024-byte aligned): A0 | A1 | ring 0 | ring 1
  static constexpr int kOffA0 = 0;
  static constexpr int kOffA1 = kStatBytes;
  static constexpr int kOffRing0 = 2 * kStatBytes;
  static constexpr int kStride0 = KV ? 2 * kTileBytes : kTileBytes;   // K side: Q | dO per stage
  static constexpr int kOffRing1 = kOffRing0 + ST0 * kStride0;         // Q side only
  static constexpr size_t kSmemBytes =
      (size_t)kBookBytes + 2 * kStatBytes + (size_t)ST0 * kStride0 + (KV ? 0 : (size_t)ST1 * kTileBytes);
  static_assert(kSmemBytes <= (size_t)kBwdSmemLimit, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kT0 = 0, kT1 = 128, kAcc0 = 256, kAcc1 = 384;
  static constexpr uint32_t kT1b = 384;   // Q side: second T1 buffer (the K side's dV columns)
};

enum {
  BB_STAT = 0,      // stationary pair landed
  BB_FULL0 = 1,     // +stage: ring 0 (K; or Q, dO and (L, D)) landed
  BB_EMPTY0 = 5,    // +stage: the products reading ring 0's stage completed
  BB_FULL1 = 9,     // +stage: ring 1 (V, Q side) landed
  BB_EMPTY1 = 13,   // +stage: the T1 product reading ring 1's stage completed
  BB_T0 = 17,       // T0 of the current moving tile is in TMEM
  BB_T0FREE = 18,   // the softmax warps have read T0 (8 warp arrivals)
  BB_T1 = 19,       // +buffer: T1 of a moving tile is in TMEM
  BB_DSRDY = 21,    // dS (and P) packed into T1 (8 warp arrivals)
  BB_ACCDONE = 22,  // +buffer: the accumulating products have read T1
  BB_ACC = 24,      // every accumulating product completed (the epilogue's signal)
  BB_TDRAIN = 25    // every T product completed (the T issuer's drain)
};

__device__ __forceinline__ bool bwd_warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                              uint64_t timeout_ns) {
  const bool ok = mbar_wait(bar, parity, abort, timeout_ns);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void bwd_drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy, timeout_ns);
}

// Packed operands in T1: T1's columns are read in chunks of 32; once a chunk
// is in registers, dS of its 32 K elements goes to its first 16 columns and
// (K side) P to the next 16, two bf16 per column.  TMEM column offsets of
// K-step kk (16 K elements) within T1:
__device__ __forceinline__ uint32_t packed_ds_col(int kk) { return (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1)); }
__device__ __forceinline__ uint32_t packed_p_col(int kk) { return packed_ds_col(kk) + 16u; }

template <int D, int BN, bool KV>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_kernel(const __grid_constant__ BwdMaps<kMaxGridMaps> M, const __grid_constant__ Geometry G,
                    const __grid_constant__ BwdArgs A) {
  using C = BwdCfg<D, BN, KV>;
  constexpr int ST0 = C::ST0, ST1 = C::ST1;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {   // CTA-uniform, before any barrier or TMEM use
    if (threadIdx.x == 0) atomicExch(&g_device_error, kErrSmemAlign);
    return;
  }
  uint8_t* ops = smem + C::kBookBytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x % G.ntmax;                // the stationary tile
  const int hb = blockIdx.x / G.ntmax;
  const int h = A.head_list[hb % A.n_group];
  const int bh = (hb / A.n_group) * G.heads + h;
  const int mi = A.map_of_head[h];
  const HeadGeom hg = G.g[h];
  if (u >= hg.nt) return;   // CTA-uniform
  const int S = G.S;

  const CUtensorMap* mA0 = &M.a0[mi];
  const CUtensorMap* mA1 = &M.a1[mi];
  const CUtensorMap* mB0 = &M.b0[mi];
  const CUtensorMap* mB1 = &M.b1[mi];
  // Tile j of a grid-order tensor: one 5D box per 64 channels, panels
  // `panel` bytes apart.
  auto load_tile = [&](uint32_t dst, int panel, const CUtensorMap* map, uint32_t b, int j) {
    const int jw = j % hg.nTw, jh = (j / hg.nTw) % hg.nTh, jt = j / (hg.nTw * hg.nTh);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tma_load_5d(dst + c * panel, map, b, 64 * c, jw * hg.pw, jh * hg.ph, jt * hg.pt, bh);
  };

  const uint32_t sA0 = smem_u32(ops + C::kOffA0);
  const uint32_t sA1 = smem_u32(ops + C::kOffA1);
  const uint32_t sRing0 = smem_u32(ops + C::kOffRing0);
  const uint32_t sRing1 = smem_u32(ops + C::kOffRing1);
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  auto bar = [&](int b) { return bar0 + 8u * (uint32_t)b; };
  int* misc = reinterpret_cast<int*>(smem + C::kOffMisc);
  float2* s_ld = reinterpret_cast<float2*>(smem + C::kOffLD);
  int16_t* s_list = reinterpret_cast<int16_t*>(smem + C::kOffList);
  volatile int* abort = misc + 1;

  // The moving tiles: the selection row of Q tile u (up to its first entry
  // outside [0, NT_h)), or the Q tiles that selected K tile u.
  const int32_t* mov;
  int n_list;
  if constexpr (KV) {
    const int32_t* off = A.inv_off + (long long)bh * (G.ntmax + 1);
    const int o0 = off[u];
    n_list = off[u + 1] - o0;
    mov = A.inv_list + (long long)bh * G.ntmax * A.k_max + o0;
  } else {
    mov = A.idx + ((long long)bh * G.ntmax + u) * A.k_max;
    n_list = A.k_max;
  }
  if (tid == 0) {
    misc[1] = 0;
    misc[2] = n_list;
  }
  __syncthreads();
  for (int c = tid; c < n_list; c += C::kThreads) {
    const int v = mov[c];
    if (!KV && (v < 0 || v >= hg.nt)) atomicMin(&misc[2], c);
    if (KV) (void)VEDA_IN_BOUNDS(v >= 0 && v < hg.nt);   // the inverse lists hold Q tiles of this head
    if (c < C::kListCap) s_list[c] = (int16_t)v;
  }
  if (tid == 0) {
    mbar_init(bar(BB_STAT), 1);
    for (int s = 0; s < ST0; ++s) {
      mbar_init(bar(BB_FULL0 + s), 1);
      mbar_init(bar(BB_EMPTY0 + s), 1);
    }
    for (int s = 0; s < ST1; ++s) {
      mbar_init(bar(BB_FULL1 + s), 1);
      mbar_init(bar(BB_EMPTY1 + s), 1);
    }
    mbar_init(bar(BB_T0), 1);
    mbar_init(bar(BB_T0FREE), 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BB_T1 + b), 1);
      mbar_init(bar(BB_ACCDONE + b), 1);
    }
    mbar_init(bar(BB_DSRDY), 8);
    mbar_init(bar(BB_ACC), 1);
    mbar_init(bar(BB_TDRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc[0]), C::kTmemCols);
    tmem_relinquish();
  }
  if (BN < 128 && warp >= 4) {
    // S = 64: the products always run 128 rows; rows 64..127 of the
    // stationary panels are zero.
    for (int t = 0; t < 2; ++t)
      for (int c = 0; c < D / 64; ++c) {
        uint4* p = reinterpret_cast<uint4*>(ops + t * C::kStatBytes + c * C::kChunk + 64 * 128);
        for (int e = tid - 128; e < 64 * 128 / 16; e += 256) p[e] = make_uint4(0, 0, 0, 0);
      }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int n_mov = misc[2];
  const uint64_t tmo = A.timeout_ns;
  auto tile_at = [&](int n) -> int { return n < C::kListCap ? (int)s_list[n] : (int)mov[n]; };

  if (warp == 0 || (!KV && warp == 2)) {
    // ------------------------------------------------------------ TMA producers
    // Warp 0: the stationary pair, then ring 0 (K; or Q, dO and (L, D)).
    // Warp 2 (Q side): ring 1 (V).
    const bool r0 = warp == 0;
    const int st_n = r0 ? ST0 : ST1;
    int issued = 0;
    bool stat_issued = false;
    if (n_mov > 0) {
      if (r0 && lane == 0) {
        tma_prefetch_desc(mA0);
        tma_prefetch_desc(mA1);
        tma_prefetch_desc(mB0);
        mbar_arrive_expect_tx(bar(BB_STAT), (uint32_t)(2 * S * D * 2));
        load_tile(sA0, C::kChunk, mA0, bar(BB_STAT), u);
        load_tile(sA1, C::kChunk, mA1, bar(BB_STAT), u);
      }
      if (!r0 && lane == 0) tma_prefetch_desc(mB1);
      stat_issued = r0;
      for (int n = 0; n < n_mov; ++n) {
        const int st = n % st_n, fill = n / st_n;
        if (fill >= 1 &&
            !bwd_warp_wait(bar((r0 ? BB_EMPTY0 : BB_EMPTY1) + st), (fill - 1) & 1, abort, tmo))
          break;
        if (lane == 0) {
          const int t = tile_at(n);
          if (r0) {
            const uint32_t dst = sRing0 + (uint32_t)(st * C::kStride0);
            if constexpr (KV) {
              mbar_arrive_expect_tx(bar(BB_FULL0 + st), (uint32_t)(2 * C::kTileBytes + BN * 8));
              load_tile(dst, BN * 128, mB0, bar(BB_FULL0 + st), t);
              load_tile(dst + C::kTileBytes, BN * 128, mB1, bar(BB_FULL0 + st), t);
              bulk_load(smem_u32(s_ld + st * BN), A.ldt + ((long long)bh * G.ntmax + t) * S, (uint32_t)(BN * 8),
                        bar(BB_FULL0 + st));
            } else {
              mbar_arrive_expect_tx(bar(BB_FULL0 + st), (uint32_t)C::kTileBytes);
              load_tile(dst, BN * 128, mB0, bar(BB_FULL0 + st), t);
            }
          } else {
            mbar_arrive_expect_tx(bar(BB_FULL1 + st), (uint32_t)C::kTileBytes);
            load_tile(sRing1 + (uint32_t)(st * C::kTileBytes), BN * 128, mB1, bar(BB_FULL1 + st), t);
          }
        }
        __syncwarp();
        issued = n + 1;
      }
    }
    if (*abort) {
      if (stat_issued) bwd_drain_wait(bar(BB_STAT), 0, tmo);
      for (int n = issued > st_n ? issued - st_n : 0; n < issued; ++n)
        bwd_drain_wait(bar((r0 ? BB_FULL0 : BB_FULL1) + n % st_n), (n / st_n) & 1, tmo);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ tcgen05 issuer: T0, T1
    if (n_mov > 0) {
      constexpr uint32_t idesc_t = make_idesc_bf16(128, BN, false);   // T = A B^T, both K-major
      const uint64_t da0 = make_sdesc_sw128(sA0, 16, 1024);
      const uint64_t da1 = make_sdesc_sw128(sA1, 16, 1024);
      // T = A x (moving tile at shared address sb)^T, K = D
      auto product_t = [&](uint32_t t_col, uint64_t da, uint32_t sb) {
        const uint64_t db = make_sdesc_sw128(sb, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * C::kChunk + (kk & 3) * 32;
          const uint32_t bo = (kk >> 2) * BN * 128 + (kk & 3) * 32;
          umma_ss(tmem + t_col, da + (ao >> 4), db + (bo >> 4), idesc_t, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = bwd_warp_wait(bar(BB_STAT), 0, abort, tmo);
      for (int n = 0; ok && n < n_mov; ++n) {
        const int s0 = n % ST0, s1 = n % ST1;
        if (!(ok = bwd_warp_wait(bar(BB_FULL0 + s0), (n / ST0) & 1, abort, tmo))) break;
        if (n >= 1 && !(ok = bwd_warp_wait(bar(BB_T0FREE), (n - 1) & 1, abort, tmo))) break;
        tc_fence_after();
        const uint32_t b0 = sRing0 + (uint32_t)(s0 * C::kStride0);
        if (lane == 0) {
          product_t(C::kT0, da0, b0);
          umma_commit(bar(BB_T0));
        }
        __syncwarp();
        if (!KV && !(ok = bwd_warp_wait(bar(BB_FULL1 + s1), (n / ST1) & 1, abort, tmo))) break;
        // T1's buffer is free once the accumulating products of the tile
        // that last used it have read it.
        const int b = KV ? 0 : (n & 1);
        const int use = KV ? n : (n >> 1);   // earlier uses of this buffer
        if (use >= 1 && !(ok = bwd_warp_wait(bar(BB_ACCDONE + b), (use - 1) & 1, abort, tmo))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t b1 = KV ? b0 + C::kTileBytes : sRing1 + (uint32_t)(s1 * C::kTileBytes);
          product_t(b == 0 ? C::kT1 : C::kT1b, da1, b1);
          umma_commit(bar(BB_T1 + b));
          if (!KV) umma_commit(bar(BB_EMPTY1 + s1));   // V is read by this product only
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit(bar(BB_TDRAIN));
      __syncwarp();
      bwd_drain_wait(bar(BB_TDRAIN), 0, tmo);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ tcgen05 issuer: accumulating products
    if (n_mov > 0) {
      constexpr uint32_t idesc_acc = make_idesc_bf16(128, D, true);   // acc += (packed T1) B, B MN-major
      bool ok = true;
      for (int n = 0; ok && n < n_mov; ++n) {
        if (!(ok = bwd_warp_wait(bar(BB_DSRDY), n & 1, abort, tmo))) break;
        tc_fence_after();
        const int b = KV ? 0 : (n & 1);
        const uint32_t t1 = tmem + (b == 0 ? C::kT1 : C::kT1b);
        if (lane == 0) {
          const uint32_t sb0 = sRing0 + (uint32_t)((n % ST0) * C::kStride0);
          const uint64_t d0 = make_sdesc_sw128(sb0, BN * 128, 1024);   // moving tile as an MN-major operand
          // dQ += dS K_n, or dK += dS^T Q_n
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_ts(tmem + C::kAcc0, t1 + packed_ds_col(kk), d0 + ((kk * 16 * 128) >> 4), idesc_acc,
                    (n > 0 || kk > 0) ? 1u : 0u);
          if constexpr (KV) {
            // dV += P^T dO_n
            const uint64_t d1 = make_sdesc_sw128(sb0 + C::kTileBytes, BN * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              umma_ts(tmem + C::kAcc1, t1 + packed_p_col(kk), d1 + ((kk * 16 * 128) >> 4), idesc_acc,
                      (n > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar(BB_EMPTY0 + n % ST0));
          umma_commit(bar(BB_ACCDONE + b));
        }
        __syncwarp();
      }
      // Completes after every accumulating product: the epilogue's signal,
      // and the drain before TMEM is released.
      if (lane == 0) umma_commit(bar(BB_ACC));
      __syncwarp();
      bwd_drain_wait(bar(BB_ACC), 0, tmo);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax and epilogue
    constexpr int HC = BN / 2;                 // columns of T per warpgroup
    const int w = (warp - 4) >> 2;             // column half
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;       // TMEM lane = stationary slot
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const int c0 = w * HC;
    const int n_row = row < BN ? slot_to_grid(G, hg, u, row) : -1;
    const bool rvalid = n_row >= 0;
    float Lrow = INFINITY, Drow = 0.f;         // Q side: per-row L and D
    if constexpr (!KV) {
      if (row < BN) {
        const float2 v = A.ldt[((long long)bh * G.ntmax + u) * S + row];
        Lrow = v.x;
        Drow = v.y;
      }
    }
    const float sl2 = A.scale_log2;
    // Q side: slot offsets of this lane's key columns c0 + 32 q + lane, for
    // the pad-key mask of edge K tiles.
    int8_t kt[HC / 32], ky[HC / 32], kx[HC / 32];
#pragma unroll
    for (int q = 0; q < HC / 32; ++q) {
      const int c = c0 + 32 * q + lane;
      kx[q] = (int8_t)(c % hg.pw);
      ky[q] = (int8_t)((c / hg.pw) % hg.ph);
      kt[q] = (int8_t)(c / (hg.pw * hg.ph));
    }
    bool ok = true;
    for (int n = 0; n < n_mov; ++n) {
      const int b = KV ? 0 : (n & 1);          // T1 buffer
      uint32_t mw[HC / 32];
#pragma unroll
      for (int q = 0; q < HC / 32; ++q) mw[q] = 0xffffffffu;
      if constexpr (!KV) {
        const int t = tile_at(n);
        const int jw = t % hg.nTw, jh = (t / hg.nTw) % hg.nTh, jt = t / (hg.nTw * hg.nTh);
        const int ct = min((int)hg.pt, G.T - jt * hg.pt);
        const int ch = min((int)hg.ph, G.H - jh * hg.ph);
        const int cw = min((int)hg.pw, G.W - jw * hg.pw);
        if (ct * ch * cw != S) {
#pragma unroll
          for (int q = 0; q < HC / 32; ++q) mw[q] = __ballot_sync(0xffffffffu, kt[q] < ct && ky[q] < ch && kx[q] < cw);
        }
      }
      // The stage's (L, D) are visible once its full barrier has completed.
      if (KV && !(ok = bwd_warp_wait(bar(BB_FULL0 + n % ST0), (n / ST0) & 1, abort, tmo))) break;
      if (!(ok = bwd_warp_wait(bar(BB_T0), n & 1, abort, tmo))) break;
      tc_fence_after();
      const float2* ld = s_ld + (n % ST0) * BN + c0;
      const uint32_t t0 = t_lane + C::kT0 + c0;
      const uint32_t t1 = t_lane + (b == 0 ? C::kT1 : C::kT1b) + c0;
      float p[HC];
#pragma unroll
      for (int q = 0; q < HC / 32; ++q) {
        float x[32];
        tmem_ld32(t0 + 32 * q, x);
        tmem_ld_wait();
        if constexpr (KV) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float4 v = *reinterpret_cast<const float4*>(ld + 32 * q + 2 * e);   // (L, D) of 2 columns
            p[32 * q + 2 * e] = rvalid ? fast_exp2(fmaf(x[2 * e], sl2, -v.x)) : 0.f;
            p[32 * q + 2 * e + 1] = rvalid ? fast_exp2(fmaf(x[2 * e + 1], sl2, -v.z)) : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float pe = fast_exp2(fmaf(x[e], sl2, -Lrow));
            p[32 * q + e] = ((mw[q] >> e) & 1u) ? pe : 0.f;
          }
        }
      }
      // T0 is in registers: the issuer may start the next tile's T0 product.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BB_T0FREE));
      if (!(ok = bwd_warp_wait(bar(BB_T1 + b), KV ? (n & 1) : ((n >> 1) & 1), abort, tmo))) break;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < HC / 32; ++q) {
        float y[32];
        tmem_ld32(t1 + 32 * q, y);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float d0 = Drow, d1 = Drow;
          if constexpr (KV) {
            const float4 v = *reinterpret_cast<const float4*>(ld + 32 * q + 2 * e);
            d0 = v.y;
            d1 = v.w;
          }
          const float g0 = p[32 * q + 2 * e] * (y[2 * e] - d0);
          const float g1 = p[32 * q + 2 * e + 1] * (y[2 * e + 1] - d1);
          pk[e] = pack_bf16x2(g0, g1);
        }
        tmem_st16u(t1 + 32 * q, pk);            // dS
        if constexpr (KV) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(p[32 * q + 2 * e], p[32 * q + 2 * e + 1]);
          tmem_st16u(t1 + 32 * q + 16, pk);     // P
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BB_DSRDY));
    }

    // Epilogue: this warpgroup's half of the accumulator columns, scaled,
    // rounded to bf16 and written to the stationary tile's grid rows.
    const bool have = n_mov > 0 && ok;
    if (have) {
      ok = bwd_warp_wait(bar(BB_ACC), 0, abort, tmo);
      tc_fence_after();
    }
    constexpr int HD = D / 2;
    const int d0 = w * HD;
    const int n_out = KV ? 2 : 1;
    for (int o = 0; o < n_out; ++o) {
      const uint32_t acc = o == 0 ? C::kAcc0 : C::kAcc1;
      const float mul = o == 0 ? A.scale : 1.0f;       // dQ and dK carry the scale, dV does not
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(o == 0 ? A.dx : A.dv);
#pragma unroll
      for (int q = 0; q < HD / 32; ++q) {
        float a[32];
        if (have && ok) {
          tmem_ld32(t_lane + acc + d0 + 32 * q, a);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0.f;
        }
        if (rvalid && VEDA_IN_BOUNDS(n_row >= 0 && n_row < G.N)) {
          uint4* dst = reinterpret_cast<uint4*>(out + ((long long)bh * G.N + n_row) * D + d0 + 32 * q);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 pkt;
            pkt.x = pack_bf16x2(a[8 * v4 + 0] * mul, a[8 * v4 + 1] * mul);
            pkt.y = pack_bf16x2(a[8 * v4 + 2] * mul, a[8 * v4 + 3] * mul);
            pkt.z = pack_bf16x2(a[8 * v4 + 4] * mul, a[8 * v4 + 5] * mul);
            pkt.w = pack_bf16x2(a[8 * v4 + 6] * mul, a[8 * v4 + 7] * mul);
            dst[v4] = pkt;
          }
        }
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

// Per tile slot of every (b, h): (L, D) = (lse log2 e, <dO, O>) of the slot's
// grid row, in fp32, or (+inf, 0) for a pad slot (a zero probability and no
// contribution).  d / 8 threads per slot, 16 bytes of each row apiece.
template <int D>
__global__ void __launch_bounds__(256)
    attn_bwd_prep_kernel(const __grid_constant__ Geometry G, const uint4* __restrict__ o, const uint4* __restrict__ g,
                         const float* __restrict__ lse, float2* __restrict__ ldt) {
  constexpr int TPR = D / 8;
  const long long slots = (long long)G.B * G.heads * G.ntmax * G.S;
  const long long total = slots * TPR;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long iters = (total + stride - 1) / stride;
  for (long long it = 0; it < iters; ++it) {   // the same trip count for every lane
    const long long x = it * stride + blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long sidx = x / TPR;
    float s = 0.f;
    int n = -1;
    bool live = false;
    long long bh = 0;
    if (x < total) {
      const int l = (int)(sidx % G.S);
      const int j = (int)((sidx / G.S) % G.ntmax);
      bh = sidx / ((long long)G.S * G.ntmax);
      const HeadGeom& hg = G.g[bh % G.heads];
      live = j < hg.nt;
      if (live) n = slot_to_grid(G, hg, j, l);
      if (n >= 0) {
        const long long r = (bh * G.N + n) * TPR + (x % TPR);
        const uint4 a = __ldg(o + r), b = __ldg(g + r);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = __bfloat1622float2(a2[e]), fb = __bfloat1622float2(b2[e]);
          s = fmaf(fa.x, fb.x, s);
          s = fmaf(fa.y, fb.y, s);
        }
      }
    }
#pragma unroll
    for (int off = TPR / 2; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (live && (x % TPR) == 0)
      ldt[sidx] = n >= 0 ? make_float2(lse[bh * G.N + n] * kLog2e, s) : make_float2(INFINITY, 0.f);
  }
}

// Bit (j, i) of the per-(b, h) matrix [NT_max, W words] is set when Q tile
// i selects K tile j.  One thread per selection row; a row is read up to its
// first entry outside [0, NT_h), as the forward reads it.
__global__ void inv_scatter_kernel(const __grid_constant__ Geometry G, const int32_t* __restrict__ idx, int k_max,
                                   uint32_t* __restrict__ bits, int W) {
  const long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (r >= (long long)G.B * G.heads * G.ntmax) return;
  const int i = (int)(r % G.ntmax);
  const long long bh = r / G.ntmax;
  const int nt = G.g[bh % G.heads].nt;
  if (i >= nt) return;
  const int32_t* row = idx + r * k_max;
  for (int c = 0; c < k_max; ++c) {
    const int j = row[c];
    if (j < 0 || j >= nt) break;
    atomicOr(&bits[(bh * G.ntmax + j) * W + (i >> 5)], 1u << (i & 31));
  }
}

// One block per (b, h): off[j] = number of (Q tile, K tile j') selections
// with j' < j, list[off[j] .. off[j+1]) = the Q tiles selecting K tile j, in
// ascending order.
__global__ void __launch_bounds__(1024)
    inv_build_kernel(const __grid_constant__ Geometry G, const uint32_t* __restrict__ bits, int W,
                     int32_t* __restrict__ off_all, int32_t* __restrict__ list_all, int k_max) {
  __shared__ int wsum[32];
  const int bh = blockIdx.x;
  const int nt = G.g[bh % G.heads].nt;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* off = off_all + (long long)bh * (G.ntmax + 1);
  const uint32_t* bb = bits + (long long)bh * G.ntmax * W;
  for (int j = warp; j < G.ntmax; j += 32) {
    int c = 0;
    if (j < nt)
      for (int x = lane; x < W; x += 32) c += __popc(bb[(long long)j * W + x]);
#pragma unroll
    for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) off[j + 1] = c;
  }
  if (threadIdx.x == 0) off[0] = 0;
  __syncthreads();
  // In-place inclusive scan of off[1 .. NT_max]: a contiguous segment per
  // thread, then a block scan of the segment totals.
  const int seg = (G.ntmax + 1023) / 1024;
  const int s0 = 1 + threadIdx.x * seg, s1 = min(G.ntmax + 1, s0 + seg);
  int local = 0;
  for (int x = s0; x < s1; ++x) local += off[x];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    wsum[lane] = v;
  }
  __syncthreads();
  int run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
  for (int x = s0; x < s1; ++x) {
    run += off[x];
    off[x] = run;
  }
  __syncthreads();
  int32_t* list = list_all + (long long)bh * G.ntmax * k_max;
  for (int j = warp; j < nt; j += 32) {
    int base = off[j];
    for (int x0 = 0; x0 < W; x0 += 32) {
      const int x = x0 + lane;
      uint32_t m = x < W ? bb[(long long)j * W + x] : 0u;
      const int c = __popc(m);
      int inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      int pos = base + inc - c;
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1;
        list[pos++] = x * 32 + b;
      }
      base += __shfl_sync(0xffffffffu, inc, 31);
    }
  }
}

// Workspace: (L, D) per tile slot [B*heads, NT_max, S] float2 | selection
// bits [B*heads, NT_max, W] | offsets [B*heads, NT_max + 1] | lists
// [B*heads, NT_max * k_max], each part starting on a 256-byte boundary.
static size_t bwd_round256(size_t x) { return (x + 255) & ~size_t(255); }

static void attn_bwd_ws_parts(const Geometry& G, int k_max, size_t* p) {
  const size_t bh = (size_t)G.B * G.heads;
  const size_t W = (size_t)(G.ntmax + 31) / 32;
  p[0] = bwd_round256(sizeof(float2) * bh * G.ntmax * G.S);
  p[1] = bwd_round256(sizeof(uint32_t) * bh * G.ntmax * W);
  p[2] = bwd_round256(sizeof(int32_t) * bh * (G.ntmax + 1));
  p[3] = bwd_round256(sizeof(int32_t) * bh * G.ntmax * (size_t)k_max);
}

size_t attn_bwd_ws_bytes(const Geometry& G, int k_max) {
  size_t p[4];
  attn_bwd_ws_parts(G, k_max, p);
  return p[0] + p[1] + p[2] + p[3];
}

cudaError_t launch_attn_bwd_prep(const Geometry& G, const void* o, const void* dout, const float* lse,
                                 const int32_t* idx, int k_max, void* ws, BwdArgs* a, cudaStream_t s) {
  size_t p[4];
  attn_bwd_ws_parts(G, k_max, p);
  char* base = static_cast<char*>(ws);
  float2* ldt = reinterpret_cast<float2*>(base);
  uint32_t* bits = reinterpret_cast<uint32_t*>(base + p[0]);
  int32_t* off = reinterpret_cast<int32_t*>(base + p[0] + p[1]);
  int32_t* list = reinterpret_cast<int32_t*>(base + p[0] + p[1] + p[2]);
  const int W = (G.ntmax + 31) / 32;
  const long long work = (long long)G.B * G.heads * G.ntmax * G.S * (G.d / 8);
  const unsigned grid_prep = (unsigned)std::min<long long>((work + 255) / 256, 148LL * 16);
  if (G.d == 128)
    attn_bwd_prep_kernel<128><<<grid_prep, 256, 0, s>>>(G, static_cast<const uint4*>(o),
                                                        static_cast<const uint4*>(dout), lse, ldt);
  else
    attn_bwd_prep_kernel<64><<<grid_prep, 256, 0, s>>>(G, static_cast<const uint4*>(o),
                                                       static_cast<const uint4*>(dout), lse, ldt);
  const long long n4 = (long long)(p[1] / 16);
  fill_zero_kernel<<<(unsigned)std::min<long long>((n4 + 255) / 256, 148 * 8), 256, 0, s>>>(
      reinterpret_cast<float4*>(bits), n4);
  const long long nrows = (long long)G.B * G.heads * G.ntmax;
  inv_scatter_kernel<<<(unsigned)((nrows + 255) / 256), 256, 0, s>>>(G, idx, k_max, bits, W);
  inv_build_kernel<<<(unsigned)(G.B * G.heads), 1024, 0, s>>>(G, bits, W, off, list, k_max);
  a->idx = idx;
  a->k_max = k_max;
  a->ldt = ldt;
  a->inv_off = off;
  a->inv_list = list;
  return cudaGetLastError();
}

template <int D, int BN, bool KV>
static cudaError_t launch_bwd_t(const Geometry& G, const BwdMaps<kMaxGridMaps>& m, const BwdArgs& a,
                                cudaStream_t s) {
  using C = BwdCfg<D, BN, KV>;
  auto kernel = attn_bwd_kernel<D, BN, KV>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes);
  if (err != cudaSuccess) return err;
  const unsigned blocks = (unsigned)(G.B * a.n_group * G.ntmax);
  kernel<<<blocks, C::kThreads, C::kSmemBytes, s>>>(m, G, a);
  return cudaGetLastError();
}

template <bool KV>
static cudaError_t launch_bwd_kind(const Geometry& G, const BwdMaps<kMaxGridMaps>& m, const BwdArgs& a,
                                   cudaStream_t s) {
  if (G.d == 128 && G.S == 128) return launch_bwd_t<128, 128, KV>(G, m, a, s);
  if (G.d == 128 && G.S == 64) return launch_bwd_t<128, 64, KV>(G, m, a, s);
  if (G.d == 64 && G.S == 128) return launch_bwd_t<64, 128, KV>(G, m, a, s);
  return launch_bwd_t<64, 64, KV>(G, m, a, s);
}

cudaError_t launch_attn_bwd_dq(const Geometry& G, const BwdMaps<kMaxGridMaps>& m, const BwdArgs& a, cudaStream_t s) {
  return launch_bwd_kind<false>(G, m, a, s);
}

cudaError_t launch_attn_bwd_dkdv(const Geometry& G, const BwdMaps<kMaxGridMaps>& m, const BwdArgs& a,
                                 cudaStream_t s) {
  return launch_bwd_kind<true>(G, m, a, s);
}

}  // namespace veda
