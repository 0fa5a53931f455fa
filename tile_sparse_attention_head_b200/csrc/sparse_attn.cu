// Tile-skipping sparse attention on the sm_100a tensor cores (section 2.3 of
// the Veda summary: a block-sparse attention kernel that fetches only the
// selected, non-contiguous K/V tiles and hides the data movement behind the
// matrix math with warp-specialised producer/consumer roles).
//
// Blackwell design: a persistent kernel, one CTA per SM, each CTA working
// through the (b, h, Q tile) items gridDim.x apart; 12 warps in 3 warpgroups.
// Every role keeps its own ring counters and barrier phases running across
// items, so one item's tail (the last PV products, the merge of the two
// softmax streams, the stores of O) overlaps the next item's Q load and first
// score products instead of being paid per CTA.
//   warp 0       K producer: loads each item's selection list into one of two
//                shared-memory slots (the next item's while the current one
//                runs), prefetches the next item's Q tile into L2, loads the Q
//                tile once the score products of the previous item are done
//                with the Q buffer, then K_j of every selected tile j into a
//                KST-stage ring.  A permuted tile is S contiguous rows, so each
//                fetch is a plain 2D TMA box; on grid-order tensors it is one 5D
//                box (the tile's pt x ph x pw tokens), which lands in shared
//                memory in the same slot order.  Panels are 128-byte swizzled
//                for the tensor cores.  A K stage is released as soon as the
//                score product has read it.
//   warp 2       V producer: V_j into a VST-stage ring, released after PV.
//   warp 1       tcgen05 issuer of the score products S_t = Q K_t^T into the
//                single TMEM S buffer, freed as soon as the owning stream has
//                loaded S_t into registers.
//   warp 3       tcgen05 issuer of the PV products O_s += P_t V_t (P read from
//                TMEM, the "TS" form).  The first PV of an item waits until the
//                previous item's epilogue has read O out of TMEM.  Each
//                issuer's tcgen05.commit tracks only its own products.
//   warps 4-7    softmax stream A: the tiles t = 0, 2, 4, ... of each list;
//   warps 8-11   softmax stream B: the tiles t = 1, 3, 5, ...
//                Each stream keeps its own online softmax (running maximum,
//                row sum) and its own O accumulator, so the two warps that
//                share a scheduler work on different tiles and never wait for
//                each other; a thread owns one query row (its TMEM lane) and
//                all BN columns of it.  Exponentials run in the log2 domain on
//                the special-function unit; O is rescaled in TMEM only
//                when the stream's maximum grows by more than 2^8; P is
//                written as packed bf16 to the stream's own P buffer.
//                At the end of an item the two partial results are merged
//                exactly:
//                O = (2^(mA-m) O_A + 2^(mB-m) O_B) / (2^(mA-m) l_A + 2^(mB-m) l_B),
//                read out of TMEM, the O buffers released, then stored.
// TMEM (512 columns): S (128), P_A and P_B (64 each), O_A and O_B (128 each).
// Registers: the producer/issuer warpgroup gives registers back
// (setmaxnreg) so the softmax warpgroups can hold a whole S row.
// Every wait is bounded (veda_common.cuh) and the item loops use mbarriers
// only (no named barriers), so on a time-out every role leaves its loops,
// in-flight copies and MMAs are drained and TMEM is freed.
#include "veda_common.cuh"
#include "kernels.h"
#undef VEDA_SRC_ID
#define VEDA_SRC_ID 4   // bounds-check site id of this file (debug builds)

namespace veda {

// Every exponential runs on the special-function unit (ex2.approx).  The
// kernel runs at the board's power cap under sustained load, where throughput
// follows energy per tile: moving a share of the exponentials to an FMA-pipe
// polynomial balances the pipes but costs more instructions, and measured at
// sustained load it is slower (1/8 of them: -3%, 3/8: -9%).
// Share of the exponentials computed on the FMA pipe (a fitted cubic,
// exp2_fma_x2) instead of the special-function unit: out of every 8 column
// pairs of a score row, the first VEDA_EXP_POLY8.
#ifndef VEDA_EXP_POLY8
#define VEDA_EXP_POLY8 0
#endif
constexpr int kSmemLimit = 232448;   // dynamic shared memory per CTA on sm_100

// Shared memory: the bookkeeping (barriers, the final (m, l) exchange, flags,
// two selection-list slots) first, then -- from the next 1024-byte boundary,
// as the 128-byte swizzle needs -- the operand region Q | K ring | V ring.
// The dynamic shared memory base must itself be 1024-byte aligned (checked).
template <int D, int BN, int KST, int VST>
struct AttnCfg {
  static constexpr int BM = 128;                 // MMA rows (query slots; S = 64 tiles use half)
  static constexpr int kThreads = 384;
  static constexpr int kChunk = 128 * 128;       // one [128 rows x 128 B] swizzle panel
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kTileBytes = BN * D * 2;  // one K or V tile
  static constexpr int kOffBar = 0;
  static constexpr int kNumBars = 40;
  static constexpr int kOffRed = kOffBar + kNumBars * 8;   // float [2 stream][2: m, l][128 rows]
  static constexpr int kOffMisc = kOffRed + 2 * 2 * 128 * 4;
  static constexpr int kOffList = kOffMisc + 64;           // int16 selection lists [2 slots][cap]
  __host__ __device__ static int list_cap(int k_max) { return (k_max + 7) & ~7; }
  __host__ __device__ static size_t bookkeeping_bytes(int k_max) {
    return (kOffList + 4 * (size_t)list_cap(k_max) + 1023) & ~size_t(1023);
  }
  // offsets inside the operand region
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + KST * kTileBytes;
  static constexpr int kOperandBytes = kOffV + VST * kTileBytes;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmemS = 0;          // S, shared by the streams
  static constexpr uint32_t kTmemP = 128;        // P of stream s at kTmemP + 64 s (packed bf16)
  static constexpr uint32_t kTmemO = 256;        // O of stream s at kTmemO + 128 s
  static size_t smem_bytes(int k_max) { return bookkeeping_bytes(k_max) + kOperandBytes; }
};

// mbarrier slots
enum {
  BAR_QFULL = 0,    // the item's Q tile is in shared memory
  BAR_QEMPTY = 1,   // the item's score products are done with the Q buffer
  BAR_KFULL = 2,    // +stage (<= 4)
  BAR_KEMPTY = 6,   // +stage
  BAR_VFULL = 10,   // +stage (<= 4)
  BAR_VEMPTY = 14,  // +stage
  BAR_SFULL = 18,   // +stream: S of the stream's current tile is in TMEM
  BAR_SFREE = 20,   // +stream: the stream has loaded its S from TMEM (4 arrivals)
  BAR_PFULL = 22,   // +stream: P of the stream's current tile is in TMEM (4 arrivals)
  BAR_PVDONE = 24,  // +stream: the stream's last PV product completed
  BAR_XFIN = 26,    // final (m, l) exchange between the streams (256 arrivals)
  BAR_OFREE = 27,   // the epilogue has read O_A and O_B out of TMEM (8 arrivals)
  BAR_LFULL = 28,   // +slot: the selection list of an item is in its slot (32 arrivals)
  BAR_LEMPTY = 30,  // +slot: every consumer is done with the slot (11 arrivals)
  BAR_DRAIN = 32,   // score-product issuer drain
  BAR_DRAIN2 = 33   // PV-product issuer drain
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

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
  static_assert(N % 16 == 0, "");
#pragma unroll
  for (int c = 0; c + 32 <= N; c += 32) tmem_ld32(taddr + c, v + c);
  if constexpr (N % 32 == 16) tmem_ld16(taddr + (N - 16), v + (N - 16));
}

template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const float* v) {
#pragma unroll
  for (int c = 0; c + 32 <= N; c += 32) tmem_st32(taddr + c, v + c);
  if constexpr (N % 32 == 16) tmem_st16(taddr + (N - 16), v + (N - 16));
}

template <int N>
__device__ __forceinline__ void tmem_st_cols_u(uint32_t taddr, const uint32_t* v) {
#pragma unroll
  for (int c = 0; c + 32 <= N; c += 32) tmem_st32u(taddr + c, v + c);
  if constexpr (N % 32 == 16) tmem_st16u(taddr + (N - 16), v + (N - 16));
}

// One work item: Q tile i of head h (batch-head row bh), whose tile boxes use
// the launch's tensor maps number mi.
struct AttnItem {
  int i, h, bh, mi;
};

// Items of a launch are numbered with the Q tile fastest: w = (b * heads of
// the launch + position in the launch's head list) * NT_max + i.  Returns
// false for an item whose Q tile does not exist in its head (i >= NT_h).
template <bool GRID>
__device__ __forceinline__ bool attn_item(const Geometry& G, const AttnArgs& A, int w, AttnItem& it) {
  it.i = w % G.ntmax;
  const int hb = w / G.ntmax;
  if constexpr (GRID) {
    it.h = A.head_list[hb % A.n_group];
    it.bh = (hb / A.n_group) * G.heads + it.h;
    it.mi = A.map_of_head[it.h];
  } else {
    it.bh = hb;
    it.h = hb % G.heads;
    it.mi = 0;
  }
  return it.i < G.g[it.h].nt;
}

// The first item of this CTA at or after w (stepping by gridDim.x) whose Q
// tile exists, or n_items when there is none.  Every role walks the same
// sequence.
template <bool GRID>
__device__ __forceinline__ int next_attn_item(const Geometry& G, const AttnArgs& A, int w, int n_items,
                                              AttnItem& it) {
  for (; w < n_items; w += gridDim.x)
    if (attn_item<GRID>(G, A, w, it)) return w;
  return n_items;
}

// Exact quotient j / n for j, n < 2^16 with the reciprocal m = ceil(2^32 / n)
// (the error j * (m - 2^32/n) / 2^32 stays below 1/n, so the floor does not
// move).
__device__ __forceinline__ uint32_t div_by_recip(uint32_t j, uint64_t m) {
  return (uint32_t)(((uint64_t)j * m) >> 32);
}
// ceil(2^32 / n) from a 32-bit division: floor((2^32 - 1) / n) + 1 for n >= 2
// (equal whether or not n divides 2^32), 2^32 for n = 1.
__device__ __forceinline__ uint64_t recip_ceil(uint32_t n) {
  return n == 1u ? 0x100000000ull : (uint64_t)(0xffffffffu / n) + 1ull;
}

// GRID = false: Q/K/V/O are tile-major [B, heads, NT_max*S, d]; tile j of a
// head is rows j*S .. j*S+S-1, fetched as one 2D box per 64 channels.
// GRID = true: Q/K/V/O stay in grid order [B, heads, T*H*W, d].  Seen as the
// 5D array [B*heads, T, H, W, d], tile j of a head with tiling (pt, ph, pw)
// is the box of pt x ph x pw tokens at (jt*pt, jh*ph, jw*pw); TMA writes the
// box to shared memory with w fastest, then h, then t -- exactly the
// within-tile slot order -- and fills the part of an edge box that lies
// outside the grid with zeros, as the permutation does for pad slots.  O and
// the LSE of each valid query slot are written straight to its grid row.
template <int D, int BN, int KST, int VST, bool GRID>
__global__ void __launch_bounds__(384, 1)
    sparse_attn_kernel(const __grid_constant__ AttnMaps<GRID ? kMaxGridMaps : 1> M,
                       const __grid_constant__ Geometry G, const __grid_constant__ AttnArgs A) {
  using C = AttnCfg<D, BN, KST, VST>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {   // CTA-uniform, before any barrier or TMEM use
    if (threadIdx.x == 0) atomicExch(&g_device_error, kErrSmemAlign);
    return;
  }
  uint8_t* ops = smem + C::bookkeeping_bytes(A.k_max);   // operand region, 1024-byte aligned

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = G.S;
  const int cap = C::list_cap(A.k_max);
  const int n_items = G.B * (GRID ? A.n_group : G.heads) * G.ntmax;
  // Channel chunk c (64 channels) of tile j of head row bh into shared memory at dst.
  auto load_tile = [&](uint32_t dst, const CUtensorMap* map, uint32_t b, int c, const HeadGeom& hg, int bh, int j,
                       uint64_t r_w, uint64_t r_h) {
    if constexpr (GRID) {
      // tile coordinates from exact reciprocals of the head's tile counts
      const uint32_t jq = div_by_recip((uint32_t)j, r_w);
      const uint32_t jt = div_by_recip(jq, r_h);
      const int jw = j - (int)jq * hg.nTw, jh = (int)jq - (int)jt * hg.nTh;
      tma_load_5d(dst, map, b, 64 * c, jw * hg.pw, jh * hg.ph, (int)jt * hg.pt, bh);
    } else {
      tma_load_2d(dst, map, b, 64 * c, (bh * G.ntmax + j) * S);
    }
  };
  auto prefetch_tile = [&](const CUtensorMap* map, int c, const HeadGeom& hg, int bh, int j) {
    if constexpr (GRID) {
      const int jw = j % hg.nTw, jh = (j / hg.nTw) % hg.nTh, jt = j / (hg.nTw * hg.nTh);
      tma_prefetch_l2_5d(map, 64 * c, jw * hg.pw, jh * hg.ph, jt * hg.pt, bh);
    } else {
      tma_prefetch_l2_2d(map, 64 * c, (bh * G.ntmax + j) * S);
    }
  };

  const uint32_t sQ = smem_u32(ops + C::kOffQ);
  const uint32_t sK = smem_u32(ops + C::kOffK);
  const uint32_t sV = smem_u32(ops + C::kOffV);
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  auto bar = [&](int b) { return bar0 + 8u * (uint32_t)b; };
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  int* misc = reinterpret_cast<int*>(smem + C::kOffMisc);  // [0] tmem base, [1] abort, [4 + slot] list length
  int16_t* s_list = reinterpret_cast<int16_t*>(smem + C::kOffList);   // [2][cap]
  volatile int* abort = misc + 1;

  if (tid == 0) {
    misc[1] = 0;
    mbar_init(bar(BAR_QFULL), 1);
    mbar_init(bar(BAR_QEMPTY), 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_KEMPTY + s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_VEMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BAR_SFULL + s), 1);
      mbar_init(bar(BAR_SFREE + s), 4);
      mbar_init(bar(BAR_PFULL + s), 4);
      mbar_init(bar(BAR_PVDONE + s), 1);
      mbar_init(bar(BAR_LFULL + s), 32);
      mbar_init(bar(BAR_LEMPTY + s), 11);
    }
    mbar_init(bar(BAR_XFIN), 256);
    mbar_init(bar(BAR_OFREE), 8);
    mbar_init(bar(BAR_DRAIN), 1);
    mbar_init(bar(BAR_DRAIN2), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&misc[0]), C::kTmemCols);
    tmem_relinquish();
  }
  if (BN < 128 && warp >= 4) {
    // S = 64: the MMA always runs 128 rows; rows 64..127 of the Q panels stay
    // zero for every item (the Q box writes rows 0..63 only).
    for (int c = 0; c < D / 64; ++c) {
      uint4* p = reinterpret_cast<uint4*>(ops + C::kOffQ + c * C::kChunk + 64 * 128);
      for (int e = tid - 128; e < 64 * 128 / 16; e += 256) p[e] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const uint64_t tmo = A.timeout_ns;

  if (warp < 4) {
  // producers and issuers need few registers; the softmax warpgroups take them
  asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
  if (warp == 0) {
    // ------------------------------------------------------------ lists, Q and K producer
    AttnItem it;
    int w = next_attn_item<GRID>(G, A, blockIdx.x, n_items, it);
    int n = 0;             // items of this CTA so far
    uint32_t kt = 0;       // K tiles issued
    int q_fills = 0;       // Q tiles issued
    bool ok = true;
    // Selection list of item x into slot `slot`: entries as int16, the list
    // length (the first entry outside [0, NT_h) ends it) in misc[4 + slot].
    // Every lane arrives on LFULL after its own writes.
    auto load_list = [&](int slot, const AttnItem& x) {
      const int nt = G.g[x.h].nt;
      const int32_t* irow = A.idx + ((long long)x.bh * G.ntmax + x.i) * A.k_max;
      int first_bad = A.k_max;
      for (int c = lane; c < A.k_max; c += 32) {
        const int v = irow[c];
        const bool good = v >= 0 && v < nt;
        s_list[slot * cap + c] = (int16_t)(good ? v : 0);
        if (!good) first_bad = min(first_bad, c);
      }
      first_bad = __reduce_min_sync(0xffffffffu, first_bad);
      if (lane == 0) misc[4 + slot] = first_bad;
      mbar_arrive(bar(BAR_LFULL + slot));
    };
    auto issue_q = [&](const AttnItem& x) {
      if (lane == 0) {
        const HeadGeom hg = G.g[x.h];
        const CUtensorMap* tmQ = &M.q[x.mi];
        tma_prefetch_desc(tmQ);
        tma_prefetch_desc(&M.k[x.mi]);
        mbar_arrive_expect_tx(bar(BAR_QFULL), (uint32_t)(S * D * 2));
        const uint64_t rw = recip_ceil((uint32_t)hg.nTw), rh = recip_ceil((uint32_t)hg.nTh);
        for (int c = 0; c < D / 64; ++c) load_tile(sQ + c * C::kChunk, tmQ, bar(BAR_QFULL), c, hg, x.bh, x.i, rw, rh);
      }
      __syncwarp();
      ++q_fills;
    };
    if (w < n_items) {
      load_list(0, it);
      issue_q(it);
    }
    while (w < n_items) {
      const int slot = n & 1;
      const HeadGeom hg = G.g[it.h];
      const CUtensorMap* tmK = &M.k[it.mi];
      const uint64_t rw = recip_ceil((uint32_t)hg.nTw), rh = recip_ceil((uint32_t)hg.nTh);
      __syncwarp();   // this warp's own list writes are visible to lane 0
      const int nsel = misc[4 + slot];
      AttnItem nx;
      const int wn = next_attn_item<GRID>(G, A, w + gridDim.x, n_items, nx);
      if (lane == 0 && wn < n_items) {
        // the next item's Q tile comes from HBM: bring it to L2 now, so its
        // load at this item's end is an L2 hit
        const HeadGeom hn = G.g[nx.h];
        for (int c = 0; c < D / 64; ++c) prefetch_tile(&M.q[nx.mi], c, hn, nx.bh, nx.i);
      }
      for (int t = 0; t < nsel; ++t, ++kt) {
        const int st = kt % KST, fill = kt / KST;
        if (fill >= 1 && !(ok = warp_wait(bar(BAR_KEMPTY + st), (fill - 1) & 1, abort, tmo))) break;
        if (lane == 0) {
          const int j = s_list[slot * cap + t];
          if (VEDA_IN_BOUNDS(j >= 0 && j < hg.nt)) {   // a skipped fetch runs the consumers' waits out
            mbar_arrive_expect_tx(bar(BAR_KFULL + st), (uint32_t)C::kTileBytes);
            for (int c = 0; c < D / 64; ++c)
              load_tile(sK + st * C::kTileBytes + c * BN * 128, tmK, bar(BAR_KFULL + st), c, hg, it.bh, j, rw, rh);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      if (wn < n_items) {
        // The other slot was last used by the item before this one.
        if (n >= 1 && !(ok = warp_wait(bar(BAR_LEMPTY + (slot ^ 1)), ((n - 1) >> 1) & 1, abort, tmo))) break;
        load_list(slot ^ 1, nx);
        if (!(ok = warp_wait(bar(BAR_QEMPTY), n & 1, abort, tmo))) break;
        issue_q(nx);
      }
      w = wn;
      it = nx;
      ++n;
    }
    if (*abort) {
      if (q_fills > 0) drain_wait(bar(BAR_QFULL), (q_fills - 1) & 1, tmo);
      for (uint32_t t = kt > (uint32_t)KST ? kt - KST : 0; t < kt; ++t)
        drain_wait(bar(BAR_KFULL + t % KST), (t / KST) & 1, tmo);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ V producer
    AttnItem it;
    int w = next_attn_item<GRID>(G, A, blockIdx.x, n_items, it);
    int n = 0;
    uint32_t vt = 0;       // V tiles issued
    bool ok = true;
    while (w < n_items) {
      const int slot = n & 1;
      if (!(ok = warp_wait(bar(BAR_LFULL + slot), (n >> 1) & 1, abort, tmo))) break;
      const int nsel = misc[4 + slot];
      const HeadGeom hg = G.g[it.h];
      const CUtensorMap* tmV = &M.v[it.mi];
      const uint64_t rw = recip_ceil((uint32_t)hg.nTw), rh = recip_ceil((uint32_t)hg.nTh);
      if (lane == 0) tma_prefetch_desc(tmV);
      for (int t = 0; t < nsel; ++t, ++vt) {
        const int st = vt % VST, fill = vt / VST;
        if (fill >= 1 && !(ok = warp_wait(bar(BAR_VEMPTY + st), (fill - 1) & 1, abort, tmo))) break;
        if (lane == 0) {
          const int j = s_list[slot * cap + t];
          if (VEDA_IN_BOUNDS(j >= 0 && j < hg.nt)) {
            mbar_arrive_expect_tx(bar(BAR_VFULL + st), (uint32_t)C::kTileBytes);
            for (int c = 0; c < D / 64; ++c)
              load_tile(sV + st * C::kTileBytes + c * BN * 128, tmV, bar(BAR_VFULL + st), c, hg, it.bh, j, rw, rh);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mbar_arrive(bar(BAR_LEMPTY + slot));
      __syncwarp();
      w = next_attn_item<GRID>(G, A, w + gridDim.x, n_items, it);
      ++n;
    }
    if (*abort) {
      for (uint32_t t = vt > (uint32_t)VST ? vt - VST : 0; t < vt; ++t)
        drain_wait(bar(BAR_VFULL + t % VST), (t / VST) & 1, tmo);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ tcgen05 issuer, score products
    constexpr uint32_t idesc_qk = make_idesc_bf16(128, BN, false);
    // Descriptors are built once; per MMA only a compile-time offset (in
    // 16-byte units, added to the start-address field) and the stage base
    // change.
    const uint64_t dq0 = make_sdesc_sw128(sQ, 16, 1024);
    const uint64_t dk0 = make_sdesc_sw128(sK, 16, 1024);
    AttnItem it;
    int w = next_attn_item<GRID>(G, A, blockIdx.x, n_items, it);
    int n = 0;
    uint32_t kt = 0;              // K tiles consumed
    uint32_t cs[2] = {0u, 0u};    // score products issued per stream
    int last_s = -1;              // stream of the last score product (its S buffer use)
    bool ok = true;
    while (w < n_items) {
      const int slot = n & 1;
      if (!(ok = warp_wait(bar(BAR_LFULL + slot), (n >> 1) & 1, abort, tmo))) break;
      const int nsel = misc[4 + slot];
      if (!(ok = warp_wait(bar(BAR_QFULL), n & 1, abort, tmo))) break;
      for (int t = 0; t < nsel; ++t, ++kt) {
        const int st = kt % KST, s = t & 1;
        if (!(ok = warp_wait(bar(BAR_KFULL + st), (kt / KST) & 1, abort, tmo))) break;
        // The single S buffer is free once the stream of the previous score
        // product has loaded it.
        if (last_s >= 0 && !(ok = warp_wait(bar(BAR_SFREE + last_s), (cs[last_s] - 1) & 1, abort, tmo))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t dk = dk0 + (uint64_t)((st * C::kTileBytes) >> 4);
          const uint32_t dS = tmem + C::kTmemS;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t da = dq0 + (uint64_t)(((kk >> 2) * C::kChunk + (kk & 3) * 32) >> 4);
            const uint64_t db = dk + (uint64_t)(((kk >> 2) * BN * 128 + (kk & 3) * 32) >> 4);
            umma_ss(dS, da, db, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(BAR_KEMPTY + st));
          umma_commit(bar(BAR_SFULL + s));
        }
        __syncwarp();
        ++cs[s];
        last_s = s;
      }
      if (!ok) break;
      if (lane == 0) {
        // The Q buffer is free once this item's score products complete.
        if (nsel > 0) umma_commit(bar(BAR_QEMPTY));
        else mbar_arrive(bar(BAR_QEMPTY));
        mbar_arrive(bar(BAR_LEMPTY + slot));
      }
      __syncwarp();
      w = next_attn_item<GRID>(G, A, w + gridDim.x, n_items, it);
      ++n;
    }
    // Every MMA issued above completes before TMEM is released.
    if (lane == 0) umma_commit(bar(BAR_DRAIN));
    __syncwarp();
    drain_wait(bar(BAR_DRAIN), 0, tmo);
  } else if (warp == 3) {
    // ------------------------------------------------------------ tcgen05 issuer, PV products
    constexpr uint32_t idesc_pv = make_idesc_bf16(128, D, true);
    const uint64_t dv0 = make_sdesc_sw128(sV, BN * 128, 1024);
    AttnItem it;
    int w = next_attn_item<GRID>(G, A, blockIdx.x, n_items, it);
    int n = 0;
    uint32_t vt = 0;              // V tiles consumed
    uint32_t cp[2] = {0u, 0u};    // PV products issued per stream
    bool ok = true;
    while (w < n_items) {
      const int slot = n & 1;
      if (!(ok = warp_wait(bar(BAR_LFULL + slot), (n >> 1) & 1, abort, tmo))) break;
      const int nsel = misc[4 + slot];
      for (int t = 0; t < nsel; ++t, ++vt) {
        const int s = t & 1;
        if (!(ok = warp_wait(bar(BAR_PFULL + s), cp[s] & 1, abort, tmo))) break;
        if (!(ok = warp_wait(bar(BAR_VFULL + vt % VST), (vt / VST) & 1, abort, tmo))) break;
        // The previous item's epilogue must have read O_A and O_B out of TMEM
        // before this item's first product overwrites them.
        if (t == 0 && n >= 1 && !(ok = warp_wait(bar(BAR_OFREE), (n - 1) & 1, abort, tmo))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t dv = dv0 + (uint64_t)(((vt % VST) * C::kTileBytes) >> 4);
          const uint32_t pbase = tmem + C::kTmemP + s * 64;
          const uint32_t dO = tmem + C::kTmemO + s * 128;
          const uint32_t acc0 = t >= 2 ? 1u : 0u;   // first tile of each stream starts its O
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t db = dv + (uint64_t)((kk * 16 * 128) >> 4);
            umma_ts(dO, pbase + kk * 8, db, idesc_pv, kk > 0 ? 1u : acc0);
          }
          umma_commit(bar(BAR_VEMPTY + vt % VST));
          umma_commit(bar(BAR_PVDONE + s));
        }
        __syncwarp();
        ++cp[s];
      }
      if (!ok) break;
      if (lane == 0) mbar_arrive(bar(BAR_LEMPTY + slot));
      __syncwarp();
      w = next_attn_item<GRID>(G, A, w + gridDim.x, n_items, it);
      ++n;
    }
    if (lane == 0) umma_commit(bar(BAR_DRAIN2));
    __syncwarp();
    drain_wait(bar(BAR_DRAIN2), 0, tmo);
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;\n" ::: "memory");
    // ------------------------------------------------------------ softmax streams
    const int s = (warp - 4) >> 2;           // stream: tiles t with t % 2 == s
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = t_lane + C::kTmemS;
    const uint32_t tP = t_lane + C::kTmemP + s * 64;
    const uint32_t tO = t_lane + C::kTmemO + s * 128;
    const float sl2 = A.scale_log2;
    AttnItem it;
    int w = next_attn_item<GRID>(G, A, blockIdx.x, n_items, it);
    int n = 0;
    uint32_t cs = 0;               // score tiles this stream has received
    uint32_t cnt[2] = {0u, 0u};    // P tiles (= PV products) of each stream so far
    bool ok = true;
    while (w < n_items) {
      const int slot = n & 1;
      if (!(ok = warp_wait(bar(BAR_LFULL + slot), (n >> 1) & 1, abort, tmo))) break;
      const int nsel = misc[4 + slot];
      const HeadGeom hg = G.g[it.h];
      // Slot coordinates (t, y, x offsets) of this lane's key columns
      // c = 32 w + lane, for the pad-key mask of edge tiles, and exact
      // reciprocals for the tile coordinates of a tile index.
      int8_t kt[BN / 32], ky[BN / 32], kx[BN / 32];
#pragma unroll
      for (int q = 0; q < BN / 32; ++q) {
        const int c = q * 32 + lane;
        kx[q] = (int8_t)(c % hg.pw);
        ky[q] = (int8_t)((c / hg.pw) % hg.ph);
        kt[q] = (int8_t)(c / (hg.pw * hg.ph));
      }
      const uint64_t r_w = recip_ceil((uint32_t)hg.nTw), r_h = recip_ceil((uint32_t)hg.nTh);
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = s; t < nsel; t += 2) {
        const int k = t >> 1;                  // this stream's k-th tile of the item
        // Valid extents of the tile (pad keys of an edge tile are masked).
        const uint32_t j = (uint32_t)s_list[slot * cap + t];
        const uint32_t jq = div_by_recip(j, r_w), jt = div_by_recip(jq, r_h);
        const int jw = (int)(j - jq * hg.nTw), jh = (int)(jq - jt * hg.nTh);
        const int ct = min((int)hg.pt, G.T - (int)jt * hg.pt);
        const int ch = min((int)hg.ph, G.H - jh * hg.ph);
        const int cw = min((int)hg.pw, G.W - jw * hg.pw);
        if (!(ok = warp_wait(bar(BAR_SFULL + s), cs & 1, abort, tmo))) break;
        ++cs;
        tc_fence_after();
        float sc[BN];
        tmem_ld_cols<BN>(tS, sc);
        tmem_ld_wait();
        // S is in registers: the score issuer may overwrite the S buffer.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_SFREE + s));

        if (ct * ch * cw != S) {
          uint32_t mw[BN / 32];
#pragma unroll
          for (int q = 0; q < BN / 32; ++q) mw[q] = __ballot_sync(0xffffffffu, kt[q] < ct && ky[q] < ch && kx[q] < cw);
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (!((mw[c >> 5] >> (c & 31)) & 1u)) sc[c] = -INFINITY;
        }
        // Row maximum: three-input max over 8 independent chains.
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
        // Lazy rescaling: keep the old reference maximum unless the new one is
        // more than 8 (log2 units) above it.
        float m_use;
        bool rescale = false;
        if (k == 0) {
          m_use = mt;
        } else if (mt > m_run + 8.0f) {
          m_use = mt;
          rescale = true;
        } else {
          m_use = m_run;
        }
        const float m_ref = (m_use == -INFINITY) ? 0.f : m_use;
        // x = s*scale*log2(e) - m_ref as packed pairs; row sum over 4 packed
        // chains.
        const uint64_t scl2 = f2(sl2, sl2), nref2 = f2(-m_ref, -m_ref);
        uint64_t r4[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          float x0, x1, p0, p1;
          f2_split(f2_fma(f2(sc[c], sc[c + 1]), scl2, nref2), x0, x1);
          if (((c >> 1) & 7) < VEDA_EXP_POLY8) {
            exp2_fma_x2(x0, x1, p0, p1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          r4[(c >> 1) & 3] = f2_add(r4[(c >> 1) & 3], f2(p0, p1));
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        float ra, rb, rc, rd;
        f2_split(f2_add(r4[0], r4[1]), ra, rb);
        f2_split(f2_add(r4[2], r4[3]), rc, rd);
        const float rs = (ra + rb) + (rc + rd);
        const float alpha = rescale ? fast_exp2(m_run - m_ref) : 1.f;
        l_run = l_run * alpha + rs;
        m_run = m_use;

        // The stream's previous PV (possibly the last one of the previous
        // item) must be done before its P buffer is rewritten and before its
        // O is rescaled.
        if (cnt[s] >= 1 && !(ok = warp_wait(bar(BAR_PVDONE + s), (cnt[s] - 1) & 1, abort, tmo))) break;
        tc_fence_after();
        // P (bf16 pairs) into the stream's P buffer: the A operand of PV.
        tmem_st_cols_u<BN / 2>(tP, pk);
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            float o[32];
            tmem_ld32(tO + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] *= alpha;
            tmem_st32(tO + c, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_PFULL + s));
        ++cnt[s];
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue: merge the streams
      const int n_own = s == 0 ? (nsel + 1) >> 1 : nsel >> 1;   // tiles per stream of this item
      const int n_oth = nsel - n_own;
      cnt[s ^ 1] += (uint32_t)n_oth;
      // Own stream first: at most its last PV is pending, so the parity wait
      // is exact.
      if (n_own > 0 && !(ok = warp_wait(bar(BAR_PVDONE + s), (cnt[s] - 1) & 1, abort, tmo))) break;
      red[(s * 2 + 0) * 128 + row] = m_run;
      red[(s * 2 + 1) * 128 + row] = l_run;
      mbar_arrive(bar(BAR_XFIN));
      if (!(ok = warp_wait(bar(BAR_XFIN), n & 1, abort, tmo))) break;
      // The other stream's warpgroup waited for its own last PV before the
      // exchange, and no PV of the next item is issued before O is released,
      // so that barrier is complete now and the wait returns at once.
      if (n_oth > 0 && !(ok = warp_wait(bar(BAR_PVDONE + (s ^ 1)), (cnt[s ^ 1] - 1) & 1, abort, tmo))) break;
      tc_fence_after();
      const float mA = red[0 * 128 + row], lA = red[1 * 128 + row];
      const float mB = red[2 * 128 + row], lB = red[3 * 128 + row];
      const float m = fmaxf(mA, mB);
      const float wA = (lA > 0.f) ? fast_exp2(mA - m) : 0.f;
      const float wB = (lB > 0.f) ? fast_exp2(mB - m) : 0.f;
      const float l_tot = wA * lA + wB * lB;
      const float inv_l = (l_tot > 0.f) ? 1.0f / l_tot : 0.f;
      const float cA = wA * inv_l, cB = wB * inv_l;
      // stream s writes output columns [s*D/2, (s+1)*D/2), reading both O's
      float o[D / 2];
#pragma unroll
      for (int c = 0; c < D / 2; c += 32) {
        float ob[32];
        tmem_ld32(t_lane + C::kTmemO + s * (D / 2) + c, o + c);
        tmem_ld32(t_lane + C::kTmemO + 128 + s * (D / 2) + c, ob);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; ++q) o[c + q] = (cA != 0.f ? cA * o[c + q] : 0.f) + (cB != 0.f ? cB * ob[q] : 0.f);
      }
      // O is in registers: the next item's PV products may overwrite it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_OFREE));
      long long grow;
      bool valid = row < S;
      const int i = it.i;
      if constexpr (GRID) {
        const int iw = i % hg.nTw, ih = (i / hg.nTw) % hg.nTh, iq = i / (hg.nTw * hg.nTh);
        const int x = iw * hg.pw + row % hg.pw;
        const int y = ih * hg.ph + (row / hg.pw) % hg.ph;
        const int tt = iq * hg.pt + row / (hg.pw * hg.ph);
        valid = valid && tt < G.T && y < G.H && x < G.W;
        grow = (long long)it.bh * G.N + ((long long)tt * G.H + y) * G.W + x;
      } else {
        grow = ((long long)it.bh * G.ntmax + i) * S + row;
      }
      if (valid) valid = VEDA_IN_BOUNDS(grow < (long long)G.B * G.heads * (GRID ? (long long)G.N : (long long)G.ntmax * S));
      if (valid) {
        uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(A.op) + grow * D + s * (D / 2));
#pragma unroll
        for (int q = 0; q < D / 16; ++q) {
          uint4 v;
          v.x = pack_bf16x2(o[q * 8 + 0], o[q * 8 + 1]);
          v.y = pack_bf16x2(o[q * 8 + 2], o[q * 8 + 3]);
          v.z = pack_bf16x2(o[q * 8 + 4], o[q * 8 + 5]);
          v.w = pack_bf16x2(o[q * 8 + 6], o[q * 8 + 7]);
          orow[q] = v;
        }
        if (A.lse != nullptr && s == 0)
          A.lse[grow] = (l_tot > 0.f) ? (m + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_LEMPTY + slot));
      w = next_attn_item<GRID>(G, A, w + gridDim.x, n_items, it);
      ++n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, int BN, int KST, int VST, bool GRID>
static cudaError_t launch_attn_t(const Geometry& G, const AttnMaps<GRID ? kMaxGridMaps : 1>& m,
                                 const AttnArgs& a, cudaStream_t s) {
  using C = AttnCfg<D, BN, KST, VST>;
  auto kernel = sparse_attn_kernel<D, BN, KST, VST, GRID>;
  const size_t smem = C::smem_bytes(a.k_max);
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  // setmaxnreg moves registers between warpgroups inside the block's launch
  // allocation: 128 threads drop to 56 and 256 threads rise to 224.  The
  // split must fit the registers the block is launched with, or the raise
  // would wait forever; refuse to launch otherwise.
  cudaFuncAttributes attr;
  if ((err = cudaFuncGetAttributes(&attr, kernel)) != cudaSuccess) return err;
  if (128 * 56 + 256 * 224 > C::kThreads * attr.numRegs) return cudaErrorInvalidConfiguration;
  // Persistent grid: one CTA per SM (the shared memory allows no second),
  // each walking the items gridDim.x apart.
  int dev = 0, sms = 148;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  const long long items = (long long)G.B * (GRID ? a.n_group : G.heads) * G.ntmax;
  const unsigned blocks = (unsigned)std::min<long long>(items, sms);
  kernel<<<blocks, C::kThreads, smem, s>>>(m, G, a);
  return cudaGetLastError();
}

// The deepest K/V rings that fit: a K/V tile fetch from L2 takes a few
// thousand cycles under load, and the V ring in particular is refilled only
// after the PV product that read its stage, so ring depth sets the tile rate.
template <int D, int BN>
static int attn_stages_t(int k_max) {   // returns 10 * K stages + V stages
  if (D * BN <= 64 * 128 && AttnCfg<D, BN, 4, 4>::smem_bytes(k_max) <= (size_t)kSmemLimit) return 44;
  if (AttnCfg<D, BN, 3, 3>::smem_bytes(k_max) <= (size_t)kSmemLimit) return 33;
  if (AttnCfg<D, BN, 3, 2>::smem_bytes(k_max) <= (size_t)kSmemLimit) return 32;
  return 22;
}

template <int D, int BN, bool GRID>
static cudaError_t launch_attn_d(const Geometry& G, const AttnMaps<GRID ? kMaxGridMaps : 1>& m,
                                 const AttnArgs& a, cudaStream_t s) {
  switch (attn_stages_t<D, BN>(a.k_max)) {
    case 44:
      if constexpr (D * BN <= 64 * 128) return launch_attn_t<D, BN, 4, 4, GRID>(G, m, a, s);
      return cudaErrorInvalidConfiguration;
    case 33: return launch_attn_t<D, BN, 3, 3, GRID>(G, m, a, s);
    case 32: return launch_attn_t<D, BN, 3, 2, GRID>(G, m, a, s);
    default: return launch_attn_t<D, BN, 2, 2, GRID>(G, m, a, s);
  }
}

// K and V ring depths and dynamic shared memory the attention launch uses.
void sparse_attn_config(int d, int S, int k_max, int* k_stages, int* v_stages, size_t* smem) {
  int ks = 22;
  size_t bytes = 0;
  auto pick = [&](auto cfg44, auto cfg33, auto cfg32, auto cfg22, int code) {
    ks = code;
    bytes = code == 44 ? decltype(cfg44)::smem_bytes(k_max)
          : code == 33 ? decltype(cfg33)::smem_bytes(k_max)
          : code == 32 ? decltype(cfg32)::smem_bytes(k_max) : decltype(cfg22)::smem_bytes(k_max);
  };
  if (d == 128 && S == 128)
    pick(AttnCfg<128, 128, 4, 4>{}, AttnCfg<128, 128, 3, 3>{}, AttnCfg<128, 128, 3, 2>{}, AttnCfg<128, 128, 2, 2>{},
         attn_stages_t<128, 128>(k_max));
  else if (d == 128)
    pick(AttnCfg<128, 64, 4, 4>{}, AttnCfg<128, 64, 3, 3>{}, AttnCfg<128, 64, 3, 2>{}, AttnCfg<128, 64, 2, 2>{},
         attn_stages_t<128, 64>(k_max));
  else if (S == 128)
    pick(AttnCfg<64, 128, 4, 4>{}, AttnCfg<64, 128, 3, 3>{}, AttnCfg<64, 128, 3, 2>{}, AttnCfg<64, 128, 2, 2>{},
         attn_stages_t<64, 128>(k_max));
  else
    pick(AttnCfg<64, 64, 4, 4>{}, AttnCfg<64, 64, 3, 3>{}, AttnCfg<64, 64, 3, 2>{}, AttnCfg<64, 64, 2, 2>{},
         attn_stages_t<64, 64>(k_max));
  *k_stages = ks / 10;
  *v_stages = ks % 10;
  *smem = bytes;
}

size_t sparse_attn_smem_bytes(int d, int S, int k_max) {
  // the smallest configuration that can run (two stages of each)
  if (d == 128 && S == 128) return AttnCfg<128, 128, 2, 2>::smem_bytes(k_max);
  if (d == 128 && S == 64) return AttnCfg<128, 64, 2, 2>::smem_bytes(k_max);
  if (d == 64 && S == 128) return AttnCfg<64, 128, 2, 2>::smem_bytes(k_max);
  return AttnCfg<64, 64, 2, 2>::smem_bytes(k_max);
}

cudaError_t launch_sparse_attn(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s) {
  AttnMaps<1> m;
  m.q[0] = tq;
  m.k[0] = tk;
  m.v[0] = tv;
  if (G.d == 128 && G.S == 128) return launch_attn_d<128, 128, false>(G, m, a, s);
  if (G.d == 128 && G.S == 64) return launch_attn_d<128, 64, false>(G, m, a, s);
  if (G.d == 64 && G.S == 128) return launch_attn_d<64, 128, false>(G, m, a, s);
  return launch_attn_d<64, 64, false>(G, m, a, s);
}

cudaError_t launch_sparse_attn_grid(const Geometry& G, const AttnMaps<kMaxGridMaps>& m, const AttnArgs& a,
                                    cudaStream_t s) {
  if (G.d == 128 && G.S == 128) return launch_attn_d<128, 128, true>(G, m, a, s);
  if (G.d == 128 && G.S == 64) return launch_attn_d<128, 64, true>(G, m, a, s);
  if (G.d == 64 && G.S == 128) return launch_attn_d<64, 128, true>(G, m, a, s);
  return launch_attn_d<64, 64, true>(G, m, a, s);
}

}  // namespace veda
