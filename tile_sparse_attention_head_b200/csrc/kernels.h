// Launchers of the sm_100a kernels (internal to the library; the public
// surface is include/veda.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "veda_common.cuh"

namespace veda {

struct EstimatorWeights {
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
};

struct TopkArgs {
  int32_t* idx;
  float* probs;
  uint64_t timeout_ns;   // bounded-wait limit of the tensor-core estimator
  int32_t k_max;
  int32_t k_per_head[VEDA_MAX_HEADS];
};

struct AttnArgs {
  const int32_t* idx;
  int32_t k_max;
  float scale_log2;   // softmax scale * log2(e)
  void* op;           // bf16 [B, heads, NT_max*S, d] (tile-major) or [B, heads, N, d] (grid order)
  float* lse;         // fp32 [B, heads, NT_max*S] or [B, heads, N]; or null
  uint64_t timeout_ns;
  // Grid-order launches only: the heads this launch covers and, per head,
  // which of the launch's tensor maps holds its tile box.
  int32_t n_group;
  int16_t head_list[VEDA_MAX_HEADS];
  int8_t map_of_head[VEDA_MAX_HEADS];
};

// Tensor maps of one attention launch.  Tile-major operands need one map
// each; grid-order operands need one per distinct tiling (the tile box is
// part of the map), up to kMaxGridMaps per launch.
constexpr int kMaxGridMaps = 8;
template <int NM>
struct AttnMaps {
  CUtensorMap q[NM], k[NM], v[NM];
};

// Attention backward (grid order).  The dQ launch holds (Q_i, dO_i) and
// streams the selected (K, V) tiles; the dK/dV launch holds (K_j, V_j) and
// streams (Q, dO) of the Q tiles that selected j.  Maps per distinct tiling:
// a0/a1 the stationary pair, b0/b1 the moving pair.
template <int NM>
struct BwdMaps {
  CUtensorMap a0[NM], a1[NM], b0[NM], b1[NM];
};

struct BwdArgs {
  const int32_t* idx;       // [B, heads, NT_max, k_max]
  int32_t k_max;
  const int32_t* inv_off;   // [B*heads, NT_max + 1]
  const int32_t* inv_list;  // [B*heads, NT_max * k_max]
  const float2* ldt;        // [B*heads, NT_max, S]: per tile slot (L, D) = (lse log2(e), rowsum(dO * O)),
                            // (+inf, 0) on pad slots
  void* dx;                 // bf16 [B, heads, N, d]: dQ (dQ launch) or dK (dK/dV launch)
  void* dv;                 // bf16 [B, heads, N, d]: dV (dK/dV launch)
  float scale;
  float scale_log2;
  uint64_t timeout_ns;
  int32_t n_group;
  int16_t head_list[VEDA_MAX_HEADS];
  int8_t map_of_head[VEDA_MAX_HEADS];
};

struct MapArgs {
  const int32_t* rows;  // [B*heads, R]
  int32_t R;
  float scale_log2;
  float* rowmax;        // scratch [B*heads, R, NT_max, S]  (scaled, log2 domain)
  float* lse2;          // scratch [B*heads, R, S]          (log2 domain)
  float* map;           // [B, heads, R, NT_max]
  uint64_t timeout_ns;
  // Grid-order pass-1 launches only: the heads this launch covers and, per
  // head, which of the launch's tensor maps holds its tile box.
  int32_t n_group;
  int16_t head_list[VEDA_MAX_HEADS];
  int8_t map_of_head[VEDA_MAX_HEADS];
};

cudaError_t launch_permute(const Geometry& G, const void* x, void* xp, cudaStream_t s, int sms);
cudaError_t launch_unpermute(const Geometry& G, const void* xp, void* x, cudaStream_t s, int sms);
cudaError_t launch_permute_tripool(const Geometry& G, const void* x, void* xp, float* desc, cudaStream_t s);
cudaError_t launch_tripool(const Geometry& G, const void* xp, float* desc, cudaStream_t s);

size_t estimator_smem_bytes(int d, int hidden, int e);
cudaError_t launch_estimator(const Geometry& G, const float* dq, const float* dk, const EstimatorWeights& wq,
                             const EstimatorWeights& wk, int hidden, int e, float* phi, float* hid,
                             uint64_t timeout_ns, cudaStream_t s);
void score_topk_config(int ntmax, int e, int* qb, int* ntpad, size_t* smem);
// Scoring and selection.  phi: the estimator features, 2*B*heads*NT_max*e
// floats.  scores: room for the fp32 score matrix (score_matrix_bytes), or
// NULL, in which case each CTA keeps its block of scores in shared memory.
size_t score_matrix_bytes(const Geometry& G, int e);
cudaError_t launch_score_topk(const Geometry& G, const float* desc_q, const float* desc_k,
                              const EstimatorWeights& wq, const EstimatorWeights& wk, int hidden,
                              int e, float* phi, float* scores, const TopkArgs& args, cudaStream_t s);

size_t sparse_attn_smem_bytes(int d, int S, int k_max);
void sparse_attn_config(int d, int S, int k_max, int* k_stages, int* v_stages, size_t* smem);
cudaError_t launch_sparse_attn(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const AttnArgs& a, cudaStream_t s);
// Grid-order variant: Q/K/V tiles are fetched as 5D boxes of the grid-order
// tensors, O and the LSE are written to grid rows.  One launch covers the
// heads a.head_list[0..a.n_group); head h uses maps m.*[a.map_of_head[h]].
cudaError_t launch_sparse_attn_grid(const Geometry& G, const AttnMaps<kMaxGridMaps>& m, const AttnArgs& a,
                                    cudaStream_t s);
cudaError_t launch_tripool_grid(const Geometry& G, const void* x, float* desc, cudaStream_t s);

cudaError_t launch_tile_map(const Geometry& G, const CUtensorMap& tq, const CUtensorMap& tk,
                            const MapArgs& a, cudaStream_t s);
// Grid-order tile map: pass 1 once per group of up to kMaxGridMaps distinct
// tilings (a.head_list / a.map_of_head), then pass 2 once for all heads.
cudaError_t launch_tile_map_pass1_grid(const Geometry& G, const AttnMaps<kMaxGridMaps>& m, const MapArgs& a,
                                       cudaStream_t s);
cudaError_t launch_tile_map_pass2(const Geometry& G, const MapArgs& a, cudaStream_t s);

size_t distill_ws_bytes(const Geometry& G, int hidden, int e, int R);
cudaError_t launch_head_error(const Geometry& G, const void* o, const void* o_ref, float* err, float* ref,
                              float* part, cudaStream_t s);
cudaError_t launch_distill(const Geometry& G, const float* desc_q, const float* desc_k, const EstimatorWeights& wq,
                           const EstimatorWeights& wk, int hidden, int e, const float* map, const int32_t* rows,
                           int R, float* loss, const EstimatorWeights& gq, const EstimatorWeights& gk, void* ws,
                           uint64_t timeout_ns, cudaStream_t s);

size_t attn_bwd_ws_bytes(const Geometry& G, int k_max);
// Per tile slot (L, D) and the inverse selection lists into the workspace;
// fills a.idx, a.k_max, a.ldt, a.inv_off and a.inv_list.
cudaError_t launch_attn_bwd_prep(const Geometry& G, const void* o, const void* dout, const float* lse,
                                 const int32_t* idx, int k_max, void* ws, BwdArgs* a, cudaStream_t s);
cudaError_t launch_attn_bwd_dq(const Geometry& G, const BwdMaps<kMaxGridMaps>& m, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_attn_bwd_dkdv(const Geometry& G, const BwdMaps<kMaxGridMaps>& m, const BwdArgs& a,
                                 cudaStream_t s);

cudaError_t launch_timeout_selftest(uint64_t timeout_ns, cudaStream_t s);
cudaError_t launch_bounds_selftest(cudaStream_t s);

}  // namespace veda
