// kernels.h -- host-side launchers of the libvsa kernels (internal to the library).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace vsa {

cudaError_t launch_permute(const void* src, bool src_f32, void* dst, const uint8_t* kinds, const Geom& g, int BH,
                           int d, int* err, cudaStream_t stream);
cudaError_t launch_unpermute(const void* src, const float* src_lse, void* dst, bool dst_f32, float* dst_lse,
                             const uint8_t* kinds, const Geom& g, int BH, int d, int* err, cudaStream_t stream);

cudaError_t launch_pattern_mask(const uint8_t* kinds, const Geom& g, int BH, int w_s, int w_t, uint32_t* bits,
                                int32_t* kv_idx, int32_t* kv_cnt, int max_kv, int* err, cudaStream_t stream);
// Workspace: 2 * BH * ncubes * d doubles.
size_t cube_mask_workspace_bytes(const Geom& g, int BH, int d);
cudaError_t launch_cube_mask(const uint8_t* kinds, const void* q_cube, const void* k_cube, const Geom& g, int BH, int d,
                             int topk, uint32_t* bits, int32_t* kv_idx, int32_t* kv_cnt, int max_kv, void* ws,
                             int* err, cudaStream_t stream);

// Attention work order per head (query blocks sorted by their first kept key block).
cudaError_t launch_block_order(const uint8_t* kinds, const Geom& g, int BH, const int32_t* kv_idx,
                               const int32_t* kv_cnt, int max_kv, int32_t* order, cudaStream_t stream);

// Semantic-aware permutation (see semantic.cu).  At most kMaxClusters clusters per tensor.
constexpr int kMaxClusters = 1024;
// k-means of x [BH, N, d] bf16: cent [BH, C, d] f32, label [BH, N], counts [BH, C], perm [BH, N]
// (slot -> token, cluster-major).  ws (kmeans_workspace_bytes): the cluster offsets and
// partial-sum chunk offsets [BH, C + 1], the centroids' squared norms [BH, C], their bf16
// halves [BH, C, d] twice, the update's chunk sums [BH, ceil(N / 128) + C, d], and the
// sort's segment histograms [BH, 8, C] with one flag per head, and the chunks' clusters.
size_t kmeans_workspace_bytes(int BH, int N, int C, int d);
cudaError_t launch_kmeans(const void* x, int BH, int N, int d, int C, int iters, float* cent, int32_t* label,
                          int32_t* counts, int32_t* perm, void* ws, int* err, cudaStream_t stream);
// Workspace of launch_semantic_mask: the cluster range of every query and key block.
size_t semantic_mask_workspace_bytes(int BH, int N, int block);
cudaError_t launch_semantic_mask(const float* cent_q, const int32_t* counts_q, const int32_t* label_q,
                                 const int32_t* perm_q, int Cq, const float* cent_k, const int32_t* counts_k,
                                 const int32_t* label_k, const int32_t* perm_k, int Ck, int BH, int N, int d,
                                 int block, double scale, double top_p, uint32_t* keep, uint32_t* bits,
                                 int32_t* kv_idx, int32_t* kv_cnt, int max_kv, void* ws, int* err,
                                 cudaStream_t stream);
cudaError_t launch_gather_rows(const void* src, const int32_t* perm, void* dst, int BH, int N, int d, int* err,
                               cudaStream_t stream);
cudaError_t launch_scatter_rows(const void* src, const float* src_lse, const int32_t* perm, void* dst, float* dst_lse,
                                int BH, int N, int d, int* err, cudaStream_t stream);

// Tensor maps of one attention problem (3D: d, rows, B*H).
struct AttnMaps {
  CUtensorMap q, k, v, o;
};

struct AttnArgs {
  const uint8_t* kinds;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  const int32_t* order;  // [B*H, nblk] query-block order, or null for natural order
  float* lse_nat;
  float* lse_perm;
  int* err;
  int BH;
  int max_kv;
  int has_perm;
  int nat_rows;  // rows per head of the natural buffers (N, or R when they hold every layout)
  int ucap;      // capacity of the per-CTA union list: min(nblk, 2 * max_kv)
  float scale_log2;
  Geom g;
  // In-kernel layout: temporal heads read Q, K, V and write O in natural order through the
  // frame-major slot map (no permuted copies); only with has_perm == 0.
  int gather;
  // e4m3 Q and K (null for bf16): per (head, block) power-of-two exponents of their scales
  const int32_t* qexp;
  const int32_t* kexp;
  const void* nat_q;
  const void* nat_k;
  const void* nat_v;
  void* nat_o;
};

cudaError_t launch_sparse_attn(const AttnMaps& nat, const AttnMaps& perm, const AttnArgs& a, int d,
                               cudaStream_t stream);

// Profiling (see profile.cu).
struct ProfilePlan {
  int r;        // sampled rows
  int r_pad;    // rounded up to the 128-row tile
  int tiles;    // r_pad / 128
  int splits;   // key-range splits per tile
  size_t off_qs, off_ranges, off_order, off_opart, off_ml, off_rowerr, bytes;
};
ProfilePlan profile_plan(const Geom& g, int BH, int d, double frac);
// Same layout as profile_plan but with an explicit number of key-range splits (>= 1).
ProfilePlan profile_plan_splits(const Geom& g, int BH, int d, double frac, int splits);
cudaError_t launch_profile(const void* q, const void* k, const void* v, const Geom& g, int BH, int d, int w_s,
                           int w_t, float scale_log2, const ProfilePlan& plan, void* ws, uint8_t* kinds_out,
                           float* mse_out, int* err, cudaStream_t stream);

// Tensor-map encoding through the driver entry point (no link-time libcuda dependency).
cudaError_t encode_rows_map(CUtensorMap* map, const void* base, int d, int rows, int BH, int box_rows);
// The same for rows of d = 128 one-byte elements (e4m3 codes): one 128-byte box per row.
cudaError_t encode_rows_map_u8(CUtensorMap* map, const void* base, int d, int rows, int BH, int box_rows);

// Per-block e4m3 quantisation (fp8.cu): dst [BH, R, d] codes, exps [BH, nblk].
cudaError_t launch_quantize_e4m3(const void* nat, const void* perm, const uint8_t* kinds, const Geom& g, int BH,
                                 int d, int nat_rows, uint8_t* dst, int32_t* exps, int* err, cudaStream_t stream);

}  // namespace vsa
