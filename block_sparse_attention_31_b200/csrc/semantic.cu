// semantic.cu -- semantic-aware permutation ("Sparse VideoGen2" page, abstract): tokens are
// clustered by k-means on their Q (respectively K) vectors, reordered so that every cluster
// is contiguous, and a top-p budget over the clusters picks the key clusters each query
// cluster attends to.  The page gives no formulas; the readings used here:
//   - Lloyd's k-means per head on the bf16 rows (as fp32), `iters` rounds of assignment then
//     update, initial centroids the rows rho_j = floor((2j+1) N / (2C));
//   - assignment: argmin_j |c_j|^2 - 2 x.c_j, ties to the smaller j: |c_j|^2 in fp32 (fused
//     multiply-adds in dimension order), x.c_j on the tensor cores as x.c_hi + x.c_lo with
//     c = c_hi + c_lo + r split into two bf16 vectors (|r| <= 2^-18 |c| per element; the bf16
//     products are exact and accumulate in fp32);
//   - update: fp64 sum of the members in token order, divided by the count, rounded to fp32;
//     an empty cluster keeps its centroid;
//   - cluster-major order: slots sorted by (cluster, token);
//   - weight of key cluster j for query cluster i: n_j exp(s_ij - max_j s_ij), s_ij = scale *
//     cq_i . ck_j in fp64 (dimension order, fused multiply-adds; CUDA's fp64 exp); kept: the
//     shortest prefix of the weights sorted in descending order (ties to the smaller j) whose
//     running sum reaches top_p times the sum of all of them;
//   - block pair (a, b) of the two cluster-major layouts is kept when some query slot of a
//     and some key slot of b belong to a kept cluster pair.
// Every floating-point step that decides an integer (assignment, order, top-p) is written
// out with explicitly rounded operations, so the result does not depend on contraction.  The
// assignment's fp32 distances can differ from exact ones by a bounded amount: where two
// centroids are that close to a tie, either label is a correct nearest-centroid choice.
#include <cuda_bf16.h>
#include <algorithm>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

namespace {

constexpr int kKeepThreads = 256;
constexpr int kRowThreads = 256;

// |c|^2 of one centroid held in shared memory: fp32, dimension order, one fused multiply-add
// per term (the first term of the assignment's distance).
__device__ __forceinline__ float sq_norm(const float* c, int D) {
  float acc = 0.f;
  for (int k = 0; k < D; ++k) acc = __fmaf_rn(c[k], c[k], acc);
  return acc;
}


// ---------------------------------------------------------------------------------------
// k-means
// ---------------------------------------------------------------------------------------

// cent[bh, j] = x[bh, rho_j] as fp32, and its squared norm.  128 threads, d <= 128.
__global__ void __launch_bounds__(128) kmeans_init_kernel(const __nv_bfloat16* __restrict__ x, int N, int d, int C,
                                                          float* __restrict__ cent, float* __restrict__ cnorm,
                                                          __nv_bfloat16* __restrict__ chi,
                                                          __nv_bfloat16* __restrict__ clo,
                                                          int32_t* __restrict__ bad) {
  __shared__ float row_s[128];
  const int j = blockIdx.x, bh = blockIdx.y;
  const long long r = ((2LL * j + 1) * N) / (2LL * C);
  const __nv_bfloat16* src = x + (static_cast<size_t>(bh) * N + r) * d;
  float* dst = cent + (static_cast<size_t>(bh) * C + j) * d;
  const size_t o = (static_cast<size_t>(bh) * C + j) * d;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    const float v = __bfloat162float(src[k]);
    dst[k] = v;
    row_s[k] = v;
    chi[o + k] = src[k];  // a bf16 row splits exactly: hi = the row, lo = 0
    clo[o + k] = __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  if (threadIdx.x == 0) cnorm[static_cast<size_t>(bh) * C + j] = sq_norm(row_s, d);
  if (threadIdx.x == 0 && j == 0) bad[bh] = 0;  // the sort's label check starts clear
}

// label[bh, t] on the tensor cores: one CTA of 128 threads per 128 tokens of one head.  For each
// tile of 128 centroids, thread 0 loads the token tile (once) and the centroids' bf16 halves
// with TMA and issues S = X C_hi^T + X C_lo^T (tcgen05, M128 N128 K16, fp32 in TMEM); then every
// thread (one token, TMEM lane = token) reads its 128 scores and keeps the running argmin of
// |c|^2 - 2 s (one rounding), ties to the smaller index.  Tokens past N and centroids past C
// are zero rows of the TMA boxes; the latter are skipped.
constexpr int kTcRows = 128;

template <int D>
struct KmTcCfg {
  static constexpr int X_BYTES = kTcRows * D * 2;
  static constexpr int C_BYTES = kTcRows * D * 2;
  static constexpr int OFF_X = 0, OFF_HI = X_BYTES, OFF_LO = X_BYTES + C_BYTES, OFF_BAR = X_BYTES + 2 * C_BYTES;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;
  static constexpr uint32_t IDESC = idesc_bf16_f32(kTcRows, kTcRows, false, false);
};

template <int D>
__global__ void __launch_bounds__(128) kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap tx,
                                                               const __grid_constant__ CUtensorMap thi,
                                                               const __grid_constant__ CUtensorMap tlo, int N, int C,
                                                               const float* __restrict__ cnorm,
                                                               int32_t* __restrict__ label, int* err) {
  using K = KmTcCfg<D>;
  extern __shared__ uint8_t km_raw[];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  __shared__ float cn[kTcRows];
  const uint32_t raw = smem_u32(km_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  const uint32_t sX = sb + K::OFF_X, sHi = sb + K::OFF_HI, sLo = sb + K::OFF_LO;
  const uint32_t bLoad = sb + K::OFF_BAR, bMma = bLoad + 8;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y, t0 = blockIdx.x * kTcRows;
  volatile int* abort_flag = &abort_s;
  if (tid == 0) {
    mbar_init(bLoad, 1);
    mbar_init(bMma, 1);
    mbar_init_fence();
    abort_s = 0;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_s), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  float best_d = INFINITY;
  int best_j = 0;
  bool ok = true;
  const int ntiles = (C + kTcRows - 1) / kTcRows;
  for (int ct = 0; ct < ntiles && ok; ++ct) {
    const int c0 = ct * kTcRows;
    if (tid == 0) {
      const uint32_t bytes = (ct == 0 ? K::X_BYTES : 0) + 2 * K::C_BYTES;
      mbar_arrive_expect_tx(bLoad, bytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        if (ct == 0) tma_load_3d(sX + c * kTcRows * 128, &tx, bLoad, c * 64, t0, bh);
        tma_load_3d(sHi + c * kTcRows * 128, &thi, bLoad, c * 64, c0, bh);
        tma_load_3d(sLo + c * kTcRows * 128, &tlo, bLoad, c * 64, c0, bh);
      }
      if (mbar_wait(bLoad, ct & 1, abort_flag, err)) {
        tc_fence_after();
        const uint64_t dx = sdesc_sw128(sX, 16, 1024), dh = sdesc_sw128(sHi, 16, 1024),
                       dl = sdesc_sw128(sLo, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) / 16);
          tc_mma_ss(tmem, dx + off, dh + off, K::IDESC, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) / 16);
          tc_mma_ss(tmem, dx + off, dl + off, K::IDESC, 1u);
        }
        tc_commit(bMma);
      } else {
        mbar_wait_drain(bLoad, ct & 1, err);  // the copies land before the CTA moves on
      }
    }
    cn[tid] = c0 + tid < C ? cnorm[static_cast<size_t>(bh) * C + c0 + tid] : 0.f;
    ok = __syncthreads_and(!*abort_flag);
    if (!ok) break;
    ok = __syncthreads_and(mbar_wait(bMma, ct & 1, abort_flag, err));
    if (!ok) {
      if (tid == 0) mbar_wait_drain(bMma, ct & 1, err);  // the MMAs were issued: let them finish
      break;
    }
    tc_fence_after();
    const int nc = min(kTcRows, C - c0);
#pragma unroll 1
    for (int q = 0; q < kTcRows / 32; ++q) {
      if (q * 32 >= nc) break;
      float sv[32];
      tmem_ld32(t_lane + q * 32, sv);
#pragma unroll
      for (int x = 0; x < 32; ++x) {  // ascending index, strict <: ties keep the smaller index
        const int jl = q * 32 + x;
        float dist = __fmaf_rn(-2.f, sv[x], cn[jl]);  // |c|^2 - 2 s, rounded once
        dist = jl < nc ? dist : INFINITY;
        const bool lt = dist < best_d;
        best_d = lt ? dist : best_d;
        best_j = lt ? c0 + jl : best_j;
      }
    }
    tc_fence_before();
    __syncthreads();  // every thread has read S and cn before the next tile overwrites them
  }
  const int t = t0 + tid;
  if (ok && t < N) label[static_cast<size_t>(bh) * N + t] = best_j;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// The same assignment with the centroids resident, for C <= 128 * NCT (NCT <= 2): CTAs are
// persistent per head (grid (ctas_per_head, BH)) and walk the head's token tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...  The centroid halves are loaded once; token tiles
// stream through two shared-memory stages and S through two TMEM buffers, so the load of the
// next tile and its MMAs overlap this tile's argmin.  Roles: warp 8 lane 0 loads (TMA),
// warp 9 lane 0 issues the MMAs; warps 0-3 and 4-7 (one token row per thread) read S buffer 0
// and 1 respectively (even and odd tiles) and write the labels.
constexpr int kPcThreads = 320;

template <int D, int NCT>
struct KmPcCfg {
  static constexpr int X_BYTES = kTcRows * D * 2;      // one token tile
  static constexpr int CT_BYTES = kTcRows * D * 2;     // one 128-centroid tile of one half
  static constexpr int OFF_C = 0;                      // [NCT][hi, lo]
  static constexpr int OFF_X = NCT * 2 * CT_BYTES;     // [2 stages]
  static constexpr int OFF_BAR = OFF_X + 2 * X_BYTES;  // 9 barriers
  static constexpr int OFF_CN = OFF_BAR + 128;         // [NCT * 128] centroid norms
  static constexpr int SMEM = OFF_CN + NCT * kTcRows * 4 + 1024;
  static constexpr int SCOLS = NCT * kTcRows;          // TMEM columns of one S buffer
  static constexpr int TMEM_COLS = 2 * SCOLS;          // 256 or 512
  static constexpr uint32_t IDESC = idesc_bf16_f32(kTcRows, kTcRows, false, false);
};

enum { KB_C = 0, KB_XF = 1, KB_XE = 3, KB_SF = 5, KB_SE = 7 };

template <int D, int NCT>
__global__ void __launch_bounds__(kPcThreads, 1)
    kmeans_assign_pc_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap thi,
                            const __grid_constant__ CUtensorMap tlo, int N, int C, const float* __restrict__ cnorm,
                            int32_t* __restrict__ label, int* err) {
  using K = KmPcCfg<D, NCT>;
  extern __shared__ uint8_t pc_raw[];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int bh = blockIdx.y;
  const int ntiles = (N + kTcRows - 1) / kTcRows;
  const int mine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;  // tiles of this CTA
  if (mine == 0) return;
  const uint32_t raw = smem_u32(pc_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  float* cn = reinterpret_cast<float*>(pc_raw + (sb - raw) + K::OFF_CN);
  auto bar = [&](int i) -> uint32_t { return sb + K::OFF_BAR + 8u * i; };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &abort_s;
  if (tid == 0) {
    mbar_init(bar(KB_C), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(KB_XF + s), 1);
      mbar_init(bar(KB_XE + s), 1);
      mbar_init(bar(KB_SF + s), 1);
      mbar_init(bar(KB_SE + s), 128);
    }
    mbar_init_fence();
    abort_s = 0;
  }
  for (int c = tid; c < NCT * kTcRows; c += kPcThreads) cn[c] = c < C ? cnorm[static_cast<size_t>(bh) * C + c] : 0.f;
  if (warp == 9) {
    tmem_alloc(smem_u32(&tmem_s), K::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;

  if (warp == 8) {  // ---- loads ----
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(KB_C), NCT * 2 * K::CT_BYTES);
#pragma unroll
      for (int ct = 0; ct < NCT; ++ct)
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const uint32_t dst = sb + K::OFF_C + (2 * ct) * K::CT_BYTES + c * kTcRows * 128;
          tma_load_3d(dst, &thi, bar(KB_C), c * 64, ct * kTcRows, bh);
          tma_load_3d(dst + K::CT_BYTES, &tlo, bar(KB_C), c * 64, ct * kTcRows, bh);
        }
      int issued = 0;
      for (int li = 0; li < mine; ++li) {
        const int s = li & 1;
        if (li >= 2 && !mbar_wait(bar(KB_XE + s), ((li - 2) >> 1) & 1, abort_flag, err)) break;
        const int t0 = (blockIdx.x + li * gridDim.x) * kTcRows;
        mbar_arrive_expect_tx(bar(KB_XF + s), K::X_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sb + K::OFF_X + s * K::X_BYTES + c * kTcRows * 128, &tx, bar(KB_XF + s), c * 64, t0, bh);
        issued = li + 1;
      }
      // every issued copy lands before the CTA exits (a copy older than the last two was
      // consumed by an MMA, whose completion freed its stage for a later copy)
      mbar_wait_drain(bar(KB_C), 0, err);
      for (int li = (issued > 2 ? issued - 2 : 0); li < issued; ++li)
        mbar_wait_drain(bar(KB_XF + (li & 1)), (li >> 1) & 1, err);
    }
    __syncwarp();
  } else if (warp == 9) {  // ---- MMAs ----
    if (lane == 0) {
      bool ok = mbar_wait(bar(KB_C), 0, abort_flag, err);
      int issued = 0;
      for (int li = 0; ok && li < mine; ++li) {
        const int s = li & 1;
        if (!mbar_wait(bar(KB_XF + s), (li >> 1) & 1, abort_flag, err)) break;
        if (li >= 2 && !mbar_wait(bar(KB_SE + s), ((li - 2) >> 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint64_t dx = sdesc_sw128(sb + K::OFF_X + s * K::X_BYTES, 16, 1024);
#pragma unroll
        for (int ct = 0; ct < NCT; ++ct) {
          const uint64_t dh = sdesc_sw128(sb + K::OFF_C + (2 * ct) * K::CT_BYTES, 16, 1024);
          const uint64_t dl = sdesc_sw128(sb + K::OFF_C + (2 * ct + 1) * K::CT_BYTES, 16, 1024);
          const uint32_t d_s = tmem + s * K::SCOLS + ct * kTcRows;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) / 16);
            tc_mma_ss(d_s, dx + off, dh + off, K::IDESC, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) / 16);
            tc_mma_ss(d_s, dx + off, dl + off, K::IDESC, 1u);
          }
        }
        tc_commit(bar(KB_XE + s));
        tc_commit(bar(KB_SF + s));
        issued = li + 1;
      }
      // every issued MMA completes before TMEM is released: the last commits cover them
      if (issued > 0) mbar_wait_drain(bar(KB_SF + ((issued - 1) & 1)), ((issued - 1) >> 1) & 1, err);
    }
    __syncwarp();
  } else {  // ---- argmin: warpgroup g = warp / 4 takes the tiles li = g, g + 2, ...; row = lane quarter ----
    const int g = warp >> 2, row = (warp & 3) * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + g * K::SCOLS;
    for (int li = g; li < mine; li += 2) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(KB_SF + g), (li >> 1) & 1, abort_flag, err))) break;
      tc_fence_after();
      // ascending centroid index with a strict < keeps the smaller index on ties
      float best_d = INFINITY;
      int best_j = 0;
#pragma unroll
      for (int ct = 0; ct < NCT; ++ct) {
        const int c0 = ct * kTcRows;
        const int nc = min(kTcRows, C - c0);
#pragma unroll 1
        for (int q = 0; q < kTcRows / 32; ++q) {
          if (q * 32 >= nc) break;
          float sv[32];
          tmem_ld32(t_lane + c0 + q * 32, sv);
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const int jl = q * 32 + x;
            float dist = __fmaf_rn(-2.f, sv[x], cn[c0 + jl]);  // |c|^2 - 2 s, rounded once
            dist = jl < nc ? dist : INFINITY;
            const bool lt = dist < best_d;
            best_d = lt ? dist : best_d;
            best_j = lt ? c0 + jl : best_j;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(KB_SE + g));  // S buffer g may be overwritten
      const int t = (blockIdx.x + li * gridDim.x) * kTcRows + row;
      if (t < N) label[static_cast<size_t>(bh) * N + t] = best_j;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, K::TMEM_COLS);
}

// Counts, offsets and the stable cluster-major order (slots sorted by (cluster, token)) of
// every head, in three launches.  A head's tokens are cut into kSortSegs contiguous segments:
//   hist     one CTA per (segment, head): the segment's label histogram;
//   scan     one CTA per head: counts, offsets, chunk offsets (exclusive scans over the
//            clusters), then every segment's first slot per cluster (segments before it);
//   scatter  one CTA per (segment, head): the segment is cut again into kSortWarps warp
//            segments with their own histograms, and every warp ranks its tokens in token
//            order, 32 per step (ranks among equal labels from __match_any_sync).
// A label outside [0, C) anywhere in a head sets VSA_DEVERR_KV_RANGE and leaves that head with
// empty clusters (counts and offsets zero, no slot written).
constexpr int kSortWarps = 16;
constexpr int kSortSegs = 8;
constexpr int kSortPrefetch = 8;  // 32-token steps whose labels are loaded ahead
constexpr int kUpdChunk = 128;    // member rows per partial-sum CTA of the update

__device__ __forceinline__ int seg_begin(int N, int nseg, int s) {
  return static_cast<int>((static_cast<long long>(N) * s) / nseg);
}

// seg_hist [BH, kSortSegs, C]; bad [BH] (set to 1 on a label outside [0, C))
__global__ void __launch_bounds__(256) kmeans_hist_kernel(const int32_t* __restrict__ label, int N, int C,
                                                          int32_t* __restrict__ seg_hist, int32_t* __restrict__ bad) {
  extern __shared__ int hist_smem[];
  const int sg = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  for (int j = tid; j < C; j += blockDim.x) hist_smem[j] = 0;
  __syncthreads();
  const int32_t* lh = label + static_cast<size_t>(bh) * N;
  const int a = seg_begin(N, kSortSegs, sg), b = seg_begin(N, kSortSegs, sg + 1);
  bool badl = false;
  for (int t = a + tid; t < b; t += blockDim.x) {
    const int l = lh[t];
    if (l >= 0 && l < C) atomicAdd(&hist_smem[l], 1);
    else badl = true;
  }
  if (badl) atomicExch(&bad[bh], 1);
  __syncthreads();
  int32_t* out = seg_hist + (static_cast<size_t>(bh) * kSortSegs + sg) * C;
  for (int j = tid; j < C; j += blockDim.x) out[j] = hist_smem[j];
}

// Turns seg_hist into every segment's first slot per cluster, in place.
__global__ void __launch_bounds__(256) kmeans_scan_kernel(int C, int32_t* __restrict__ seg_hist,
                                                          int32_t* __restrict__ bad,
                                                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ chunk_off,
                                                          int32_t* __restrict__ chunk_cl, int max_chunks, int* err) {
  extern __shared__ int tot[];  // [C]
  const int bh = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* hh = seg_hist + static_cast<size_t>(bh) * kSortSegs * C;
  const bool is_bad = bad[bh] != 0;
  __syncthreads();
  if (tid == 0) bad[bh] = 0;  // clear for the next round (the scatter tests offsets[C] instead)
  if (is_bad) {  // empty clusters: the update and the mask read nothing
    if (tid == 0) atomicOr(err, kDevErrKvRange);
    for (int j = tid; j < C; j += blockDim.x) {
      counts[static_cast<size_t>(bh) * C + j] = 0;
      offsets[static_cast<size_t>(bh) * (C + 1) + j] = 0;
    }
    for (int j = tid; j <= C; j += blockDim.x) {
      chunk_off[static_cast<size_t>(bh) * (C + 1) + j] = 0;
      if (j == C) offsets[static_cast<size_t>(bh) * (C + 1) + C] = 0;
    }
    return;
  }
  for (int j = tid; j < C; j += blockDim.x) {
    int sum = 0;
    for (int sg = 0; sg < kSortSegs; ++sg) sum += hh[sg * C + j];
    tot[j] = sum;
    counts[static_cast<size_t>(bh) * C + j] = sum;
  }
  __syncthreads();
  // exclusive scans over the clusters (warp 0, 32 clusters per step): of tot (the offsets) and
  // of each cluster's number of kUpdChunk-row chunks (the update's partial sums)
  if (warp == 0) {
    int carry = 0, ccarry = 0;
    for (int j0 = 0; j0 < C; j0 += 32) {
      const int j = j0 + lane;
      const int v = j < C ? tot[j] : 0;
      const int cv = (v + kUpdChunk - 1) / kUpdChunk;
      int incl = v, cincl = cv;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        const int co = __shfl_up_sync(0xffffffffu, cincl, off);
        if (lane >= off) {
          incl += o;
          cincl += co;
        }
      }
      if (j < C) {
        tot[j] = carry + incl - v;
        offsets[static_cast<size_t>(bh) * (C + 1) + j] = carry + incl - v;
        chunk_off[static_cast<size_t>(bh) * (C + 1) + j] = ccarry + cincl - cv;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
      ccarry += __shfl_sync(0xffffffffu, cincl, 31);
    }
    if (lane == 0) {
      offsets[static_cast<size_t>(bh) * (C + 1) + C] = carry;
      chunk_off[static_cast<size_t>(bh) * (C + 1) + C] = ccarry;
    }
  }
  __syncthreads();
  for (int j = tid; j < C; j += blockDim.x) {
    int run = tot[j];
    for (int sg = 0; sg < kSortSegs; ++sg) {
      const int c = hh[sg * C + j];
      hh[sg * C + j] = run;
      run += c;
    }
    // the cluster of every partial-sum chunk (the chunks of j follow its chunk offset)
    const int32_t* co = chunk_off + static_cast<size_t>(bh) * (C + 1);
    for (int k = co[j]; k < co[j + 1]; ++k) chunk_cl[static_cast<size_t>(bh) * max_chunks + k] = j;
  }
}

// Shared memory: kSortWarps * C ints.  A head whose labels were bad has offsets[C] = 0 != N.
__global__ void __launch_bounds__(kSortWarps * 32) kmeans_scatter_kernel(const int32_t* __restrict__ label, int N,
                                                                         int C, const int32_t* __restrict__ seg_start,
                                                                         const int32_t* __restrict__ offsets,
                                                                         int32_t* __restrict__ perm) {
  extern __shared__ int sort_smem[];
  int* hist = sort_smem;  // [kSortWarps][C]: counts, then first free slot, per warp segment
  const int sg = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (offsets[static_cast<size_t>(bh) * (C + 1) + C] != N) return;
  const int32_t* lh = label + static_cast<size_t>(bh) * N;
  const int a = seg_begin(N, kSortSegs, sg), b = seg_begin(N, kSortSegs, sg + 1);
  const int s0 = a + seg_begin(b - a, kSortWarps, warp), s1 = a + seg_begin(b - a, kSortWarps, warp + 1);
  for (int e = tid; e < kSortWarps * C; e += kSortWarps * 32) hist[e] = 0;
  __syncthreads();
  for (int t = s0 + lane; t < s1; t += 32) atomicAdd(&hist[warp * C + lh[t]], 1);  // labels checked by hist
  __syncthreads();
  const int32_t* base = seg_start + (static_cast<size_t>(bh) * kSortSegs + sg) * C;
  for (int j = tid; j < C; j += kSortWarps * 32) {
    int run = base[j];
    for (int w = 0; w < kSortWarps; ++w) {
      const int c = hist[w * C + j];
      hist[w * C + j] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  int* cur = hist + warp * C;
  int32_t* ph = perm + static_cast<size_t>(bh) * N;
  for (int base_t = s0; base_t < s1; base_t += 32 * kSortPrefetch) {
    int lab[kSortPrefetch];
#pragma unroll
    for (int u = 0; u < kSortPrefetch; ++u) {
      const int t = base_t + u * 32 + lane;
      lab[u] = t < s1 ? lh[t] : -1;
    }
#pragma unroll
    for (int u = 0; u < kSortPrefetch; ++u) {
      const int t = base_t + u * 32 + lane;
      const int l = lab[u];
      const unsigned peers = __match_any_sync(0xffffffffu, l);
      const int rank = __popc(peers & lt);
      const int slot = l >= 0 ? cur[l] + rank : 0;
      __syncwarp();
      if (l >= 0) {
        ph[slot] = t;
        if (rank == 0) cur[l] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

// New centroids.  The reading is the members' fp64 sum in token order, divided by the count.
// That sum is computed in parallel and still exactly: every member value is a bf16 number, so
// all of a cluster's values in one dimension are integer multiples of 2^q, q the smallest
// unit in the last place among them (ulp(v) = 2^(E - 7) for a normal bf16 value of exponent
// E, 2^-133 for a subnormal one).  Every partial sum, in any order, is then a multiple of 2^q
// of magnitude at most A = sum |v|, and fp64 holds every such number exactly while
// A < 2^(q + 53).  Under that condition the ordered sum and any grouping of it are the same
// exact number.  kmeans_partial_kernel sums chunks of kUpdChunk members (and their |v| and
// q); kmeans_combine_kernel adds a cluster's chunks, checks the condition, and where it fails
// (values spread over more than 53 binades, an infinity or a NaN) adds the members again one
// by one in token order.  A sum of non-negative fp64 numbers reaches 2^(q+53) in floating
// point exactly when it does in exact arithmetic, so the check itself is exact.
constexpr int kNoUlp = 1000;  // q of a dimension with no nonzero member

// One CTA of kPartThreads per chunk k of a head's chunk list (chunk_cl[k]: the chunk's cluster,
// written by the scan).  Thread (row lane rl, dimension group g) loads 16-byte pieces (8
// dimensions) of rows rl, rl + RL, ... all at once (the member index of a row is one load the
// G threads of a row share), so a CTA waits for one round of memory latency; the row lanes'
// partial sums are then added with shuffles inside each warp and through shared memory across
// the warps (any order: see above).
constexpr int kPartThreads = 128;

template <int D>
__global__ void __launch_bounds__(kPartThreads, 4) kmeans_partial_kernel(const __nv_bfloat16* __restrict__ x, int N,
                                                                      int C, const int32_t* __restrict__ offsets,
                                                                      const int32_t* __restrict__ chunk_off,
                                                                      const int32_t* __restrict__ chunk_cl,
                                                                      const int32_t* __restrict__ perm, int max_chunks,
                                                                      double* __restrict__ psum,
                                                                      double* __restrict__ pabs,
                                                                      int32_t* __restrict__ pq) {
  constexpr int G = D / 8;               // dimension groups of 8
  constexpr int RL = kPartThreads / G;   // row lanes
  constexpr int PER = kUpdChunk / RL;    // rows per thread
  constexpr int NW = kPartThreads / 32;  // warps
  static_assert(G <= 32 && 32 % G == 0, "a warp holds whole rows");
  __shared__ double red_s[NW][D];
  __shared__ double reda_s[NW][D];
  __shared__ int redq_s[NW][D];
  const int k = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t* co = chunk_off + static_cast<size_t>(bh) * (C + 1);
  if (k >= co[C]) return;
  const int j = chunk_cl[static_cast<size_t>(bh) * max_chunks + k];
  const int32_t* off = offsets + static_cast<size_t>(bh) * (C + 1);
  const int first = (k - co[j]) * kUpdChunk;
  const int cnt = min(kUpdChunk, off[j + 1] - off[j] - first);
  const int32_t* ph = perm + static_cast<size_t>(bh) * N + off[j] + first;
  const int g = tid % G, rl = tid / G;
  const uint4* xh = reinterpret_cast<const uint4*>(x + static_cast<size_t>(bh) * N * D);
  int rows[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int r = rl + i * RL;
    const int t = r < cnt ? __ldg(ph + r) : -1;
    rows[i] = (t >= 0 && t < N) ? t : -1;
  }
  uint4 w[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i)
    w[i] = rows[i] >= 0 ? __ldg(xh + static_cast<size_t>(rows[i]) * G + g) : make_uint4(0u, 0u, 0u, 0u);
  // Per dimension: the fp32 sum and |v| sum of this thread's PER rows, and the smallest nonzero
  // magnitude (15-bit bf16 pattern, packed in 16-bit halves, zeros counted as 0xffff).  The
  // fp32 sums are exact while the |v| sum stays below 2^(q + 24) (the argument above with a
  // 24-bit significand); a thread whose sums may not be exact adds its rows again in fp64.
  uint64_t s2[4], a2[4];
  uint32_t mm[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    s2[p] = 0ull;
    a2[p] = 0ull;
    mm[p] = 0xffffffffu;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const uint32_t ww[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // dimensions 2p (low half) and 2p + 1 (high half)
      const uint32_t lo = ww[p] << 16, hi = ww[p] & 0xffff0000u;
      s2[p] = f2_add(s2[p], f2_make(__uint_as_float(lo), __uint_as_float(hi)));
      a2[p] = f2_add(a2[p], f2_make(__uint_as_float(lo & 0x7fffffffu), __uint_as_float(hi & 0x7fffffffu)));
      const uint32_t mag = ww[p] & 0x7fff7fffu;
      mm[p] = __vminu2(mm[p], mag | __vcmpeq2(mag, 0u));
    }
  }
  double sa[8], aa[8];
  int qa[8];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    float f0, f1, g0, g1;
    f2_split(s2[p], f0, f1);
    f2_split(a2[p], g0, g1);
    const uint32_t m0 = mm[p] & 0xffffu, m1 = mm[p] >> 16;
    // ulp exponent of the smallest nonzero magnitude: max(exponent field, 1) - 134
    qa[2 * p] = m0 == 0xffffu ? kNoUlp : max(static_cast<int>(m0 >> 7), 1) - 134;
    qa[2 * p + 1] = m1 == 0xffffu ? kNoUlp : max(static_cast<int>(m1 >> 7), 1) - 134;
    sa[2 * p] = f0;
    sa[2 * p + 1] = f1;
    aa[2 * p] = g0;
    aa[2 * p + 1] = g1;
  }
  bool exact = true;
#pragma unroll
  for (int e = 0; e < 8; ++e) exact = exact && (aa[e] < ldexp(1.0, min(qa[e], 200) + 24));
  if (!exact) {  // rare: the same rows again in fp64
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sa[e] = 0.0;
      aa[e] = 0.0;
    }
#pragma unroll 1
    for (int i = 0; i < PER; ++i) {
      const int r = rl + i * RL;
      const int t = r < cnt ? __ldg(ph + r) : -1;
      const uint4 v4 = (t >= 0 && t < N) ? __ldg(xh + static_cast<size_t>(t) * G + g) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t ww[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t bits = (e & 1) ? (ww[e >> 1] & 0xffff0000u) : (ww[e >> 1] << 16);
        const double v = static_cast<double>(__uint_as_float(bits));
        sa[e] += v;
        aa[e] += fabs(v);
      }
    }
  }
  // row lanes of one warp (lanes g, g + G, ...), then the warps
#pragma unroll
  for (int o = G; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sa[e] += __shfl_xor_sync(0xffffffffu, sa[e], o);
      aa[e] += __shfl_xor_sync(0xffffffffu, aa[e], o);
      qa[e] = min(qa[e], __shfl_xor_sync(0xffffffffu, qa[e], o));
    }
  }
  if (lane < G) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red_s[warp][g * 8 + e] = sa[e];
      reda_s[warp][g * 8 + e] = aa[e];
      redq_s[warp][g * 8 + e] = qa[e];
    }
  }
  __syncthreads();
  for (int dd = tid; dd < D; dd += kPartThreads) {
    double sm = 0.0, am = 0.0;
    int q = kNoUlp;
#pragma unroll
    for (int l = 0; l < NW; ++l) {
      sm += red_s[l][dd];
      am += reda_s[l][dd];
      q = min(q, redq_s[l][dd]);
    }
    const size_t o = (static_cast<size_t>(bh) * max_chunks + k) * D + dd;
    psum[o] = sm;
    pabs[o] = am;
    pq[o] = q;
  }
}

// One CTA (d threads) per (cluster, head): the cluster's chunk sums in order, the exactness
// check, the fallback, then the centroid as fp32(sum / n), its bf16 halves and its norm.  An
// empty cluster keeps its centroid.
template <int D>
__global__ void __launch_bounds__(D) kmeans_combine_kernel(const __nv_bfloat16* __restrict__ x, int N, int C,
                                                           const int32_t* __restrict__ counts,
                                                           const int32_t* __restrict__ offsets,
                                                           const int32_t* __restrict__ chunk_off,
                                                           const int32_t* __restrict__ perm, int max_chunks,
                                                           const double* __restrict__ psum,
                                                           const double* __restrict__ pabs,
                                                           const int32_t* __restrict__ pq, float* __restrict__ cent,
                                                           float* __restrict__ cnorm, __nv_bfloat16* __restrict__ chi,
                                                           __nv_bfloat16* __restrict__ clo) {
  __shared__ float cnew[D];
  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int n = counts[static_cast<size_t>(bh) * C + j];
  if (n <= 0) return;
  const int32_t* co = chunk_off + static_cast<size_t>(bh) * (C + 1);
  double sum = 0.0, abs_sum = 0.0;
  int q = kNoUlp;
  for (int k = co[j]; k < co[j + 1]; ++k) {
    const size_t o = (static_cast<size_t>(bh) * max_chunks + k) * D + tid;
    sum = __dadd_rn(sum, psum[o]);
    abs_sum = __dadd_rn(abs_sum, pabs[o]);
    q = min(q, pq[o]);
  }
  if (!(abs_sum < ldexp(1.0, q + 53))) {  // not provably exact: the ordered sum itself
    const int32_t* ph = perm + static_cast<size_t>(bh) * N + offsets[static_cast<size_t>(bh) * (C + 1) + j];
    const __nv_bfloat16* xh = x + static_cast<size_t>(bh) * N * D;
    sum = 0.0;
    for (int m = 0; m < n; ++m) {
      const int t = ph[m];
      if (t >= 0 && t < N) sum = __dadd_rn(sum, static_cast<double>(__bfloat162float(xh[static_cast<size_t>(t) * D + tid])));
    }
  }
  const float c = __double2float_rn(__ddiv_rn(sum, static_cast<double>(n)));
  const size_t o = (static_cast<size_t>(bh) * C + j) * D + tid;
  cent[o] = c;
  cnew[tid] = c;
  const __nv_bfloat16 h = __float2bfloat16_rn(c);
  chi[o] = h;
  clo[o] = __float2bfloat16_rn(__fsub_rn(c, __bfloat162float(h)));
  __syncthreads();
  if (tid == 0) cnorm[static_cast<size_t>(bh) * C + j] = sq_norm(cnew, D);
}

// ---------------------------------------------------------------------------------------
// top-p budget
// ---------------------------------------------------------------------------------------

// Kept key clusters of query cluster blockIdx.x of head blockIdx.y: keep[bh, i, ceil(Ck/32)].
__global__ void __launch_bounds__(kKeepThreads) semantic_keep_kernel(const float* __restrict__ cq,
                                                                     const int32_t* __restrict__ nq, int Cq,
                                                                     const float* __restrict__ ck,
                                                                     const int32_t* __restrict__ nk, int Ck, int D,
                                                                     double scale, double top_p, int n2,
                                                                     uint32_t* __restrict__ keep) {
  extern __shared__ double ks_w[];                 // [n2] weights, then [n2] cluster indices
  int* ks_i = reinterpret_cast<int*>(ks_w + n2);
  __shared__ double red[kKeepThreads / 32];
  __shared__ uint32_t row_s[kMaxClusters / 32];
  constexpr int kNone = 0x7fffffff;
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int words = (Ck + 31) >> 5;
  for (int w = tid; w < words; w += kKeepThreads) row_s[w] = 0u;
  const bool live_row = nq[static_cast<size_t>(bh) * Cq + i] > 0;
  const float* qi = cq + (static_cast<size_t>(bh) * Cq + i) * D;
  const int32_t* nkh = nk + static_cast<size_t>(bh) * Ck;
  double lmax = -INFINITY;
  for (int j = tid; j < n2; j += kKeepThreads) {
    double s = -1.0;
    int id = kNone;
    if (live_row && j < Ck && nkh[j] > 0) {
      const float* kj = ck + (static_cast<size_t>(bh) * Ck + j) * D;
      double acc = 0.0;
      for (int x = 0; x < D; ++x) acc = __fma_rn(static_cast<double>(qi[x]), static_cast<double>(kj[x]), acc);
      s = __dmul_rn(scale, acc);
      id = j;
      lmax = fmax(lmax, s);
    }
    ks_w[j] = s;
    ks_i[j] = id;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lmax = fmax(lmax, __shfl_xor_sync(0xffffffffu, lmax, off));
  if ((tid & 31) == 0) red[tid >> 5] = lmax;
  __syncthreads();
  double m = red[0];
#pragma unroll
  for (int w = 1; w < kKeepThreads / 32; ++w) m = fmax(m, red[w]);
  for (int j = tid; j < n2; j += kKeepThreads) {
    if (ks_i[j] != kNone)
      ks_w[j] = __dmul_rn(static_cast<double>(nkh[ks_i[j]]), exp(__dsub_rn(ks_w[j], m)));  // CUDA fp64 exp
    else
      ks_w[j] = -1.0;  // below every weight (weights are >= 0)
  }
  __syncthreads();
  // bitonic sort: weight descending, then cluster index ascending
  for (int k = 2; k <= n2; k <<= 1)
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int e = tid; e < n2; e += kKeepThreads) {
        const int p = e ^ jj;
        if (p > e) {
          const double wa = ks_w[e], wb = ks_w[p];
          const int ia = ks_i[e], ib = ks_i[p];
          const bool a_first = wa > wb || (wa == wb && ia < ib);
          const bool up = (e & k) == 0;
          if (up != a_first) {
            ks_w[e] = wb;
            ks_w[p] = wa;
            ks_i[e] = ib;
            ks_i[p] = ia;
          }
        }
      }
      __syncthreads();
    }
  if (tid == 0 && live_row) {
    double total = 0.0;
    int live = 0;
    while (live < n2 && ks_i[live] != kNone) total = __dadd_rn(total, ks_w[live++]);
    const double target = __dmul_rn(top_p, total);
    double cum = 0.0;
    for (int e = 0; e < live; ++e) {
      const int j = ks_i[e];
      row_s[j >> 5] |= 1u << (j & 31);
      cum = __dadd_rn(cum, ks_w[e]);
      if (cum >= target) break;
    }
  }
  __syncthreads();
  uint32_t* krow = keep + (static_cast<size_t>(bh) * Cq + i) * words;
  for (int w = tid; w < words; w += kKeepThreads) krow[w] = row_s[w];
}

// ---------------------------------------------------------------------------------------
// block mask over the cluster-major layouts
// ---------------------------------------------------------------------------------------

// Cluster of the first and last slot of every block: in a cluster-major layout the clusters
// present in a block are exactly the non-empty ones between these two.
__global__ void block_cluster_range_kernel(const int32_t* __restrict__ label, const int32_t* __restrict__ perm,
                                           int N, int block, int nblk, int C, int2* __restrict__ range, int* err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x, bh = blockIdx.y;
  if (b >= nblk) return;
  const int s0 = b * block, s1 = min(N, (b + 1) * block) - 1;
  const int32_t* ph = perm + static_cast<size_t>(bh) * N;
  const int32_t* lh = label + static_cast<size_t>(bh) * N;
  const int t0 = ph[s0], t1 = ph[s1];
  int2 r = make_int2(0, -1);  // empty range
  if (t0 >= 0 && t0 < N && t1 >= 0 && t1 < N) {
    const int l0 = lh[t0], l1 = lh[t1];
    if (l0 >= 0 && l0 <= l1 && l1 < C) r = make_int2(l0, l1);
    else atomicOr(err, kDevErrKvRange);
  } else {
    atomicOr(err, kDevErrKvRange);
  }
  range[static_cast<size_t>(bh) * nblk + b] = r;
}

__device__ __forceinline__ bool any_bit_in_range(const uint32_t* bits, int lo, int hi) {
  for (int w = lo >> 5; w <= (hi >> 5); ++w) {
    uint32_t m = bits[w];
    if (w == (lo >> 5)) m &= ~0u << (lo & 31);
    if (w == (hi >> 5) && (hi & 31) != 31) m &= (1u << ((hi & 31) + 1)) - 1u;
    if (m) return true;
  }
  return false;
}

// One warp per (head, query block): the key clusters reachable from the block's query
// clusters, then every key block tested against its cluster range.
__global__ void __launch_bounds__(32) semantic_block_mask_kernel(
    const int2* __restrict__ qrange, const int2* __restrict__ krange, const int32_t* __restrict__ nq, int Cq,
    const int32_t* __restrict__ nk, int Ck, const uint32_t* __restrict__ keep, int nblk, uint32_t* __restrict__ bits,
    int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, int max_kv, int* err) {
  __shared__ uint32_t reach[kMaxClusters / 32];
  const int bq = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
  const int words = (Ck + 31) >> 5, nwb = (nblk + 31) >> 5;
  const int2 qr = qrange[static_cast<size_t>(bh) * nblk + bq];
  uint32_t acc = 0u;
  for (int i = qr.x; i <= qr.y; ++i) {
    if (nq[static_cast<size_t>(bh) * Cq + i] <= 0) continue;
    if (lane < words) acc |= keep[(static_cast<size_t>(bh) * Cq + i) * words + lane];
  }
  if (lane < words) {
    uint32_t ne = 0u;
    for (int b = 0; b < 32; ++b) {
      const int j = lane * 32 + b;
      if (j < Ck && nk[static_cast<size_t>(bh) * Ck + j] > 0) ne |= 1u << b;
    }
    reach[lane] = acc & ne;
  }
  __syncwarp();
  const size_t row = static_cast<size_t>(bh) * nblk + bq;
  const unsigned lt = (1u << lane) - 1u;
  int cnt = 0;
  for (int b0 = 0; b0 < nblk; b0 += 32) {
    const int bk = b0 + lane;
    bool kept = false;
    if (bk < nblk) {
      const int2 kr = krange[static_cast<size_t>(bh) * nblk + bk];
      kept = kr.x <= kr.y && any_bit_in_range(reach, kr.x, kr.y);
    }
    const unsigned ball = __ballot_sync(0xffffffffu, kept);
    if (lane == 0) bits[row * nwb + (b0 >> 5)] = ball;
    const int pos = cnt + __popc(ball & lt);
    if (kept && pos < max_kv) kv_idx[row * max_kv + pos] = bk;
    cnt += __popc(ball);
  }
  if (lane == 0) {
    if (cnt > max_kv) atomicOr(err, kDevErrOverflow);
    kv_cnt[row] = min(cnt, max_kv);
  }
}

// ---------------------------------------------------------------------------------------
// row gather / scatter through a per-head permutation (16-byte vectors)
// ---------------------------------------------------------------------------------------

__global__ void __launch_bounds__(kRowThreads) gather_rows_kernel(const uint4* __restrict__ src,
                                                                  const int32_t* __restrict__ perm,
                                                                  uint4* __restrict__ dst, int N, int vpr, int* err) {
  const int bh = blockIdx.y;
  const size_t total = static_cast<size_t>(N) * vpr;
  const size_t head = static_cast<size_t>(bh) * total;
  for (size_t e = static_cast<size_t>(blockIdx.x) * kRowThreads + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * kRowThreads) {
    const int s = static_cast<int>(e / vpr), v = static_cast<int>(e - static_cast<size_t>(s) * vpr);
    const int t = perm[static_cast<size_t>(bh) * N + s];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t >= 0 && t < N) val = src[head + static_cast<size_t>(t) * vpr + v];
    else if (v == 0) atomicOr(err, kDevErrKvRange);
    dst[head + e] = val;
  }
}

__global__ void __launch_bounds__(kRowThreads) scatter_rows_kernel(const uint4* __restrict__ src,
                                                                   const float* __restrict__ src_lse,
                                                                   const int32_t* __restrict__ perm,
                                                                   uint4* __restrict__ dst, float* __restrict__ dst_lse,
                                                                   int N, int vpr, int* err) {
  const int bh = blockIdx.y;
  const size_t total = static_cast<size_t>(N) * vpr;
  const size_t head = static_cast<size_t>(bh) * total;
  for (size_t e = static_cast<size_t>(blockIdx.x) * kRowThreads + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * kRowThreads) {
    const int s = static_cast<int>(e / vpr), v = static_cast<int>(e - static_cast<size_t>(s) * vpr);
    const int t = perm[static_cast<size_t>(bh) * N + s];
    if (t < 0 || t >= N) {
      if (v == 0) atomicOr(err, kDevErrKvRange);
      continue;
    }
    dst[head + static_cast<size_t>(t) * vpr + v] = src[head + e];
    if (v == 0 && dst_lse != nullptr)
      dst_lse[static_cast<size_t>(bh) * N + t] = src_lse[static_cast<size_t>(bh) * N + s];
  }
}

int rows_grid_x(int N, int vpr, int BH) {
  const long long want = (static_cast<long long>(N) * vpr + kRowThreads - 1) / kRowThreads;
  const long long cap = (148LL * 16 + BH - 1) / BH;
  return static_cast<int>(want < cap ? want : cap);
}

// k-means scratch, carved from the caller's workspace (256-byte aligned pieces).
struct KmWork {
  int32_t* offsets;    // [BH, C + 1] cluster offsets in the cluster-major order
  int32_t* chunk_off;  // [BH, C + 1] first partial-sum chunk of every cluster
  float* cnorm;        // [BH, C] squared centroid norms
  __nv_bfloat16* chi;  // [BH, C, d] bf16 high halves of the centroids
  __nv_bfloat16* clo;  // [BH, C, d] bf16 low halves
  double* psum;        // [BH, max_chunks, d] chunk sums
  double* pabs;        // [BH, max_chunks, d] chunk sums of |v|
  int32_t* pq;         // [BH, max_chunks, d] chunk ulp exponents
  int32_t* seg_hist;   // [BH, kSortSegs, C] segment histograms, then segment first slots
  int32_t* chunk_cl;   // [BH, max_chunks] cluster of every partial-sum chunk
  int32_t* bad;        // [BH] a label outside [0, C) was seen
  int max_chunks;      // ceil(N / kUpdChunk) + C bounds a head's chunk count
  size_t bytes;
};

KmWork kmeans_layout(void* ws, int BH, int N, int C, int d) {
  KmWork w{};
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    void* p = base ? base + off : nullptr;
    off += (bytes + 255) & ~static_cast<size_t>(255);
    return p;
  };
  const size_t bh = static_cast<size_t>(BH);
  w.max_chunks = (N + kUpdChunk - 1) / kUpdChunk + C;
  w.offsets = static_cast<int32_t*>(take(bh * (C + 1) * sizeof(int32_t)));
  w.chunk_off = static_cast<int32_t*>(take(bh * (C + 1) * sizeof(int32_t)));
  w.cnorm = static_cast<float*>(take(bh * C * sizeof(float)));
  w.chi = static_cast<__nv_bfloat16*>(take(bh * C * d * sizeof(__nv_bfloat16)));
  w.clo = static_cast<__nv_bfloat16*>(take(bh * C * d * sizeof(__nv_bfloat16)));
  w.psum = static_cast<double*>(take(bh * w.max_chunks * d * sizeof(double)));
  w.pabs = static_cast<double*>(take(bh * w.max_chunks * d * sizeof(double)));
  w.pq = static_cast<int32_t*>(take(bh * w.max_chunks * d * sizeof(int32_t)));
  w.seg_hist = static_cast<int32_t*>(take(bh * kSortSegs * C * sizeof(int32_t)));
  w.bad = static_cast<int32_t*>(take(bh * sizeof(int32_t)));
  w.chunk_cl = static_cast<int32_t*>(take(bh * w.max_chunks * sizeof(int32_t)));
  w.bytes = off;
  return w;
}

template <int D>
cudaError_t kmeans_d(const __nv_bfloat16* x, int BH, int N, int C, int iters, float* cent, int32_t* label,
                     int32_t* counts, int32_t* perm, const KmWork& w, int* err, cudaStream_t stream) {
  using K = KmTcCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(kmeans_assign_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM);
  if (e != cudaSuccess) return e;
  const size_t ssmem = sizeof(int) * kSortWarps * static_cast<size_t>(C);
  if (ssmem > 48 * 1024) {
    e = cudaFuncSetAttribute(kmeans_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(ssmem));
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tx, thi, tlo;
  if ((e = encode_rows_map(&tx, x, D, N, BH, kTcRows)) != cudaSuccess) return e;
  if ((e = encode_rows_map(&thi, w.chi, D, C, BH, kTcRows)) != cudaSuccess) return e;
  if ((e = encode_rows_map(&tlo, w.clo, D, C, BH, kTcRows)) != cudaSuccess) return e;
  kmeans_init_kernel<<<dim3(C, BH), 128, 0, stream>>>(x, N, D, C, cent, w.cnorm, w.chi, w.clo, w.bad);
  const dim3 agrid((N + kTcRows - 1) / kTcRows, BH), pgrid(w.max_chunks, BH), cgrid(C, BH);
  // resident centroids (C <= 256): persistent CTAs, one per SM, spread evenly over the heads;
  // the shared-memory request keeps one CTA per SM so that TMEM never oversubscribes
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const int ntiles = (N + kTcRows - 1) / kTcRows;
  const dim3 pcgrid(std::min(ntiles, std::max(1, sms / BH)), BH);
  const int pc1 = std::max(KmPcCfg<D, 1>::SMEM, 120 * 1024), pc2 = std::max(KmPcCfg<D, 2>::SMEM, 120 * 1024);
  if (C <= kTcRows) {
    if ((e = cudaFuncSetAttribute(kmeans_assign_pc_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, pc1)) !=
        cudaSuccess)
      return e;
  } else if (C <= 2 * kTcRows) {
    if ((e = cudaFuncSetAttribute(kmeans_assign_pc_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, pc2)) !=
        cudaSuccess)
      return e;
  }
  for (int it = 0; it < iters; ++it) {
    if (C <= kTcRows)
      kmeans_assign_pc_kernel<D, 1><<<pcgrid, kPcThreads, pc1, stream>>>(tx, thi, tlo, N, C, w.cnorm, label, err);
    else if (C <= 2 * kTcRows)
      kmeans_assign_pc_kernel<D, 2><<<pcgrid, kPcThreads, pc2, stream>>>(tx, thi, tlo, N, C, w.cnorm, label, err);
    else
      kmeans_assign_tc_kernel<D><<<agrid, 128, K::SMEM, stream>>>(tx, thi, tlo, N, C, w.cnorm, label, err);
    const dim3 sgrid(kSortSegs, BH);
    kmeans_hist_kernel<<<sgrid, 256, sizeof(int) * C, stream>>>(label, N, C, w.seg_hist, w.bad);
    kmeans_scan_kernel<<<BH, 256, sizeof(int) * C, stream>>>(C, w.seg_hist, w.bad, counts, w.offsets, w.chunk_off,
                                                             w.chunk_cl, w.max_chunks, err);
    kmeans_scatter_kernel<<<sgrid, kSortWarps * 32, ssmem, stream>>>(label, N, C, w.seg_hist, w.offsets, perm);
    kmeans_partial_kernel<D><<<pgrid, kPartThreads, 0, stream>>>(x, N, C, w.offsets, w.chunk_off, w.chunk_cl, perm,
                                                                 w.max_chunks, w.psum, w.pabs, w.pq);
    kmeans_combine_kernel<D><<<cgrid, D, 0, stream>>>(x, N, C, counts, w.offsets, w.chunk_off, perm, w.max_chunks,
                                                      w.psum, w.pabs, w.pq, cent, w.cnorm, w.chi, w.clo);
  }
  return cudaGetLastError();
}

}  // namespace

size_t kmeans_workspace_bytes(int BH, int N, int C, int d) {
  KmWork w = kmeans_layout(nullptr, BH, N, C, d);
  return w.bytes;
}

cudaError_t launch_kmeans(const void* x, int BH, int N, int d, int C, int iters, float* cent, int32_t* label,
                          int32_t* counts, int32_t* perm, void* ws, int* err, cudaStream_t stream) {
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  const KmWork w = kmeans_layout(ws, BH, N, C, d);
  if (d == 128) return kmeans_d<128>(xb, BH, N, C, iters, cent, label, counts, perm, w, err, stream);
  if (d == 64) return kmeans_d<64>(xb, BH, N, C, iters, cent, label, counts, perm, w, err, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_semantic_mask(const float* cent_q, const int32_t* counts_q, const int32_t* label_q,
                                 const int32_t* perm_q, int Cq, const float* cent_k, const int32_t* counts_k,
                                 const int32_t* label_k, const int32_t* perm_k, int Ck, int BH, int N, int d,
                                 int block, double scale, double top_p, uint32_t* keep, uint32_t* bits,
                                 int32_t* kv_idx, int32_t* kv_cnt, int max_kv, void* ws, int* err,
                                 cudaStream_t stream) {
  const int nblk = (N + block - 1) / block;
  int n2 = 1;
  while (n2 < Ck) n2 <<= 1;
  const size_t ksmem = static_cast<size_t>(n2) * (sizeof(double) + sizeof(int));
  semantic_keep_kernel<<<dim3(Cq, BH), kKeepThreads, ksmem, stream>>>(cent_q, counts_q, Cq, cent_k, counts_k, Ck,
                                                                      d, scale, top_p, n2, keep);
  int2* qr = static_cast<int2*>(ws);
  int2* kr = qr + static_cast<size_t>(BH) * nblk;
  const dim3 rgrid((nblk + 127) / 128, BH);
  block_cluster_range_kernel<<<rgrid, 128, 0, stream>>>(label_q, perm_q, N, block, nblk, Cq, qr, err);
  block_cluster_range_kernel<<<rgrid, 128, 0, stream>>>(label_k, perm_k, N, block, nblk, Ck, kr, err);
  semantic_block_mask_kernel<<<dim3(nblk, BH), 32, 0, stream>>>(qr, kr, counts_q, Cq, counts_k, Ck, keep, nblk, bits,
                                                                kv_idx, kv_cnt, max_kv, err);
  return cudaGetLastError();
}

size_t semantic_mask_workspace_bytes(int BH, int N, int block) {
  const size_t nblk = (static_cast<size_t>(N) + block - 1) / block;
  return 2 * static_cast<size_t>(BH) * nblk * sizeof(int2);
}

cudaError_t launch_gather_rows(const void* src, const int32_t* perm, void* dst, int BH, int N, int d, int* err,
                               cudaStream_t stream) {
  const int vpr = d * 2 / 16;
  gather_rows_kernel<<<dim3(rows_grid_x(N, vpr, BH), BH), kRowThreads, 0, stream>>>(
      static_cast<const uint4*>(src), perm, static_cast<uint4*>(dst), N, vpr, err);
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const void* src, const float* src_lse, const int32_t* perm, void* dst, float* dst_lse,
                                int BH, int N, int d, int* err, cudaStream_t stream) {
  const int vpr = d * 2 / 16;
  scatter_rows_kernel<<<dim3(rows_grid_x(N, vpr, BH), BH), kRowThreads, 0, stream>>>(
      static_cast<const uint4*>(src), src_lse, perm, static_cast<uint4*>(dst), dst_lse, N, vpr, err);
  return cudaGetLastError();
}

}  // namespace vsa
