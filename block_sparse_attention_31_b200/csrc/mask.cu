// mask.cu -- block-mask builder (vsa_build_mask).
//
// Pattern heads ("Sparse Video-Gen" summary page, "Approach" and "Limitations"): a spatial
// head keeps key blocks whose frame interval is within w_s frames of the query block's
// (natural order, S tokens per frame); a temporal head keeps key blocks whose position
// interval is within w_t positions (frame-major order, F slots per position).  Block i
// spans slots [i*B, min(N,(i+1)*B)-1] and covers groups [first/G, last/G].
//
// Cube heads ("USV" page, Figure 2: top-k cube selection on coarse attention): every cube
// is pooled to the fp64 mean of its real tokens' Q and K; the coarse score of (c, c') is
// their dot product; each query cube keeps itself plus the top-k key cubes by score
// (ties to the smaller index).  The pooled sums are accumulated in slot order and the dot
// products in dimension order with separately rounded multiply and add, so the scores are
// reproducible to the last bit.
//
// Every mask row is written three ways: a bitset, an ascending index list padded with -1,
// and a count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

constexpr int kMaskThreads = 256;

__global__ void __launch_bounds__(kMaskThreads) pattern_mask_kernel(const uint8_t* __restrict__ kinds, Geom g, int BH,
                                                                    int w_s, int w_t, uint32_t* __restrict__ bits,
                                                                    int32_t* __restrict__ kv_idx,
                                                                    int32_t* __restrict__ kv_cnt, int max_kv,
                                                                    int* err) {
  const int warp = (blockIdx.x * kMaskThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= BH * g.nblk) return;
  const int bh = warp / g.nblk, i = warp - bh * g.nblk;
  const int kind = kinds[bh];
  if (kind == kCube && g.ncubes > 0) return;  // written by the cube kernels
  const int nwords = (g.nblk + 31) >> 5;
  const size_t row = static_cast<size_t>(bh) * g.nblk + i;
  uint32_t* brow = bits + row * nwords;
  int32_t* irow = kv_idx + row * max_kv;
  const int nb = (g.N + g.block - 1) / g.block;
  if (kind >= kCube || i >= nb) {
    if (kind >= kCube && lane == 0 && i == 0) atomicOr(err, kDevErrKind);
    for (int x = lane; x < nwords; x += 32) brow[x] = 0u;
    for (int x = lane; x < max_kv; x += 32) irow[x] = -1;
    if (lane == 0) kv_cnt[row] = 0;
    return;
  }
  const int G = kind == kSpatial ? g.S : g.F;
  const int w = kind == kSpatial ? w_s : w_t;
  const int ai = (i * g.block) / G;
  const int bi = (min(g.N, (i + 1) * g.block) - 1) / G;
  int count = 0;
  for (int wd = 0; wd < nwords; ++wd) {
    const int j = wd * 32 + lane;
    bool keep = false;
    if (j < nb) {
      const int aj = (j * g.block) / G;
      const int bj = (min(g.N, (j + 1) * g.block) - 1) / G;
      keep = max(0, max(aj - bi, ai - bj)) <= w;
    }
    const uint32_t ball = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) brow[wd] = ball;
    const int pos = count + __popc(ball & ((1u << lane) - 1u));
    if (keep && pos < max_kv) irow[pos] = j;
    count += __popc(ball);
  }
  for (int x = count + lane; x < max_kv; x += 32) irow[x] = -1;
  if (lane == 0) {
    kv_cnt[row] = count;
    if (count > max_kv) atomicOr(err, kDevErrOverflow);
  }
}

cudaError_t launch_pattern_mask(const uint8_t* kinds, const Geom& g, int BH, int w_s, int w_t, uint32_t* bits,
                                int32_t* kv_idx, int32_t* kv_cnt, int max_kv, int* err, cudaStream_t stream) {
  const long long warps = static_cast<long long>(BH) * g.nblk;
  const int grid = static_cast<int>((warps * 32 + kMaskThreads - 1) / kMaskThreads);
  pattern_mask_kernel<<<grid, kMaskThreads, 0, stream>>>(kinds, g, BH, w_s, w_t, bits, kv_idx, kv_cnt, max_kv, err);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Cube heads
// ---------------------------------------------------------------------------------------
constexpr int kPoolThreads = 64;

// One CTA per (cube, head); thread x owns dimensions 2x, 2x+1 (+128 per pass).  The sums run
// over the cube's real tokens in slot order, i.e. increasing natural token index.
__global__ void __launch_bounds__(kPoolThreads) cube_pool_kernel(const __nv_bfloat16* __restrict__ qc,
                                                                 const __nv_bfloat16* __restrict__ kc,
                                                                 const uint8_t* __restrict__ kinds, Geom g, int d,
                                                                 double* __restrict__ qbar,
                                                                 double* __restrict__ kbar) {
  const int cube = blockIdx.x, bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int cw_i = cube % g.ncw, ch_i = (cube / g.ncw) % g.nch, cf_i = cube / (g.ncw * g.nch);
  const int nf = min(g.cf, g.F - cf_i * g.cf), nh = min(g.ch, g.Hl - ch_i * g.ch), nw = min(g.cw, g.Wl - cw_i * g.cw);
  const double n = static_cast<double>(nf * nh * nw);
  const size_t base = (static_cast<size_t>(bh) * g.R + static_cast<size_t>(cube) * g.vol) * d;
  const size_t out = (static_cast<size_t>(bh) * g.ncubes + cube) * d;
  for (int x = threadIdx.x * 2; x < d; x += kPoolThreads * 2) {
    double sq0 = 0.0, sq1 = 0.0, sk0 = 0.0, sk1 = 0.0;
    for (int df = 0; df < nf; ++df)
      for (int dh = 0; dh < nh; ++dh)
        for (int dw = 0; dw < nw; ++dw) {
          const size_t r = static_cast<size_t>((df * g.ch + dh) * g.cw + dw);
          const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(qc + base + r * d + x);
          const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(kc + base + r * d + x);
          sq0 = __dadd_rn(sq0, static_cast<double>(__low2float(a)));
          sq1 = __dadd_rn(sq1, static_cast<double>(__high2float(a)));
          sk0 = __dadd_rn(sk0, static_cast<double>(__low2float(b)));
          sk1 = __dadd_rn(sk1, static_cast<double>(__high2float(b)));
        }
    qbar[out + x] = __ddiv_rn(sq0, n);
    qbar[out + x + 1] = __ddiv_rn(sq1, n);
    kbar[out + x] = __ddiv_rn(sk0, n);
    kbar[out + x + 1] = __ddiv_rn(sk1, n);
  }
}

// Coarse scores S[c][c'] = qbar_c . kbar_c' of one head: 64 x 64 outputs per CTA, 4 x 4 per
// thread (rows ty + 16i, columns tx + 16j), dimensions staged 32 at a time in shared memory
// (transposed, so a warp's column reads are consecutive).  Every output accumulates its
// products in dimension order with separately rounded multiply and add.
constexpr int kScoreTile = 64, kScoreK = 32;

__global__ void __launch_bounds__(256) cube_score_kernel(const double* __restrict__ qbar,
                                                         const double* __restrict__ kbar,
                                                         const uint8_t* __restrict__ kinds, int C, int d,
                                                         double* __restrict__ scores) {
  __shared__ double sq[kScoreK][kScoreTile + 1];
  __shared__ double sk[kScoreK][kScoreTile + 1];
  const int bh = blockIdx.z;
  if (kinds[bh] != kCube) return;
  const int r0 = blockIdx.y * kScoreTile, c0 = blockIdx.x * kScoreTile;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const double* qh = qbar + static_cast<size_t>(bh) * C * d;
  const double* kh = kbar + static_cast<size_t>(bh) * C * d;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int e0 = 0; e0 < d; e0 += kScoreK) {
    __syncthreads();
    for (int x = tid; x < kScoreTile * kScoreK; x += 256) {
      const int r = x / kScoreK, e = x - r * kScoreK;
      sq[e][r] = r0 + r < C ? qh[static_cast<size_t>(r0 + r) * d + e0 + e] : 0.0;
      sk[e][r] = c0 + r < C ? kh[static_cast<size_t>(c0 + r) * d + e0 + e] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int e = 0; e < kScoreK; ++e) {
      double a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sq[e][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sk[e][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __dadd_rn(acc[i][j], __dmul_rn(a[i], b[j]));
    }
  }
  double* sh = scores + static_cast<size_t>(bh) * C * C;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty + 16 * i;
    if (r >= C) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + tx + 16 * j;
      if (c < C) sh[static_cast<size_t>(r) * C + c] = acc[i][j];
    }
  }
}

// Top-k of one score row per warp (score descending, ties to the smaller index) plus the own
// cube; emits the bitset, the ascending list and the count.
constexpr int kTopkWarps = 4;

__global__ void __launch_bounds__(kTopkWarps * 32) cube_topk_kernel(const double* __restrict__ scores,
                                                                    const uint8_t* __restrict__ kinds, Geom g,
                                                                    int topk, uint32_t* __restrict__ bits,
                                                                    int32_t* __restrict__ kv_idx,
                                                                    int32_t* __restrict__ kv_cnt, int max_kv,
                                                                    int* err) {
  extern __shared__ __align__(16) uint8_t topk_smem[];  // [kTopkWarps][C] doubles, then [kTopkWarps][nwords]
  const int bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int C = g.ncubes;
  const int nwords = (g.nblk + 31) >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kTopkWarps + warp;
  double* srow = reinterpret_cast<double*>(topk_smem) + static_cast<size_t>(warp) * C;
  uint32_t* sel = reinterpret_cast<uint32_t*>(reinterpret_cast<double*>(topk_smem) + static_cast<size_t>(kTopkWarps) * C) +
                  warp * nwords;
  for (int x = lane; x < nwords; x += 32) sel[x] = 0u;
  if (row >= C) return;
  const double* grow = scores + (static_cast<size_t>(bh) * C + row) * C;
  for (int c = lane; c < C; c += 32) srow[c] = __ldg(grow + c);
  __syncwarp();
  const int picks = topk < C ? topk : C;
  for (int p = 0; p < picks; ++p) {
    double best = -DBL_MAX;
    int best_c = 0x7fffffff;
    for (int c = lane; c < C; c += 32) {
      if ((sel[c >> 5] >> (c & 31)) & 1u) continue;
      const double s = srow[c];
      if (s > best || (s == best && c < best_c)) {
        best = s;
        best_c = c;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oc = __shfl_xor_sync(0xffffffffu, best_c, off);
      if (ob > best || (ob == best && oc < best_c)) {
        best = ob;
        best_c = oc;
      }
    }
    if (lane == 0 && best_c < C) sel[best_c >> 5] |= 1u << (best_c & 31);
    __syncwarp();
  }
  if (lane == 0) sel[row >> 5] |= 1u << (row & 31);
  __syncwarp();
  const size_t orow = static_cast<size_t>(bh) * g.nblk + row;
  for (int x = lane; x < nwords; x += 32) bits[orow * nwords + x] = sel[x];
  // ascending list: per word prefix counts across the warp
  int32_t* irow = kv_idx + orow * max_kv;
  int base = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32) {
    const int w = w0 + lane;
    uint32_t m = w < nwords ? sel[w] : 0u;
    const int c = __popc(m);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += n;
    }
    int pos = base + incl - c;
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1u;
      if (pos < max_kv) irow[pos] = w * 32 + b;
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int x = base + lane; x < max_kv; x += 32) irow[x] = -1;
  if (lane == 0) {
    kv_cnt[orow] = base;
    if (base > max_kv) atomicOr(err, kDevErrOverflow);
  }
}

// Work order for the attention kernel, per head: the query blocks sorted by (smallest kept key
// block, block index); rows of a head past its own block count, then empty rows, go last.
// Consecutive entries then share most key blocks (neighbouring windows for pattern heads,
// the same cube slab or position for cube heads), which the attention kernel turns into
// shared K/V loads within a CTA and L2 reuse across concurrently running CTAs.
constexpr int kOrderThreads = 1024;

__global__ void __launch_bounds__(kOrderThreads) block_order_kernel(const uint8_t* __restrict__ kinds, Geom g,
                                                                    const int32_t* __restrict__ kv_idx,
                                                                    const int32_t* __restrict__ kv_cnt, int max_kv,
                                                                    int n2, int32_t* __restrict__ order) {
  extern __shared__ uint32_t keys[];  // n2 = next power of two >= nblk
  const int bh = blockIdx.x;
  const int kind = kinds[bh];
  const int rows = kind <= kCube ? layout_rows(g, kind) : 0;
  const int nb_head = (rows + g.block - 1) / g.block;
  for (int i = threadIdx.x; i < n2; i += kOrderThreads) {
    uint32_t key = 0xffffffffu;
    if (i < g.nblk) {
      const size_t row = static_cast<size_t>(bh) * g.nblk + i;
      const int cnt = kv_cnt[row];
      uint32_t hi;
      if (i >= nb_head) hi = 0xffffu;
      else if (cnt <= 0) hi = 0xfffeu;
      else hi = min(static_cast<uint32_t>(kv_idx[row * max_kv]), 0xfffdu);
      key = (hi << 16) | static_cast<uint32_t>(i);
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += kOrderThreads) {
        const int p = i ^ j;
        if (p > i) {
          const uint32_t a = keys[i], b = keys[p];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            keys[i] = b;
            keys[p] = a;
          }
        }
      }
      __syncthreads();
    }
  for (int i = threadIdx.x; i < g.nblk; i += kOrderThreads)
    order[static_cast<size_t>(bh) * g.nblk + i] = static_cast<int32_t>(keys[i] & 0xffffu);
}

cudaError_t launch_block_order(const uint8_t* kinds, const Geom& g, int BH, const int32_t* kv_idx,
                               const int32_t* kv_cnt, int max_kv, int32_t* order, cudaStream_t stream) {
  if (g.nblk > 0xffff) return cudaErrorInvalidValue;
  int n2 = 1;
  while (n2 < g.nblk) n2 <<= 1;
  const size_t smem = sizeof(uint32_t) * n2;
  if (smem > 232448) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e =
        cudaFuncSetAttribute(block_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  block_order_kernel<<<BH, kOrderThreads, smem, stream>>>(kinds, g, kv_idx, kv_cnt, max_kv, n2, order);
  return cudaGetLastError();
}

size_t cube_mask_workspace_bytes(const Geom& g, int BH, int d) {
  return sizeof(double) * (2 * static_cast<size_t>(BH) * g.ncubes * d +
                           static_cast<size_t>(BH) * g.ncubes * g.ncubes);
}

cudaError_t launch_cube_mask(const uint8_t* kinds, const void* q_cube, const void* k_cube, const Geom& g, int BH, int d,
                             int topk, uint32_t* bits, int32_t* kv_idx, int32_t* kv_cnt, int max_kv, void* ws,
                             int* err, cudaStream_t stream) {
  const int C = g.ncubes;
  double* qbar = static_cast<double*>(ws);
  double* kbar = qbar + static_cast<size_t>(BH) * C * d;
  double* scores = kbar + static_cast<size_t>(BH) * C * d;
  cube_pool_kernel<<<dim3(C, BH), kPoolThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(q_cube),
                                                              static_cast<const __nv_bfloat16*>(k_cube), kinds, g, d,
                                                              qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nt = (C + kScoreTile - 1) / kScoreTile;
  cube_score_kernel<<<dim3(nt, nt, BH), 256, 0, stream>>>(qbar, kbar, kinds, C, d, scores);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nwords = (g.nblk + 31) >> 5;
  const size_t smem = sizeof(double) * kTopkWarps * C + sizeof(uint32_t) * kTopkWarps * nwords;
  if (smem > 232448) return cudaErrorInvalidConfiguration;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(cube_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  cube_topk_kernel<<<dim3((C + kTopkWarps - 1) / kTopkWarps, BH), kTopkWarps * 32, smem, stream>>>(
      scores, kinds, g, topk, bits, kv_idx, kv_cnt, max_kv, err);
  return cudaGetLastError();
}

}  // namespace vsa
