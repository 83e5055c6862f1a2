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
// (ties to the smaller index).  The pooled sums are accumulated in slot order with one
// rounded add per token and the dot products in dimension order with one fused multiply-add
// per term, so the scores are reproducible to the last bit.
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
// Exact widening of a bf16 bit pattern to double.  Normal numbers are rebuilt with integer
// operations (exponent rebias 127 -> 1023, mantissa moved to the top of the 52-bit field);
// zero, subnormals, infinities and NaN take the float path.  Both are exact.
__device__ __forceinline__ double bf16_bits_to_double(uint32_t x) {
  const uint32_t e = x & 0x7F80u;
  if (e != 0u && e != 0x7F80u)
    return __hiloint2double(static_cast<int>(((x & 0x8000u) << 16) | (((x & 0x7FFFu) << 13) + (896u << 20))), 0);
  return static_cast<double>(__uint_as_float(x << 16));
}

constexpr int kPoolWarps = 4;  // one cube per warp
constexpr int kPoolBatch = 8;  // rows loaded ahead of the sequential adds

// Pooled means of one cube per warp: lanes 0-15 own Q, lanes 16-31 own K, each lane eight
// consecutive dimensions (one 16-byte load per row).  Per dimension the sum runs over the
// cube's real tokens in slot order, i.e. increasing natural token index, one rounded add per
// token; kPoolBatch rows are loaded before they are added so that the loads overlap.
__global__ void __launch_bounds__(kPoolWarps * 32) cube_pool_kernel(const __nv_bfloat16* __restrict__ qc,
                                                                   const __nv_bfloat16* __restrict__ kc,
                                                                   const uint8_t* __restrict__ kinds, Geom g, int d,
                                                                   double* __restrict__ qbar,
                                                                   double* __restrict__ kbar) {
  const int bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int lane = threadIdx.x & 31;
  const int cube = blockIdx.x * kPoolWarps + (threadIdx.x >> 5);
  const int x = (lane & 15) * 8;  // first dimension of this lane
  if (cube >= g.ncubes || x >= d) return;
  const __nv_bfloat16* src = lane < 16 ? qc : kc;
  double* dst = lane < 16 ? qbar : kbar;
  const int cw_i = cube % g.ncw, ch_i = (cube / g.ncw) % g.nch, cf_i = cube / (g.ncw * g.nch);
  const int nf = min(g.cf, g.F - cf_i * g.cf), nh = min(g.ch, g.Hl - ch_i * g.ch), nw = min(g.cw, g.Wl - cw_i * g.cw);
  const int cnt = nf * nh * nw;
  const bool full = cnt == g.vol;
  const __nv_bfloat16* base = src + (static_cast<size_t>(bh) * g.R + static_cast<size_t>(cube) * g.vol) * d + x;
  double acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0;
  for (int i0 = 0; i0 < cnt; i0 += kPoolBatch) {
    uint4 buf[kPoolBatch];
#pragma unroll
    for (int u = 0; u < kPoolBatch; ++u) {
      const int i = i0 + u;
      if (i < cnt) {
        int slot = i;
        if (!full) {  // token i of the cube's nf x nh x nw real tokens -> slot (df*ch + dh)*cw + dw
          const int dw = i % nw, t = i / nw;
          slot = ((t / nh) * g.ch + t % nh) * g.cw + dw;
        }
        buf[u] = *reinterpret_cast<const uint4*>(base + static_cast<size_t>(slot) * d);
      }
    }
#pragma unroll
    for (int u = 0; u < kPoolBatch; ++u) {
      if (i0 + u < cnt) {
        const uint32_t w[4] = {buf[u].x, buf[u].y, buf[u].z, buf[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] = __dadd_rn(acc[2 * j], bf16_bits_to_double(w[j] & 0xFFFFu));
          acc[2 * j + 1] = __dadd_rn(acc[2 * j + 1], bf16_bits_to_double(w[j] >> 16));
        }
      }
    }
  }
  const double n = static_cast<double>(cnt);
  double* out = dst + (static_cast<size_t>(bh) * g.ncubes + cube) * d + x;
#pragma unroll
  for (int j = 0; j < 8; ++j) out[j] = __ddiv_rn(acc[j], n);
}

// Coarse scores S[c][c'] = qbar_c . kbar_c' of one head: 128 x 128 outputs per CTA, 8 x 8
// per thread (rows ty + 16i, columns tx + 16j), dimensions staged 16 at a time in shared
// memory (transposed, so a warp's column reads are consecutive).  Every output accumulates
// its products in dimension order, one fused multiply-add per term.  Eight outputs per
// operand load keep the FP64 pipe, not shared memory, the limit.
constexpr int kScoreTile = 128, kScoreK = 16, kScoreThreads = 256;

__global__ void __launch_bounds__(kScoreThreads, 1) cube_score_kernel(const double* __restrict__ qbar,
                                                                      const double* __restrict__ kbar,
                                                                      const uint8_t* __restrict__ kinds, int C,
                                                                      int d, double* __restrict__ scores) {
  __shared__ double sq[kScoreK][kScoreTile + 1];
  __shared__ double sk[kScoreK][kScoreTile + 1];
  const int bh = blockIdx.z;
  if (kinds[bh] != kCube) return;
  const int r0 = blockIdx.y * kScoreTile, c0 = blockIdx.x * kScoreTile;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const double* qh = qbar + static_cast<size_t>(bh) * C * d;
  const double* kh = kbar + static_cast<size_t>(bh) * C * d;
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  for (int e0 = 0; e0 < d; e0 += kScoreK) {
    __syncthreads();
#pragma unroll
    for (int it = 0; it < kScoreTile * kScoreK / kScoreThreads; ++it) {
      const int x = tid + it * kScoreThreads;
      const int r = x / kScoreK, e = x % kScoreK;
      sq[e][r] = r0 + r < C ? qh[static_cast<size_t>(r0 + r) * d + e0 + e] : 0.0;
      sk[e][r] = c0 + r < C ? kh[static_cast<size_t>(c0 + r) * d + e0 + e] : 0.0;
    }
    __syncthreads();
#pragma unroll 2
    for (int e = 0; e < kScoreK; ++e) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = sq[e][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = sk[e][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = __fma_rn(a[i], b[j], acc[i][j]);
    }
  }
  double* sh = scores + static_cast<size_t>(bh) * C * C;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + ty + 16 * i;
    if (r >= C) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = c0 + tx + 16 * j;
      if (c < C) sh[static_cast<size_t>(r) * C + c] = acc[i][j];
    }
  }
}

constexpr int kTopkWarps = 4;
constexpr int kTopkCap = 512;  // candidates per row kept for the exact selection
constexpr int kLaneTop = 8;    // largest keys each lane keeps for the candidate bound

// Order-preserving integer key of a finite double (larger value <-> larger key); -0 and +0,
// equal as doubles, get the same key.
__device__ __forceinline__ uint64_t score_key(double s) {
  uint64_t b = static_cast<uint64_t>(__double_as_longlong(s));
  if (b == 0x8000000000000000ull) b = 0ull;
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Warp-wide maximum of (key desc, index asc) pairs; every lane gets the winning index.
__device__ __forceinline__ int warp_argmax_key(uint64_t k, int c) {
  const uint32_t hi = static_cast<uint32_t>(k >> 32), lo = static_cast<uint32_t>(k);
  const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
  const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
  const bool top = hi == mhi && lo == mlo;
  return static_cast<int>(__reduce_min_sync(0xffffffffu, top ? static_cast<uint32_t>(c) : 0x7fffffffu));
}

// Top-k of one score row per warp (score descending, ties to the smaller index) plus the own
// cube; emits the bitset, the ascending list and the count.
//
// Fast path (topk <= 32): every lane keeps its kLaneTop largest keys; the k-th largest of those
// 32*kLaneTop keys is a lower bound L on the row's k-th largest score, since k distinct entries
// are >= L.  Only entries >= L (about k, unless a lane held more than kLaneTop of the winners)
// are gathered, and the exact selection runs on them.  With more than kTopkCap candidates, or
// topk > 32, every round scans the whole row.
__global__ void __launch_bounds__(kTopkWarps * 32, 1) cube_topk_kernel(const double* __restrict__ scores,
                                                                    const uint8_t* __restrict__ kinds, Geom g,
                                                                    int topk, uint32_t* __restrict__ bits,
                                                                    int32_t* __restrict__ kv_idx,
                                                                    int32_t* __restrict__ kv_cnt, int max_kv,
                                                                    int* err) {
  // per warp: kTopkCap keys, kTopkCap indices, nwords selection words
  extern __shared__ __align__(16) uint8_t topk_smem[];
  const int bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int C = g.ncubes;
  const int nwords = (g.nblk + 31) >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kTopkWarps + warp;
  uint64_t* ck = reinterpret_cast<uint64_t*>(topk_smem) + static_cast<size_t>(warp) * kTopkCap;
  int* ci = reinterpret_cast<int*>(reinterpret_cast<uint64_t*>(topk_smem) + kTopkWarps * kTopkCap) + warp * kTopkCap;
  uint32_t* sel = reinterpret_cast<uint32_t*>(reinterpret_cast<int*>(reinterpret_cast<uint64_t*>(topk_smem) +
                                                                     kTopkWarps * kTopkCap) +
                                              kTopkWarps * kTopkCap) +
                  warp * nwords;
  for (int x = lane; x < nwords; x += 32) sel[x] = 0u;
  if (row >= C) return;
  const double* grow = scores + (static_cast<size_t>(bh) * C + row) * C;
  const int picks = topk < C ? topk : C;
  bool exact_scan = picks > 32;
  if (!exact_scan && picks > 0) {
    // each lane's kLaneTop largest keys, descending (0: empty, below every finite key)
    uint64_t tk[kLaneTop];
#pragma unroll
    for (int j = 0; j < kLaneTop; ++j) tk[j] = 0ull;
    for (int c = lane; c < C; c += 32) {
      const uint64_t k = score_key(__ldg(grow + c));
      if (k > tk[kLaneTop - 1]) {
#pragma unroll
        for (int j = kLaneTop - 1; j > 0; --j) tk[j] = max(tk[j], min(k, tk[j - 1]));
        tk[0] = max(tk[0], k);
      }
    }
    // the picks-th largest key of all lanes' lists: picks real entries are >= it, so it bounds
    // the picks-th largest score of the row from below
    uint64_t bound = 0ull;
    for (int p = 0; p < picks; ++p) {
      const uint32_t hi = static_cast<uint32_t>(tk[0] >> 32), lo = static_cast<uint32_t>(tk[0]);
      const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
      const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
      bound = (static_cast<uint64_t>(mhi) << 32) | mlo;
      const uint32_t holders = __ballot_sync(0xffffffffu, tk[0] == bound);
      if (lane == __ffs(holders) - 1) {  // that lane's head is taken
#pragma unroll
        for (int j = 0; j < kLaneTop - 1; ++j) tk[j] = tk[j + 1];
        tk[kLaneTop - 1] = 0ull;
      }
    }
    int n = 0;
    for (int c0 = 0; c0 < C; c0 += 32) {
      const int c = c0 + lane;
      const uint64_t k = c < C ? score_key(__ldg(grow + c)) : 0ull;
      const bool cand = c < C && k >= bound;
      const uint32_t m = __ballot_sync(0xffffffffu, cand);
      const int pos = n + __popc(m & ((1u << lane) - 1u));
      if (cand && pos < kTopkCap) {
        ck[pos] = k;
        ci[pos] = c;
      }
      n += __popc(m);
    }
    __syncwarp();
    if (n > kTopkCap) {
      exact_scan = true;
    } else {
      // exact selection among the n candidates; lane owns slots lane + 32 m
      const int M = (n + 31) >> 5;  // <= kTopkCap / 32 = 16
      uint32_t taken = 0u;
      for (int p = 0; p < picks; ++p) {
        uint64_t bk = 0ull;
        int bc = 0x7fffffff, bm = -1;
        for (int m = 0; m < M; ++m) {
          const int x = lane + 32 * m;
          if (x >= n || ((taken >> m) & 1u)) continue;
          const uint64_t k = ck[x];
          const int c = ci[x];
          if (bm < 0 || k > bk || (k == bk && c < bc)) {
            bk = k;
            bc = c;
            bm = m;
          }
        }
        const int win = warp_argmax_key(bm < 0 ? 0ull : bk, bm < 0 ? 0x7fffffff : bc);
        if (bm >= 0 && bc == win) {
          taken |= 1u << bm;
          sel[win >> 5] |= 1u << (win & 31);
        }
        __syncwarp();
      }
    }
  }
  if (exact_scan) {  // every round scans the whole row (topk > 32 or too many candidates)
    for (int p = 0; p < picks; ++p) {
      double best = -DBL_MAX;
      int best_c = 0x7fffffff;
      for (int c = lane; c < C; c += 32) {
        if ((sel[c >> 5] >> (c & 31)) & 1u) continue;
        const double s = __ldg(grow + c);
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
  cube_pool_kernel<<<dim3((C + kPoolWarps - 1) / kPoolWarps, BH), kPoolWarps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q_cube), static_cast<const __nv_bfloat16*>(k_cube), kinds, g, d, qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nt = (C + kScoreTile - 1) / kScoreTile;
  cube_score_kernel<<<dim3(nt, nt, BH), kScoreThreads, 0, stream>>>(qbar, kbar, kinds, C, d, scores);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nwords = (g.nblk + 31) >> 5;
  const size_t smem = (sizeof(uint64_t) + sizeof(int)) * kTopkWarps * kTopkCap + sizeof(uint32_t) * kTopkWarps * nwords;
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
