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

// One CTA per (cube, head); thread x owns dimensions 2x, 2x+1 (+128 per pass).
__global__ void __launch_bounds__(kPoolThreads) cube_pool_kernel(const __nv_bfloat16* __restrict__ qc,
                                                                 const __nv_bfloat16* __restrict__ kc,
                                                                 const uint8_t* __restrict__ kinds, Geom g, int d,
                                                                 double* __restrict__ qbar,
                                                                 double* __restrict__ kbar) {
  const int cube = blockIdx.x, bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int count = cube_tokens(g, cube);
  const size_t base = (static_cast<size_t>(bh) * g.R + static_cast<size_t>(cube) * g.vol) * d;
  const size_t out = (static_cast<size_t>(bh) * g.ncubes + cube) * d;
  for (int x = threadIdx.x * 2; x < d; x += kPoolThreads * 2) {
    double sq0 = 0.0, sq1 = 0.0, sk0 = 0.0, sk1 = 0.0;
    for (int r = 0; r < g.vol; ++r) {
      if (token_of_slot(g, kCube, cube * g.vol + r) < 0) continue;
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(qc + base + static_cast<size_t>(r) * d + x);
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(kc + base + static_cast<size_t>(r) * d + x);
      sq0 = __dadd_rn(sq0, static_cast<double>(__low2float(a)));
      sq1 = __dadd_rn(sq1, static_cast<double>(__high2float(a)));
      sk0 = __dadd_rn(sk0, static_cast<double>(__low2float(b)));
      sk1 = __dadd_rn(sk1, static_cast<double>(__high2float(b)));
    }
    const double n = static_cast<double>(count);
    qbar[out + x] = __ddiv_rn(sq0, n);
    qbar[out + x + 1] = __ddiv_rn(sq1, n);
    kbar[out + x] = __ddiv_rn(sk0, n);
    kbar[out + x + 1] = __ddiv_rn(sk1, n);
  }
}

constexpr int kTopkRows = 8;       // query cubes per CTA (one warp each for the selection)
constexpr int kTopkChunk = 32;     // key cubes staged per pass
constexpr int kTopkThreads = 256;  // kTopkRows * 32

static size_t topk_smem_bytes(int C, int d, int nwords) {
  return sizeof(double) * (static_cast<size_t>(kTopkRows) * C + static_cast<size_t>(kTopkRows) * d +
                           static_cast<size_t>(kTopkChunk) * (d + 1)) +
         sizeof(uint32_t) * static_cast<size_t>(kTopkRows) * nwords;
}

__global__ void __launch_bounds__(kTopkThreads) cube_topk_kernel(const double* __restrict__ qbar,
                                                                 const double* __restrict__ kbar,
                                                                 const uint8_t* __restrict__ kinds, Geom g, int d,
                                                                 int topk, uint32_t* __restrict__ bits,
                                                                 int32_t* __restrict__ kv_idx,
                                                                 int32_t* __restrict__ kv_cnt, int max_kv, int* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int C = g.ncubes;
  const int nwords = (g.nblk + 31) >> 5;
  const int row0 = blockIdx.x * kTopkRows;
  double* sc = reinterpret_cast<double*>(smem_raw);  // [kTopkRows][C]
  double* qs = sc + static_cast<size_t>(kTopkRows) * C;  // [kTopkRows][d]
  double* ks = qs + static_cast<size_t>(kTopkRows) * d;  // [kTopkChunk][d + 1]
  uint32_t* sel = reinterpret_cast<uint32_t*>(ks + static_cast<size_t>(kTopkChunk) * (d + 1));  // [rows][nwords]
  const int tid = threadIdx.x;
  for (int x = tid; x < kTopkRows * d; x += kTopkThreads) {
    const int r = x / d, c = x - r * d;
    qs[x] = row0 + r < C ? qbar[(static_cast<size_t>(bh) * C + row0 + r) * d + c] : 0.0;
  }
  for (int x = tid; x < kTopkRows * nwords; x += kTopkThreads) sel[x] = 0u;
  const int r = tid >> 5, lane = tid & 31;
  for (int c0 = 0; c0 < C; c0 += kTopkChunk) {
    __syncthreads();
    for (int x = tid; x < kTopkChunk * d; x += kTopkThreads) {
      const int c = x / d, e = x - c * d;
      ks[c * (d + 1) + e] = c0 + c < C ? kbar[(static_cast<size_t>(bh) * C + c0 + c) * d + e] : 0.0;
    }
    __syncthreads();
    if (c0 + lane < C) {
      double acc = 0.0;
      for (int e = 0; e < d; ++e) acc = __dadd_rn(acc, __dmul_rn(qs[r * d + e], ks[lane * (d + 1) + e]));
      sc[static_cast<size_t>(r) * C + c0 + lane] = acc;
    }
  }
  __syncthreads();
  const int row = row0 + r;
  if (row >= C) return;
  const double* srow = sc + static_cast<size_t>(r) * C;
  uint32_t* srow_sel = sel + r * nwords;
  const int picks = topk < C ? topk : C;
  for (int p = 0; p < picks; ++p) {
    double best = -DBL_MAX;
    int best_c = 0x7fffffff;
    for (int c = lane; c < C; c += 32) {
      if ((srow_sel[c >> 5] >> (c & 31)) & 1u) continue;
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
    if (lane == 0 && best_c < C) srow_sel[best_c >> 5] |= 1u << (best_c & 31);
    __syncwarp();
  }
  if (lane == 0) srow_sel[row >> 5] |= 1u << (row & 31);
  __syncwarp();
  const size_t orow = static_cast<size_t>(bh) * g.nblk + row;
  for (int x = lane; x < nwords; x += 32) bits[orow * nwords + x] = srow_sel[x];
  if (lane == 0) {
    int n = 0;
    int32_t* irow = kv_idx + orow * max_kv;
    for (int wd = 0; wd < nwords; ++wd) {
      uint32_t m = srow_sel[wd];
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1u;
        if (n < max_kv) irow[n] = wd * 32 + b;
        ++n;
      }
    }
    for (int x = n; x < max_kv; ++x) irow[x] = -1;
    kv_cnt[orow] = n;
    if (n > max_kv) atomicOr(err, kDevErrOverflow);
  }
}

size_t cube_mask_workspace_bytes(const Geom& g, int BH, int d) {
  return 2 * sizeof(double) * static_cast<size_t>(BH) * g.ncubes * d;
}

cudaError_t launch_cube_mask(const uint8_t* kinds, const void* q_cube, const void* k_cube, const Geom& g, int BH, int d,
                             int topk, uint32_t* bits, int32_t* kv_idx, int32_t* kv_cnt, int max_kv, void* ws,
                             int* err, cudaStream_t stream) {
  double* qbar = static_cast<double*>(ws);
  double* kbar = qbar + static_cast<size_t>(BH) * g.ncubes * d;
  cube_pool_kernel<<<dim3(g.ncubes, BH), kPoolThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(q_cube),
                                                                     static_cast<const __nv_bfloat16*>(k_cube), kinds,
                                                                     g, d, qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nwords = (g.nblk + 31) >> 5;
  const size_t smem = topk_smem_bytes(g.ncubes, d, nwords);
  e = cudaFuncSetAttribute(cube_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cube_topk_kernel<<<dim3((g.ncubes + kTopkRows - 1) / kTopkRows, BH), kTopkThreads, smem, stream>>>(
      qbar, kbar, kinds, g, d, topk, bits, kv_idx, kv_cnt, max_kv, err);
  return cudaGetLastError();
}

size_t cube_topk_smem_bytes(const Geom& g, int d) { return topk_smem_bytes(g.ncubes, d, (g.nblk + 31) >> 5); }

}  // namespace vsa
