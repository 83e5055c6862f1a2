// permute.cu -- layout gather (vsa_permute) and scatter (vsa_unpermute).
//
// "Sparse Video-Gen" summary page, "Approach": temporal heads attend to the same spatial
// position across frames; re-laying their tokens out frame-major (slot s*F + f) makes
// those keys contiguous so the attention kernel runs dense blocks on them.  "USV" page,
// Figure 2: cube heads use local 3D cubes, laid out cube by cube.
//
// Both kernels are HBM-bound row copies: each thread moves one 16-byte vector (8 bf16) of
// a row and every thread keeps four rows in flight.  Rows are 128 or 256 bytes, so each
// warp touches whole 128-byte lines.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

constexpr int kPermThreads = 256;
constexpr int kPermUnroll = 4;

__device__ __forceinline__ uint4 load8_as_bf16(const void* src, size_t elem_off, bool f32) {
  if (!f32) return __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + elem_off));
  const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + elem_off);
  const float4 a = __ldg(p), b = __ldg(p + 1);
  uint4 r;
  r.x = pack_bf16x2(a.x, a.y);
  r.y = pack_bf16x2(a.z, a.w);
  r.z = pack_bf16x2(b.x, b.y);
  r.w = pack_bf16x2(b.z, b.w);
  return r;
}

__device__ __forceinline__ void store8_from_bf16(void* dst, size_t elem_off, uint4 v, bool f32) {
  if (!f32) {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + elem_off) = v;
    return;
  }
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  float4* p = reinterpret_cast<float4*>(static_cast<float*>(dst) + elem_off);
  p[0] = make_float4(f[0], f[1], f[2], f[3]);
  p[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// dst[bh, slot] = bf16(src[bh, token_of_slot(slot)]), zero where the slot holds no token.
template <bool kSrcF32>
__global__ void __launch_bounds__(kPermThreads) permute_kernel(const void* __restrict__ src,
                                                               __nv_bfloat16* __restrict__ dst,
                                                               const uint8_t* __restrict__ kinds, Geom g, int d,
                                                               int* err) {
  const int bh = blockIdx.y;
  const int kind = kinds[bh];
  if (kind > kCube) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, kDevErrKind);
    return;
  }
  if (!kSrcF32 && kind == kSpatial) return;
  if (kind == kCube && g.ncubes > 0) return;  // cube_permute_kernel
  const int vpr = d / 8;  // 16-byte vectors per row
  const int rows_per_pass = kPermThreads / vpr;
  const int v = threadIdx.x % vpr;
  const int r0 = threadIdx.x / vpr;
  const size_t src_head = static_cast<size_t>(bh) * g.N * d;
  const size_t dst_head = static_cast<size_t>(bh) * g.R * d;
  const int stride = gridDim.x * rows_per_pass * kPermUnroll;
  for (int base = blockIdx.x * rows_per_pass * kPermUnroll; base < g.R; base += stride) {
    uint4 val[kPermUnroll];
    int slot[kPermUnroll];
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      slot[u] = base + u * rows_per_pass + r0;
      const int t = slot[u] < g.R ? token_of_slot(g, kind, slot[u]) : -1;
      val[u] = t >= 0 ? load8_as_bf16(src, src_head + static_cast<size_t>(t) * d + v * 8, kSrcF32)
                      : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u)
      if (slot[u] < g.R) *reinterpret_cast<uint4*>(dst + dst_head + static_cast<size_t>(slot[u]) * d + v * 8) = val[u];
  }
}

// dst[bh, t] = src[bh, slot_of_token(t)] (converted to the destination type); same for LSE.
template <bool kDstF32>
__global__ void __launch_bounds__(kPermThreads) unpermute_kernel(const __nv_bfloat16* __restrict__ src,
                                                                 const float* __restrict__ src_lse,
                                                                 void* __restrict__ dst, float* __restrict__ dst_lse,
                                                                 const uint8_t* __restrict__ kinds, Geom g, int d,
                                                                 int* err) {
  const int bh = blockIdx.y;
  const int kind = kinds[bh];
  if (kind > kCube) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, kDevErrKind);
    return;
  }
  if (!kDstF32 && kind == kSpatial) return;
  if (kind == kCube && g.ncubes > 0) return;  // cube_unpermute_kernel
  const int vpr = d / 8;
  const int rows_per_pass = kPermThreads / vpr;
  const int v = threadIdx.x % vpr;
  const int r0 = threadIdx.x / vpr;
  const size_t src_head = static_cast<size_t>(bh) * g.R * d;
  const size_t dst_head = static_cast<size_t>(bh) * g.N * d;
  const int stride = gridDim.x * rows_per_pass * kPermUnroll;
  for (int base = blockIdx.x * rows_per_pass * kPermUnroll; base < g.N; base += stride) {
    uint4 val[kPermUnroll];
    int tok[kPermUnroll], slot[kPermUnroll];
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      tok[u] = base + u * rows_per_pass + r0;
      slot[u] = tok[u] < g.N ? slot_of_token(g, kind, tok[u]) : 0;
      val[u] = tok[u] < g.N ? __ldg(reinterpret_cast<const uint4*>(src + src_head + static_cast<size_t>(slot[u]) * d +
                                                                   v * 8))
                            : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      if (tok[u] >= g.N) continue;
      store8_from_bf16(dst, dst_head + static_cast<size_t>(tok[u]) * d + v * 8, val[u], kDstF32);
      if (src_lse != nullptr && dst_lse != nullptr && v == 0)
        dst_lse[static_cast<size_t>(bh) * g.N + tok[u]] = src_lse[static_cast<size_t>(bh) * g.R + slot[u]];
    }
  }
}

// Cube heads: one warp per cube.  A lane keeps one 16-byte column v of the row and walks the
// cube's slots r = r_lane, r_lane + 32/vpr, ...; the slot's (df, dh, dw) offsets are advanced
// incrementally, so no division runs per row.  Consecutive slots of a cube line (fixed df, dh)
// are consecutive tokens, so every warp access is contiguous on both sides.
constexpr int kCubeWarps = 8;
constexpr int kCubeUnroll = 8;

struct CubeWalk {
  int dw, dh, df;
  __device__ __forceinline__ void init(const Geom& g, int r) {
    dw = r % g.cw;
    const int t = r / g.cw;
    dh = t % g.ch;
    df = t / g.ch;
  }
  __device__ __forceinline__ void advance(const Geom& g, int step) {
    dw += step;
    while (dw >= g.cw) {
      dw -= g.cw;
      if (++dh == g.ch) {
        dh = 0;
        ++df;
      }
    }
  }
};

// dst[bh, cube*vol + r] = bf16(src[bh, token of slot r of the cube]), zero for padding slots.
template <bool kSrcF32>
__global__ void __launch_bounds__(kCubeWarps * 32) cube_permute_kernel(const void* __restrict__ src,
                                                                      __nv_bfloat16* __restrict__ dst,
                                                                      const uint8_t* __restrict__ kinds, Geom g,
                                                                      int d) {
  const int bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int cube = blockIdx.x * kCubeWarps + (threadIdx.x >> 5);
  if (cube >= g.ncubes) return;
  const int lane = threadIdx.x & 31;
  const int vpr = d / 8, rstep = 32 / vpr;
  const int v = lane % vpr;
  const int cw_i = cube % g.ncw, ch_i = (cube / g.ncw) % g.nch, cf_i = cube / (g.ncw * g.nch);
  const int f0 = cf_i * g.cf, h0 = ch_i * g.ch, w0 = cw_i * g.cw;
  const size_t src_head = static_cast<size_t>(bh) * g.N * d + v * 8;
  const size_t dst_cube = (static_cast<size_t>(bh) * g.R + static_cast<size_t>(cube) * g.vol) * d + v * 8;
  const int r_lane = lane / vpr;
  CubeWalk c;
  c.init(g, r_lane);
  const int steps = g.vol / rstep;
  for (int k0 = 0; k0 < steps; k0 += kCubeUnroll) {
    uint4 val[kCubeUnroll];
#pragma unroll
    for (int u = 0; u < kCubeUnroll; ++u) {
      const int f = f0 + c.df, h = h0 + c.dh, w = w0 + c.dw;
      const bool ok = k0 + u < steps && f < g.F && h < g.Hl && w < g.Wl;
      val[u] = ok ? load8_as_bf16(src, src_head + static_cast<size_t>((f * g.Hl + h) * g.Wl + w) * d, kSrcF32)
                  : make_uint4(0, 0, 0, 0);
      c.advance(g, rstep);
    }
#pragma unroll
    for (int u = 0; u < kCubeUnroll; ++u)
      if (k0 + u < steps)
        *reinterpret_cast<uint4*>(dst + dst_cube + static_cast<size_t>(r_lane + (k0 + u) * rstep) * d) = val[u];
  }
}

// dst[bh, token] = src[bh, cube*vol + r] for every real token of the cube; same for LSE.
template <bool kDstF32>
__global__ void __launch_bounds__(kCubeWarps * 32) cube_unpermute_kernel(const __nv_bfloat16* __restrict__ src,
                                                                        const float* __restrict__ src_lse,
                                                                        void* __restrict__ dst,
                                                                        float* __restrict__ dst_lse,
                                                                        const uint8_t* __restrict__ kinds, Geom g,
                                                                        int d) {
  const int bh = blockIdx.y;
  if (kinds[bh] != kCube) return;
  const int cube = blockIdx.x * kCubeWarps + (threadIdx.x >> 5);
  if (cube >= g.ncubes) return;
  const int lane = threadIdx.x & 31;
  const int vpr = d / 8, rstep = 32 / vpr;
  const int v = lane % vpr;
  const int cw_i = cube % g.ncw, ch_i = (cube / g.ncw) % g.nch, cf_i = cube / (g.ncw * g.nch);
  const int f0 = cf_i * g.cf, h0 = ch_i * g.ch, w0 = cw_i * g.cw;
  const size_t src_cube = (static_cast<size_t>(bh) * g.R + static_cast<size_t>(cube) * g.vol) * d + v * 8;
  const size_t dst_head = static_cast<size_t>(bh) * g.N * d + v * 8;
  const bool lse = src_lse != nullptr && dst_lse != nullptr && v == 0;
  const int r_lane = lane / vpr;
  CubeWalk c;
  c.init(g, r_lane);
  const int steps = g.vol / rstep;
  for (int k0 = 0; k0 < steps; k0 += kCubeUnroll) {
    uint4 val[kCubeUnroll];
    int tok[kCubeUnroll];
#pragma unroll
    for (int u = 0; u < kCubeUnroll; ++u) {
      const int f = f0 + c.df, h = h0 + c.dh, w = w0 + c.dw;
      const bool ok = k0 + u < steps && f < g.F && h < g.Hl && w < g.Wl;
      tok[u] = ok ? (f * g.Hl + h) * g.Wl + w : -1;
      val[u] = ok ? __ldg(reinterpret_cast<const uint4*>(src + src_cube +
                                                         static_cast<size_t>(r_lane + (k0 + u) * rstep) * d))
                  : make_uint4(0, 0, 0, 0);
      c.advance(g, rstep);
    }
#pragma unroll
    for (int u = 0; u < kCubeUnroll; ++u) {
      if (tok[u] < 0) continue;
      store8_from_bf16(dst, dst_head + static_cast<size_t>(tok[u]) * d, val[u], kDstF32);
      if (lse)
        dst_lse[static_cast<size_t>(bh) * g.N + tok[u]] =
            src_lse[static_cast<size_t>(bh) * g.R + static_cast<size_t>(cube) * g.vol + r_lane + (k0 + u) * rstep];
    }
  }
}

// Row-copy grid: enough CTAs for every row, except with cube dims set, where the cube kernels
// do the cube heads and the row kernel (grid-stride) only needs enough CTAs to fill the GPU
// for the other heads; its CTAs of cube heads exit at once.
static int perm_grid_x(const Geom& g, int rows, int d, int BH) {
  const int rows_per_cta = (kPermThreads / (d / 8)) * kPermUnroll;
  int x = (rows + rows_per_cta - 1) / rows_per_cta;
  if (g.ncubes > 0) x = std::min(x, (148 * 16 + BH - 1) / BH);
  return x < 1 ? 1 : x;
}

cudaError_t launch_permute(const void* src, bool src_f32, void* dst, const uint8_t* kinds, const Geom& g, int BH,
                           int d, int* err, cudaStream_t stream) {
  dim3 grid(perm_grid_x(g, g.R, d, BH), BH);
  if (src_f32)
    permute_kernel<true><<<grid, kPermThreads, 0, stream>>>(src, static_cast<__nv_bfloat16*>(dst), kinds, g, d, err);
  else
    permute_kernel<false><<<grid, kPermThreads, 0, stream>>>(src, static_cast<__nv_bfloat16*>(dst), kinds, g, d, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || g.ncubes == 0) return e;
  const dim3 cgrid((g.ncubes + kCubeWarps - 1) / kCubeWarps, BH);
  auto* out = static_cast<__nv_bfloat16*>(dst);
  if (src_f32)
    cube_permute_kernel<true><<<cgrid, kCubeWarps * 32, 0, stream>>>(src, out, kinds, g, d);
  else
    cube_permute_kernel<false><<<cgrid, kCubeWarps * 32, 0, stream>>>(src, out, kinds, g, d);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* src, const float* src_lse, void* dst, bool dst_f32, float* dst_lse,
                             const uint8_t* kinds, const Geom& g, int BH, int d, int* err, cudaStream_t stream) {
  dim3 grid(perm_grid_x(g, g.N, d, BH), BH);
  const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(src);
  if (dst_f32)
    unpermute_kernel<true><<<grid, kPermThreads, 0, stream>>>(s, src_lse, dst, dst_lse, kinds, g, d, err);
  else
    unpermute_kernel<false><<<grid, kPermThreads, 0, stream>>>(s, src_lse, dst, dst_lse, kinds, g, d, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || g.ncubes == 0) return e;
  const dim3 cgrid((g.ncubes + kCubeWarps - 1) / kCubeWarps, BH);
  if (dst_f32)
    cube_unpermute_kernel<true><<<cgrid, kCubeWarps * 32, 0, stream>>>(s, src_lse, dst, dst_lse, kinds, g, d);
  else
    cube_unpermute_kernel<false><<<cgrid, kCubeWarps * 32, 0, stream>>>(s, src_lse, dst, dst_lse, kinds, g, d);
  return cudaGetLastError();
}

}  // namespace vsa
