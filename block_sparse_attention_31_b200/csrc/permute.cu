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

static int perm_grid_x(int rows, int d) {
  const int rows_per_cta = (kPermThreads / (d / 8)) * kPermUnroll;
  int x = (rows + rows_per_cta - 1) / rows_per_cta;
  return x < 1 ? 1 : x;
}

cudaError_t launch_permute(const void* src, bool src_f32, void* dst, const uint8_t* kinds, const Geom& g, int BH,
                           int d, int* err, cudaStream_t stream) {
  dim3 grid(perm_grid_x(g.R, d), BH);
  if (src_f32)
    permute_kernel<true><<<grid, kPermThreads, 0, stream>>>(src, static_cast<__nv_bfloat16*>(dst), kinds, g, d, err);
  else
    permute_kernel<false><<<grid, kPermThreads, 0, stream>>>(src, static_cast<__nv_bfloat16*>(dst), kinds, g, d, err);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const void* src, const float* src_lse, void* dst, bool dst_f32, float* dst_lse,
                             const uint8_t* kinds, const Geom& g, int BH, int d, int* err, cudaStream_t stream) {
  dim3 grid(perm_grid_x(g.N, d), BH);
  const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(src);
  if (dst_f32)
    unpermute_kernel<true><<<grid, kPermThreads, 0, stream>>>(s, src_lse, dst, dst_lse, kinds, g, d, err);
  else
    unpermute_kernel<false><<<grid, kPermThreads, 0, stream>>>(s, src_lse, dst, dst_lse, kinds, g, d, err);
  return cudaGetLastError();
}

}  // namespace vsa
