// fp8.cu -- per-block e4m3 quantisation of Q and K for the FP8 Q.K^T attention
// ("Sparse Video-Gen" summary page, "Measured effects": FP8 quantisation added on top of the
// sparse attention).  The page gives no format; the reading used here: e4m3 codes (round to
// nearest even, saturating at 448) of x / 2^e, with one power-of-two scale 2^e per block of
// `block` rows of a head's layout, the smallest with max |x| <= 448 * 2^e (e = 0 for an
// all-zero block).  The attention multiplies each block pair's scores by 2^(e_q + e_k).
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

constexpr int kQuantThreads = 512;

// Smallest e with a <= 448 * 2^e for a > 0: with a = f * 2^E, f in [0.5, 1), and
// 448 = 0.875 * 2^9, that is E - 9 when f <= 0.875 and E - 8 otherwise.
__device__ __forceinline__ int e4m3_block_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int E;
  const float f = frexpf(amax, &E);
  return f <= 0.875f ? E - 9 : E - 8;
}

// One CTA per (head, block of BN rows of the head's layout): the block's max |x|, its
// exponent, then the codes.  Rows past the head's own rows are written as zeros.
template <int D, int BN>
__global__ void __launch_bounds__(kQuantThreads) quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ nat,
                                                                      const __nv_bfloat16* __restrict__ perm,
                                                                      const uint8_t* __restrict__ kinds, Geom g,
                                                                      int nat_rows, uint8_t* __restrict__ dst,
                                                                      int32_t* __restrict__ exps, int* err) {
  constexpr int CH = BN * D / 8;                       // 16-byte chunks of a block
  constexpr int PER = CH / kQuantThreads;              // chunks per thread
  static_assert(CH % kQuantThreads == 0, "whole chunks per thread");
  __shared__ float red[kQuantThreads / 32];
  const int b = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int kind = kinds[bh];
  uint8_t* out = dst + (static_cast<size_t>(bh) * g.R + static_cast<size_t>(b) * BN) * D;
  if (kind > kCube) {
    if (tid == 0 && b == 0) atomicOr(err, kDevErrKind);
    return;
  }
  const int rows = layout_rows(g, kind);
  const bool use_perm = perm != nullptr && kind != kSpatial;
  const __nv_bfloat16* src = use_perm ? perm + static_cast<size_t>(bh) * g.R * D
                                      : nat + static_cast<size_t>(bh) * nat_rows * D;
  uint4 v[PER];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = tid + i * kQuantThreads;
    const int r = b * BN + c / (D / 8);
    v[i] = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows) v[i] = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * D + (c % (D / 8)) * 8);
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[q] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[q] & 0xffff0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) m = fmaxf(m, red[w]);
  const int e = e4m3_block_exponent(m);
  if (tid == 0) exps[static_cast<size_t>(bh) * g.nblk + b] = e;
  // 2^-e as a float (exact for -126 <= -e <= 127; other exponents go through ldexpf)
  const bool plain = e >= -127 && e <= 126;
  const float inv = plain ? __int_as_float((127 - e) << 23) : 1.f;
  auto scaled = [&](float x) { return plain ? x * inv : ldexpf(x, -e); };
  // x / 2^e is exact (a power-of-two scaling of a bf16 value); the conversion rounds to the
  // nearest e4m3 value, ties to even, saturating at 448
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = tid + i * kQuantThreads;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint32_t packed[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x0 = scaled(__uint_as_float(w[2 * h] << 16)), x1 = scaled(__uint_as_float(w[2 * h] & 0xffff0000u));
      const float x2 = scaled(__uint_as_float(w[2 * h + 1] << 16)),
                  x3 = scaled(__uint_as_float(w[2 * h + 1] & 0xffff0000u));
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x2, x3), __NV_SATFINITE, __NV_E4M3);
      packed[h] = (lo & 0xffffu) | (hi << 16);
    }
    if (b * BN + c / (D / 8) < g.R)  // the last block of a head may reach past its R rows
      *reinterpret_cast<uint2*>(out + static_cast<size_t>(c / (D / 8)) * D + (c % (D / 8)) * 8) =
          make_uint2(packed[0], packed[1]);
  }
}

cudaError_t launch_quantize_e4m3(const void* nat, const void* perm, const uint8_t* kinds, const Geom& g, int BH,
                                 int d, int nat_rows, uint8_t* dst, int32_t* exps, int* err, cudaStream_t stream) {
  if (d != 128) return cudaErrorInvalidValue;
  const dim3 grid(g.nblk, BH);
  const auto* n = static_cast<const __nv_bfloat16*>(nat);
  const auto* p = static_cast<const __nv_bfloat16*>(perm);
  if (g.block == 128)
    quantize_e4m3_kernel<128, 128><<<grid, kQuantThreads, 0, stream>>>(n, p, kinds, g, nat_rows, dst, exps, err);
  else if (g.block == 64)
    quantize_e4m3_kernel<128, 64><<<grid, kQuantThreads, 0, stream>>>(n, p, kinds, g, nat_rows, dst, exps, err);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace vsa
