// api.cu -- the C ABI of libvsa.so (declared in include/vsa.h): host-side validation,
// planning helpers, TMA descriptor encoding and the launch sequence of one attention call.
// No device memory is allocated here; every buffer comes from the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "vsa.h"

namespace vsa {

// ---------------------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point
// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3D view (d, rows, B*H) of a [B*H, rows, d] bf16 tensor; box = 64 columns x box_rows rows,
// 128-byte swizzle; out-of-range rows read as zero and are clipped on store.
cudaError_t encode_rows_map(CUtensorMap* map, const void* base, int d, int rows, int BH, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_rows_map_u8(CUtensorMap* map, const void* base, int d, int rows, int BH, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  if (d != 128) return cudaErrorInvalidValue;  // one 128-byte swizzled row per box row
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows) * d};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every non-null pointer is device (or managed) memory.  Kernels and TMA copies fault on a
// pageable host address, so a host pointer is refused here, before anything is launched.
static bool on_device(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (p == nullptr) continue;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return false;
  }
  return true;
}

// Validate the shape and derive the geometry.
static vsa_status make_geom(const vsa_shape* s, Geom* g) {
  if (s == nullptr || g == nullptr) return VSA_ERR_INVALID_ARG;
  if (s->B <= 0 || s->H <= 0 || s->F <= 0 || s->Hl <= 0 || s->Wl <= 0 || s->d <= 0 || s->block <= 0)
    return VSA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return VSA_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return VSA_ERR_UNSUPPORTED;
  const long long N = static_cast<long long>(s->F) * s->Hl * s->Wl;
  if (N > (1LL << 28)) return VSA_ERR_UNSUPPORTED;
  const bool cubes = s->cube_f != 0 || s->cube_h != 0 || s->cube_w != 0;
  Geom r{};
  r.F = s->F;
  r.Hl = s->Hl;
  r.Wl = s->Wl;
  r.S = s->Hl * s->Wl;
  r.N = static_cast<int>(N);
  r.block = s->block;
  if (cubes) {
    if (s->cube_f <= 0 || s->cube_h <= 0 || s->cube_w <= 0) return VSA_ERR_INVALID_ARG;
    if (s->cube_f * s->cube_h * s->cube_w != s->block) return VSA_ERR_UNSUPPORTED;
    r.cf = s->cube_f;
    r.ch = s->cube_h;
    r.cw = s->cube_w;
    r.vol = r.cf * r.ch * r.cw;
    r.ncf = (r.F + r.cf - 1) / r.cf;
    r.nch = (r.Hl + r.ch - 1) / r.ch;
    r.ncw = (r.Wl + r.cw - 1) / r.cw;
    const long long nc = static_cast<long long>(r.ncf) * r.nch * r.ncw;
    if (nc * r.vol > (1LL << 28)) return VSA_ERR_UNSUPPORTED;
    r.ncubes = static_cast<int>(nc);
    r.R = r.ncubes * r.vol;
  } else {
    r.cf = r.ch = r.cw = r.vol = 1;  // unused; keeps the cube arithmetic division-safe
    r.ncf = r.nch = r.ncw = 1;
    r.ncubes = 0;
    r.R = r.N;
  }
  r.nblk = (r.R + r.block - 1) / r.block;
  *g = r;
  return VSA_OK;
}

static float scale_log2_of(float scale, int d) {
  const float s = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  return s * 1.4426950408889634f;
}

// ---------------------------------------------------------------------------------------
// Window planning on the host: per-query-block kept ranges are contiguous, so the kept
// count for window w is a sum of range lengths found by binary search.
// ---------------------------------------------------------------------------------------
struct BlockIntervals {
  std::vector<int> a, b;  // group interval [a_i, b_i] of block i
};

static BlockIntervals intervals(const Geom& g, int kind) {
  const int G = kind == kSpatial ? g.S : g.F;
  const int nb = (g.N + g.block - 1) / g.block;
  BlockIntervals iv;
  iv.a.resize(nb);
  iv.b.resize(nb);
  for (int i = 0; i < nb; ++i) {
    iv.a[i] = (i * g.block) / G;
    iv.b[i] = (std::min(g.N, (i + 1) * g.block) - 1) / G;
  }
  return iv;
}

// Kept blocks of row i: j with a_j <= b_i + w and b_j >= a_i - w (both sequences nondecreasing).
static int kept_in_row(const BlockIntervals& iv, int i, long long w) {
  const int nb = static_cast<int>(iv.a.size());
  const long long hi_val = iv.b[i] + w, lo_val = iv.a[i] - w;
  int lo = 0, hi = nb;  // first j with b_j >= lo_val
  while (lo < hi) {
    const int mid = (lo + hi) / 2;
    if (iv.b[mid] >= lo_val) hi = mid; else lo = mid + 1;
  }
  const int j0 = lo;
  lo = 0;
  hi = nb;  // first j with a_j > hi_val
  while (lo < hi) {
    const int mid = (lo + hi) / 2;
    if (iv.a[mid] > hi_val) hi = mid; else lo = mid + 1;
  }
  const int j1 = lo;  // exclusive
  return j1 > j0 ? j1 - j0 : 0;
}

static long long kept_total(const BlockIntervals& iv, long long w, int* row_max) {
  long long tot = 0;
  int mx = 0;
  for (int i = 0; i < static_cast<int>(iv.a.size()); ++i) {
    const int k = kept_in_row(iv, i, w);
    tot += k;
    mx = std::max(mx, k);
  }
  if (row_max) *row_max = mx;
  return tot;
}

}  // namespace vsa

using namespace vsa;

extern "C" {

const char* vsa_status_string(vsa_status s) {
  switch (s) {
    case VSA_OK: return "ok";
    case VSA_ERR_INVALID_ARG: return "invalid argument";
    case VSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case VSA_ERR_WORKSPACE: return "workspace too small";
    case VSA_ERR_CUDA: return "CUDA call failed";
    case VSA_ERR_DEVICE: return "device-side error flagged";
    case VSA_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int vsa_version(void) { return 100; }

vsa_status vsa_layout_rows(const vsa_shape* shape, int64_t* rows) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (rows == nullptr) return VSA_ERR_INVALID_ARG;
  *rows = g.R;
  return VSA_OK;
}

vsa_status vsa_num_blocks(const vsa_shape* shape, int* nblk) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (nblk == nullptr) return VSA_ERR_INVALID_ARG;
  *nblk = g.nblk;
  return VSA_OK;
}

vsa_status vsa_pattern_window(const vsa_shape* shape, vsa_kind kind, double target, int* w, double* kept) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (w == nullptr || (kind != VSA_SPATIAL && kind != VSA_TEMPORAL) || !(target >= 0.0) || target > 1.0)
    return VSA_ERR_INVALID_ARG;
  const BlockIntervals iv = intervals(g, kind);
  const double nb = static_cast<double>(iv.a.size());
  const long long wmax = kind == VSA_SPATIAL ? g.F - 1 : g.S - 1;
  long long lo = 0, hi = wmax;  // smallest w in [0, wmax] with kept(w)/nb^2 >= target
  while (lo < hi) {
    const long long mid = (lo + hi) / 2;
    if (static_cast<double>(kept_total(iv, mid, nullptr)) / (nb * nb) >= target) hi = mid; else lo = mid + 1;
  }
  *w = static_cast<int>(lo);
  if (kept) *kept = static_cast<double>(kept_total(iv, lo, nullptr)) / (nb * nb);
  return VSA_OK;
}

vsa_status vsa_max_kv(const vsa_shape* shape, const vsa_params* params, int* max_kv) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (params == nullptr || max_kv == nullptr || params->w_s < 0 || params->w_t < 0) return VSA_ERR_INVALID_ARG;
  int mx = 0, m1 = 0;
  kept_total(intervals(g, kSpatial), params->w_s, &m1);
  mx = std::max(mx, m1);
  kept_total(intervals(g, kTemporal), params->w_t, &m1);
  mx = std::max(mx, m1);
  if (g.ncubes > 0) {
    if (params->topk < 0) return VSA_ERR_INVALID_ARG;
    mx = std::max(mx, std::min(params->topk + 1, g.ncubes));
  }
  *max_kv = mx;
  return VSA_OK;
}

vsa_status vsa_profile_rows(const vsa_shape* shape, const vsa_params* params, int* rows) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (params == nullptr || rows == nullptr || !(params->profile_frac > 0.0) || params->profile_frac > 1.0)
    return VSA_ERR_INVALID_ARG;
  *rows = profile_plan(g, shape->B * shape->H, shape->d, params->profile_frac).r;
  return VSA_OK;
}

size_t vsa_profile_workspace_size(const vsa_shape* shape, const vsa_params* params) {
  Geom g;
  if (make_geom(shape, &g) != VSA_OK || params == nullptr || !(params->profile_frac > 0.0)) return 0;
  return profile_plan(g, shape->B * shape->H, shape->d, params->profile_frac).bytes;
}

size_t vsa_mask_workspace_size(const vsa_shape* shape, const vsa_params* params) {
  Geom g;
  if (make_geom(shape, &g) != VSA_OK || params == nullptr) return 0;
  return g.ncubes > 0 ? cube_mask_workspace_bytes(g, shape->B * shape->H, shape->d) : 0;
}

vsa_status vsa_permute(const void* src, vsa_dtype src_dtype, void* dst, const uint8_t* d_kind, const vsa_shape* shape,
                       int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!src || !dst || !d_kind || !d_err || !aligned16(src) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  if (src_dtype != VSA_F32 && src_dtype != VSA_BF16) return VSA_ERR_INVALID_ARG;
  if (!on_device({src, dst, d_kind, d_err})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e =
      launch_permute(src, src_dtype == VSA_F32, dst, d_kind, g, shape->B * shape->H, shape->d, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_unpermute(const void* src, const float* src_lse, void* dst, vsa_dtype dst_dtype, float* dst_lse,
                         const uint8_t* d_kind, const vsa_shape* shape, int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!src || !dst || !d_kind || !d_err || !aligned16(src) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  if ((src_lse == nullptr) != (dst_lse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (dst_dtype != VSA_F32 && dst_dtype != VSA_BF16) return VSA_ERR_INVALID_ARG;
  if (!on_device({src, src_lse, dst, dst_lse, d_kind, d_err})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e = launch_unpermute(src, src_lse, dst, dst_dtype == VSA_F32, dst_lse, d_kind, g,
                                         shape->B * shape->H, shape->d, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_profile_heads(const void* q, const void* k, const void* v, const vsa_shape* shape,
                             const vsa_params* params, uint8_t* d_kind, float* d_mse, void* ws, size_t ws_bytes,
                             int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!q || !k || !v || !params || !d_kind || !d_mse || !ws || !d_err) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(ws)) return VSA_ERR_INVALID_ARG;
  if (!(params->profile_frac > 0.0) || params->profile_frac > 1.0 || params->w_s < 0 || params->w_t < 0)
    return VSA_ERR_INVALID_ARG;
  const int BH = shape->B * shape->H;
  const ProfilePlan plan = profile_plan(g, BH, shape->d, params->profile_frac);
  if (ws_bytes < plan.bytes) return VSA_ERR_WORKSPACE;
  if (!on_device({q, k, v, d_kind, d_mse, ws, d_err})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e = launch_profile(q, k, v, g, BH, shape->d, params->w_s, params->w_t,
                                       scale_log2_of(params->scale, shape->d), plan, ws, d_kind, d_mse, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_build_mask(const uint8_t* d_kind, const void* q_cube, const void* k_cube, const vsa_shape* shape,
                          const vsa_params* params, uint32_t* d_bits, int32_t* d_kv_idx, int32_t* d_kv_cnt, int max_kv,
                          void* ws, size_t ws_bytes, int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!d_kind || !params || !d_bits || !d_kv_idx || !d_kv_cnt || !d_err || max_kv <= 0) return VSA_ERR_INVALID_ARG;
  if (params->w_s < 0 || params->w_t < 0) return VSA_ERR_INVALID_ARG;
  const int BH = shape->B * shape->H;
  if (!on_device({d_kind, d_bits, d_kv_idx, d_kv_cnt, d_err})) return VSA_ERR_INVALID_ARG;
  if (g.ncubes > 0 && !on_device({q_cube, k_cube, ws})) return VSA_ERR_INVALID_ARG;
  cudaError_t e = launch_pattern_mask(d_kind, g, BH, params->w_s, params->w_t, d_bits, d_kv_idx, d_kv_cnt, max_kv,
                                      d_err, stream);
  if (e != cudaSuccess) return VSA_ERR_CUDA;
  if (g.ncubes > 0) {
    if (!q_cube || !k_cube || !ws || !aligned16(q_cube) || !aligned16(k_cube) || !aligned16(ws) || params->topk < 0)
      return VSA_ERR_INVALID_ARG;
    if (ws_bytes < cube_mask_workspace_bytes(g, BH, shape->d)) return VSA_ERR_WORKSPACE;
    e = launch_cube_mask(d_kind, q_cube, k_cube, g, BH, shape->d, params->topk, d_bits, d_kv_idx, d_kv_cnt, max_kv,
                         ws, d_err, stream);
    if (e != cudaSuccess) return VSA_ERR_CUDA;
  }
  return VSA_OK;
}

static vsa_status check_qkvo(const vsa_qkvo* t) {
  if (t == nullptr || !t->q || !t->k || !t->v || !t->o) return VSA_ERR_INVALID_ARG;
  if (!aligned16(t->q) || !aligned16(t->k) || !aligned16(t->v) || !aligned16(t->o)) return VSA_ERR_INVALID_ARG;
  return VSA_OK;
}

static vsa_status encode_set(AttnMaps* m, const vsa_qkvo* t, const Geom& g, int rows, int BH, int d) {
  if (encode_rows_map(&m->q, t->q, d, rows, BH, 128) != cudaSuccess) return VSA_ERR_CUDA;
  if (encode_rows_map(&m->k, t->k, d, rows, BH, g.block) != cudaSuccess) return VSA_ERR_CUDA;
  if (encode_rows_map(&m->v, t->v, d, rows, BH, g.block) != cudaSuccess) return VSA_ERR_CUDA;
  if (encode_rows_map(&m->o, t->o, d, rows, BH, g.block) != cudaSuccess) return VSA_ERR_CUDA;
  return VSA_OK;
}

vsa_status vsa_block_order(const uint8_t* d_kind, const int32_t* d_kv_idx, const int32_t* d_kv_cnt, int max_kv,
                           const vsa_shape* shape, int32_t* d_order, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!d_kind || !d_kv_idx || !d_kv_cnt || !d_order || max_kv <= 0) return VSA_ERR_INVALID_ARG;
  if (g.nblk > 32768) return VSA_ERR_UNSUPPORTED;
  if (!on_device({d_kind, d_kv_idx, d_kv_cnt, d_order})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e = launch_block_order(d_kind, g, shape->B * shape->H, d_kv_idx, d_kv_cnt, max_kv, d_order,
                                           stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// e4m3 Q and K for vsa_sparse_attn_fwd_fp8qk (all null for bf16).
struct Fp8QK {
  const uint8_t* q8;
  const int32_t* qexp;
  const uint8_t* k8;
  const int32_t* kexp;
};

static vsa_status sparse_attn_fwd_impl(const vsa_qkvo* natural, const vsa_qkvo* permuted, const Fp8QK& f8,
                                       const uint8_t* d_kind, const int32_t* d_kv_idx, const int32_t* d_kv_cnt,
                                       int max_kv, const int32_t* d_order, const vsa_shape* shape, float scale,
                                       int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if ((st = check_qkvo(natural)) != VSA_OK) return st;
  if (permuted != nullptr && (st = check_qkvo(permuted)) != VSA_OK) return st;
  if (!d_kind || !d_kv_idx || !d_kv_cnt || !d_err || max_kv <= 0 || !(scale >= 0.f)) return VSA_ERR_INVALID_ARG;
  const bool qk8 = f8.q8 != nullptr;
  if (qk8) {
    if (!f8.qexp || !f8.k8 || !f8.kexp || !aligned16(f8.q8) || !aligned16(f8.k8)) return VSA_ERR_INVALID_ARG;
    if (shape->d != 128 || shape->block != 128) return VSA_ERR_UNSUPPORTED;
    if (!on_device({f8.q8, f8.qexp, f8.k8, f8.kexp})) return VSA_ERR_INVALID_ARG;
  }
  const int BH = shape->B * shape->H;
  if (!on_device({natural->q, natural->k, natural->v, natural->o, natural->lse, d_kind, d_kv_idx, d_kv_cnt, d_order,
                  d_err}))
    return VSA_ERR_INVALID_ARG;
  if (permuted != nullptr &&
      !on_device({permuted->q, permuted->k, permuted->v, permuted->o, permuted->lse}))
    return VSA_ERR_INVALID_ARG;
  AttnMaps nat, perm;
  // Without a permuted set every head reads the `natural` buffers, whose rows must then
  // cover every head's layout (R rows per head).
  const int nat_rows = permuted != nullptr ? g.N : g.R;
  if ((st = encode_set(&nat, natural, g, nat_rows, BH, shape->d)) != VSA_OK) return st;
  if (permuted != nullptr) {
    if ((st = encode_set(&perm, permuted, g, g.R, BH, shape->d)) != VSA_OK) return st;
  } else {
    perm = nat;
  }
  if (qk8) {  // every head's Q and K come from the e4m3 buffers (R rows per head, its own layout)
    if (encode_rows_map_u8(&nat.q, f8.q8, shape->d, g.R, BH, 128) != cudaSuccess) return VSA_ERR_CUDA;
    if (encode_rows_map_u8(&nat.k, f8.k8, shape->d, g.R, BH, g.block) != cudaSuccess) return VSA_ERR_CUDA;
    perm.q = nat.q;
    perm.k = nat.k;
  }
  AttnArgs a;
  a.kinds = d_kind;
  a.kv_idx = d_kv_idx;
  a.kv_cnt = d_kv_cnt;
  a.order = d_order;
  a.lse_nat = natural->lse;
  a.lse_perm = permuted != nullptr ? permuted->lse : natural->lse;
  a.err = d_err;
  a.BH = BH;
  a.max_kv = max_kv;
  a.has_perm = permuted != nullptr ? 1 : 0;
  a.scale_log2 = scale_log2_of(scale, shape->d);
  a.g = g;
  a.nat_rows = nat_rows;
  a.ucap = std::min(g.nblk, 2 * max_kv);
  a.gather = 0;
  a.qexp = qk8 ? f8.qexp : nullptr;
  a.kexp = qk8 ? f8.kexp : nullptr;
  a.nat_q = a.nat_k = a.nat_v = nullptr;
  a.nat_o = natural->o;  // written only for a head with an invalid kind byte (zero rows)
  const cudaError_t e = launch_sparse_attn(nat, perm, a, shape->d, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_sparse_attn_fwd(const vsa_qkvo* natural, const vsa_qkvo* permuted, const uint8_t* d_kind,
                               const int32_t* d_kv_idx, const int32_t* d_kv_cnt, int max_kv,
                               const int32_t* d_order, const vsa_shape* shape, float scale, int* d_err,
                               cudaStream_t stream) {
  return sparse_attn_fwd_impl(natural, permuted, Fp8QK{nullptr, nullptr, nullptr, nullptr}, d_kind, d_kv_idx,
                              d_kv_cnt, max_kv, d_order, shape, scale, d_err, stream);
}

vsa_status vsa_sparse_attn_fwd_fp8qk(const vsa_qkvo* natural, const vsa_qkvo* permuted, const uint8_t* q8,
                                     const int32_t* d_qexp, const uint8_t* k8, const int32_t* d_kexp,
                                     const uint8_t* d_kind, const int32_t* d_kv_idx, const int32_t* d_kv_cnt,
                                     int max_kv, const int32_t* d_order, const vsa_shape* shape, float scale,
                                     int* d_err, cudaStream_t stream) {
  if (!q8) return VSA_ERR_INVALID_ARG;
  return sparse_attn_fwd_impl(natural, permuted, Fp8QK{q8, d_qexp, k8, d_kexp}, d_kind, d_kv_idx, d_kv_cnt, max_kv,
                              d_order, shape, scale, d_err, stream);
}

vsa_status vsa_quantize_fp8(const void* natural, const void* permuted, const uint8_t* d_kind,
                            const vsa_shape* shape, uint8_t* dst, int32_t* d_exp, int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!natural || !d_kind || !dst || !d_exp || !d_err) return VSA_ERR_INVALID_ARG;
  if (!aligned16(natural) || (permuted && !aligned16(permuted)) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  if (shape->d != 128) return VSA_ERR_UNSUPPORTED;
  if (!on_device({natural, permuted, d_kind, dst, d_exp, d_err})) return VSA_ERR_INVALID_ARG;
  const int nat_rows = permuted != nullptr ? g.N : g.R;
  const cudaError_t e = launch_quantize_e4m3(natural, permuted, d_kind, g, shape->B * shape->H, shape->d, nat_rows,
                                             dst, d_exp, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_sparse_attn_fwd_natural(const vsa_qkvo* natural, const uint8_t* d_kind, const int32_t* d_kv_idx,
                                       const int32_t* d_kv_cnt, int max_kv, const int32_t* d_order,
                                       const vsa_shape* shape, float scale, int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (g.ncubes > 0) return VSA_ERR_UNSUPPORTED;  // cube heads read cube-major copies
  if ((st = check_qkvo(natural)) != VSA_OK) return st;
  if (!d_kind || !d_kv_idx || !d_kv_cnt || !d_err || max_kv <= 0 || !(scale >= 0.f)) return VSA_ERR_INVALID_ARG;
  const int BH = shape->B * shape->H;
  if (!on_device({natural->q, natural->k, natural->v, natural->o, natural->lse, d_kind, d_kv_idx, d_kv_cnt, d_order,
                  d_err}))
    return VSA_ERR_INVALID_ARG;
  AttnMaps nat;
  if ((st = encode_set(&nat, natural, g, g.N, BH, shape->d)) != VSA_OK) return st;
  AttnArgs a;
  a.kinds = d_kind;
  a.kv_idx = d_kv_idx;
  a.kv_cnt = d_kv_cnt;
  a.order = d_order;
  a.lse_nat = natural->lse;
  a.lse_perm = natural->lse;
  a.err = d_err;
  a.BH = BH;
  a.max_kv = max_kv;
  a.has_perm = 0;
  a.scale_log2 = scale_log2_of(scale, shape->d);
  a.g = g;
  a.nat_rows = g.N;
  a.ucap = std::min(g.nblk, 2 * max_kv);
  a.gather = 1;
  a.qexp = a.kexp = nullptr;
  a.nat_q = natural->q;
  a.nat_k = natural->k;
  a.nat_v = natural->v;
  a.nat_o = natural->o;
  const cudaError_t e = launch_sparse_attn(nat, nat, a, shape->d, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Semantic-aware permutation ("Sparse VideoGen2" page, abstract)
// ---------------------------------------------------------------------------------------
// Shapes of the semantic path: no cube dims (every head has N rows).
static vsa_status semantic_geom(const vsa_shape* shape, Geom* g) {
  vsa_status st = make_geom(shape, g);
  if (st != VSA_OK) return st;
  if (g->ncubes > 0) return VSA_ERR_UNSUPPORTED;
  return VSA_OK;
}

static bool clusters_ok(const Geom& g, int C) { return C >= 1 && C <= kMaxClusters && C <= g.N; }

size_t vsa_kmeans_workspace_size(const vsa_shape* shape, int n_clusters) {
  Geom g;
  if (semantic_geom(shape, &g) != VSA_OK || !clusters_ok(g, n_clusters)) return 0;
  return kmeans_workspace_bytes(shape->B * shape->H, g.N, n_clusters, shape->d);
}

vsa_status vsa_kmeans(const void* x, const vsa_shape* shape, int n_clusters, int iters, float* d_centroids,
                      int32_t* d_labels, int32_t* d_counts, int32_t* d_perm, void* ws, size_t ws_bytes, int* d_err,
                      cudaStream_t stream) {
  Geom g;
  vsa_status st = semantic_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!clusters_ok(g, n_clusters) || iters < 1 || iters > 1000) return VSA_ERR_INVALID_ARG;
  if (!x || !d_centroids || !d_labels || !d_counts || !d_perm || !ws || !d_err || !aligned16(x) ||
      !aligned16(d_centroids))
    return VSA_ERR_INVALID_ARG;
  if (ws_bytes < vsa_kmeans_workspace_size(shape, n_clusters)) return VSA_ERR_WORKSPACE;
  if (!on_device({x, d_centroids, d_labels, d_counts, d_perm, ws, d_err})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e = launch_kmeans(x, shape->B * shape->H, g.N, shape->d, n_clusters, iters, d_centroids,
                                      d_labels, d_counts, d_perm, ws, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

size_t vsa_semantic_mask_workspace_size(const vsa_shape* shape) {
  Geom g;
  if (semantic_geom(shape, &g) != VSA_OK) return 0;
  return align256(semantic_mask_workspace_bytes(shape->B * shape->H, g.N, g.block));
}

vsa_status vsa_semantic_mask(const float* d_cent_q, const int32_t* d_counts_q, const int32_t* d_labels_q,
                             const int32_t* d_perm_q, int cq, const float* d_cent_k, const int32_t* d_counts_k,
                             const int32_t* d_labels_k, const int32_t* d_perm_k, int ck, const vsa_shape* shape,
                             float top_p, float scale, uint32_t* d_keep, uint32_t* d_bits, int32_t* d_kv_idx,
                             int32_t* d_kv_cnt, int max_kv, void* ws, size_t ws_bytes, int* d_err,
                             cudaStream_t stream) {
  Geom g;
  vsa_status st = semantic_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!clusters_ok(g, cq) || !clusters_ok(g, ck)) return VSA_ERR_INVALID_ARG;
  if (!(top_p > 0.f && top_p <= 1.f) || !(scale >= 0.f) || max_kv <= 0) return VSA_ERR_INVALID_ARG;
  if (!d_cent_q || !d_counts_q || !d_labels_q || !d_perm_q || !d_cent_k || !d_counts_k || !d_labels_k ||
      !d_perm_k || !d_keep || !d_bits || !d_kv_idx || !d_kv_cnt || !ws || !d_err || !aligned16(ws))
    return VSA_ERR_INVALID_ARG;
  if (ws_bytes < vsa_semantic_mask_workspace_size(shape)) return VSA_ERR_WORKSPACE;
  if (!on_device({d_cent_q, d_counts_q, d_labels_q, d_perm_q, d_cent_k, d_counts_k, d_labels_k, d_perm_k, d_keep,
                  d_bits, d_kv_idx, d_kv_cnt, ws, d_err}))
    return VSA_ERR_INVALID_ARG;
  const double sc = scale > 0.f ? static_cast<double>(scale) : 1.0 / std::sqrt(static_cast<double>(shape->d));
  const cudaError_t e = launch_semantic_mask(d_cent_q, d_counts_q, d_labels_q, d_perm_q, cq, d_cent_k, d_counts_k,
                                             d_labels_k, d_perm_k, ck, shape->B * shape->H, g.N, shape->d, g.block,
                                             sc, static_cast<double>(top_p), d_keep, d_bits, d_kv_idx, d_kv_cnt,
                                             max_kv, ws, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_gather_rows(const void* src, const int32_t* d_perm, void* dst, const vsa_shape* shape, int* d_err,
                           cudaStream_t stream) {
  Geom g;
  vsa_status st = semantic_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!src || !d_perm || !dst || !d_err || !aligned16(src) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  if (!on_device({src, d_perm, dst, d_err})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e = launch_gather_rows(src, d_perm, dst, shape->B * shape->H, g.N, shape->d, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status vsa_scatter_rows(const void* src, const float* src_lse, const int32_t* d_perm, void* dst, float* dst_lse,
                            const vsa_shape* shape, int* d_err, cudaStream_t stream) {
  Geom g;
  vsa_status st = semantic_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!src || !d_perm || !dst || !d_err || !aligned16(src) || !aligned16(dst)) return VSA_ERR_INVALID_ARG;
  if ((src_lse == nullptr) != (dst_lse == nullptr)) return VSA_ERR_INVALID_ARG;
  if (!on_device({src, src_lse, d_perm, dst, dst_lse, d_err})) return VSA_ERR_INVALID_ARG;
  const cudaError_t e =
      launch_scatter_rows(src, src_lse, d_perm, dst, dst_lse, shape->B * shape->H, g.N, shape->d, d_err, stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// Workspace of the whole semantic call.
struct SemLayout {
  size_t kinds, cent_q, lab_q, cnt_q, perm_q, cent_k, lab_k, cnt_k, perm_k, offs, keep, bits, idx, cnt, mws, pq, pk,
      pv, po, plse, bytes;
  int max_kv;
};

static vsa_status semantic_layout(const vsa_shape* shape, const vsa_semantic_params* sp, SemLayout* L) {
  Geom g;
  vsa_status st = semantic_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (sp == nullptr || L == nullptr) return VSA_ERR_INVALID_ARG;
  if (!clusters_ok(g, sp->cq) || !clusters_ok(g, sp->ck) || sp->iters < 1 || sp->iters > 1000) return VSA_ERR_INVALID_ARG;
  if (!(sp->top_p > 0.f && sp->top_p <= 1.f) || !(sp->scale >= 0.f)) return VSA_ERR_INVALID_ARG;
  const size_t BH = static_cast<size_t>(shape->B) * shape->H, N = g.N, d = shape->d, nb = g.nblk;
  const size_t kwords = (sp->ck + 31) / 32, bwords = (nb + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L->kinds = take(BH);
  L->cent_q = take(BH * sp->cq * d * 4);
  L->lab_q = take(BH * N * 4);
  L->cnt_q = take(BH * sp->cq * 4);
  L->perm_q = take(BH * N * 4);
  L->cent_k = take(BH * sp->ck * d * 4);
  L->lab_k = take(BH * N * 4);
  L->cnt_k = take(BH * sp->ck * 4);
  L->perm_k = take(BH * N * 4);
  L->offs = take(kmeans_workspace_bytes(static_cast<int>(BH), g.N, std::max(sp->cq, sp->ck), static_cast<int>(d)));
  L->keep = take(BH * sp->cq * kwords * 4);
  L->bits = take(BH * nb * bwords * 4);
  L->idx = take(BH * nb * nb * 4);
  L->cnt = take(BH * nb * 4);
  L->mws = take(semantic_mask_workspace_bytes(static_cast<int>(BH), g.N, g.block));
  L->pq = take(BH * N * d * 2);
  L->pk = take(BH * N * d * 2);
  L->pv = take(BH * N * d * 2);
  L->po = take(BH * N * d * 2);
  L->plse = take(BH * N * 4);
  L->bytes = off;
  L->max_kv = static_cast<int>(nb);
  return VSA_OK;
}

size_t vsa_semantic_workspace_size(const vsa_shape* shape, const vsa_semantic_params* params) {
  SemLayout L;
  return semantic_layout(shape, params, &L) == VSA_OK ? L.bytes : 0;
}

vsa_status vsa_semantic_attention(const vsa_qkvo* io, const vsa_shape* shape, const vsa_semantic_params* params,
                                  void* ws, size_t ws_bytes, int* d_err, cudaStream_t stream) {
  SemLayout L;
  vsa_status st = semantic_layout(shape, params, &L);
  if (st != VSA_OK) return st;
  if ((st = check_qkvo(io)) != VSA_OK) return st;
  if (!ws || !d_err || !aligned16(ws)) return VSA_ERR_INVALID_ARG;
  if (ws_bytes < L.bytes) return VSA_ERR_WORKSPACE;
  if (!on_device({io->q, io->k, io->v, io->o, io->lse, ws, d_err})) return VSA_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(ws);
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(w + off); };
  auto i32 = [&](size_t off) { return reinterpret_cast<int32_t*>(w + off); };
  const size_t kmws = L.keep - L.offs;  // bytes reserved for the k-means scratch
  // 1. clusters and cluster-major orders of Q and of K
  if ((st = vsa_kmeans(io->q, shape, params->cq, params->iters, f32(L.cent_q), i32(L.lab_q), i32(L.cnt_q),
                       i32(L.perm_q), w + L.offs, kmws, d_err, stream)) != VSA_OK)
    return st;
  if ((st = vsa_kmeans(io->k, shape, params->ck, params->iters, f32(L.cent_k), i32(L.lab_k), i32(L.cnt_k),
                       i32(L.perm_k), w + L.offs, kmws, d_err, stream)) != VSA_OK)
    return st;
  // 2. rows in cluster-major order: Q by its clusters, K and V by the key clusters
  void *pq = w + L.pq, *pk = w + L.pk, *pv = w + L.pv, *po = w + L.po;
  if ((st = vsa_gather_rows(io->q, i32(L.perm_q), pq, shape, d_err, stream)) != VSA_OK) return st;
  if ((st = vsa_gather_rows(io->k, i32(L.perm_k), pk, shape, d_err, stream)) != VSA_OK) return st;
  if ((st = vsa_gather_rows(io->v, i32(L.perm_k), pv, shape, d_err, stream)) != VSA_OK) return st;
  // 3. top-p cluster budget and the block mask over the two layouts
  if ((st = vsa_semantic_mask(f32(L.cent_q), i32(L.cnt_q), i32(L.lab_q), i32(L.perm_q), params->cq, f32(L.cent_k),
                              i32(L.cnt_k), i32(L.lab_k), i32(L.perm_k), params->ck, shape, params->top_p,
                              params->scale, reinterpret_cast<uint32_t*>(w + L.keep),
                              reinterpret_cast<uint32_t*>(w + L.bits), i32(L.idx), i32(L.cnt), L.max_kv, w + L.mws,
                              ws_bytes - L.mws, d_err, stream)) != VSA_OK)
    return st;
  // 4. attention on the permuted rows.  The kernel reads a VSA_TEMPORAL head's N rows from the
  // permuted set; which permutation produced them does not matter to it.
  uint8_t* kinds = w + L.kinds;
  if (cudaMemsetAsync(kinds, kTemporal, static_cast<size_t>(shape->B) * shape->H, stream) != cudaSuccess)
    return VSA_ERR_CUDA;
  float* plse = io->lse ? f32(L.plse) : nullptr;
  const vsa_qkvo perm_set{pq, pk, pv, po, plse};
  if ((st = vsa_sparse_attn_fwd(io, &perm_set, kinds, i32(L.idx), i32(L.cnt), L.max_kv, nullptr, shape,
                                params->scale, d_err, stream)) != VSA_OK)
    return st;
  // 5. output rows back to token order through the query permutation
  return vsa_scatter_rows(po, plse, i32(L.perm_q), io->o, io->lse, shape, d_err, stream);
}

// ---------------------------------------------------------------------------------------
// Whole call
// ---------------------------------------------------------------------------------------
struct AttnLayout {
  size_t off_bits, off_idx, off_cnt, off_order, off_q, off_k, off_v, off_o, off_lse, off_prof, off_mask;
  size_t off_q8, off_k8, off_qe, off_ke, bytes;
  int max_kv;
};

static vsa_status attention_layout(const vsa_shape* shape, const vsa_params* params, vsa_dtype dtype,
                                   vsa_select select, AttnLayout* L) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (params == nullptr || L == nullptr) return VSA_ERR_INVALID_ARG;
  if (select != VSA_SELECT_PROFILE && select != VSA_SELECT_GIVEN && select != VSA_SELECT_CUBE)
    return VSA_ERR_INVALID_ARG;
  if (select == VSA_SELECT_CUBE && g.ncubes == 0) return VSA_ERR_INVALID_ARG;
  if (select == VSA_SELECT_PROFILE && dtype != VSA_BF16) return VSA_ERR_UNSUPPORTED;
  const bool qk8 = params->qk_fp8 != 0;
  if (qk8 && (dtype != VSA_BF16 || shape->d != 128 || shape->block != 128 || params->layout_in_kernel != 0))
    return VSA_ERR_UNSUPPORTED;
  int max_kv = 0;
  if ((st = vsa_max_kv(shape, params, &max_kv)) != VSA_OK) return st;
  if (max_kv <= 0) max_kv = 1;
  const size_t BH = static_cast<size_t>(shape->B) * shape->H, d = shape->d;
  const size_t nwords = (g.nblk + 31) / 32;
  size_t off = 0;
  L->off_bits = off;
  off = align256(off + BH * g.nblk * nwords * 4);
  L->off_idx = off;
  off = align256(off + BH * g.nblk * max_kv * 4);
  L->off_cnt = off;
  off = align256(off + BH * g.nblk * 4);
  L->off_order = off;
  if (g.ncubes > 0) off = align256(off + BH * g.nblk * 4);
  const bool fused = params->layout_in_kernel != 0 && dtype == VSA_BF16 && g.ncubes == 0;
  const size_t tbytes = fused ? 0 : BH * g.R * d * 2;  // permuted copies (none when fused)
  L->off_q = off;
  off = align256(off + tbytes);
  L->off_k = off;
  off = align256(off + tbytes);
  L->off_v = off;
  off = align256(off + tbytes);
  L->off_o = off;
  off = align256(off + tbytes);
  L->off_lse = off;
  off = align256(off + (fused ? BH * 2 * 4 : BH * g.R * 4));  // fused: only the profiling MSE scratch
  L->off_prof = off;
  if (select == VSA_SELECT_PROFILE) off = align256(off + vsa_profile_workspace_size(shape, params));
  L->off_mask = off;
  off = align256(off + vsa_mask_workspace_size(shape, params));
  // e4m3 Q and K with their per-block scale exponents
  L->off_q8 = off;
  if (qk8) off = align256(off + BH * g.R * d);
  L->off_k8 = off;
  if (qk8) off = align256(off + BH * g.R * d);
  L->off_qe = off;
  if (qk8) off = align256(off + BH * g.nblk * 4);
  L->off_ke = off;
  if (qk8) off = align256(off + BH * g.nblk * 4);
  L->bytes = off;
  L->max_kv = max_kv;
  return VSA_OK;
}

size_t vsa_attention_workspace_size(const vsa_shape* shape, const vsa_params* params, vsa_dtype dtype,
                                    vsa_select select) {
  AttnLayout L;
  return attention_layout(shape, params, dtype, select, &L) == VSA_OK ? L.bytes : 0;
}

vsa_status vsa_attention_workspace_layout(const vsa_shape* shape, const vsa_params* params, vsa_dtype dtype,
                                          vsa_select select, size_t* off_bits, size_t* off_kv_idx,
                                          size_t* off_kv_cnt, int* max_kv) {
  AttnLayout L;
  vsa_status st = attention_layout(shape, params, dtype, select, &L);
  if (st != VSA_OK) return st;
  if (off_bits) *off_bits = L.off_bits;
  if (off_kv_idx) *off_kv_idx = L.off_idx;
  if (off_kv_cnt) *off_kv_cnt = L.off_cnt;
  if (max_kv) *max_kv = L.max_kv;
  return VSA_OK;
}

vsa_status vsa_attention(const vsa_qkvo* io, vsa_dtype dtype, const vsa_shape* shape, const vsa_params* params,
                         vsa_select select, uint8_t* d_kind, float* d_mse, void* ws, size_t ws_bytes, int* d_err,
                         cudaStream_t stream) {
  AttnLayout L;
  vsa_status st = attention_layout(shape, params, dtype, select, &L);
  if (st != VSA_OK) return st;
  if ((st = check_qkvo(io)) != VSA_OK) return st;
  if (!d_kind || !ws || !d_err || !aligned16(ws)) return VSA_ERR_INVALID_ARG;
  if (ws_bytes < L.bytes) return VSA_ERR_WORKSPACE;
  if (dtype != VSA_F32 && dtype != VSA_BF16) return VSA_ERR_INVALID_ARG;
  if (!on_device({io->q, io->k, io->v, io->o, io->lse, d_kind, d_mse, ws, d_err})) return VSA_ERR_INVALID_ARG;
  Geom g;
  make_geom(shape, &g);
  const int BH = shape->B * shape->H;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* bits = reinterpret_cast<uint32_t*>(w + L.off_bits);
  int32_t* kv_idx = reinterpret_cast<int32_t*>(w + L.off_idx);
  int32_t* kv_cnt = reinterpret_cast<int32_t*>(w + L.off_cnt);
  void *pq = w + L.off_q, *pk = w + L.off_k, *pv = w + L.off_v, *po = w + L.off_o;
  float* plse = io->lse ? reinterpret_cast<float*>(w + L.off_lse) : nullptr;

  // 1. kinds
  if (select == VSA_SELECT_PROFILE) {
    float* mse = d_mse;
    if (mse == nullptr) mse = reinterpret_cast<float*>(w + L.off_lse);  // scratch before the LSE is written
    if ((st = vsa_profile_heads(io->q, io->k, io->v, shape, params, d_kind, mse, w + L.off_prof,
                                ws_bytes - L.off_prof, d_err, stream)) != VSA_OK)
      return st;
  } else if (select == VSA_SELECT_CUBE) {
    if (cudaMemsetAsync(d_kind, kCube, BH, stream) != cudaSuccess) return VSA_ERR_CUDA;
  }
  // In-kernel layout: no permuted copies for pattern heads; the attention gathers them.
  const bool fused = params->layout_in_kernel != 0 && dtype == VSA_BF16 && g.ncubes == 0;
  if (fused) {
    if ((st = vsa_build_mask(d_kind, nullptr, nullptr, shape, params, bits, kv_idx, kv_cnt, L.max_kv, nullptr, 0,
                             d_err, stream)) != VSA_OK)
      return st;
    return vsa_sparse_attn_fwd_natural(io, d_kind, kv_idx, kv_cnt, L.max_kv, nullptr, shape, params->scale, d_err,
                                       stream);
  }
  // 2. layouts
  const vsa_dtype src_t = dtype;
  if ((st = vsa_permute(io->q, src_t, pq, d_kind, shape, d_err, stream)) != VSA_OK) return st;
  if ((st = vsa_permute(io->k, src_t, pk, d_kind, shape, d_err, stream)) != VSA_OK) return st;
  if ((st = vsa_permute(io->v, src_t, pv, d_kind, shape, d_err, stream)) != VSA_OK) return st;
  // 3. masks
  if ((st = vsa_build_mask(d_kind, pq, pk, shape, params, bits, kv_idx, kv_cnt, L.max_kv, w + L.off_mask,
                           ws_bytes - L.off_mask, d_err, stream)) != VSA_OK)
    return st;
  // 4. attention: fp32 inputs run every head from the converted buffers.  With cube heads
  // possible, query blocks are paired and scheduled by their first kept key block.
  int32_t* order = nullptr;
  if (g.ncubes > 0) {
    order = reinterpret_cast<int32_t*>(w + L.off_order);
    if ((st = vsa_block_order(d_kind, kv_idx, kv_cnt, L.max_kv, shape, order, stream)) != VSA_OK) return st;
  }
  const vsa_qkvo perm_set{pq, pk, pv, po, plse};
  if (params->qk_fp8 != 0) {  // e4m3 Q and K (bf16 inputs only, checked by attention_layout)
    uint8_t *q8 = w + L.off_q8, *k8 = w + L.off_k8;
    int32_t *qe = reinterpret_cast<int32_t*>(w + L.off_qe), *ke = reinterpret_cast<int32_t*>(w + L.off_ke);
    if ((st = vsa_quantize_fp8(io->q, pq, d_kind, shape, q8, qe, d_err, stream)) != VSA_OK) return st;
    if ((st = vsa_quantize_fp8(io->k, pk, d_kind, shape, k8, ke, d_err, stream)) != VSA_OK) return st;
    st = vsa_sparse_attn_fwd_fp8qk(io, &perm_set, q8, qe, k8, ke, d_kind, kv_idx, kv_cnt, L.max_kv, order, shape,
                                   params->scale, d_err, stream);
  } else if (dtype == VSA_F32) {
    st = vsa_sparse_attn_fwd(&perm_set, nullptr, d_kind, kv_idx, kv_cnt, L.max_kv, order, shape, params->scale,
                             d_err, stream);
  } else {
    st = vsa_sparse_attn_fwd(io, &perm_set, d_kind, kv_idx, kv_cnt, L.max_kv, order, shape, params->scale, d_err,
                             stream);
  }
  if (st != VSA_OK) return st;
  // 5. back to natural order
  return vsa_unpermute(po, plse, io->o, dtype, io->lse, d_kind, shape, d_err, stream);
}

vsa_status vsa_attention_host(const vsa_host_batch* host, int n, const vsa_qkvo* sets, vsa_dtype dtype,
                              const vsa_shape* shape, const vsa_params* params, vsa_select select, uint8_t* d_kind,
                              float* d_mse, void* ws, size_t ws_bytes, int* d_err, cudaStream_t stream_up,
                              cudaStream_t stream_compute, cudaStream_t stream_down) {
  if (host == nullptr || sets == nullptr || n < 0 || shape == nullptr) return VSA_ERR_INVALID_ARG;
  if (dtype != VSA_F32 && dtype != VSA_BF16) return VSA_ERR_INVALID_ARG;
  if (shape->B <= 0 || shape->H <= 0 || shape->F <= 0 || shape->Hl <= 0 || shape->Wl <= 0 || shape->d <= 0)
    return VSA_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(shape->B) * shape->H * shape->F * shape->Hl * shape->Wl * shape->d *
                       (dtype == VSA_F32 ? 4 : 2);
  for (int i = 0; i < n; ++i)
    if (!host[i].q || !host[i].k || !host[i].v || !host[i].o) return VSA_ERR_INVALID_ARG;
  for (int s = 0; s < 2; ++s) {
    vsa_status st = check_qkvo(&sets[s]);
    if (st != VSA_OK) return st;
  }
  if (n == 0) return VSA_OK;
  // events: uploaded[i], computed[i], downloaded[i] (host-side objects)
  std::vector<cudaEvent_t> ev(3 * static_cast<size_t>(n), nullptr);
  auto cleanup = [&]() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
  };
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      cleanup();
      return VSA_ERR_CUDA;
    }
  vsa_status st = VSA_OK;
  for (int i = 0; i < n && st == VSA_OK; ++i) {
    const vsa_qkvo& d = sets[i % 2];
    cudaEvent_t up = ev[3 * i], comp = ev[3 * i + 1], down = ev[3 * i + 2];
    // upload: the set must no longer be read by batch i-2's compute
    if (i >= 2 && cudaStreamWaitEvent(stream_up, ev[3 * (i - 2) + 1], 0) != cudaSuccess) st = VSA_ERR_CUDA;
    if (st == VSA_OK &&
        (cudaMemcpyAsync(const_cast<void*>(d.q), host[i].q, bytes, cudaMemcpyHostToDevice, stream_up) != cudaSuccess ||
         cudaMemcpyAsync(const_cast<void*>(d.k), host[i].k, bytes, cudaMemcpyHostToDevice, stream_up) != cudaSuccess ||
         cudaMemcpyAsync(const_cast<void*>(d.v), host[i].v, bytes, cudaMemcpyHostToDevice, stream_up) != cudaSuccess ||
         cudaEventRecord(up, stream_up) != cudaSuccess))
      st = VSA_ERR_CUDA;
    // compute: inputs uploaded, and batch i-2's output has left this set's o
    if (st == VSA_OK && cudaStreamWaitEvent(stream_compute, up, 0) != cudaSuccess) st = VSA_ERR_CUDA;
    if (st == VSA_OK && i >= 2 && cudaStreamWaitEvent(stream_compute, ev[3 * (i - 2) + 2], 0) != cudaSuccess)
      st = VSA_ERR_CUDA;
    if (st == VSA_OK)
      st = vsa_attention(&d, dtype, shape, params, select, d_kind, d_mse, ws, ws_bytes, d_err, stream_compute);
    if (st == VSA_OK && cudaEventRecord(comp, stream_compute) != cudaSuccess) st = VSA_ERR_CUDA;
    // download
    if (st == VSA_OK && (cudaStreamWaitEvent(stream_down, comp, 0) != cudaSuccess ||
                         cudaMemcpyAsync(host[i].o, d.o, bytes, cudaMemcpyDeviceToHost, stream_down) != cudaSuccess ||
                         cudaEventRecord(down, stream_down) != cudaSuccess))
      st = VSA_ERR_CUDA;
  }
  cleanup();
  return st;
}

vsa_status vsa_get_device_error(const int* d_err, cudaStream_t stream, int* host_err) {
  if (d_err == nullptr) return VSA_ERR_INVALID_ARG;
  int h = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return VSA_ERR_CUDA;
  if (cudaMemcpy(&h, d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return VSA_ERR_CUDA;
  if (host_err) *host_err = h;
  if (h == 0) return VSA_OK;
  return (h & VSA_DEVERR_TIMEOUT) ? VSA_ERR_TIMEOUT : VSA_ERR_DEVICE;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Profiling without caller-provided scratch
// ---------------------------------------------------------------------------------------
// Some callers cannot allocate device memory for a workspace: a host framework that has
// reserved all device memory for its own pool and hands out only the tensors it owns, or
// a latency-critical path where cudaMalloc's implicit device synchronisation is not
// acceptable.  For them vsa_profile_heads_static keeps its scratch in a fixed device array
// of this file (kStaticProfileScratchBytes, held by every GPU that loads the library until
// the process exits).  The array's host-side name is only a stand-in for the device
// address.  Each call asks the runtime for the array's device address in the current context
// (cudaGetSymbolAddress, a host-side lookup) and passes it to the kernels; no address is
// cached, so a context that was reset and created again gets its own array's address.
namespace vsa {
constexpr size_t kStaticProfileScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_profile_scratch[kStaticProfileScratchBytes];

// Device address of the scratch array in the current device's context.
static cudaError_t profile_scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_profile_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}
}  // namespace vsa

extern "C" {

size_t vsa_profile_static_scratch_bytes(void) { return vsa::kStaticProfileScratchBytes; }

vsa_status vsa_profile_heads_static(const void* q, const void* k, const void* v, const vsa_shape* shape,
                                    const vsa_params* params, uint8_t* d_kind, float* d_mse, int* d_err,
                                    cudaStream_t stream) {
  Geom g;
  vsa_status st = make_geom(shape, &g);
  if (st != VSA_OK) return st;
  if (!q || !k || !v || !params || !d_kind || !d_mse || !d_err) return VSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return VSA_ERR_INVALID_ARG;
  if (!(params->profile_frac > 0.0) || params->profile_frac > 1.0 || params->w_s < 0 || params->w_t < 0)
    return VSA_ERR_INVALID_ARG;
  const int BH = shape->B * shape->H;
  // Fewer key-range splits need less scratch; use the largest count that fits.
  ProfilePlan plan = profile_plan(g, BH, shape->d, params->profile_frac);
  for (int s = plan.splits; s >= 1; --s) {
    plan = profile_plan_splits(g, BH, shape->d, params->profile_frac, s);
    if (plan.bytes <= kStaticProfileScratchBytes) break;
  }
  if (plan.bytes > kStaticProfileScratchBytes) return VSA_ERR_WORKSPACE;
  if (!on_device({q, k, v, d_kind, d_mse, d_err})) return VSA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (profile_scratch_address(&scratch) != cudaSuccess) return VSA_ERR_CUDA;
  const cudaError_t e = launch_profile(q, k, v, g, BH, shape->d, params->w_s, params->w_t,
                                       scale_log2_of(params->scale, shape->d), plan, scratch, d_kind, d_mse, d_err,
                                       stream);
  return e == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

}  // extern "C"
