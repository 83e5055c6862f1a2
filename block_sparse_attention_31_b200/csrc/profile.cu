// profile.cu -- online head profiling (vsa_profile_heads).
//
// "Sparse Video-Gen" summary page, "Approach": a profiling step on about 1% of the query
// rows picks, per head, the pattern (spatial or temporal) with the lower error; its
// "Measured effects" table reports 1% as the profiled share.  Reading used here: the
// sampled rows are rho_i = floor((2i+1)N/(2r)), r = ceil(frac*N); the error of a pattern
// is the mean squared difference between its output and dense attention over those rows
// and all d outputs, under the block masks that the attention kernel would execute;
// ties pick the spatial pattern.
//
// Three kernels:
//   prep     gathers the sampled Q rows of every head into a 128-row-padded tile buffer
//            and, per sampled row, the contiguous key range each pattern allows (spatial:
//            a natural-order token range; temporal: a frame-major slot range);
//   attn3    one CTA per (head, 128-row tile, key split): S = Q K^T on tcgen05 into TMEM,
//            one online softmax whose probabilities serve the dense, spatial-masked and
//            temporal-masked variants, and three P.V products into three TMEM accumulators
//            (the masked ones with rows switched off by the MMA's lane mask); the softmax runs
//            on two warpgroups, each owning one half of every row's columns; writes the
//            partial (max, sum, unnormalised O) of each variant;
//   row_error one CTA per (sampled row, head): merges the splits, forms the three outputs and
//            the row's two squared errors (fp64);
//   reduce   one CTA per head: sums the rows' errors in a fixed order and picks the kind.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

constexpr int kProfThreads = 320;  // producer, MMA issuer, two softmax warpgroups
constexpr int kPM = 128;  // rows per tile
constexpr int kNumSMs = 148;
constexpr int kMaxSplits = 16;  // key-range splits per row tile, at most
// The margin the recompute rule below guarantees: a masked variant that is not recomputed has
// its largest allowed logit within this many base-2 units of every split's dense maximum, so
// every probability the 2^-126 flush can remove is below 2^-46 of the variant's own largest one.
constexpr float kProfFlushMargin = 80.0f;
// Merged masked-variant sums below this (2^-60 of the dense maximum) trigger the recompute:
// 60 + 18 (at most 2^18 keys) stays inside kProfFlushMargin.
constexpr float kProfLowSum = 8.673617379884035e-19f;  // 2^-60
static_assert(60.0f + 18.0f < kProfFlushMargin, "low-sum threshold outside the flush margin");

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

ProfilePlan profile_plan(const Geom& g, int BH, int d, double frac) {
  ProfilePlan p{};
  long long r = static_cast<long long>(ceil(frac * static_cast<double>(g.N)));
  if (r < 1) r = 1;
  if (r > g.N) r = g.N;
  p.r = static_cast<int>(r);
  p.r_pad = (p.r + kPM - 1) / kPM * kPM;
  p.tiles = p.r_pad / kPM;
  const int nb = (g.N + g.block - 1) / g.block;
  // Key-range splits: the smallest count that fills at least one wave of 148 SMs with a last
  // wave at least 90% full; otherwise the count (up to 16) with the fullest last wave.
  const long long tiles = static_cast<long long>(BH) * p.tiles;
  auto wave_eff = [&](int s) {
    const double w = static_cast<double>(tiles * s) / kNumSMs;
    return w / std::ceil(w);
  };
  int splits = 0;
  for (int s = 1; s <= kMaxSplits && s <= nb; ++s)
    if (tiles * s >= kNumSMs && wave_eff(s) >= 0.9) {
      splits = s;
      break;
    }
  if (splits == 0) {
    splits = 1;
    for (int s = 2; s <= kMaxSplits && s <= nb; ++s)
      if (wave_eff(s) > wave_eff(splits) + 1e-9) splits = s;
  }
  p.splits = splits;
  size_t off = 0;
  p.off_qs = off;
  off = align256(off + static_cast<size_t>(BH) * p.r_pad * d * 2);
  p.off_ranges = off;
  off = align256(off + static_cast<size_t>(p.r_pad) * 4 * sizeof(int));
  p.off_order = off;
  off = align256(off + static_cast<size_t>(p.r_pad) * sizeof(int));
  p.off_opart = off;
  off = align256(off + static_cast<size_t>(BH) * splits * 3 * p.r_pad * d * sizeof(float));
  p.off_ml = off;
  off = align256(off + static_cast<size_t>(BH) * splits * 3 * p.r_pad * 2 * sizeof(float));
  p.off_rowerr = off;
  off = align256(off + static_cast<size_t>(BH) * p.r_pad * 2 * sizeof(double));
  p.bytes = off;
  return p;
}

ProfilePlan profile_plan_splits(const Geom& g, int BH, int d, double frac, int splits) {
  ProfilePlan p = profile_plan(g, BH, d, frac);
  const int nb = (g.N + g.block - 1) / g.block;
  p.splits = splits < 1 ? 1 : (splits > nb ? nb : splits);
  if (p.splits > kMaxSplits) p.splits = kMaxSplits;
  size_t off = p.off_opart;
  off = align256(off + static_cast<size_t>(BH) * p.splits * 3 * p.r_pad * d * sizeof(float));
  p.off_ml = off;
  off = align256(off + static_cast<size_t>(BH) * p.splits * 3 * p.r_pad * 2 * sizeof(float));
  p.off_rowerr = off;
  off = align256(off + static_cast<size_t>(BH) * p.r_pad * 2 * sizeof(double));
  p.bytes = off;
  return p;
}

// Contiguous range [lo, hi] of key blocks kept for query block i, groups of G slots.
// Block j spans groups [a_j, b_j]; both ends are non-decreasing in j, so the blocks kept for
// block i (max(0, a_j - b_i, a_i - b_j) <= w) are the contiguous run from the first j with
// b_j >= a_i - w to the last j with a_j <= b_i + w.  Two binary searches find it.
__device__ __forceinline__ void kept_block_range(int i, int N, int B, int G, int w, int& lo, int& hi) {
  const int nb = (N + B - 1) / B;
  const int ai = (i * B) / G, bi = (min(N, (i + 1) * B) - 1) / G;
  int l = 0, h = nb;  // first j in [0, nb) with b_j >= ai - w
  while (l < h) {
    const int m = (l + h) >> 1;
    if ((min(N, (m + 1) * B) - 1) / G >= ai - w) h = m;
    else l = m + 1;
  }
  lo = l;
  l = 0;
  h = nb;  // first j with a_j > bi + w
  while (l < h) {
    const int m = (l + h) >> 1;
    if ((m * B) / G > bi + w) h = m;
    else l = m + 1;
  }
  hi = l - 1;
}

// Order of the sampled rows inside each 128-row tile: ascending temporal slot (spatial
// position, then frame), padding rows last.  Rows that share a warp then have nearby
// temporal key ranges, so whole 32-key words of a block fall outside all of them and the
// softmax skips their temporal masking.  One CTA of 128 threads per tile; order[slot] = row.
__global__ void __launch_bounds__(kPM) profile_order_kernel(Geom g, int r, int32_t* __restrict__ order) {
  __shared__ long long key_s[kPM];
  const int p = threadIdx.x, i = blockIdx.x * kPM + p;
  long long key = (1LL << 40) + i;
  if (i < r) {
    const long long t = (static_cast<long long>(2 * i + 1) * g.N) / (2LL * r);
    key = static_cast<long long>(slot_of_token(g, kTemporal, static_cast<int>(t))) * kPM + p;
  }
  key_s[p] = key;
  __syncthreads();
  int rank = 0;
  for (int q = 0; q < kPM; ++q) rank += key_s[q] < key ? 1 : 0;  // keys are distinct
  order[blockIdx.x * kPM + rank] = i;
}

// Slot s of the sampled-row buffers holds row order[s] (profile_order_kernel).
__global__ void __launch_bounds__(256) profile_prep_kernel(const __nv_bfloat16* __restrict__ q, Geom g, int d, int r,
                                                           int r_pad, int w_s, int w_t, const int32_t* __restrict__ order,
                                                           __nv_bfloat16* __restrict__ qs, int4* __restrict__ ranges) {
  const int bh = blockIdx.y;
  const int vpr = d / 8;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int slot = idx / vpr, v = idx - (idx / vpr) * vpr;
  if (slot >= r_pad) return;
  const int i = order[slot];
  const long long t = i < r ? (static_cast<long long>(2 * i + 1) * g.N) / (2LL * r) : -1;
  uint4 val = make_uint4(0, 0, 0, 0);
  if (t >= 0) val = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<size_t>(bh) * g.N + t) * d + v * 8));
  *reinterpret_cast<uint4*>(qs + (static_cast<size_t>(bh) * r_pad + slot) * d + v * 8) = val;
  if (bh == 0 && v == 0) {
    int4 rg = make_int4(0, 0, 0, 0);
    if (t >= 0) {
      int lo, hi;
      kept_block_range(static_cast<int>(t) / g.block, g.N, g.block, g.S, w_s, lo, hi);
      rg.x = lo * g.block;
      rg.y = min(g.N, (hi + 1) * g.block);
      const int p = slot_of_token(g, kTemporal, static_cast<int>(t));
      kept_block_range(p / g.block, g.N, g.block, g.F, w_t, lo, hi);
      rg.z = lo * g.block;
      rg.w = min(g.N, (hi + 1) * g.block);
    }
    ranges[slot] = rg;
  }
}

template <int D, int BN>
struct ProfCfg {
  static constexpr int Q_BYTES = kPM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int P_BYTES = kPM * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;       // 2 stages
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;  // 2 stages
  static constexpr int OFF_PD = OFF_V + 2 * KV_BYTES; // dense P
  static constexpr int OFF_PT = OFF_PD + P_BYTES;     // temporal-masked P
  static constexpr int OFF_BAR = OFF_PT + P_BYTES;
  static constexpr int OFF_MISC = OFF_BAR + 16 * 8;
  static constexpr int BYTES = OFF_MISC + 128;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  // TMEM: S, then O of dense, spatial, temporal
  static constexpr int TMEM_S = 0, TMEM_O = BN;
  static constexpr int TMEM_COLS = (BN + 3 * D) <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(kPM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kPM, D, false, true);
};

enum { PB_Q = 0, PB_FULL_K = 1, PB_FULL_V = 3, PB_EMPTY_K = 5, PB_EMPTY_V = 7, PB_S_FULL = 9, PB_S_FREE = 10,
       PB_P_FULL = 11, PB_O_DONE = 12, PB_DRAIN = 13 };

struct ProfArgs {
  const int4* ranges;
  float* opart;
  float* ml;
  int* err;
  int r_pad, tiles, splits, per_split;
  float scale_log2;
  Geom g;
};

// Set bits [lo, hi] (inclusive, columns) of a BN-bit mask.
template <int BN>
__device__ __forceinline__ void set_bit_range(uint32_t (&m)[BN / 32], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < BN / 32; ++w) {
    const int a = max(lo - 32 * w, 0), b = min(hi - 32 * w, 31);
    if (a <= b) m[w] |= (0xffffffffu >> (31 - b)) & (0xffffffffu << a);
  }
}

// Three attention variants of 128 sampled query rows over a range of natural key blocks:
// dense, spatial (the row's kept natural blocks: whole blocks on or off) and temporal (the
// row's kept frame-major slots).  All three use the dense running max, so their
// probabilities are masked copies of the dense ones and each score is exponentiated once.
// The spatial P.V reads the dense P with the rows outside the window disabled (the MMA's
// output-lane mask); the temporal P.V reads a masked copy with rows that allow no key of the
// block disabled.  Probabilities more than 2^126 below the running dense maximum flush to
// zero; the row-error kernel detects a masked variant that could have lost weight that way
// from its merged sum and recomputes it with its own maximum.  Both P tiles live in shared
// memory so that Q.K^T of block j+1 runs while the softmax of block j computes.
template <int D, int BN>
__global__ void __launch_bounds__(kProfThreads, 1)
    profile_attn3_kernel(const __grid_constant__ CUtensorMap tqs, const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv, const ProfArgs a) {
  using C = ProfCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_u32);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  const uint32_t sPD = sbase + C::OFF_PD, sPT = sbase + C::OFF_PT;
  uint8_t* pPD = smem + C::OFF_PD;
  uint8_t* pPT = smem + C::OFF_PT;
  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* abort_flag = misc + 1;
  // per block parity: [slot][variant 0 = spatial, 1 = temporal][quad] ballots of rows using it
  volatile uint32_t* rowuse = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geom& g = a.g;
  const int split = blockIdx.x % a.splits;
  const int tile = (blockIdx.x / a.splits) % a.tiles;
  const int bh = blockIdx.x / (a.splits * a.tiles);
  const int nb = (g.N + BN - 1) / BN;
  const int kb0 = split * a.per_split;
  const int cnt = max(0, min(nb, kb0 + a.per_split) - kb0);
  bool stop = false;
  if (tid == 0) stop = (*reinterpret_cast<volatile int*>(a.err) & kDevErrTimeout) != 0;
  if (__syncthreads_or(stop)) return;

  if (tid == 0) {
    mbar_init(bar(PB_Q), 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar(PB_FULL_K + st), 1);
      mbar_init(bar(PB_FULL_V + st), 1);
      mbar_init(bar(PB_EMPTY_K + st), 1);
      mbar_init(bar(PB_EMPTY_V + st), 1);
    }
    mbar_init(bar(PB_S_FULL), 1);
    mbar_init(bar(PB_S_FREE), 256);
    mbar_init(bar(PB_P_FULL), 256);
    mbar_init(bar(PB_O_DONE), 1);
    mbar_init(bar(PB_DRAIN), 1);
    misc[1] = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  if (warp == 0) {
    if (lane == 0 && cnt > 0) {
      int nk = 0, nv = 0;
      mbar_arrive_expect_tx(bar(PB_Q), C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_3d(sQ + c * kPM * 128, &tqs, bar(PB_Q), c * 64, tile * kPM, bh);
      for (int j = 0; j < cnt; ++j) {
        const int kb = kb0 + j, st = j & 1;
        const uint32_t u = j >> 1;
        if (j >= 2 && !mbar_wait(bar(PB_EMPTY_K + st), (u - 1) & 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(bar(PB_FULL_K + st), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sK + st * C::KV_BYTES + c * BN * 128, &tk, bar(PB_FULL_K + st), c * 64, kb * BN, bh);
        nk = j + 1;
        if (j >= 2 && !mbar_wait(bar(PB_EMPTY_V + st), (u - 1) & 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(bar(PB_FULL_V + st), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sV + st * C::KV_BYTES + c * BN * 128, &tv, bar(PB_FULL_V + st), c * 64, kb * BN, bh);
        nv = j + 1;
      }
      if (*abort_flag) {
        mbar_wait_drain(bar(PB_Q), 0, a.err);
        for (int st = 0; st < 2; ++st) {
          int lk = -1, lv = -1;
          for (int j = st; j < nk; j += 2) lk = j;
          for (int j = st; j < nv; j += 2) lv = j;
          if (lk >= 0) mbar_wait_drain(bar(PB_FULL_K + st), (lk >> 1) & 1, a.err);
          if (lv >= 0) mbar_wait_drain(bar(PB_FULL_V + st), (lv >> 1) & 1, a.err);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && cnt > 0) {
      const uint64_t dq = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024), dk1 = sdesc_sw128(sK + C::KV_BYTES, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, BN * 128, 1024), dv1 = sdesc_sw128(sV + C::KV_BYTES, BN * 128, 1024);
      const uint64_t dpd = sdesc_sw128(sPD, 16, 1024), dpt = sdesc_sw128(sPT, 16, 1024);
      auto issue_qk = [&](int j) -> bool {
        if (!mbar_wait(bar(PB_FULL_K + (j & 1)), (j >> 1) & 1, abort_flag, a.err)) return false;
        if (j >= 1 && !mbar_wait(bar(PB_S_FREE), (j - 1) & 1, abort_flag, a.err)) return false;
        tc_fence_after();
        const uint64_t kd = (j & 1) ? dk1 : dk0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma_ss(tmem + C::TMEM_S, dq + static_cast<uint64_t>(((kk >> 2) * (kPM * 128) + (kk & 3) * 32) / 16),
                    kd + static_cast<uint64_t>(((kk >> 2) * (BN * 128) + (kk & 3) * 32) / 16), C::IDESC_QK,
                    kk > 0 ? 1u : 0u);
        tc_commit(bar(PB_EMPTY_K + (j & 1)));
        tc_commit(bar(PB_S_FULL));
        return true;
      };
      auto issue_pv = [&](int jp) -> bool {
        if (!mbar_wait(bar(PB_P_FULL), jp & 1, abort_flag, a.err)) return false;
        if (!mbar_wait(bar(PB_FULL_V + (jp & 1)), (jp >> 1) & 1, abort_flag, a.err)) return false;
        uint32_t dis_sp[4], dis_tp[4];
        uint32_t any_sp = 0u, any_tp = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t us = rowuse[(jp & 1) * 8 + q], ut = rowuse[(jp & 1) * 8 + 4 + q];
          dis_sp[q] = ~us;
          dis_tp[q] = ~ut;
          any_sp |= us;
          any_tp |= ut;
        }
        tc_fence_after();
        const uint64_t vd = (jp & 1) ? dv1 : dv0;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t poff = static_cast<uint64_t>(((kk >> 2) * (kPM * 128) + (kk & 3) * 32) / 16);
          tc_mma_ss(tmem + C::TMEM_O, dpd + poff, vd + static_cast<uint64_t>(kk * 16 * 128 / 16), C::IDESC_PV,
                    (jp > 0 || kk > 0) ? 1u : 0u);
        }
        if (any_sp) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t poff = static_cast<uint64_t>(((kk >> 2) * (kPM * 128) + (kk & 3) * 32) / 16);
            tc_mma_ss_masked(tmem + C::TMEM_O + D, dpd + poff, vd + static_cast<uint64_t>(kk * 16 * 128 / 16),
                             C::IDESC_PV, dis_sp, 1u);
          }
        }
        if (any_tp) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t poff = static_cast<uint64_t>(((kk >> 2) * (kPM * 128) + (kk & 3) * 32) / 16);
            tc_mma_ss_masked(tmem + C::TMEM_O + 2 * D, dpt + poff, vd + static_cast<uint64_t>(kk * 16 * 128 / 16),
                             C::IDESC_PV, dis_tp, 1u);
          }
        }
        tc_commit(bar(PB_EMPTY_V + (jp & 1)));
        tc_commit(bar(PB_O_DONE));
        return true;
      };
      bool ok = mbar_wait(bar(PB_Q), 0, abort_flag, a.err) && issue_qk(0);
      for (int j = 0; ok && j < cnt; ++j) {
        // Q.K^T of the next block first: it overlaps this block's softmax
        if (j + 1 < cnt && !issue_qk(j + 1)) {
          ok = false;
          break;
        }
        if (!issue_pv(j)) ok = false;
      }
      tc_commit(bar(PB_DRAIN));
      mbar_wait_drain(bar(PB_DRAIN), 0, a.err);
    }
    __syncwarp();
  } else {
    // Two softmax warpgroups split every S row by columns: warp w (2..9) serves the TMEM lane
    // quarter w % 4 and the column half h = (w - 2) / 4.  Both threads of a row read the whole
    // row for its maximum (so they take the same rescale decisions without exchanging
    // anything), exponentiate their own half, write their half of each P tile and keep partial
    // sums, which are added at the end (half 0 + half 1).
    constexpr int HB = BN / 2;
    const int quad = warp & 3, half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const int c_own = half * HB;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t t_s = t_lane + C::TMEM_S, t_o = t_lane + C::TMEM_O;
    const float sl2 = a.scale_log2;
    // Allowed keys of this row: spatial = natural tokens [rg.x, rg.y) (whole blocks),
    // temporal = frame-major slots [rg.z, rg.w), i.e. (s, f) from (ts_lo, tf_lo) to (ts_hi, tf_hi).
    const int4 rg = a.ranges[tile * kPM + row];
    const bool t_any = rg.w > rg.z;
    const int ts_lo = rg.z / g.F, tf_lo = rg.z - (rg.z / g.F) * g.F;
    const int ts_hi = t_any ? (rg.w - 1) / g.F : -1, tf_hi = t_any ? (rg.w - 1) - ((rg.w - 1) / g.F) * g.F : -1;
    float m = -INFINITY, l[3] = {0.f, 0.f, 0.f};
    {  // the spatial and temporal accumulators only ever accumulate: start them at zero
      float z[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) z[x] = 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) tmem_st32(t_o + D + half * D + c * 32, z);
    }
    bool ok = true;
    for (int j = 0; j < cnt; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(PB_S_FULL), j & 1, abort_flag, a.err));
      if (!ok) break;
      tc_fence_after();
      // both halves of the row: this thread's own, and the other one for the row maximum only
      // (reading it costs less than exchanging partial maxima between the warps)
      uint32_t rs_own[HB], rs_oth[HB];
#pragma unroll
      for (int c = 0; c < HB / 32; ++c) {
        tmem_ld32_async(t_s + c_own + c * 32, rs_own + c * 32);
        tmem_ld32_async(t_s + (HB - c_own) + c * 32, rs_oth + c * 32);
      }
      tmem_wait_ld();
      reg_fence<HB>(rs_own);
      reg_fence<HB>(rs_oth);
      tc_fence_before();
      mbar_arrive(bar(PB_S_FREE));  // S may be overwritten by the next block's Q.K^T
      const int t0 = (kb0 + j) * BN;
      const int nvalid = min(BN, g.N - t0);
      float s[HB], so[HB];
#pragma unroll
      for (int c = 0; c < HB; ++c) {
        s[c] = __uint_as_float(rs_own[c]);
        so[c] = __uint_as_float(rs_oth[c]);
      }
      if (nvalid < BN) {  // the ragged last block
#pragma unroll
        for (int c = 0; c < HB; ++c) {
          if (c_own + c >= nvalid) s[c] = -INFINITY;
          if (HB - c_own + c >= nvalid) so[c] = -INFINITY;
        }
      }
      float mx8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) mx8[x] = fmax3(s[2 * x], s[2 * x + 1], so[2 * x]);
#pragma unroll
      for (int x = 0; x < 8; ++x) mx8[x] = fmax3(mx8[x], so[2 * x + 1], -INFINITY);
#pragma unroll
      for (int c = 16; c < HB; c += 2) {
        mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], s[c], s[c + 1]);
        mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], so[c], so[c + 1]);
      }
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      const float m_new = fmaxf(m, mx * sl2);
      const bool grow = m_new > m + kRescaleLog2;
      // masks: spatial whole block; temporal as contiguous column ranges per frame segment
      // (the whole row, so both halves know whether the row uses the temporal P tile)
      const bool sp_on = t0 >= rg.x && t0 < rg.y;
      // this half's temporal mask words (bit c = own column c); tp_on: the row has a temporal
      // key anywhere in the block (both halves compute it the same way)
      uint32_t mh[HB / 32];
#pragma unroll
      for (int w = 0; w < HB / 32; ++w) mh[w] = 0u;
      bool tp_on = false;
      if (t_any) {
        int f = t0 / g.S, s0 = t0 - (t0 / g.S) * g.S;
        for (int c = 0; c < nvalid;) {
          const int seg = min(nvalid - c, g.S - s0);
          const int lo_s = ts_lo + (f < tf_lo ? 1 : 0), hi_s = ts_hi - (f > tf_hi ? 1 : 0);
          const int x0 = max(lo_s, s0), x1 = min(hi_s, s0 + seg - 1);
          if (x0 <= x1) {
            tp_on = true;
            set_bit_range<HB>(mh, c + x0 - s0 - c_own, c + x1 - s0 - c_own);
          }
          c += seg;
          ++f;
          s0 = 0;
        }
      }
      // Exponentials of this half first, into registers (packed bf16 pairs): this overlaps the
      // previous block's P.V products, which still read the P tiles.
      const float m_next = grow ? m_new : m;
      const float m_use = m_next == -INFINITY ? 0.f : m_next;
      const bool warp_tp = __any_sync(0xffffffffu, tp_on);
      const uint64_t sl2x2 = f2_make(sl2, sl2), negm2 = f2_make(-m_use, -m_use);
      uint64_t rs2[2] = {0ull, 0ull};
      uint64_t rt2[2] = {0ull, 0ull};
      uint32_t pk[HB / 2], pt[HB / 2];  // packed P and its temporal-masked copy
#pragma unroll
      for (int w = 0; w < HB / 32; ++w) {
        // one branch per 32-key word: the masking runs only where some row of the warp has
        // a temporal key
        if (__any_sync(0xffffffffu, mh[w] != 0u)) {
#pragma unroll
          for (int c = 16 * w; c < 16 * w + 16; ++c) {
            const uint64_t x = f2_fma(f2_make(s[2 * c], s[2 * c + 1]), sl2x2, negm2);
            float x0, x1;
            f2_split(x, x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            rs2[c & 1] = f2_add(rs2[c & 1], f2_make(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
            const uint32_t b = (mh[w] >> ((2 * c) & 31)) & 3u;
            const float q0 = (b & 1u) ? p0 : 0.f, q1 = (b & 2u) ? p1 : 0.f;  // temporal-masked pair
            rt2[c & 1] = f2_add(rt2[c & 1], f2_make(q0, q1));
            pt[c] = pack_bf16x2(q0, q1);
          }
        } else {
#pragma unroll
          for (int c = 16 * w; c < 16 * w + 16; ++c) {
            const uint64_t x = f2_fma(f2_make(s[2 * c], s[2 * c + 1]), sl2x2, negm2);
            float x0, x1;
            f2_split(x, x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            rs2[c & 1] = f2_add(rs2[c & 1], f2_make(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
            pt[c] = 0u;
          }
        }
      }
      // the previous block's P.V products must be done: O stable, P tiles free
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(PB_O_DONE), (j - 1) & 1, abort_flag, a.err));
        if (!ok) break;
        tc_fence_after();
      }
      if (j > 0 && __any_sync(0xffffffffu, grow && m != -INFINITY)) {
        // this half rescales its 3D/2 of the three accumulators' columns
        const float alpha = grow ? fast_exp2(m - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 3 * D / 64; ++c) {
          float o[32];
          const uint32_t col = static_cast<uint32_t>(half * (3 * D / 2) + c * 32);
          tmem_ld32(t_o + col, o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] *= alpha;
          tmem_st32(t_o + col, o);
        }
      }
      if (grow) {
        const float alpha = fast_exp2(m - m_new);
        l[0] *= alpha;
        l[1] *= alpha;
        l[2] *= alpha;
        m = m_new;
      }
      // 8 probabilities -> one 16-byte chunk of each P tile; the temporal tile is written for
      // every row of a warp with some temporal key (rows without one are switched off in the
      // temporal P.V)
#pragma unroll
      for (int ch = 0; ch < HB / 8; ++ch) {
        const int gch = half * (HB / 8) + ch;
        const int off = (gch >> 3) * (kPM * 128) + row * 128 + (((gch & 7) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(pPD + off) = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      if (warp_tp) {
#pragma unroll
        for (int ch = 0; ch < HB / 8; ++ch) {
          const int gch = half * (HB / 8) + ch;
          const int off = (gch >> 3) * (kPM * 128) + row * 128 + (((gch & 7) ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(pPT + off) = make_uint4(pt[4 * ch], pt[4 * ch + 1], pt[4 * ch + 2], pt[4 * ch + 3]);
        }
      }
      float rs0, rs1;
      f2_split(f2_add(rs2[0], rs2[1]), rs0, rs1);
      const float rs = rs0 + rs1;
      float rt0, rt1;
      f2_split(f2_add(rt2[0], rt2[1]), rt0, rt1);
      const float rt = rt0 + rt1;
      l[0] += rs;
      if (sp_on) l[1] += rs;
      l[2] += rt;
      const uint32_t bs = __ballot_sync(0xffffffffu, sp_on), bt = __ballot_sync(0xffffffffu, tp_on);
      if (lane == 0 && half == 0) {
        rowuse[(j & 1) * 8 + quad] = bs;
        rowuse[(j & 1) * 8 + 4 + quad] = bt;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(PB_P_FULL));
    }
    if (ok && cnt > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(PB_O_DONE), (cnt - 1) & 1, abort_flag, a.err));
      tc_fence_after();
    }
    const bool have = ok && cnt > 0;
    // the halves' partial sums, added as half 0 + half 1 (the last P.V has read the dense P
    // tile, which now holds half 1's sums)
    float* lx = reinterpret_cast<float*>(pPD);
    if (half == 1) {
#pragma unroll
      for (int vv = 0; vv < 3; ++vv) lx[vv * kPM + row] = have ? l[vv] : 0.f;
    }
    named_barrier_sync(1, 8 * 32);
    if (half == 0) {
#pragma unroll
      for (int vv = 0; vv < 3; ++vv) l[vv] += lx[vv * kPM + row];
    }
    // partials: (m, l) and unnormalised O of each variant (m is the dense max for all three);
    // each half writes its D/2 output columns
    const size_t base = ((static_cast<size_t>(bh) * a.splits + split) * 3) * a.r_pad + tile * kPM + row;
#pragma unroll
    for (int vv = 0; vv < 3; ++vv) {
      const size_t prow = base + static_cast<size_t>(vv) * a.r_pad;
      if (half == 0) {
        a.ml[prow * 2 + 0] = have ? m : -INFINITY;
        a.ml[prow * 2 + 1] = have ? l[vv] : 0.f;
      }
      float4* dst = reinterpret_cast<float4*>(a.opart + prow * D + half * (D / 2));
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        float o[32];
        if (have) {
          tmem_ld32(t_o + vv * D + half * (D / 2) + c * 32, o);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = 0.f;
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) dst[c * 8 + x] = make_float4(o[4 * x], o[4 * x + 1], o[4 * x + 2], o[4 * x + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Output x of one masked variant of sampled row i recomputed with the variant's own maximum
// (used when a split marked the variant: its allowed logits sit far below the dense maximum).
// The d threads of the CTA form d/32 warps; each warp takes every (d/32)-th allowed key, its
// lanes hold d/32 dimensions each and reduce q.k with shuffles.  Two passes: the maximum, then the
// exponentials, their sum and sum p*v.  Spatial keys are the natural tokens [lo, hi);
// temporal keys the frame-major slots [lo, hi), slot p being token (p % F) * S + p / F.
__device__ float profile_variant_exact(const __nv_bfloat16* __restrict__ qrow, const __nv_bfloat16* __restrict__ kh,
                                       const __nv_bfloat16* __restrict__ vh, int lo, int hi, bool frame_major,
                                       const Geom& g, int d, float scale_log2) {
  __shared__ float red_m[4], red_l[4];
  __shared__ float red_o[4][128];
  const int x = threadIdx.x, warp = x >> 5, lane = x & 31, nw = blockDim.x >> 5;  // nw = d / 32
  const int per = d / 32;  // dimensions per lane (2 or 4)
  float qv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) qv[e] = e < per ? __bfloat162float(qrow[lane * per + e]) : 0.f;
  auto logit = [&](int slot) -> float {
    const int t = frame_major ? (slot % g.F) * g.S + slot / g.F : slot;
    const __nv_bfloat16* kr = kh + static_cast<size_t>(t) * d + lane * per;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < per) acc = fmaf(qv[e], __bfloat162float(kr[e]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    return acc * scale_log2;
  };
  float mx = -INFINITY;
  for (int u = lo + warp; u < hi; u += nw) mx = fmaxf(mx, logit(u));
  if (lane == 0) red_m[warp] = mx;
  __syncthreads();
  float M = red_m[0];
  for (int w = 1; w < nw; ++w) M = fmaxf(M, red_m[w]);
  float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  if (M != -INFINITY)
    for (int u = lo + warp; u < hi; u += nw) {
      const float p = exp2f(logit(u) - M);
      L += p;
      const int t = frame_major ? (u % g.F) * g.S + u / g.F : u;
      const __nv_bfloat16* vr = vh + static_cast<size_t>(t) * d + lane * per;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e < per) o[e] = fmaf(p, __bfloat162float(vr[e]), o[e]);
    }
  if (lane == 0) red_l[warp] = L;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (e < per) red_o[warp][lane * per + e] = o[e];
  __syncthreads();
  float Lt = 0.f, ot = 0.f;
  for (int w = 0; w < nw; ++w) {
    Lt += red_l[w];
    ot += red_o[w][x];
  }
  __syncthreads();  // the shared partials may be reused by the next call
  return Lt > 0.f ? ot / Lt : 0.f;
}

// Merge the key splits of one sampled row of one head and accumulate its two squared errors
// (one CTA of d threads per (row, head)); the per-row sums are reduced in fixed order below.
// Every split's sums are based on its dense max md.  A masked variant's merged sum L, taken
// against the largest md, is at least 2^(M_v - max md) with M_v the variant's largest logit
// (base 2), and at most its key count times that.  When L >= kProfLowSum, M_v lies within
// -log2(kProfLowSum) + 18 < kProfFlushMargin of every split's md, so no probability above
// 2^-46 of the variant's own maximum was flushed; otherwise the variant of this row is
// recomputed with its own maximum.
__global__ void __launch_bounds__(128) profile_row_error_kernel(const float* __restrict__ opart,
                                                                const float* __restrict__ ml, int r_pad,
                                                                int splits, int d, double* __restrict__ row_err,
                                                                const __nv_bfloat16* __restrict__ qs,
                                                                const __nv_bfloat16* __restrict__ k,
                                                                const __nv_bfloat16* __restrict__ v,
                                                                const int4* __restrict__ ranges, Geom g,
                                                                float scale_log2) {
  __shared__ double red[2][4];
  const int i = blockIdx.x, bh = blockIdx.y, x = threadIdx.x;
  float o[3];
#pragma unroll
  for (int vv = 0; vv < 3; ++vv) {
    // all splits' partials are loaded before they are combined (at most kMaxSplits)
    float ms[kMaxSplits], ls[kMaxSplits], os[kMaxSplits];
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) {
      ms[sp] = -INFINITY;
      ls[sp] = os[sp] = 0.f;
      if (sp < splits) {
        const size_t prow = ((static_cast<size_t>(bh) * splits + sp) * 3 + vv) * r_pad + i;
        ms[sp] = __ldg(ml + prow * 2);
        ls[sp] = __ldg(ml + prow * 2 + 1);
        os[sp] = __ldg(opart + prow * d + x);
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) M = fmaxf(M, ms[sp]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) {
      if (ms[sp] == -INFINITY) continue;
      const float w = exp2f(ms[sp] - M);
      L += ls[sp] * w;
      acc += os[sp] * w;
    }
    if (vv > 0 && !(L >= kProfLowSum)) {  // uniform across the CTA: every thread read the same sums
      const int4 rg = ranges[i];
      const bool tp = vv == 2;
      o[vv] = profile_variant_exact(qs + (static_cast<size_t>(bh) * r_pad + i) * d,
                                    k + static_cast<size_t>(bh) * g.N * d, v + static_cast<size_t>(bh) * g.N * d,
                                    tp ? rg.z : rg.x, tp ? rg.w : rg.y, tp, g, d, scale_log2);
      continue;
    }
    o[vv] = L > 0.f ? acc / L : 0.f;
  }
  const double ds = static_cast<double>(o[1]) - o[0], dt = static_cast<double>(o[2]) - o[0];
  double es = ds * ds, et = dt * dt;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    es += __shfl_xor_sync(0xffffffffu, es, off);
    et += __shfl_xor_sync(0xffffffffu, et, off);
  }
  if ((x & 31) == 0) {
    red[0][x >> 5] = es;
    red[1][x >> 5] = et;
  }
  __syncthreads();
  if (x == 0) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < d / 32; ++w) {
      a += red[0][w];
      b += red[1][w];
    }
    row_err[(static_cast<size_t>(bh) * r_pad + i) * 2 + 0] = a;
    row_err[(static_cast<size_t>(bh) * r_pad + i) * 2 + 1] = b;
  }
}

constexpr int kRedThreads = 256;

// Sum the per-row errors of one head in a fixed order, form the two MSEs, pick the kind.
__global__ void __launch_bounds__(kRedThreads) profile_reduce_kernel(const double* __restrict__ row_err, int r,
                                                                     int r_pad, int d, uint8_t* __restrict__ kinds,
                                                                     float* __restrict__ mse) {
  __shared__ double red[2][kRedThreads];
  const int bh = blockIdx.x;
  double es = 0.0, et = 0.0;
  for (int i = threadIdx.x; i < r; i += kRedThreads) {
    es += row_err[(static_cast<size_t>(bh) * r_pad + i) * 2 + 0];
    et += row_err[(static_cast<size_t>(bh) * r_pad + i) * 2 + 1];
  }
  red[0][threadIdx.x] = es;
  red[1][threadIdx.x] = et;
  __syncthreads();
  for (int off = kRedThreads / 2; off > 0; off >>= 1) {
    if (threadIdx.x < off) {
      red[0][threadIdx.x] += red[0][threadIdx.x + off];
      red[1][threadIdx.x] += red[1][threadIdx.x + off];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double n = static_cast<double>(r) * d;
    const double ms = red[0][0] / n, mt = red[1][0] / n;
    mse[bh * 2 + 0] = static_cast<float>(ms);
    mse[bh * 2 + 1] = static_cast<float>(mt);
    kinds[bh] = mt < ms ? kTemporal : kSpatial;
  }
}

template <int D, int BN>
static cudaError_t launch_prof_attn(const CUtensorMap& tqs, const CUtensorMap& tk, const CUtensorMap& tv,
                                    const ProfArgs& pa, int BH, cudaStream_t stream) {
  using C = ProfCfg<D, BN>;
  auto kern = profile_attn3_kernel<D, BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(BH) * pa.tiles * pa.splits;
  kern<<<grid, kProfThreads, C::SMEM_ALLOC, stream>>>(tqs, tk, tv, pa);
  return cudaGetLastError();
}

cudaError_t launch_profile(const void* q, const void* k, const void* v, const Geom& g, int BH, int d, int w_s,
                           int w_t, float scale_log2, const ProfilePlan& plan, void* ws, uint8_t* kinds_out,
                           float* mse_out, int* err, cudaStream_t stream) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(w + plan.off_qs);
  int4* ranges = reinterpret_cast<int4*>(w + plan.off_ranges);
  int32_t* order = reinterpret_cast<int32_t*>(w + plan.off_order);
  float* opart = reinterpret_cast<float*>(w + plan.off_opart);
  float* ml = reinterpret_cast<float*>(w + plan.off_ml);
  if (plan.splits < 1 || plan.splits > kMaxSplits) return cudaErrorInvalidValue;
  {
    const int vpr = d / 8;
    profile_order_kernel<<<plan.tiles, kPM, 0, stream>>>(g, plan.r, order);
    dim3 grid((plan.r_pad * vpr + 255) / 256, BH);
    profile_prep_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q), g, d, plan.r, plan.r_pad,
                                                  w_s, w_t, order, qs, ranges);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tqs, tk, tv;
  cudaError_t e = encode_rows_map(&tqs, qs, d, plan.r_pad, BH, kPM);
  if (e == cudaSuccess) e = encode_rows_map(&tk, k, d, g.N, BH, g.block);
  if (e == cudaSuccess) e = encode_rows_map(&tv, v, d, g.N, BH, g.block);
  if (e != cudaSuccess) return e;
  ProfArgs pa;
  pa.ranges = ranges;
  pa.opart = opart;
  pa.ml = ml;
  pa.err = err;
  pa.r_pad = plan.r_pad;
  pa.tiles = plan.tiles;
  pa.splits = plan.splits;
  const int nb = (g.N + g.block - 1) / g.block;
  pa.per_split = (nb + plan.splits - 1) / plan.splits;
  pa.scale_log2 = scale_log2;
  pa.g = g;
  if (d == 128 && g.block == 128) e = launch_prof_attn<128, 128>(tqs, tk, tv, pa, BH, stream);
  else if (d == 64 && g.block == 128) e = launch_prof_attn<64, 128>(tqs, tk, tv, pa, BH, stream);
  else if (d == 128 && g.block == 64) e = launch_prof_attn<128, 64>(tqs, tk, tv, pa, BH, stream);
  else if (d == 64 && g.block == 64) e = launch_prof_attn<64, 64>(tqs, tk, tv, pa, BH, stream);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  double* row_err = reinterpret_cast<double*>(w + plan.off_rowerr);
  profile_row_error_kernel<<<dim3(plan.r, BH), d, 0, stream>>>(opart, ml, plan.r_pad, plan.splits, d, row_err, qs,
                                                                static_cast<const __nv_bfloat16*>(k),
                                                                static_cast<const __nv_bfloat16*>(v), ranges, g,
                                                                scale_log2);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  profile_reduce_kernel<<<BH, kRedThreads, 0, stream>>>(row_err, plan.r, plan.r_pad, d, kinds_out, mse_out);
  return cudaGetLastError();
}

}  // namespace vsa
