// attn.cu -- block-sparse attention forward (vsa_sparse_attn_fwd) for sm_100a.
//
// For a query block i of head (b, h): O_i = softmax(Q_i K_J^T * scale) V_J with J the kept
// key blocks kv_idx[b,h,i,0..cnt) ("OSP-Next" page, "Method": sparse attention that stays
// compatible with FlashAttention kernels; "Sparse Video-Gen" summary, "Approach": block-wise
// spatial and temporal masks).  Online softmax in the base-2 domain, fp32 accumulation.
//
// One CTA per (head, query block), 192 threads in three roles:
//   warp 0  (one lane)  TMA producer: Q once, then K_j and V_j into a 2-stage ring
//   warp 1  (one lane)  tcgen05 issuer: S = Q K_j^T into a double-buffered TMEM tile,
//                       O += P_j V_j into a TMEM accumulator; warp 1 also owns TMEM
//   warps 2-5           softmax: one query row per thread (TMEM lane = row); reads S from
//                       TMEM, rescales O in TMEM when the running max grows, writes
//                       P = exp2(S*scale*log2e - m) as bf16 into shared memory, and at the
//                       end normalises O and stores it through shared memory with TMA
//
// All operand tiles use the 128-byte swizzle (TMA SWIZZLE_128B == UMMA SWIZZLE_128B):
// a tile of R rows x 64 bf16 is R*128 bytes, 16-byte chunk c of row r at ((c ^ r%8)*16).
// QK^T: A = Q (K-major), B = K (K-major).  PV: A = P (K-major over keys), B = V (MN-major:
// keys are rows, d contiguous).  Every wait is bounded; on a timeout the CTA raises its
// abort flag, drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

constexpr int kAttnThreads = 192;
constexpr int kBM = 128;  // MMA M: query rows per tile

template <int D, int BN>
struct AttnCfg {
  static constexpr int NS = 2;  // K/V ring stages
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int P_BYTES = kBM * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int NBAR = 16;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int SMEM_ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr int TMEM_S0 = 0, TMEM_S1 = BN, TMEM_O = 2 * BN;
  static constexpr int TMEM_COLS = (2 * BN + D) <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(kBM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kBM, D, false, true);
};

// Barrier slots.
enum {
  B_Q = 0,
  B_FULL_K = 1,   // +stage
  B_FULL_V = 3,   // +stage
  B_EMPTY_K = 5,  // +stage
  B_EMPTY_V = 7,  // +stage
  B_S_FULL = 9,   // +buffer
  B_S_FREE = 11,  // +buffer
  B_P_FULL = 13,
  B_O_DONE = 14,
  B_DRAIN = 15
};

// Validity of the key columns of block kb for one head: a ragged tail (natural and
// frame-major layouts) or cube padding slots are not real tokens.
template <int BN>
__device__ __forceinline__ void key_valid_bits(const Geom& g, int kind, int kb, uint32_t (&vb)[BN / 32]) {
#pragma unroll
  for (int w = 0; w < BN / 32; ++w) {
    uint32_t m = 0;
    for (int c = 0; c < 32; ++c) {
      const int slot = kb * BN + w * 32 + c;
      bool ok;
      if (kind == kCube)
        ok = token_of_slot(g, kCube, slot) >= 0;
      else
        ok = slot < g.N;
      m |= (ok ? 1u : 0u) << c;
    }
    vb[w] = m;
  }
}

template <int D, int BN>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tq_n, const __grid_constant__ CUtensorMap tk_n,
                           const __grid_constant__ CUtensorMap tv_n, const __grid_constant__ CUtensorMap to_n,
                           const __grid_constant__ CUtensorMap tq_p, const __grid_constant__ CUtensorMap tk_p,
                           const __grid_constant__ CUtensorMap tv_p, const __grid_constant__ CUtensorMap to_p,
                           const AttnArgs a) {
  using C = AttnCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_u32);
  const uint32_t sQ = sbase + C::OFF_Q, sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sP = sbase + C::OFF_P;
  uint8_t* pP = smem + C::OFF_P;
  uint8_t* pQ = smem + C::OFF_Q;
  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  // misc[0]: TMEM base address, misc[1]: abort flag, misc[2]: bad-list flag
  volatile int* abort_flag = misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Geom& g = a.g;
  const int bh = blockIdx.x / g.nblk;
  const int qb = blockIdx.x - bh * g.nblk;
  const int kind = a.kinds[bh];
  if (kind > kCube) {
    if (tid == 0 && qb == 0) atomicOr(a.err, kDevErrKind);
    return;
  }
  const int rows = layout_rows(g, kind);
  const int nb_head = (rows + BN - 1) / BN;
  if (qb >= nb_head) return;
  const bool use_perm = a.has_perm && kind != kSpatial;
  const CUtensorMap* tq = use_perm ? &tq_p : &tq_n;
  const CUtensorMap* tk = use_perm ? &tk_p : &tk_n;
  const CUtensorMap* tv = use_perm ? &tv_p : &tv_n;
  const CUtensorMap* to = use_perm ? &to_p : &to_n;
  float* lse = use_perm ? a.lse_perm : a.lse_nat;
  const int lse_stride = use_perm ? g.R : a.nat_rows;

  // ---- validate this row's list ----
  const size_t mrow = static_cast<size_t>(bh) * g.nblk + qb;
  const int32_t* kvl = a.kv_idx + mrow * a.max_kv;
  int cnt = a.kv_cnt[mrow];
  bool bad = cnt < 0 || cnt > a.max_kv;
  if (!bad)
    for (int j = tid; j < cnt; j += kAttnThreads) {
      const int kb = kvl[j];
      bad |= kb < 0 || kb >= nb_head;
    }
  bool stop = false;  // drain quickly once some CTA has timed out
  if (tid == 0) stop = (*reinterpret_cast<volatile int*>(a.err) & kDevErrTimeout) != 0;
  if (__syncthreads_or(stop)) return;
  bad = __syncthreads_or(bad);
  if (bad) {
    if (tid == 0) atomicOr(a.err, kDevErrKvRange);
    cnt = 0;
  }

  // ---- setup: barriers and TMEM ----
  if (tid == 0) {
    mbar_init(bar(B_Q), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(B_FULL_K + s), 1);
      mbar_init(bar(B_FULL_V + s), 1);
      mbar_init(bar(B_EMPTY_K + s), 1);
      mbar_init(bar(B_EMPTY_V + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_S_FULL + s), 1);
      mbar_init(bar(B_S_FREE + s), 128);
    }
    mbar_init(bar(B_P_FULL), 128);
    mbar_init(bar(B_O_DONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    misc[1] = 0;
    mbar_init_fence();
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tk);
    tma_prefetch_desc(tv);
    tma_prefetch_desc(to);
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
    // ================= TMA producer =================
    if (lane == 0 && cnt > 0) {
      int issued = 0;
      mbar_arrive_expect_tx(bar(B_Q), C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_3d(sQ + c * kBM * 128, tq, bar(B_Q), c * 64, qb * BN, bh);
      for (int j = 0; j < cnt; ++j) {
        const int s = j % C::NS;
        const uint32_t u = j / C::NS;
        const int kb = kvl[j];
        if (j >= C::NS && !mbar_wait(bar(B_EMPTY_K + s), (u - 1) & 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(bar(B_FULL_K + s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sK + s * C::KV_BYTES + c * BN * 128, tk, bar(B_FULL_K + s), c * 64, kb * BN, bh);
        if (j >= C::NS && !mbar_wait(bar(B_EMPTY_V + s), (u - 1) & 1, abort_flag, a.err)) {
          // K of this stage is in flight; account for it on the drain path below
          issued = -(j + 1);
          break;
        }
        mbar_arrive_expect_tx(bar(B_FULL_V + s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sV + s * C::KV_BYTES + c * BN * 128, tv, bar(B_FULL_V + s), c * 64, kb * BN, bh);
        issued = j + 1;
      }
      if (*abort_flag) {
        // Drain: wait for every copy this thread issued that nobody may have consumed.
        mbar_wait_drain(bar(B_Q), 0, a.err);
        const int nk = issued >= 0 ? issued : -issued;        // K copies issued
        const int nv = issued >= 0 ? issued : -issued - 1;    // V copies issued
        for (int s = 0; s < C::NS; ++s) {
          // last use of stage s among the first nk (nv) iterations
          int lk = -1, lv = -1;
          for (int j = s; j < nk; j += C::NS) lk = j;
          for (int j = s; j < nv; j += C::NS) lv = j;
          if (lk >= 0) mbar_wait_drain(bar(B_FULL_K + s), (lk / C::NS) & 1, a.err);
          if (lv >= 0) mbar_wait_drain(bar(B_FULL_V + s), (lv / C::NS) & 1, a.err);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================= tcgen05 issuer =================
    if (lane == 0 && cnt > 0) {
      auto issue_pv = [&](int jp) -> bool {
        const int sp = jp % C::NS;
        if (!mbar_wait(bar(B_P_FULL), jp & 1, abort_flag, a.err)) return false;
        if (!mbar_wait(bar(B_FULL_V + sp), (jp / C::NS) & 1, abort_flag, a.err)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sP + (kk >> 2) * (kBM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sV + sp * C::KV_BYTES + kk * 16 * 128, BN * 128, 1024);
          tc_mma_ss(tmem + C::TMEM_O, ad, bd, C::IDESC_PV, (jp > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_EMPTY_V + sp));
        tc_commit(bar(B_O_DONE));
        return true;
      };
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, a.err);
      for (int j = 0; ok && j < cnt; ++j) {
        const int s = j % C::NS, sb = j & 1;
        if (!mbar_wait(bar(B_FULL_K + s), (j / C::NS) & 1, abort_flag, a.err)) {
          ok = false;
          break;
        }
        if (j >= 2 && !mbar_wait(bar(B_S_FREE + sb), ((j - 2) >> 1) & 1, abort_flag, a.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * (kBM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(sK + s * C::KV_BYTES + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16, 1024);
          tc_mma_ss(tmem + (sb ? C::TMEM_S1 : C::TMEM_S0), ad, bd, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_EMPTY_K + s));
        tc_commit(bar(B_S_FULL + sb));
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_pv(cnt - 1);
      // Drain: all MMAs issued by this thread complete before TMEM is released.
      tc_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0, a.err);
    }
    __syncwarp();
  } else {
    // ================= softmax (warps 2..5, one row per thread) =================
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;  // query row within the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < cnt; ++j) {
      const int sb = j & 1;
      ok = mbar_wait(bar(B_S_FULL + sb), (j >> 1) & 1, abort_flag, a.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_lane + (sb ? C::TMEM_S1 : C::TMEM_S0) + c * 32, s + c * 32);
      tc_fence_before();
      mbar_arrive(bar(B_S_FREE + sb));
      const int kb = kvl[j];
      if (!block_full(g, kind, kb)) {
        uint32_t vb[BN / 32];
        key_valid_bits<BN>(g, kind, kb, vb);
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (!((vb[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m, mx * sl2);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      if (j >= 1) {
        ok = mbar_wait(bar(B_O_DONE), (j - 1) & 1, abort_flag, a.err);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float alpha = fast_exp2(m - m_use);
        if (__any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(t_lane + C::TMEM_O + c * 32, o);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= alpha;
            tmem_st32(t_lane + C::TMEM_O + c * 32, o);
          }
        }
        l *= alpha;
      }
      // P = exp2(S * scale * log2(e) - m), bf16 into the swizzled K-major P tile
      float rs = 0.f;
#pragma unroll
      for (int ch = 0; ch < BN / 8; ++ch) {
        float p[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          p[x] = fast_exp2(fmaf(s[ch * 8 + x], sl2, -m_use));
          rs += p[x];
        }
        uint4 pk;
        pk.x = pack_bf16x2(p[0], p[1]);
        pk.y = pack_bf16x2(p[2], p[3]);
        pk.z = pack_bf16x2(p[4], p[5]);
        pk.w = pack_bf16x2(p[6], p[7]);
        const int kc = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4*>(pP + kc * (kBM * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = pk;
      }
      l += rs;
      m = m_new;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_P_FULL));
    }
    // ---- epilogue ----
    if (ok && cnt > 0) {
      ok = mbar_wait(bar(B_O_DONE), (cnt - 1) & 1, abort_flag, a.err);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    const bool have = ok && cnt > 0 && l > 0.f;
    const float inv = have ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      if (ok && cnt > 0) {
        tmem_ld32(t_lane + C::TMEM_O + c * 32, o);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) o[x] = 0.f;
      }
      if (row < BN) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 pk;
          pk.x = pack_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
          pk.y = pack_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
          pk.z = pack_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
          pk.w = pack_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
          const int col = c * 32 + q4 * 8;  // element column
          const int dc = col >> 6, cc = (col & 63) >> 3;
          *reinterpret_cast<uint4*>(pQ + dc * (BN * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = pk;
        }
      }
    }
    fence_proxy_async_smem();
    named_barrier_sync(1, 128);
    if (warp == 2 && lane == 0) {
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_store_3d(to, sQ + c * BN * 128, c * 64, qb * BN, bh);
      tma_store_commit();
      tma_store_wait_all();
    }
    if (lse != nullptr && row < BN && qb * BN + row < rows)
      lse[static_cast<size_t>(bh) * lse_stride + qb * BN + row] =
          have ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int BN>
static cudaError_t launch_attn_t(const AttnMaps& nat, const AttnMaps& perm, const AttnArgs& a, cudaStream_t stream) {
  using C = AttnCfg<D, BN>;
  auto kern = sparse_attn_fwd_kernel<D, BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(a.BH) * a.g.nblk;
  if (grid <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(grid), kAttnThreads, C::SMEM_ALLOC, stream>>>(nat.q, nat.k, nat.v, nat.o, perm.q, perm.k,
                                                                              perm.v, perm.o, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnMaps& nat, const AttnMaps& perm, const AttnArgs& a, int d,
                               cudaStream_t stream) {
  const int bn = a.g.block;
  if (d == 128 && bn == 128) return launch_attn_t<128, 128>(nat, perm, a, stream);
  if (d == 64 && bn == 128) return launch_attn_t<64, 128>(nat, perm, a, stream);
  if (d == 128 && bn == 64) return launch_attn_t<128, 64>(nat, perm, a, stream);
  if (d == 64 && bn == 64) return launch_attn_t<64, 64>(nat, perm, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace vsa
