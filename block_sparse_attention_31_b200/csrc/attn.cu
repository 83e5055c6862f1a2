// attn.cu -- block-sparse attention forward (vsa_sparse_attn_fwd) for sm_100a.
//
// For a query block i of head (b, h): O_i = softmax(Q_i K_J^T * scale) V_J with J the kept
// key blocks kv_idx[b,h,i,0..cnt) ("OSP-Next" page, "Method": sparse attention that stays
// compatible with FlashAttention kernels; "Sparse Video-Gen" summary, "Approach": block-wise
// spatial and temporal masks).  Online softmax in the base-2 domain, fp32 accumulation.
//
// One CTA per pair of query blocks of a head (tiles 0 and 1), 384 threads in three
// warpgroups whose registers are rebalanced at the start (setmaxnreg: the softmax warpgroups
// grow to kRegsSoftmax, the control warpgroup shrinks to kRegsCtl; the sum equals the launch's):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1, one query row per thread (TMEM lane = row):
//                    all of a key block's scores are read from TMEM with one wait, then the
//                    row max, the lazy rescale of O (only when the max grows by more than
//                    2^16), and P = exp2(S*scale*log2e - m) written as packed bf16 over the
//                    tile's S columns in TMEM in two halves, each announced on its own
//                    barrier so that the P.V of the first half overlaps the exponentials of
//                    the second; at the end O / l goes through shared memory to a TMA store.
//   warp 8 (one lane) TMA producer: both Q tiles once, then K and V of every key block in the
//                    union of the two lists through a 2-stage ring (each K/V tile is loaded
//                    once and serves both query tiles); with the in-kernel layout warp 8
//                    gathers Q and K rows and warp 10 gathers V rows instead.
//   warp 9 (one lane) tcgen05 issuer, per union entry: P.V of tile 0's previous block (first
//                    half as soon as it is written), Q.K^T of tile 0, then the same for tile
//                    1; the tensor core works on one tile while the other tile's softmax runs.
//                    Warp 9 also owns TMEM.
// TMEM: S0, S1 (BN columns each), O0, O1 (D columns each).
//
// Shared-memory operand tiles use the 128-byte swizzle (TMA SWIZZLE_128B == UMMA SWIZZLE_128B):
// a tile of R rows x 64 bf16 is R*128 bytes, 16-byte chunk c of row r at ((c ^ r%8)*16).
// Q.K^T: A = Q (K-major), B = K (K-major).  P.V: A = P from TMEM, B = V (MN-major: keys are
// rows, d contiguous).  Every wait is bounded; on a timeout the CTA raises its abort flag,
// drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace vsa {

// warps 0-3 softmax tile 0, 4-7 tile 1; warp 8 TMA (or Q and K gather), warp 9 MMA, warp 10 V
// gather (in-kernel layout only), warp 11 idle
constexpr int kAttnThreads = 384;
constexpr int kWarpLoad = 8, kWarpMma = 9, kWarpVGather = 10;
constexpr int kBM = 128;           // MMA M: query rows per tile
// Register split: 384 threads launch with 168 registers each (64,512 in all); the control
// warpgroup gives up 80 per thread and the two softmax warpgroups take 40 more each:
// 2 * 128 * 208 + 128 * 88 = 64,512 (88 keeps the producer and issuer code free of spills).
constexpr int kRegsSoftmax = 208, kRegsCtl = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsCtl == 384 * 168, "register split must equal the launch total");

// QK8: Q and K are e4m3 codes with one power-of-two scale per block (Q.K^T on kind::f8f6f4);
// V, P and O stay bf16.
template <int D, int BN, bool QK8>
struct AttnCfg {
  static constexpr int NS = 2;  // K/V ring stages
  static constexpr int QK_ES = QK8 ? 1 : 2;            // bytes per Q / K element
  static constexpr int Q_BYTES = kBM * D * QK_ES;
  static constexpr int K_BYTES = BN * D * QK_ES;
  static constexpr int V_BYTES = BN * D * 2;
  static constexpr int O_BYTES = kBM * D * 2;           // one tile of bf16 output
  static constexpr int QK_PANEL = 128 / QK_ES;          // elements in one 128-byte swizzled row
  static constexpr int QK_PANELS = D / QK_PANEL;
  static constexpr int QK_KSTEP = QK8 ? 32 : 16;        // K of one MMA instruction (32 bytes)
  static constexpr int OFF_Q = 0;  // two Q tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  // output staging: over the tile's Q buffer for bf16; a region of its own for e4m3 Q, whose
  // tile is half the size of the bf16 output tile
  static constexpr int OFF_OST = OFF_V + NS * V_BYTES;
  static constexpr int OFF_BAR = OFF_OST + (QK8 ? 2 * O_BYTES : 0);
  static constexpr int NBAR = 24;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_UNION = OFF_MISC + 64;  // union list, two bitsets, key-validity masks
  static constexpr int TMEM_S = 0;                  // S of tile t at t*BN (P aliases its first BN/2 columns)
  static constexpr int TMEM_O = 2 * BN;             // O of tile t at 2*BN + t*D
  static constexpr int TMEM_COLS = (2 * BN + 2 * D) <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_QK = QK8 ? idesc_e4m3_f32(kBM, BN) : idesc_bf16_f32(kBM, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kBM, D, false, true);
  static int smem_bytes(int ucap, int nwords) {
    return OFF_UNION + 4 * ucap + 8 * nwords + 4 * ucap * (BN / 32) + 4 * nwords + 1024;
  }
};

// Barrier slots.
enum {
  B_Q = 0,         // +tile
  B_FULL_K = 2,    // +stage
  B_FULL_V = 4,    // +stage
  B_REL = 6,       // +entry parity: K of entry n and V of entry n - 1 consumed (one commit per entry)
  B_S_FULL = 10,   // +tile
  B_P_FULL = 12,   // +tile
  B_O_FINAL = 14,  // +tile
  B_DRAIN = 16
};
constexpr uint32_t kInTile0 = 1u << 30, kInTile1 = 1u << 31, kPartial = 1u << 29, kKbMask = (1u << 29) - 1u;
// Probability pairs (2 columns) whose exponentials run on the FMA pipe: kPolyPairs8 in 8.
#ifndef VSA_POLY_PAIRS8
#define VSA_POLY_PAIRS8 1
#endif
constexpr int kPolyPairs8 = VSA_POLY_PAIRS8;

// One CTA per pair of consecutive query blocks (tiles 0 and 1) of one head.  The K/V blocks
// of the union of the two lists stream through a 2-stage ring once and serve both tiles; the
// MMA issuer interleaves the tiles (P.V of one, then Q.K^T of the same tile, then the other
// tile) so the tensor core works on one tile while the other tile's softmax runs.  P is
// written as packed bf16 over the tile's S columns in TMEM and read from there by the P.V MMA.
template <int D, int BN, bool QK8>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tq_n, const __grid_constant__ CUtensorMap tk_n,
                           const __grid_constant__ CUtensorMap tv_n, const __grid_constant__ CUtensorMap to_n,
                           const __grid_constant__ CUtensorMap tq_p, const __grid_constant__ CUtensorMap tk_p,
                           const __grid_constant__ CUtensorMap tv_p, const __grid_constant__ CUtensorMap to_p,
                           const AttnArgs a) {
  using C = AttnCfg<D, BN, QK8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_u32);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  // misc[0]: TMEM base address, misc[1]: abort flag, misc[2]: union length
  volatile int* abort_flag = misc + 1;
  const int nwords = (a.g.nblk + 31) >> 5;
  uint32_t* uni = reinterpret_cast<uint32_t*>(smem + C::OFF_UNION);
  uint32_t* bits0 = uni + a.ucap;
  uint32_t* bits1 = bits0 + nwords;
  uint32_t* uvalid = bits1 + nwords;  // [ucap][BN/32] valid-key bits of partial union entries

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthr = blockDim.x;
  const Geom& g = a.g;
  const int npairs = (g.nblk + 1) >> 1;
  const int bh = blockIdx.x / npairs;
  const int pair = blockIdx.x - bh * npairs;
  const int kind = a.kinds[bh];
  if (kind > kCube || (a.gather && kind == kCube)) {  // in-kernel layout: cube heads need their copies
    // The head's layout is unknown: its rows of the natural-order output (the buffer the caller
    // reads) are written as zeros and LSE -inf, and the kind bit is raised.
    if (tid == 0 && pair == 0) atomicOr(a.err, kDevErrKind);
    const int r0 = 2 * pair * BN, r1 = min(r0 + 2 * BN, a.nat_rows);
    if (a.nat_o != nullptr)
      for (int x = tid; x < (r1 - r0) * (D / 8); x += blockDim.x) {
        const size_t row = static_cast<size_t>(bh) * a.nat_rows + r0 + x / (D / 8);
        reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.nat_o) + row * D)[x % (D / 8)] = make_uint4(0, 0, 0, 0);
      }
    if (a.lse_nat != nullptr)
      for (int x = r0 + tid; x < r1; x += blockDim.x) a.lse_nat[static_cast<size_t>(bh) * a.nat_rows + x] = -INFINITY;
    return;
  }
  const int rows = layout_rows(g, kind);
  const int nb_head = (rows + BN - 1) / BN;
  if (2 * pair >= nb_head) return;
  const bool has1 = 2 * pair + 1 < nb_head;
  int qb0 = 2 * pair, qb1 = 2 * pair + 1;
  if (a.order != nullptr) {  // locality-aware pairing from vsa_build_mask
    const int32_t* ord = a.order + static_cast<size_t>(bh) * g.nblk;
    qb0 = ord[2 * pair];
    qb1 = has1 ? ord[2 * pair + 1] : nb_head;
    if (qb0 < 0 || qb0 >= nb_head || (has1 && (qb1 < 0 || qb1 >= nb_head || qb1 == qb0))) {
      if (tid == 0) atomicOr(a.err, kDevErrKvRange);
      return;
    }
  }
  const bool use_perm = a.has_perm && kind != kSpatial;
  const bool gather = a.gather && kind == kTemporal;  // rows through the frame-major map, in-kernel
  const CUtensorMap* tq = use_perm ? &tq_p : &tq_n;
  const CUtensorMap* tk = use_perm ? &tk_p : &tk_n;
  const CUtensorMap* tv = use_perm ? &tv_p : &tv_n;
  const CUtensorMap* to = use_perm ? &to_p : &to_n;
  float* lse = use_perm ? a.lse_perm : a.lse_nat;
  const int lse_stride = use_perm ? g.R : a.nat_rows;

  // ---- the two lists: validate, then build their union in ascending order ----
  const size_t mrow0 = static_cast<size_t>(bh) * g.nblk + qb0;
  const size_t mrow1 = static_cast<size_t>(bh) * g.nblk + (has1 ? qb1 : qb0);
  const int32_t* kvl0 = a.kv_idx + mrow0 * a.max_kv;
  const int32_t* kvl1 = a.kv_idx + mrow1 * a.max_kv;
  int cnt0 = a.kv_cnt[mrow0];
  int cnt1 = has1 ? a.kv_cnt[mrow1] : 0;
  bool bad0 = cnt0 < 0 || cnt0 > a.max_kv, bad1 = cnt1 < 0 || cnt1 > a.max_kv;
  for (int x = tid; x < 2 * nwords; x += nthr) bits0[x] = 0u;  // bits1 follows bits0
  bool stop = false;
  if (tid == 0) stop = (*reinterpret_cast<volatile int*>(a.err) & kDevErrTimeout) != 0;
  if (__syncthreads_or(stop)) return;
  // Q tiles by TMA before anything else, so that their load overlaps the list validation and
  // the union (TMA layout only; a tile whose list then turns out invalid drains its copy).
  const bool q_early0 = !gather && !bad0 && cnt0 > 0, q_early1 = !gather && !bad1 && cnt1 > 0;
  if (tid == 0 && !gather) {
    mbar_init(bar(B_Q + 0), 1);
    mbar_init(bar(B_Q + 1), 1);
    mbar_init_fence();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (!(t ? q_early1 : q_early0)) continue;
      mbar_arrive_expect_tx(bar(B_Q + t), C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::QK_PANELS; ++c)
        tma_load_3d(sbase + C::OFF_Q + t * C::Q_BYTES + c * kBM * 128, tq, bar(B_Q + t), c * C::QK_PANEL,
                    (t ? qb1 : qb0) * BN, bh);
    }
  }
  // Lists must be strictly ascending block indices in [0, nb_head).
  if (!bad0)
    for (int j = tid; j < cnt0; j += nthr) {
      const int kb = kvl0[j];
      if (kb < 0 || kb >= nb_head || (j > 0 && kvl0[j - 1] >= kb)) bad0 = true;
      else atomicOr(&bits0[kb >> 5], 1u << (kb & 31));
    }
  if (!bad1)
    for (int j = tid; j < cnt1; j += nthr) {
      const int kb = kvl1[j];
      if (kb < 0 || kb >= nb_head || (j > 0 && kvl1[j - 1] >= kb)) bad1 = true;
      else atomicOr(&bits1[kb >> 5], 1u << (kb & 31));
    }
  bad0 = __syncthreads_or(bad0);
  bad1 = __syncthreads_or(bad1);
  if (bad0 || bad1) {
    if (tid == 0) {
      atomicOr(a.err, kDevErrKvRange);
      if (bad0 && q_early0) mbar_wait_drain(bar(B_Q + 0), 0, a.err);  // the copy lands before the tile is dropped
      if (bad1 && q_early1) mbar_wait_drain(bar(B_Q + 1), 0, a.err);
    }
    if (bad0) {
      cnt0 = 0;
      for (int x = tid; x < nwords; x += nthr) bits0[x] = 0u;
    }
    if (bad1) {
      cnt1 = 0;
      for (int x = tid; x < nwords; x += nthr) bits1[x] = 0u;
    }
    __syncthreads();
  }
  // Union of the two lists in ascending order: warp 0 turns the per-word counts of the OR-ed
  // bitsets into word offsets; then every thread places the blocks of its bit positions.
  uint32_t* woff = uvalid + a.ucap * (BN / 32);  // [nwords] offset of each word's first entry
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int w = w0 + lane;
      const int c = w < nwords ? __popc(bits0[w] | bits1[w]) : 0;
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
      }
      if (w < nwords) woff[w] = static_cast<uint32_t>(base + incl - c);
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) misc[2] = base;
  }
  __syncthreads();
  for (int kb = tid; kb < nwords * 32; kb += nthr) {
    const uint32_t u0 = bits0[kb >> 5], u1 = bits1[kb >> 5], b = kb & 31;
    const uint32_t u = u0 | u1;
    if (!((u >> b) & 1u)) continue;
    const int pos = static_cast<int>(woff[kb >> 5]) + __popc(u & ((1u << b) - 1u));
    uni[pos] = static_cast<uint32_t>(kb) | (((u0 >> b) & 1u) ? kInTile0 : 0u) | (((u1 >> b) & 1u) ? kInTile1 : 0u) |
               (block_full(g, kind, kb) ? 0u : kPartial);
  }
  __syncthreads();
  {
    // valid-key bits of the blocks that are not full (ragged tail, cube padding), one union
    // entry per warp at a time.  A cube block is one cube (V == BN); its slot
    // r = (df*ch + dh)*cw + dw holds a token when the offsets fall inside the cube's real
    // extent, and the offsets of r = 32w + lane are the same for every cube.
    const int base = misc[2];
    int cdw[BN / 32], cdh[BN / 32], cdf[BN / 32];
    if (kind == kCube) {
#pragma unroll
      for (int w = 0; w < BN / 32; ++w) {
        const int r = w * 32 + lane;
        cdw[w] = r % g.cw;
        cdh[w] = (r / g.cw) % g.ch;
        cdf[w] = r / (g.cw * g.ch);
      }
    }
    for (int n = warp; n < base; n += nthr >> 5) {
      const uint32_t e = uni[n];
      if (!(e & kPartial)) continue;
      const int kb = static_cast<int>(e & kKbMask);
      int nf = 0, nh = 0, nw = 0;
      if (kind == kCube) {
        const int cw_i = kb % g.ncw, ch_i = (kb / g.ncw) % g.nch, cf_i = kb / (g.ncw * g.nch);
        nf = min(g.cf, g.F - cf_i * g.cf);
        nh = min(g.ch, g.Hl - ch_i * g.ch);
        nw = min(g.cw, g.Wl - cw_i * g.cw);
      }
#pragma unroll
      for (int w = 0; w < BN / 32; ++w) {
        const bool ok = kind == kCube ? (cdf[w] < nf && cdh[w] < nh && cdw[w] < nw) : kb * BN + w * 32 + lane < g.N;
        const uint32_t m = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) uvalid[n * (BN / 32) + w] = m;
      }
    }
  }

  // ---- setup: barriers and TMEM ----
  if (tid == 0) {
    const uint32_t nload = gather ? 32u : 1u;  // gather: one cp.async arrival per producer lane
    for (int t = 0; t < 2; ++t) {
      if (gather) mbar_init(bar(B_Q + t), nload);  // TMA layout: initialised above, copy in flight
      mbar_init(bar(B_S_FULL + t), 1);
      mbar_init(bar(B_P_FULL + t), 128);
      mbar_init(bar(B_O_FINAL + t), 1);
    }
    for (int st = 0; st < C::NS; ++st) {
      mbar_init(bar(B_FULL_K + st), nload);
      mbar_init(bar(B_FULL_V + st), nload);
      mbar_init(bar(B_REL + st), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    misc[1] = 0;
    mbar_init_fence();
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tk);
    tma_prefetch_desc(tv);
    tma_prefetch_desc(to);
  }
  if (warp == kWarpMma) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int U = misc[2];

  if (warp >= 8) {
  setmaxnreg_dec<kRegsCtl>();
  if ((warp == kWarpLoad || warp == kWarpVGather) && gather) {
    // ================= gather producers (temporal head, natural-order buffers) =================
    // Warp 8 copies the Q and K tiles, warp 10 the V tiles, 16 bytes per copy: slot p of the
    // frame-major layout is token (p % F) * S + p / F; copies land in the 128-byte-swizzled
    // layout a TMA tile load would produce, slots past N are zero-filled.  Each lane's copies
    // signal the stage's barrier when they land.  Lane l owns 16-byte column c = l % CPR of rows
    // r = l / CPR + k * RSTEP, and walks them with incremental (frame, position) and source
    // offsets, so no division runs per copy.
    if (U > 0) {
      constexpr int CPR = D / 8, RSTEP = 32 / CPR;
      const int c = lane % CPR, r0 = lane / CPR;
      const size_t head = static_cast<size_t>(bh) * g.N * D;
      const size_t fstep = static_cast<size_t>(RSTEP) * g.S * D;  // RSTEP frames further
      const size_t wrap = static_cast<size_t>(g.F) * g.S * D - D;  // frame F -> frame 0, next position
      auto gather_tile = [&](uint32_t sdst, int rows_tile, int slot0, const __nv_bfloat16* src) {
        const uint32_t panel = sdst + (c >> 3) * (rows_tile * 128);
        int slot = slot0 + r0;
        const int sp = slot / g.F;
        int f = slot - sp * g.F;
        const __nv_bfloat16* from = src + (static_cast<size_t>(f) * g.S + sp) * D + c * 8;
#pragma unroll 4
        for (int r = r0; r < rows_tile; r += RSTEP) {
          const bool in = slot < g.N;
          cp_async_16(panel + r * 128 + (((c & 7) ^ (r & 7)) << 4), in ? from : src, in ? 16u : 0u);
          slot += RSTEP;
          f += RSTEP;
          from += fstep;
          while (f >= g.F) {
            f -= g.F;
            from -= wrap;
          }
        }
      };
      const __nv_bfloat16* gq = static_cast<const __nv_bfloat16*>(a.nat_q) + head;
      const __nv_bfloat16* gk = static_cast<const __nv_bfloat16*>(a.nat_k) + head;
      const __nv_bfloat16* gv = static_cast<const __nv_bfloat16*>(a.nat_v) + head;
      const int cnts[2] = {cnt0, cnt1};
      const bool qk = warp == kWarpLoad;
      if (qk) {
        for (int t = 0; t < 2; ++t) {
          if (cnts[t] == 0) continue;
          gather_tile(sbase + C::OFF_Q + t * C::Q_BYTES, kBM, (t ? qb1 : qb0) * BN, gq);
          cp_async_mbar_arrive_noinc(bar(B_Q + t));
        }
      }
      const int fb = qk ? B_FULL_K : B_FULL_V;
      const uint32_t sdst0 = qk ? sK : sV;
      const __nv_bfloat16* gsrc = qk ? gk : gv;
      for (int n = 0; n < U; ++n) {
        const int st = n % C::NS;
        const int kb = static_cast<int>(uni[n] & kKbMask);
        // K(n) replaces K(n-2): free after entry n-2's MMAs; V(n) replaces V(n-2): free after entry n-1's
        const int re = qk ? n - 2 : n - 1;
        if (n >= C::NS &&
            !__all_sync(0xffffffffu, mbar_wait(bar(B_REL + re % C::NS), (re / C::NS) & 1, abort_flag, a.err)))
          break;
        gather_tile(sdst0 + st * (qk ? C::K_BYTES : C::V_BYTES), BN, kb * BN, gsrc);
        cp_async_mbar_arrive_noinc(bar(fb + st));
      }
      // every copy lands before the CTA can exit (they always complete; nothing to bound)
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncwarp();
  } else if (warp == kWarpLoad) {
    // ================= TMA producer =================
    if (lane == 0 && U > 0) {
      int nk = 0, nv = 0;  // copies issued (the Q tiles were issued in the prologue)
      const int cnts[2] = {cnt0, cnt1};
      for (int n = 0; n < U; ++n) {
        const int st = n % C::NS;
        const uint32_t u = n / C::NS;
        const int kb = static_cast<int>(uni[n] & kKbMask);
        // K(n) goes where K(n-2) was: free once entry n-2's MMAs complete
        if (n >= C::NS && !mbar_wait(bar(B_REL + st), (u - 1) & 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(bar(B_FULL_K + st), C::K_BYTES);
#pragma unroll
        for (int c = 0; c < C::QK_PANELS; ++c)
          tma_load_3d(sK + st * C::K_BYTES + c * BN * 128, tk, bar(B_FULL_K + st), c * C::QK_PANEL, kb * BN, bh);
        nk = n + 1;
        // V(n) goes where V(n-2) was: free once entry n-1's MMAs (which include P.V of n-2) complete
        if (n >= C::NS && !mbar_wait(bar(B_REL + (n - 1) % C::NS), ((n - 1) / C::NS) & 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(bar(B_FULL_V + st), C::V_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sV + st * C::V_BYTES + c * BN * 128, tv, bar(B_FULL_V + st), c * 64, kb * BN, bh);
        nv = n + 1;
      }
      if (*abort_flag) {
        // Drain: every copy this thread issued must land before the CTA exits.
        for (int t = 0; t < 2; ++t)
          if (cnts[t] > 0) mbar_wait_drain(bar(B_Q + t), 0, a.err);
        for (int st = 0; st < C::NS; ++st) {
          int lk = -1, lv = -1;
          for (int n = st; n < nk; n += C::NS) lk = n;
          for (int n = st; n < nv; n += C::NS) lv = n;
          if (lk >= 0) mbar_wait_drain(bar(B_FULL_K + st), (lk / C::NS) & 1, a.err);
          if (lv >= 0) mbar_wait_drain(bar(B_FULL_V + st), (lv / C::NS) & 1, a.err);
        }
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ================= tcgen05 issuer =================
    if (lane == 0 && U > 0) {
      const int cnts[2] = {cnt0, cnt1};
      int pend[2] = {-1, -1};   // union entry whose Q.K^T is issued and P.V is not
      int pvc[2] = {0, 0};      // P.V products issued per tile
      bool qready[2] = {false, false};
      bool ok = true;
      // Descriptor bases; each K step adds a compile-time offset (in 16-byte units) to the
      // start-address field, which never carries out of its 14 bits (shared memory < 256 KB).
      static_assert(C::NS == 2, "descriptor selection below assumes two stages");
      const uint64_t dq0 = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t dq1 = sdesc_sw128(sbase + C::OFF_Q + C::Q_BYTES, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sK, 16, 1024), dk1 = sdesc_sw128(sK + C::K_BYTES, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sV, BN * 128, 1024), dv1 = sdesc_sw128(sV + C::V_BYTES, BN * 128, 1024);
      // P.V of tile t's pending block (its V was waited for at the start of the entry)
      auto issue_pv = [&](int t) -> bool {
        const int np = pend[t];
        if (!mbar_wait(bar(B_P_FULL + t), pvc[t] & 1, abort_flag, a.err)) return false;
        if (gather) fence_proxy_async_smem();  // cp.async data, written by the generic proxy
        tc_fence_after();
        const uint64_t vd = (np & 1) ? dv1 : dv0;
        const uint32_t d_o = tmem + C::TMEM_O + t * D, a_p = tmem + C::TMEM_S + t * BN;
        tc_mma_ts(d_o, a_p, vd, C::IDESC_PV, pvc[t] > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < BN / 16; ++kk)
          tc_mma_ts(d_o, a_p + kk * 8, vd + static_cast<uint64_t>(kk * 16 * 128 / 16), C::IDESC_PV, 1u);
        pend[t] = -1;
        if (++pvc[t] == cnts[t]) tc_commit(bar(B_O_FINAL + t));
        return true;
      };
      // Every wait and commit of this thread can leave the tensor core idle, so an entry makes
      // few of them: K of the entry and V of the previous one up front, one P per tile, one
      // S commit per tile and one release of both stages.
      for (int n = 0; ok && n < U; ++n) {
        const int st = n % C::NS;
        if (!mbar_wait(bar(B_FULL_K + st), (n / C::NS) & 1, abort_flag, a.err) ||
            (n >= 1 && !mbar_wait(bar(B_FULL_V + (n - 1) % C::NS), ((n - 1) / C::NS) & 1, abort_flag, a.err))) {
          ok = false;
          break;
        }
        const uint32_t e = uni[n];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (pend[t] >= 0 && !issue_pv(t)) {
            ok = false;
            break;
          }
          if (!((e >> (30 + t)) & 1u)) continue;
          if (!qready[t]) {
            if (!mbar_wait(bar(B_Q + t), 0, abort_flag, a.err)) {
              ok = false;
              break;
            }
            qready[t] = true;
          }
          if (gather) fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t d_s = tmem + C::TMEM_S + t * BN;
          const uint64_t qd = t ? dq1 : dq0, kd = st ? dk1 : dk0;
          // each instruction takes 32 bytes of K: four per 128-byte swizzled row of a panel
#pragma unroll
          for (int kk = 0; kk < D / C::QK_KSTEP; ++kk) {
            const uint64_t qa = qd + static_cast<uint64_t>(((kk >> 2) * (kBM * 128) + (kk & 3) * 32) / 16);
            const uint64_t kb_ = kd + static_cast<uint64_t>(((kk >> 2) * (BN * 128) + (kk & 3) * 32) / 16);
            if constexpr (QK8) tc_mma_ss_f8(d_s, qa, kb_, C::IDESC_QK, kk > 0 ? 1u : 0u);
            else tc_mma_ss(d_s, qa, kb_, C::IDESC_QK, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_S_FULL + t));
          pend[t] = n;
        }
        if (!ok) break;
        tc_commit(bar(B_REL + st));  // K(n) and V(n-1) are free once these MMAs complete
      }
      if (ok && U >= 1 && !mbar_wait(bar(B_FULL_V + (U - 1) % C::NS), ((U - 1) / C::NS) & 1, abort_flag, a.err))
        ok = false;
      for (int t = 0; ok && t < 2; ++t)
        if (pend[t] >= 0 && !issue_pv(t)) ok = false;
      // Drain: all MMAs issued by this thread complete before TMEM is released.
      tc_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0, a.err);
    }
    __syncwarp();
  }
  } else {
    // ================= softmax: warps 0-3 tile 0, warps 4-7 tile 1; one row per thread =================
    setmaxnreg_inc<kRegsSoftmax>();
    const int t = warp >> 2;
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;   // query row within the tile
    if (t == 0 || has1) {
      const int cnt = t ? cnt1 : cnt0;
      const int qb = t ? qb1 : qb0;
      const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
      const uint32_t t_s = t_lane + C::TMEM_S + t * BN, t_o = t_lane + C::TMEM_O + t * D;
      const float sl2_base = a.scale_log2;
      // e4m3 Q and K: the block pair's scores carry the scales 2^(e_q + e_k)
      const int eq = QK8 ? a.qexp[static_cast<size_t>(bh) * g.nblk + qb] : 0;
      float m = -INFINITY, l = 0.f;  // m: the (lazily updated) max used for the exponentials
      bool ok = true;
      int cur = 0;  // cursor into the union list (this tile's entries are the ones with its bit)
      const uint32_t tbit = t ? kInTile1 : kInTile0;
      for (int k = 0; k < cnt; ++k) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + t), k & 1, abort_flag, a.err));
        if (!ok) break;
        while (!(uni[cur] & tbit)) ++cur;
        const uint32_t ent = uni[cur];
        tc_fence_after();
        // every score of the row with one wait
        uint32_t r[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32_async(t_s + c * 32, r + c * 32);
        tmem_wait_ld();
        reg_fence<BN>(r);
        if (ent & kPartial) {  // same block for every row: invalid key columns (tail, padding) -> -inf
#pragma unroll
          for (int w = 0; w < BN / 32; ++w) {
            const uint32_t vb = uvalid[cur * (BN / 32) + w];
#pragma unroll
            for (int x = 0; x < 32; ++x) r[w * 32 + x] = ((vb >> x) & 1u) ? r[w * 32 + x] : 0xff800000u;
          }
        }
        ++cur;
        const float sl2 = QK8 ? ldexpf(sl2_base, eq + a.kexp[static_cast<size_t>(bh) * g.nblk + (ent & kKbMask)])
                              : sl2_base;
        // row max: eight independent partial maxima keep the dependency chains short
        float mx8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) mx8[x] = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN / 2; ++c)
          mx8[c & 7] = fmax3(mx8[c & 7], __uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float m_new = fmaxf(m, mx * sl2);
        // Rescale only when the running max grows by more than 2^kRescaleLog2; otherwise keep the
        // old max (the final 1/l normalisation is exact either way).  O is stable here: the
        // Q.K^T whose completion signalled S was issued after the previous P.V of this tile.
        const bool grow = m_new > m + kRescaleLog2;
        if (k > 0 && __any_sync(0xffffffffu, grow && m != -INFINITY)) {
          const float alpha = grow ? fast_exp2(m - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(t_o + c * 32, o);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= alpha;
            tmem_st32(t_o + c * 32, o);
          }
        }
        if (grow) {
          l *= fast_exp2(m - m_new);
          m = m_new;
        }
        const float m_use = m == -INFINITY ? 0.f : m;
        // exponentials in two halves of the keys: each half's packed bf16 P goes over the
        // consumed S columns and is announced on its own barrier, so the P.V of the first half
        // runs while the second half is computed (scale and max subtraction, row sums and the
        // polynomial exponentials on packed pairs)
        uint64_t rs4[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) rs4[x] = 0ull;
        const uint64_t sl2x2 = f2_make(sl2, sl2), negm2 = f2_make(-m_use, -m_use);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[BN / 4];
#pragma unroll
          for (int c = 0; c < BN / 4; ++c) {
            const int cc = hf * (BN / 4) + c;  // key pair
            const uint64_t x =
                f2_fma(f2_make(__uint_as_float(r[2 * cc]), __uint_as_float(r[2 * cc + 1])), sl2x2, negm2);
            uint64_t p;
            if ((cc & 7) >= 8 - kPolyPairs8) {
              p = exp2_poly2(x);
            } else {
              float x0, x1;
              f2_split(x, x0, x1);
              p = f2_make(fast_exp2(x0), fast_exp2(x1));
            }
            rs4[cc & 3] = f2_add(rs4[cc & 3], p);
            float p0, p1;
            f2_split(p, p0, p1);
            pk[c] = pack_bf16x2(p0, p1);
          }
          tmem_st_cols<BN / 4>(t_s + hf * (BN / 4), pk);
        }
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + t));
        {
          const uint64_t s2 = f2_add(f2_add(rs4[0], rs4[1]), f2_add(rs4[2], rs4[3]));
          float s0, s1;
          f2_split(s2, s0, s1);
          l += s0 + s1;
        }
      }
      // ---- epilogue: O / l -> bf16 -> swizzled smem (over this tile's Q) -> TMA store ----
      if (ok && cnt > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FINAL + t), 0, abort_flag, a.err));
        tc_fence_after();
      }
      const bool have = ok && cnt > 0 && l > 0.f;
      const float inv = have ? 1.f / l : 0.f;
      uint8_t* stage = smem + (QK8 ? C::OFF_OST + t * C::O_BYTES : C::OFF_Q + t * C::Q_BYTES);
      // in-kernel layout: this row's natural token (slot p -> (p % F) * S + p / F)
      const int slot = qb * BN + row;
      const bool row_live = row < BN && slot < rows;
      const int tok = gather ? (slot % g.F) * g.S + slot / g.F : slot;
      __nv_bfloat16* orow = gather ? static_cast<__nv_bfloat16*>(a.nat_o) + (static_cast<size_t>(bh) * g.N + tok) * D
                                   : nullptr;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (ok && cnt > 0) {
          tmem_ld32(t_o + c * 32, o);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = 0.f;
        }
        if (row < BN) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v4;
            v4.x = pack_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
            v4.y = pack_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
            v4.z = pack_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
            v4.w = pack_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
            const int col = c * 32 + q4 * 8;
            if (gather) {
              if (row_live) *reinterpret_cast<uint4*>(orow + col) = v4;
            } else {
              const int dc = col >> 6, cc = (col & 63) >> 3;
              *reinterpret_cast<uint4*>(stage + dc * (BN * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = v4;
            }
          }
        }
      }
      if (!gather) {
        fence_proxy_async_smem();
        named_barrier_sync(1 + t, 128);
        if (quad == 2 && lane == 0) {
          const uint32_t sstage = sbase + (QK8 ? C::OFF_OST + t * C::O_BYTES : C::OFF_Q + t * C::Q_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) tma_store_3d(to, sstage + c * BN * 128, c * 64, qb * BN, bh);
          tma_store_commit();
          tma_store_wait_all();
        }
      }
      if (lse != nullptr && row_live)
        lse[static_cast<size_t>(bh) * lse_stride + tok] =
            have ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, C::TMEM_COLS);
}

template <int D, int BN, bool QK8>
static cudaError_t launch_attn_t(const AttnMaps& nat, const AttnMaps& perm, const AttnArgs& a, cudaStream_t stream) {
  using C = AttnCfg<D, BN, QK8>;
  auto kern = sparse_attn_fwd_kernel<D, BN, QK8>;
  const int nwords = (a.g.nblk + 31) / 32;
  const int smem = C::smem_bytes(a.ucap, nwords);
  if (smem > 232448) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(a.BH) * ((a.g.nblk + 1) / 2);
  if (grid <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(grid), kAttnThreads, smem, stream>>>(nat.q, nat.k, nat.v, nat.o, perm.q, perm.k, perm.v,
                                                                   perm.o, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnMaps& nat, const AttnMaps& perm, const AttnArgs& a, int d,
                               cudaStream_t stream) {
  const int bn = a.g.block;
  if (a.qexp != nullptr) {  // e4m3 Q and K: d = 128, block 128, no in-kernel layout
    if (d == 128 && bn == 128 && !a.gather) return launch_attn_t<128, 128, true>(nat, perm, a, stream);
    return cudaErrorInvalidValue;
  }
  if (d == 128 && bn == 128) return launch_attn_t<128, 128, false>(nat, perm, a, stream);
  if (d == 64 && bn == 128) return launch_attn_t<64, 128, false>(nat, perm, a, stream);
  if (d == 128 && bn == 64) return launch_attn_t<128, 64, false>(nat, perm, a, stream);
  if (d == 64 && bn == 64) return launch_attn_t<64, 64, false>(nat, perm, a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace vsa
