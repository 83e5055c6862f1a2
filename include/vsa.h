/*
 * vsa.h -- C ABI of libvsa.so: spatial-temporal block-sparse self-attention for video
 * diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * One attention call over a latent grid of F x Hl x Wl tokens (S = Hl*Wl tokens per frame,
 * N = F*S, natural token t = (f*Hl + h)*Wl + w = f*S + s) runs these steps, each a CUDA
 * kernel behind one entry point below:
 *
 *   vsa_profile_heads   pick a spatial or temporal pattern per head from ~1% of the query
 *                       rows ("Sparse Video-Gen" summary page, section "Approach"; its
 *                       "Measured effects" table gives the 1% profiling fraction)
 *   vsa_permute         gather temporal heads into frame-major order (same page,
 *                       "Approach": the token-major to frame-major layout transformation
 *                       that makes temporal blocks contiguous), cube heads into cube-major
 *                       order ("USV" page, Figure 2: local 3D cubes)
 *   vsa_build_mask      block masks: spatial/temporal windows ("Sparse Video-Gen",
 *                       "Approach" and "Limitations": hand-fixed ratios c_s, c_t), or the
 *                       own cube plus the top-k cubes of mean-pooled Q K^T ("USV",
 *                       Figure 2: top-k cube selection)
 *   vsa_sparse_attn_fwd softmax(Q K^T * scale) V restricted to the kept KV blocks, online
 *                       softmax ("OSP-Next" page, section "Method": sparse attention kept
 *                       compatible with FlashAttention kernels)
 *   vsa_unpermute       scatter the output back to natural order
 *   vsa_attention       all of the above on one stream
 *
 * A second way to choose the kept blocks, the semantic-aware permutation ("Sparse
 * VideoGen2" page, abstract), runs on the same attention kernel:
 *
 *   vsa_kmeans          per-head k-means of Q (or K) and the cluster-major order
 *   vsa_gather_rows     rows in a per-head order (Q by its clusters, K and V by theirs)
 *   vsa_semantic_mask   top-p budget over cluster pairs -> block mask of the two layouts
 *   vsa_scatter_rows    the output back to token order
 *   vsa_semantic_attention  all of them with vsa_sparse_attn_fwd on one stream
 *
 * Conventions
 *   - Tensors are [B, H, rows, d] row-major (d fastest), bf16 unless stated otherwise.
 *     A head's buffer holds N rows in natural or frame-major order, or C*V rows in
 *     cube-major order (C cubes of V = cube_f*cube_h*cube_w slots, padding slots zero).
 *   - Ownership: the caller owns every buffer (inputs, outputs, workspace, error word).
 *     The library never allocates or frees device memory and keeps no mutable global
 *     state; every call is asynchronous on `stream` (NULL = legacy default stream) and
 *     never synchronises, except vsa_get_device_error.
 *   - All device pointers must be 16-byte aligned; tensors must be contiguous.  Each one
 *     must be device (or managed) memory: a host address is refused with
 *     VSA_ERR_INVALID_ARG before any launch.
 *   - Errors: arguments are validated on the host before any launch (VSA_ERR_INVALID_ARG,
 *     VSA_ERR_UNSUPPORTED, VSA_ERR_WORKSPACE); a failed launch returns VSA_ERR_CUDA.
 *     Kernels that detect a bad device-side input (an index or count out of range) or a
 *     bounded wait that ran out set bits of the caller's device error word `d_err`
 *     (VSA_DEVERR_*) and return without trapping; vsa_get_device_error reads it.
 *   - No C++ exception crosses this interface.
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define VSA_API __attribute__((visibility("default")))
#else
#define VSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, bad enum */
    VSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d not in {64,128}) */
    VSA_ERR_WORKSPACE = 3,     /* workspace smaller than the matching *_workspace_size */
    VSA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    VSA_ERR_DEVICE = 5,        /* the device error word holds an error bit */
    VSA_ERR_TIMEOUT = 6        /* the device error word holds the timeout bit */
} vsa_status;

/* Bits of the device error word. */
#define VSA_DEVERR_KV_RANGE 0x1   /* kv index outside [0, blocks) or count outside [0, max_kv] */
#define VSA_DEVERR_TIMEOUT 0x2    /* a bounded wait inside a kernel gave up */
#define VSA_DEVERR_KIND 0x4       /* head kind byte not one of vsa_kind */
#define VSA_DEVERR_OVERFLOW 0x8   /* a mask row kept more blocks than max_kv */

typedef enum { VSA_F32 = 0, VSA_BF16 = 1 } vsa_dtype;

typedef enum { VSA_SPATIAL = 0, VSA_TEMPORAL = 1, VSA_CUBE = 2 } vsa_kind;

/* How vsa_attention chooses each head's kind. */
typedef enum {
    VSA_SELECT_PROFILE = 0,    /* run vsa_profile_heads (bf16 input only) */
    VSA_SELECT_GIVEN = 1,      /* read the caller's kinds from d_kind */
    VSA_SELECT_CUBE = 2        /* every head is a cube head (own cube + top-k) */
} vsa_select;

typedef struct {
    int B, H;                     /* batch, heads */
    int F, Hl, Wl;                /* latent grid: frames x height x width tokens */
    int d;                        /* head dimension: 64 or 128 */
    int block;                    /* tokens per query block and per key block: 64 or 128 */
    int cube_f, cube_h, cube_w;   /* cube dims for cube heads, or all 0 when unused;
                                     cube_f*cube_h*cube_w must equal block */
} vsa_shape;

typedef struct {
    int w_s;                      /* spatial window in frames (blocks whose frame
                                     intervals are at most w_s apart are kept) */
    int w_t;                      /* temporal window in positions, frame-major order */
    double profile_frac;          /* profiled share of query rows: r = ceil(frac*N) */
    int topk;                     /* long-range cubes per query cube (cube heads) */
    float scale;                  /* softmax scale; 0 selects 1/sqrt(d) */
    int layout_in_kernel;         /* vsa_attention only: 1 = temporal heads are read and written
                                     in natural order through the frame-major map inside the
                                     attention kernel (no permute / unpermute copies); used
                                     for bf16 inputs without cube dims, ignored otherwise */
    int qk_fp8;                   /* vsa_attention only: 1 = Q.K^T on e4m3 codes with one
                                     power-of-two scale per block (vsa_quantize_fp8,
                                     vsa_sparse_attn_fwd_fp8qk); bf16 inputs, d = 128, block 128,
                                     not with layout_in_kernel (VSA_ERR_UNSUPPORTED otherwise) */
} vsa_params;

/* Pointers of one attention problem; o and lse are written. lse may be NULL. */
typedef struct {
    const void *q, *k, *v;        /* [B, H, rows, d] */
    void *o;                      /* [B, H, rows, d] */
    float *lse;                   /* [B, H, rows] natural-log log-sum-exp, or NULL */
} vsa_qkvo;

VSA_API const char *vsa_status_string(vsa_status s);
VSA_API int vsa_version(void);

/* ---------------------------------------------------------------------------------
 * Host-side planning helpers (no device work)
 * --------------------------------------------------------------------------------- */

/* Rows of a permuted buffer per head: N, or C*V when cube dims are set. */
VSA_API vsa_status vsa_layout_rows(const vsa_shape *shape, int64_t *rows);

/* Blocks per head in the permuted buffers: ceil(rows / block). Masks are [B,H,nblk,...]. */
VSA_API vsa_status vsa_num_blocks(const vsa_shape *shape, int *nblk);

/* Smallest window whose kept-block fraction reaches `target` for a spatial or temporal
 * head ("Sparse Video-Gen" summary, "Measured effects": sparsity given as kept fraction).
 * Writes the window and its exact kept fraction (kept may be NULL). */
VSA_API vsa_status vsa_pattern_window(const vsa_shape *shape, vsa_kind kind, double target, int *w, double *kept);

/* Largest number of kept KV blocks of any query block: max over the spatial window w_s and
 * the temporal window w_t, or topk + 1 for cube shapes (cube dims set). */
VSA_API vsa_status vsa_max_kv(const vsa_shape *shape, const vsa_params *params, int *max_kv);

/* Profiling rows r = ceil(profile_frac * N) clamped to [1, N]. */
VSA_API vsa_status vsa_profile_rows(const vsa_shape *shape, const vsa_params *params, int *rows);

/* Workspace bytes of vsa_profile_heads / vsa_build_mask / vsa_attention.  For cube shapes the
 * mask workspace holds the fp64 pooled means (2*B*H*C*d) and coarse scores (B*H*C*C). */
VSA_API size_t vsa_profile_workspace_size(const vsa_shape *shape, const vsa_params *params);
VSA_API size_t vsa_mask_workspace_size(const vsa_shape *shape, const vsa_params *params);
VSA_API size_t vsa_attention_workspace_size(const vsa_shape *shape, const vsa_params *params, vsa_dtype dtype,
                                    vsa_select select);

/* ---------------------------------------------------------------------------------
 * Kernels (asynchronous on `stream`)
 * --------------------------------------------------------------------------------- */

/*
 * Gather natural-order rows into each head's layout ("Sparse Video-Gen" summary,
 * "Approach": token-major to frame-major transformation; "USV" Figure 2: 3D cubes).
 *   src      [B, H, N, d] in src_dtype (VSA_F32 or VSA_BF16), natural order
 *   dst      [B, H, R, d] bf16, R from vsa_layout_rows; temporal heads get frame-major
 *            order (slot s*F + f), cube heads cube-major order with zeroed padding slots
 *   d_kind   [B*H] device bytes (vsa_kind)
 * Spatial heads are left untouched when src is bf16; when src is fp32 they are copied in
 * natural order so that dst holds bf16 values (round to nearest even) for every head.
 */
VSA_API vsa_status vsa_permute(const void *src, vsa_dtype src_dtype, void *dst, const uint8_t *d_kind,
                       const vsa_shape *shape, int *d_err, cudaStream_t stream);

/*
 * Inverse of vsa_permute for outputs: dst[b,h,t] = src[b,h,slot(t)].
 *   src      [B, H, R, d] bf16 in each head's layout;  src_lse [B, H, R] fp32 or NULL
 *   dst      [B, H, N, d] in dst_dtype, natural order;  dst_lse [B, H, N] or NULL
 * Spatial heads are left untouched when dst is bf16 (their output is written in place by
 * vsa_sparse_attn_fwd); when dst is fp32 every head is converted.
 */
VSA_API vsa_status vsa_unpermute(const void *src, const float *src_lse, void *dst, vsa_dtype dst_dtype, float *dst_lse,
                         const uint8_t *d_kind, const vsa_shape *shape, int *d_err, cudaStream_t stream);

/*
 * Online profiling ("Sparse Video-Gen" summary, "Approach"; "Measured effects" rows on the
 * profiling fraction).  For r = ceil(profile_frac*N) evenly strided query rows
 * rho_i = floor((2i+1)N/(2r)) of every head it computes dense attention and attention
 * under the spatial (w_s) and temporal (w_t) block masks, the mean squared difference of
 * each to dense over the r*d outputs, and picks the smaller (ties: spatial).
 *   q, k, v  [B, H, N, d] bf16, natural order
 *   d_kind   [B*H] out: VSA_SPATIAL or VSA_TEMPORAL
 *   d_mse    [B*H*2] out: (spatial, temporal) mean squared error, fp32
 *   ws       at least vsa_profile_workspace_size bytes of device memory
 */
VSA_API vsa_status vsa_profile_heads(const void *q, const void *k, const void *v, const vsa_shape *shape,
                             const vsa_params *params, uint8_t *d_kind, float *d_mse, void *ws, size_t ws_bytes,
                             int *d_err, cudaStream_t stream);

/*
 * vsa_profile_heads without a workspace argument (the pages have no counterpart; this is
 * an interface convenience).  For callers that cannot allocate device memory themselves,
 * e.g. code running under a host framework that owns all device memory through its own
 * pool, or a latency-critical path that must not call cudaMalloc.  The scratch lives in a
 * fixed array of vsa_profile_static_scratch_bytes() (16 MiB) inside the library, held by
 * every GPU that loads the library until the process exits; nothing is allocated.
 *   - Same arguments as vsa_profile_heads, minus ws / ws_bytes.
 *   - To fit the array it may use fewer key-range splits than vsa_profile_heads, so its
 *     fp32 partial sums combine in another order: the MSE values agree with those of
 *     vsa_profile_heads within the profiling tolerance, and a head's kind can differ only
 *     where its two MSEs are a near-tie.
 *   - Shapes whose scratch does not fit (after lowering the number of key-range splits to
 *     1) return VSA_ERR_WORKSPACE without launching anything.
 *   - Every call looks up the array's device address in the current context
 *     (cudaGetSymbolAddress; nothing is cached, so a reset context is handled).  The first
 *     call on a device may load the library's device code: make it before any stream
 *     capture.
 *   - Every call shares the one array per device and leaves its contents behind; each call
 *     writes every scratch byte it reads, so no clearing is needed.  Calls that overlap on
 *     the GPU (different streams, or different host threads on the same device) race on
 *     the array: serialise them.
 */
VSA_API size_t vsa_profile_static_scratch_bytes(void);
VSA_API vsa_status vsa_profile_heads_static(const void *q, const void *k, const void *v, const vsa_shape *shape,
                                            const vsa_params *params, uint8_t *d_kind, float *d_mse, int *d_err,
                                            cudaStream_t stream);

/*
 * Block masks in three equivalent forms, per (b, h, query block i):
 *   d_bits   [B, H, nblk, ceil(nblk/32)] uint32: bit j%32 of word j/32 set when block j is kept
 *   d_kv_idx [B, H, nblk, max_kv] int32: kept key blocks ascending, unused entries -1
 *   d_kv_cnt [B, H, nblk] int32: number of kept key blocks
 * Spatial head: blocks of the natural order, kept when their frame intervals are at most
 * w_s apart.  Temporal head: blocks of the frame-major order, kept when their position
 * intervals are at most w_t apart.  Cube head ("USV", Figure 2): the own cube plus the
 * topk cubes with the largest fp64 score mean(Q over cube) . mean(K over cube'), ties to
 * the smaller index; q_cube / k_cube are the cube-major bf16 Q and K from vsa_permute
 * (required when cube dims are set, else ignored).  Rows past a head's own block count
 * get count 0.  A row that keeps more than max_kv blocks sets VSA_DEVERR_OVERFLOW.
 */
VSA_API vsa_status vsa_build_mask(const uint8_t *d_kind, const void *q_cube, const void *k_cube, const vsa_shape *shape,
                          const vsa_params *params, uint32_t *d_bits, int32_t *d_kv_idx, int32_t *d_kv_cnt,
                          int max_kv, void *ws, size_t ws_bytes, int *d_err, cudaStream_t stream);

/*
 * Work order for vsa_sparse_attn_fwd (no counterpart in the pages; it changes only which
 * query blocks share a CTA and which run at the same time, never a result): per head, the
 * query blocks 0..nb-1 sorted by (first kept key block, block index), where nb is the
 * head's own block count; blocks past nb follow in ascending order.  Query blocks that
 * keep the same key blocks (a cube slab for per-frame heads, a cube position across
 * slabs for per-position heads) then land in the same CTA and in CTAs that run together.
 *   d_kind, d_kv_idx, d_kv_cnt, max_kv   as for vsa_sparse_attn_fwd (device)
 *   d_order  [B, H, nblk] int32 out (device, caller-owned); nblk <= 32768
 */
VSA_API vsa_status vsa_block_order(const uint8_t *d_kind, const int32_t *d_kv_idx, const int32_t *d_kv_cnt,
                                   int max_kv, const vsa_shape *shape, int32_t *d_order, cudaStream_t stream);

/*
 * Block-sparse attention forward ("OSP-Next", "Method"; "Sparse Video-Gen", "Approach"):
 * for every query block i of every head, O_i = softmax(Q_i K_J^T * scale) V_J over the
 * key blocks J = kv_idx[b,h,i,0..cnt), keys past the head's real rows (ragged tail,
 * cube padding) excluded; fp32 accumulation, bf16 output, natural-log LSE.  A row with no
 * key gets O = 0 and LSE = -inf.
 *   natural   q, k, v, o, lse of spatial heads ([B, H, N, d], natural order)
 *   permuted  q, k, v, o, lse of temporal and cube heads ([B, H, R, d]); may be NULL,
 *             in which case every head uses `natural`.  The kernel reads a VSA_TEMPORAL
 *             head's N rows from here whatever order they are in (vsa_semantic_attention
 *             passes its cluster-major rows this way)
 *   d_kind    [B*H] head kinds; d_kv_idx / d_kv_cnt from vsa_build_mask (each list strictly
 *             ascending; a malformed list sets VSA_DEVERR_KV_RANGE and its rows are zero)
 *   d_order   NULL (query blocks paired as 2i, 2i+1) or the [B, H, nblk] permutation from
 *             vsa_block_order (its first nb entries per head must be distinct blocks < nb,
 *             else VSA_DEVERR_KV_RANGE)
 *   scale     softmax scale, 0 selects 1/sqrt(d)
 */
VSA_API vsa_status vsa_sparse_attn_fwd(const vsa_qkvo *natural, const vsa_qkvo *permuted, const uint8_t *d_kind,
                               const int32_t *d_kv_idx, const int32_t *d_kv_cnt, int max_kv,
                               const int32_t *d_order, const vsa_shape *shape, float scale, int *d_err,
                               cudaStream_t stream);

/*
 * vsa_sparse_attn_fwd with every head in natural order ("Sparse Video-Gen" summary page,
 * "Approach": the frame-major layout of temporal heads, applied inside the kernel): temporal
 * heads gather their Q, K, V rows through the frame-major slot map (slot p = s*F + f is token
 * f*S + s) while loading tiles, and write O and LSE rows back to their natural tokens, so no
 * permuted copies exist.  Spatial heads are as in vsa_sparse_attn_fwd.
 *   natural   q, k, v, o, lse ([B, H, N, d] bf16, natural order; lse may be NULL)
 *   the rest  as vsa_sparse_attn_fwd; masks of temporal heads are over frame-major blocks
 * Shapes with cube dims return VSA_ERR_UNSUPPORTED; a cube kind byte sets VSA_DEVERR_KIND.
 */
VSA_API vsa_status vsa_sparse_attn_fwd_natural(const vsa_qkvo *natural, const uint8_t *d_kind,
                                               const int32_t *d_kv_idx, const int32_t *d_kv_cnt, int max_kv,
                                               const int32_t *d_order, const vsa_shape *shape, float scale,
                                               int *d_err, cudaStream_t stream);

/*
 * FP8 Q and K ("Sparse Video-Gen" summary page, "Measured effects": FP8 quantisation added to
 * the sparse attention, 1.92x -> 2.33x end to end; its "Limitations" report no gain at head
 * dimension 64).  The page gives no format; the reading used here: e4m3 codes (round to
 * nearest even, saturating at 448) of x / 2^e, with one power-of-two scale 2^e per block of
 * `block` rows of a head's layout, the smallest with max |x| <= 448 * 2^e (e = 0 for an
 * all-zero block).  P.V stays bf16.
 *
 * vsa_quantize_fp8: codes of one tensor (Q or K) for every head, read as the attention reads
 * them: spatial heads (or every head when `permuted` is NULL) from `natural`, temporal and cube
 * heads from `permuted`.
 *   natural   [B, H, N, d] bf16 (or [B, H, R, d] when permuted is NULL);  permuted [B, H, R, d]
 *   dst       [B, H, R, d] e4m3 codes (caller-owned device memory); rows past a head's own
 *             rows are zero
 *   d_exp     [B*H, nblk] int32 out: the exponent e of every block's scale
 * d must be 128 (VSA_ERR_UNSUPPORTED otherwise); a bad kind byte sets VSA_DEVERR_KIND.
 */
VSA_API vsa_status vsa_quantize_fp8(const void *natural, const void *permuted, const uint8_t *d_kind,
                                    const vsa_shape *shape, uint8_t *dst, int32_t *d_exp, int *d_err,
                                    cudaStream_t stream);

/*
 * vsa_sparse_attn_fwd with Q.K^T on e4m3 codes (tcgen05 kind::f8f6f4, fp32 accumulation): the
 * scores of query block i and key block j are scaled by 2^(qexp[i] + kexp[j]) before the
 * softmax; V, P and O are as in vsa_sparse_attn_fwd.
 *   q8, k8          [B, H, R, d] e4m3 codes from vsa_quantize_fp8 (every head in its layout)
 *   d_qexp, d_kexp  [B*H, nblk] their exponents
 *   the rest        as vsa_sparse_attn_fwd (V, O and LSE from the natural / permuted sets)
 * d = 128 and block = 128 only (VSA_ERR_UNSUPPORTED otherwise).
 */
VSA_API vsa_status vsa_sparse_attn_fwd_fp8qk(const vsa_qkvo *natural, const vsa_qkvo *permuted, const uint8_t *q8,
                                             const int32_t *d_qexp, const uint8_t *k8, const int32_t *d_kexp,
                                             const uint8_t *d_kind, const int32_t *d_kv_idx, const int32_t *d_kv_cnt,
                                             int max_kv, const int32_t *d_order, const vsa_shape *shape,
                                             float scale, int *d_err, cudaStream_t stream);

/*
 * The whole call: kinds (profiled, given or cube) -> permute -> masks -> sparse attention
 * -> unpermute, all on `stream`.
 *   io        natural q, k, v (dtype), o (dtype), lse (fp32, may be NULL)
 *   d_kind    [B*H]: read for VSA_SELECT_GIVEN, written otherwise
 *   d_mse     [B*H*2] written by profiling (may be NULL)
 *   ws        vsa_attention_workspace_size bytes; the masks and permuted tensors live there
 */
VSA_API vsa_status vsa_attention(const vsa_qkvo *io, vsa_dtype dtype, const vsa_shape *shape, const vsa_params *params,
                         vsa_select select, uint8_t *d_kind, float *d_mse, void *ws, size_t ws_bytes, int *d_err,
                         cudaStream_t stream);

/*
 * The whole call on host batches: for every batch i, upload q, k, v from host memory into a
 * device buffer set, run vsa_attention on it and download o back to host memory.  Two buffer
 * sets alternate so that the upload of batch i+1 and the download of batch i-1 overlap the
 * compute of batch i, on three caller streams.  Returns once everything is enqueued; the
 * caller synchronises stream_down (the last download is on it) before reading the outputs.
 * The library allocates no device memory: the sets and the workspace are the caller's.
 *   host      [n] host pointers: q, k, v (read), o (written), each [B, H, N, d] in dtype; they
 *             should be pinned (cudaHostAlloc or registered), else the copies do not overlap
 *   sets      [2] device buffer sets: q, k, v, o [B, H, N, d] in dtype (lse NULL or [B, H, N])
 *   the rest  as vsa_attention (one workspace, kind and MSE array for every batch: batches run
 *             one after the other on stream_compute); for VSA_SELECT_GIVEN the kinds in d_kind
 *             serve every batch
 * Events that order the three streams are created and destroyed inside the call (host-side
 * objects; the destroy calls release them once their work has completed).
 */
typedef struct {
    const void *q, *k, *v;
    void *o;
} vsa_host_batch;

VSA_API vsa_status vsa_attention_host(const vsa_host_batch *host, int n, const vsa_qkvo *sets, vsa_dtype dtype,
                                      const vsa_shape *shape, const vsa_params *params, vsa_select select,
                                      uint8_t *d_kind, float *d_mse, void *ws, size_t ws_bytes, int *d_err,
                                      cudaStream_t stream_up, cudaStream_t stream_compute,
                                      cudaStream_t stream_down);

/* Byte offsets of the mask arrays inside vsa_attention's workspace (for inspection). */
VSA_API vsa_status vsa_attention_workspace_layout(const vsa_shape *shape, const vsa_params *params, vsa_dtype dtype,
                                          vsa_select select, size_t *off_bits, size_t *off_kv_idx,
                                          size_t *off_kv_cnt, int *max_kv);

/* ---------------------------------------------------------------------------------------
 * Semantic-aware permutation ("Sparse VideoGen2" page, abstract: tokens clustered by
 * k-means and reordered by cluster, a top-p budget over clusters).  The page gives no
 * formulas; the readings:
 *   - Lloyd's k-means per head on the bf16 rows (as fp32), `iters` rounds of assignment then
 *     update, starting from the rows floor((2j+1) N / (2C)), j < C;
 *   - assignment: argmin_j |c_j|^2 - 2 x.c_j, ties to the smaller j; |c_j|^2 in fp32 (fused
 *     multiply-adds in dimension order), x.c_j on the tensor cores from the two bf16 halves
 *     of c_j (c_hi + c_lo, within 2^-18 |c_j| per element), fp32 accumulation.  Where two
 *     centroids are within the rounding error of a tie, either label is a correct answer;
 *   - update: fp64 sum of the members in token order / count, rounded to fp32; an empty
 *     cluster keeps its centroid;
 *   - cluster-major order: slots sorted by (cluster, token);
 *   - weight of key cluster j for query cluster i: n_j exp(s_ij - max_j s_ij), s_ij =
 *     scale * cq_i . ck_j in fp64; kept: the shortest prefix of the weights in descending
 *     order (ties to the smaller j) whose running sum reaches top_p of their total;
 *   - block pair (a, b) of the query and key layouts is kept when some query slot of a and
 *     some key slot of b belong to a kept cluster pair.
 * These entry points take shapes without cube dims (VSA_ERR_UNSUPPORTED otherwise), bf16
 * rows, 1 <= C <= min(N, 1024) clusters and 1 <= iters <= 1000.
 * ------------------------------------------------------------------------------------- */

/* Scratch bytes of vsa_kmeans, each piece 256-byte aligned: cluster offsets and chunk offsets
 * [B*H, C+1] int32 each, centroid norms [B*H, C] fp32, the centroids' bf16 halves [B*H, C, d]
 * twice, the update's partial sums over chunks of 128 members ([B*H, M, d] fp64 twice and
 * int32 once, M = ceil(N / 128) + C), the sort's segment histograms [B*H, 8, C] int32, one
 * int32 flag per head and the chunks' clusters [B*H, M] int32.  0 for an invalid shape or
 * count. */
VSA_API size_t vsa_kmeans_workspace_size(const vsa_shape *shape, int n_clusters);

/*
 * k-means of x and its cluster-major order.
 *   x            [B, H, N, d] bf16, natural order (device)
 *   d_centroids  [B*H, C, d] fp32 out: centroids after the last update (16-byte aligned)
 *   d_labels     [B*H, N] int32 out: cluster of every token (last assignment)
 *   d_counts     [B*H, C] int32 out: members per cluster
 *   d_perm       [B*H, N] int32 out: token at each slot of the cluster-major order
 *   ws           vsa_kmeans_workspace_size bytes of scratch
 */
VSA_API vsa_status vsa_kmeans(const void *x, const vsa_shape *shape, int n_clusters, int iters, float *d_centroids,
                              int32_t *d_labels, int32_t *d_counts, int32_t *d_perm, void *ws, size_t ws_bytes,
                              int *d_err, cudaStream_t stream);

/* Scratch bytes of vsa_semantic_mask (the cluster range of every block). */
VSA_API size_t vsa_semantic_mask_workspace_size(const vsa_shape *shape);

/*
 * Top-p cluster budget and the block mask over the two cluster-major layouts.
 *   d_cent_*, d_counts_*, d_labels_*, d_perm_*  vsa_kmeans outputs of Q (cq clusters) and K
 *   top_p        in (0, 1];  scale  the score scale, 0 selects 1/sqrt(d) (fp64)
 *   d_keep       [B*H, cq, ceil(ck/32)] uint32 out: bit j of row i set when key cluster j
 *                is kept for query cluster i
 *   d_bits, d_kv_idx, d_kv_cnt  as vsa_build_mask writes them, with nblk = ceil(N/block)
 *                blocks of the query layout (rows) and of the key layout (columns); a row
 *                keeping more than max_kv blocks sets VSA_DEVERR_OVERFLOW
 *   ws           vsa_semantic_mask_workspace_size bytes of scratch
 * Labels or orders out of range set VSA_DEVERR_KV_RANGE.
 */
VSA_API vsa_status vsa_semantic_mask(const float *d_cent_q, const int32_t *d_counts_q, const int32_t *d_labels_q,
                                     const int32_t *d_perm_q, int cq, const float *d_cent_k, const int32_t *d_counts_k,
                                     const int32_t *d_labels_k, const int32_t *d_perm_k, int ck,
                                     const vsa_shape *shape, float top_p, float scale, uint32_t *d_keep,
                                     uint32_t *d_bits, int32_t *d_kv_idx, int32_t *d_kv_cnt, int max_kv, void *ws,
                                     size_t ws_bytes, int *d_err, cudaStream_t stream);

/* dst[b, h, s] = src[b, h, d_perm[b*H + h, s]] for [B, H, N, d] bf16 rows.  An order entry
 * outside [0, N) sets VSA_DEVERR_KV_RANGE and that row is written as zeros. */
VSA_API vsa_status vsa_gather_rows(const void *src, const int32_t *d_perm, void *dst, const vsa_shape *shape,
                                   int *d_err, cudaStream_t stream);

/* dst[b, h, d_perm[b*H + h, s]] = src[b, h, s] (and the same for the fp32 LSE when both
 * src_lse and dst_lse are given).  An order entry outside [0, N) sets VSA_DEVERR_KV_RANGE. */
VSA_API vsa_status vsa_scatter_rows(const void *src, const float *src_lse, const int32_t *d_perm, void *dst,
                                    float *dst_lse, const vsa_shape *shape, int *d_err, cudaStream_t stream);

typedef struct {
    int cq, ck;    /* clusters of Q and of K per head */
    int iters;     /* k-means rounds */
    float top_p;   /* budget, in (0, 1] */
    float scale;   /* softmax and score scale, 0 selects 1/sqrt(d) */
} vsa_semantic_params;

VSA_API size_t vsa_semantic_workspace_size(const vsa_shape *shape, const vsa_semantic_params *params);

/*
 * The whole semantic call on `stream`: vsa_kmeans of Q and of K, vsa_gather_rows (Q by the
 * query order, K and V by the key order), vsa_semantic_mask, vsa_sparse_attn_fwd with every
 * head read from the permuted rows, vsa_scatter_rows of O (and LSE) through the query order.
 *   io   natural q, k, v, o bf16 [B, H, N, d]; lse fp32 [B, H, N] or NULL
 *   ws   vsa_semantic_workspace_size bytes (clusters, orders, masks and permuted rows)
 */
VSA_API vsa_status vsa_semantic_attention(const vsa_qkvo *io, const vsa_shape *shape,
                                          const vsa_semantic_params *params, void *ws, size_t ws_bytes, int *d_err,
                                          cudaStream_t stream);

/* Self-test hook (the pages have no counterpart): evaluates the kernels' two base-2
 * exponentials, the FMA-pipe polynomial (y_poly) and the hardware approximation (y_mufu),
 * on n device floats, so that tests can bound the polynomial's error. */
VSA_API vsa_status vsa_selftest_exp2(const float *x, float *y_poly, float *y_mufu, int n, cudaStream_t stream);

/* Self-test hook for failure handling (no counterpart in the pages): one thread runs the
 * bounded mbarrier wait all kernels use on a barrier that nothing completes.  After the wait
 * limit (1 s of %globaltimer) it sets VSA_DEVERR_TIMEOUT in *d_err, writes 0 to *d_waited and
 * returns; vsa_get_device_error then reports VSA_ERR_TIMEOUT and the context stays usable.
 *   d_err, d_waited  device ints (d_waited: 1 if the wait succeeded, 0 if it gave up) */
VSA_API vsa_status vsa_selftest_wait_timeout(int *d_err, int *d_waited, cudaStream_t stream);

/* Self-test hook (no counterpart in the pages): cudaDeviceReset of the current device through
 * the library's own CUDA runtime.  It ends the calling process's context on that device, so
 * every device buffer of the process becomes invalid; tests use it to check that entry points
 * work again afterwards on new buffers (vsa_profile_heads_static looks its array's address up
 * per call). */
VSA_API vsa_status vsa_selftest_device_reset(void);

/* Synchronise `stream`, copy the device error word to *host_err and map it to a status
 * (VSA_OK when zero, VSA_ERR_TIMEOUT when the timeout bit is set, else VSA_ERR_DEVICE). */
VSA_API vsa_status vsa_get_device_error(const int *d_err, cudaStream_t stream, int *host_err);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
