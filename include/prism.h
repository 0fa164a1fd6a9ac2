/*
 * prism.h — C ABI of the Prism dynamic block-sparse attention hot path for
 * NVIDIA B200 (sm_100a).
 *
 * Prism ("Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio
 * Generation Model Training"; README of Tencent-Hunyuan/Prism, section
 * "Overview") organises the video token grid into spatiotemporal macro-zones,
 * gives every zone one 64-token block shape chosen from the video features'
 * channel variance and the norm of the audio-to-video (a2v) bridge residual,
 * represents blocks by block-level (mean-pooled) features, selects key blocks
 * per query block with a hybrid top-k + cumulative-mass rule, and runs exact
 * attention over the selected blocks only, forward and backward.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Token order is raster over the latent grid (T, H, W):
 *   token n = (t * H + h) * W + w.
 * - Zones tile the grid in raster (zt, zh, zw) order; zone z covers
 *   [zt*Zt, zt*Zt+Zt) x [zh*Zh, ...) x [zw*Zw, ...).
 * - A block shape is (bt, bh, bw) with bt*bh*bw == 64 dividing the zone
 *   extents. The blocks of zone z are numbered raster over the zone's
 *   (Zt/bt, Zh/bh, Zw/bw) sub-grid; global block id = z * blocks_per_zone +
 *   local id, blocks_per_zone = Zt*Zh*Zw/64. Tokens inside a block are raster
 *   (t, h, w). Query and key blocks use the same partition.
 * - Grids that are not a whole number of zones (real video latents, e.g. 45
 *   latent rows at 720p; the Prism pages train at 720p, 1080p and 2K and do
 *   not say how edges are tiled; this is the library's reading): zones tile
 *   the grid rounded up to whole zones, so n_zones = prod ceil(extent/zone),
 *   and the last zone along a clipped axis covers only the grid's remainder.
 *   Block boxes tile the unclipped zone as above and keep their ids; a block's
 *   members are the slots of its box inside the grid (fewer than 64 at the
 *   edge), and a box with no member is an empty block. Zone statistics use the
 *   member tokens (lines clipped), pooling averages the members (an empty
 *   block's pooled row is NaN), the selection never keeps an empty block and
 *   leaves its row empty, and attention runs over member tokens only.
 * - Q, K, V, O, dO, dQ, dK, dV are token-major [N, heads, head_dim] with a
 *   token stride of `tok_stride` elements (>= heads*head_dim, a multiple of 8)
 *   and contiguous heads and channels.
 * - Pointers marked "device" must be device memory of the current device;
 *   "host" pointers are read (or written) before the call returns. The
 *   library never allocates or frees device memory: scratch comes from the
 *   caller's workspace `ws` of `ws_bytes` bytes (256-byte aligned), sized by
 *   prism_workspace_size(). Work is enqueued on `stream` (a cudaStream_t; NULL
 *   is the legacy default stream) and is asynchronous unless stated.
 * - Every call validates its arguments on the host and returns a status; no
 *   exception crosses the ABI. Device-side faults are avoided by design:
 *   device waits are bounded and report PRISM_ERR_TIMEOUT, index checks
 *   report PRISM_ERR_DEVICE, through prism_check_device_status().
 * - Not re-entrant on one workspace: calls that share `ws` must be ordered on
 *   one stream.
 */
#ifndef PRISM_H_
#define PRISM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PRISM_API __attribute__((visibility("default")))
#else
#define PRISM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PRISM_OK = 0,
  PRISM_ERR_ARG = 1,         /* NULL where a pointer is required, bad scalar */
  PRISM_ERR_SHAPE = 2,       /* grid / zone / candidate geometry invalid */
  PRISM_ERR_DTYPE = 3,       /* dtype not supported for this argument */
  PRISM_ERR_WORKSPACE = 4,   /* ws NULL, misaligned or smaller than required */
  PRISM_ERR_CAPACITY = 5,    /* col_cap smaller than the number of kept pairs */
  PRISM_ERR_CUDA = 6,        /* a CUDA runtime / driver call failed */
  PRISM_ERR_TIMEOUT = 7,     /* a bounded device wait gave up */
  PRISM_ERR_DEVICE = 8,      /* a device-side index check failed */
  PRISM_ERR_UNSUPPORTED = 9  /* size outside what the kernels implement */
} prism_status;

typedef enum { PRISM_BF16 = 0, PRISM_FP32 = 1 } prism_dtype;

typedef struct {
  int32_t t, h, w;
} prism_dim3;

/* Token-grid geometry shared by the block-level entry points.
 * grid: latent token grid (T, H, W); zone: macro-zone extents (Zt, Zh, Zw)
 * (need not divide the grid, see above), with Zt*Zh*Zw a multiple of 64 and
 * at most 512;
 * cand: host array of n_cand (1..16) candidate block shapes. */
typedef struct {
  prism_dim3 grid;
  prism_dim3 zone;
  const prism_dim3* cand;
  int32_t n_cand;
} prism_geometry;

/* Constants of the zone shape rule (see prism_zone_shapes). */
typedef struct {
  float w_audio;  /* weight of the audio term, default 1 */
  float gamma;    /* isotropy penalty, default 0.25 */
  float gate_max; /* cap G of the audio gate, default 4 */
} prism_shape_params;

/* Which call a workspace is sized for. */
typedef enum {
  PRISM_OP_ZONE_SHAPES = 0,
  PRISM_OP_BLOCK_SELECT = 1,
  PRISM_OP_BSA_FWD = 2,
  PRISM_OP_BSA_BWD = 3
} prism_op;

/* Human-readable name of a status. Never NULL. */
PRISM_API const char* prism_status_string(prism_status s);

/* Library version, major*10000 + minor*100 + patch. */
PRISM_API int32_t prism_version(void);

/* Number of zones and of blocks for a geometry (host only, no GPU work). */
PRISM_API prism_status prism_geometry_counts(const prism_geometry* geo, int32_t* n_zones, int32_t* n_blocks);

/* Workspace bytes needed by `op`. `nnz` is the number of selected
 * (query block, key block) pairs summed over heads (row_ptr[heads*n_blocks]),
 * used by PRISM_OP_BSA_BWD only. `in_dtype` is the dtype of Q/K/V (fp32
 * inputs need bf16 staging copies). Host only. */
PRISM_API prism_status prism_workspace_size(prism_op op, const prism_geometry* geo, int32_t heads, int32_t head_dim,
                                  int32_t feat_c, int32_t res_c, prism_dtype in_dtype, int64_t nnz,
                                  size_t* bytes);

/* Reads and clears the device status word kept in `ws` (synchronises
 * `stream`). Returns PRISM_ERR_TIMEOUT or PRISM_ERR_DEVICE if a kernel that
 * used this workspace reported one, else PRISM_OK. */
PRISM_API prism_status prism_check_device_status(void* ws, void* stream);

/*
 * a1 + a2 — macro-zone tiling and per-zone block shape.
 * Cites: README "Overview" (zones; video feature variance along the channel
 * and a2v feature norms; finer partitioning along axes of rapid visual change
 * and strong audio-visual coupling); walkthrough (wmrh.cn/news/72296) section
 * "桥接残差反哺稀疏注意力" (per-token L2 norm of the unscaled a2v residual as
 * the audio-influence proxy; sounding regions get finer blocks) and section
 * "三者如何协同" (candidate shapes, one per zone).
 *
 * The rule (no formula is printed; this is the library's documented
 * reading): for zone z and axis a in (t, h, w), V_a = mean over channels and
 * over lines parallel to a of the population variance of the feature along
 * the line; r(n) = ||res[n, :]||_2, A_a = mean over lines parallel to a of
 * the population variance of r; g = clamp(mean_z r / mean_grid r - 1, 0,
 * gate_max); S_a = 3 V_a / (sum V + 1e-12) + w_audio * g * 3 A_a / (sum A +
 * 1e-12), renormalised to sum 3 (all ones when zero); cost(c) = sum_a S_a *
 * log2(ext_{c,a}) + gamma * sum_a (log2(ext_{c,a}) - 2)^2; the zone takes the
 * argmin, ties to the lower candidate index.
 *
 * feat: device [N, feat_c] row stride feat_ld elements (bf16 or fp32), or
 *       NULL; res: device [N, res_c] row stride res_ld, or NULL. Both NULL:
 *       every zone takes candidate 0. Row strides are multiples of 8 elements
 *       and feat_c / res_c multiples of 64.
 * params: host, NULL for the defaults.
 * zone_shape: device int32 [n_zones] out (candidate index per zone).
 * zone_margin: device float [n_zones] out (second-best minus best cost), or
 *       NULL.
 * A statistics kernel whose bounded wait for its copies ran out leaves every
 * zone_shape entry -1 (and every margin NaN) besides setting PRISM_ERR_TIMEOUT
 * in the workspace status word.
 */
PRISM_API prism_status prism_zone_shapes(const prism_geometry* geo, const void* feat, int64_t feat_ld, int32_t feat_c,
                               prism_dtype feat_dtype, const void* res, int64_t res_ld, int32_t res_c,
                               prism_dtype res_dtype, const prism_shape_params* params, int32_t* zone_shape,
                               float* zone_margin, void* ws, size_t ws_bytes, void* stream);

/*
 * prism_zone_shapes without a workspace (the Prism pages have no counterpart
 * to this entry point; it is a deployment variant of a1 + a2).
 *
 * For callers that cannot allocate device memory: code that runs inside a
 * host framework owning every device allocation (a serving runtime's fixed
 * pool, a plugin interface that hands out no scratch buffer), or code that must
 * not call cudaMalloc after start-up because it would synchronise the device
 * in the middle of its work. Inputs, outputs and the result are exactly those
 * of prism_zone_shapes; only the scratch differs: it lives in one static
 * device array of 4 MiB inside the library, which every GPU that loads the
 * library holds until the process exits. That bounds the grid: about 7 bytes
 * per token plus 32 per zone with 3072 bf16 channels (the 2K grid of 294,912
 * tokens needs 2.1 MB); a call that needs more returns PRISM_ERR_UNSUPPORTED.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine). The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress with that device current), and looks it up again when
 * the device's context has changed (after cudaDeviceReset the module is
 * reloaded and the array may move); make that first call before any stream
 * capture. All calls share the array and it keeps the last call's contents, so
 * calls that overlap on the GPU (different streams, or several host threads)
 * race and must be serialised by the caller. There is no workspace status word
 * to read back: a device-side wait that ran out shows as zone_shape entries of
 * -1 (margins NaN), which the downstream entry points reject as out of range.
 */
PRISM_API prism_status prism_zone_shapes_static(const prism_geometry* geo, const void* feat, int64_t feat_ld,
                                                int32_t feat_c, prism_dtype feat_dtype, const void* res,
                                                int64_t res_ld, int32_t res_c, prism_dtype res_dtype,
                                                const prism_shape_params* params, int32_t* zone_shape,
                                                float* zone_margin, void* stream);

/*
 * a3 — block partition and mean pooling ("block-level features", README
 * "Overview"): q_pool[h, b, :] = mean of the 64 rows Q[n, h, :] of block b,
 * likewise k_pool.
 * zone_shape: device int32 [n_zones] (from prism_zone_shapes).
 * q, k: device [N, heads, head_dim], bf16 or fp32, token stride tok_stride.
 * q_pool, k_pool: device float [heads, n_blocks, head_dim] out.
 * head_dim is 64 or 128; heads * head_dim <= 8192.
 * ws: workspace of at least prism_workspace_size(PRISM_OP_BLOCK_SELECT, ...)
 *       bytes; only its status word is used (an out-of-range zone_shape entry
 *       leaves that block's pooled rows as NaN and reports PRISM_ERR_DEVICE).
 */
PRISM_API prism_status prism_block_pool(const prism_geometry* geo, const int32_t* zone_shape, const void* q, const void* k,
                              prism_dtype dtype, int32_t heads, int32_t head_dim, int64_t tok_stride, float* q_pool,
                              float* k_pool, void* ws, size_t ws_bytes, void* stream);

/*
 * a4 + a5 — block scoring and hybrid selection (walkthrough section
 * "三者如何协同": the gating step takes the k highest-scoring blocks, then
 * extends along the CDF until cdf_threshold, default 0.20; README "Overview":
 * hybrid selection sets each query's sparsity; Sol-Attn abstract on the
 * Prism paper page: blocks ranked by a block proxy score).
 *
 * For head h and query block I: s_J = scale * q_pool[h,I] . k_pool[h,J] over
 * all key blocks J; p = softmax(s); blocks ranked by p descending, ties to the
 * lower J; m = max(top_k, min{m : p_(1) + ... + p_(m) >= cdf_threshold});
 * top_k >= n_blocks or cdf_threshold >= 1 keeps every block. The logits are
 * formed on the tensor cores in split tf32 precision (hi.hi + hi.lo + lo.hi,
 * relative error about 2^-20) for a round of heads at a time and held in the
 * workspace (a round of heads whose logits fit in 1 GiB) until that round's
 * selection has read them; they are not an output.
 *
 * q_pool, k_pool: device float [heads, n_blocks, head_dim]; n_blocks at most
 *       10240 and heads * n_blocks^2 below 2^31 (PRISM_ERR_UNSUPPORTED
 *       otherwise). A NaN pooled row marks an empty block (see the
 *       conventions): never kept as a key; as a query its row is empty.
 * top_k >= 1; cdf_threshold >= 0.
 * mask: device uint32 [heads, n_blocks, ceil(n_blocks/32)] out; bit (J % 32)
 *       of word J / 32 of row (h, I) is set when J is kept.
 * kept: device int32 [heads, n_blocks] out (m per row).
 * row_ptr: device int32 [heads*n_blocks + 1] out, CSR offsets over the rows
 *       taken in (h, I) order.
 * col_idx: device int32 [col_cap] out, kept J of each row ascending; NULL to
 *       skip (then col_cap is ignored).
 * total_kept: host int64 out (synchronises `stream`), or NULL. When col_idx
 *       is given and the total exceeds col_cap the call returns
 *       PRISM_ERR_CAPACITY after the sync, with col_idx untouched (this check
 *       needs total_kept != NULL; without it the fill clips at col_cap and
 *       reports PRISM_ERR_DEVICE through prism_check_device_status).
 * ws: at least prism_workspace_size(PRISM_OP_BLOCK_SELECT, geo, heads,
 *       head_dim, ...) bytes (equivalently prism_block_select_workspace_size):
 *       the status word, the tf32 halves of q_pool and k_pool (4 * heads *
 *       n_blocks * head_dim floats) and one round's logits (R * n_blocks *
 *       ceil4(n_blocks) floats, R = the heads whose logits fit in 1 GiB, at
 *       least 1).
 */
PRISM_API prism_status prism_block_select(const float* q_pool, const float* k_pool, int32_t heads, int32_t n_blocks,
                                int32_t head_dim, float scale, int32_t top_k, float cdf_threshold, uint32_t* mask,
                                int32_t* kept, int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                                int64_t* total_kept, void* ws, size_t ws_bytes, void* stream);

/* Per-call selection settings of prism_block_select_ex. */
typedef struct {
  int32_t top_k;                   /* k of every head when head_top_k is NULL (>= 1) */
  float cdf_threshold;             /* tau of every head when head_cdf_threshold is NULL (>= 0) */
  const int32_t* head_top_k;       /* host int32 [heads] (each >= 1), or NULL */
  const float* head_cdf_threshold; /* host float [heads] (each >= 0), or NULL */
  const float* key_bias;           /* device float [n_blocks], or NULL: b_J added to s_J */
} prism_select_params;

/*
 * a4 + a5 with per-head settings and an optional key-block scoring bias.
 *
 * Per-head k and tau: the walkthrough (wmrh.cn/news/72296) section
 * "实际案例与上手参考" exposes the selection as a tunable knob
 * (BSA_SPARSITY, a top-k sparsity ratio); this entry point lets every head
 * carry its own floor k_h and mass threshold tau_h. Scoring bias: the same
 * walkthrough, section "桥接残差反哺稀疏注意力", says the per-token norm of the
 * a2v residual is read when BSA scores blocks and that sounding regions keep
 * more attention; with key_bias (e.g. from prism_block_audio_bias) the logits
 * become s_J = scale * q_pool[h,I] . k_pool[h,J] + b_J for every head before
 * the ranking and the softmax. Otherwise the rule, outputs and their layout
 * are those of prism_block_select, with k = k_h and tau = tau_h in row (h, I).
 * With head_top_k = head_cdf_threshold = key_bias = NULL the result is
 * identical to prism_block_select(top_k, cdf_threshold).
 *
 * params: host, required. Per-head arrays need heads <= 128
 *       (PRISM_ERR_UNSUPPORTED above); any k < 1 or tau < 0 (or NaN) returns
 *       PRISM_ERR_ARG before any work is enqueued. key_bias must be 4-byte
 *       aligned; a NaN entry gives its key block no mass.
 */
PRISM_API prism_status prism_block_select_ex(const float* q_pool, const float* k_pool, int32_t heads,
                                             int32_t n_blocks, int32_t head_dim, float scale,
                                             const prism_select_params* params, uint32_t* mask, int32_t* kept,
                                             int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                                             int64_t* total_kept, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of prism_block_select / prism_block_select_ex for pooled
 * features of `heads` x `n_blocks` x `head_dim` (the same value as
 * prism_workspace_size(PRISM_OP_BLOCK_SELECT, ...) for that geometry's block
 * count), for callers that hold only the pooled shapes. Host only. */
PRISM_API prism_status prism_block_select_workspace_size(int32_t heads, int32_t n_blocks, int32_t head_dim,
                                                         size_t* bytes);

/*
 * Top-k floor from a top-k sparsity ratio (walkthrough section
 * "实际案例与上手参考": BSA_SPARSITY sets the top-k sparsity ratio). The library's
 * reading: the ratio is the fraction of key blocks the top-k part drops, so
 * k = n_blocks - floor(sparsity * n_blocks) with the product formed in double
 * from the float argument, at least 1; that is the smallest count that keeps
 * at least the fraction 1 - sparsity of the blocks. Host only.
 * sparsity in [0, 1), n_blocks >= 1, top_k: host out. PRISM_ERR_ARG otherwise.
 */
PRISM_API prism_status prism_topk_from_sparsity(float sparsity, int32_t n_blocks, int32_t* top_k);

/*
 * Audio-norm bias of every key block, for prism_block_select_ex (walkthrough
 * section "桥接残差反哺稀疏注意力": the per-token L2 norm of the unscaled a2v
 * residual is the proxy of how strongly audio drives a visual region, read
 * when BSA scores blocks; sounding regions keep more attention). The library's
 * reading: b_J = beta * mean_{n in block J} r(n) / mean_{all n} r(n),
 * r(n) = ||res[n, :]||_2 (fp32 per token, fp64 grid mean). The ratio makes
 * the bias independent of the residual's scale; a zero residual gives b = 0.
 *
 * zone_shape: device int32 [n_zones] (from prism_zone_shapes); the blocks are
 *       those of prism_block_pool.
 * res: device [N, res_c] (bf16 or fp32), row stride res_ld elements (a
 *       multiple of 8), res_c a positive multiple of 8, 16-byte aligned.
 * beta: finite scale of the bias (0 gives b = 0).
 * key_bias: device float [n_blocks] out.
 * ws: at least prism_workspace_size(PRISM_OP_BLOCK_SELECT, ...) bytes; only
 *       its status word is used (an out-of-range zone_shape entry leaves the
 *       whole bias NaN and reports PRISM_ERR_DEVICE).
 */
PRISM_API prism_status prism_block_audio_bias(const prism_geometry* geo, const int32_t* zone_shape, const void* res,
                                              int64_t res_ld, int32_t res_c, prism_dtype res_dtype, float beta,
                                              float* key_bias, void* ws, size_t ws_bytes, void* stream);

/*
 * Expands a selection bitmask (as written by prism_block_select) into the
 * CSR column lists: col_idx[row_ptr[r] .. row_ptr[r+1]) = the set bits of row
 * r, ascending. Use it after a prism_block_select call made with
 * col_idx = NULL and total_kept to size col_idx. Rows past col_cap are left
 * unwritten and reported through prism_check_device_status.
 * mask: device uint32 [rows, ceil(n_blocks/32)]; row_ptr: device int32
 * [rows+1]; col_idx: device int32 [col_cap] out.
 */
PRISM_API prism_status prism_mask_to_csr(const uint32_t* mask, const int32_t* row_ptr, int32_t rows, int32_t n_blocks,
                                         int32_t* col_idx, int64_t col_cap, void* ws, size_t ws_bytes, void* stream);

/*
 * a6 — block-sparse attention forward (Sol-Attn abstract: compute only the
 * selected key/value blocks): for every query token i of block I,
 * O_i = sum over key tokens j of the blocks in row (h, I) of the CSR of
 * softmax_j(scale * q_i . k_j) v_j, and lse[h, i] = log sum_j exp(scale q_i.k_j)
 * (natural log). Exact up to bf16 operand rounding; fp32 accumulation.
 *
 * zone_shape: device int32 [n_zones].
 * q, k, v: device [N, heads, head_dim], bf16 (fp32 inputs are rounded to bf16
 *       in the workspace), token stride tok_stride. head_dim 64 or 128.
 * row_ptr, col_idx: device CSR from prism_block_select (rows with no block
 *       give O = 0 and lse = -inf).
 * nnz: row_ptr[heads*n_blocks] (the total_kept of prism_block_select), or -1
 *       when the caller does not know it. It only chooses how the work is
 *       laid out: with at most 32 selected key blocks per row on average the
 *       kernel gathers K and V straight from k and v, row after row, and the
 *       workspace's block images go unused; otherwise (and for -1) K and V
 *       are first made block images. Any value >= -1 gives the same result;
 *       below -1 is PRISM_ERR_ARG.
 * o: device [N, heads, head_dim] out, same dtype as q, token stride tok_stride.
 * lse: device float [heads, N] out.
 * o_lo: optional device bf16 [N, heads, head_dim] out (token stride
 *       tok_stride), or NULL: the rounding residual of the bf16 output,
 *       O_fp32 - bf16(O_fp32), so that O_fp32 = o + o_lo to about 16 bits.
 *       Passing it to prism_bsa_bwd makes D_i = dO_i . O_i exact to that
 *       precision; with a nearly one-hot softmax, dS = P (dP - D) cancels
 *       and bf16 rounding of O alone would dominate dQ and dK. Ignored (may be
 *       NULL) for fp32 outputs, which carry no rounding.
 * ws: at least prism_workspace_size(PRISM_OP_BSA_FWD, ...) bytes. It holds
 *       block-major copies of K and V (2 * heads * n_blocks * head_dim * 128
 *       bytes: each 64-token block of each head as one contiguous, already
 *       swizzled operand tile, so the kernel gathers a key block with one bulk
 *       copy) and, for fp32 inputs, the bf16 copies of Q, K and V.
 */
PRISM_API prism_status prism_bsa_fwd(const prism_geometry* geo, const int32_t* zone_shape, const void* q, const void* k,
                           const void* v, prism_dtype dtype, int32_t heads, int32_t head_dim, int64_t tok_stride,
                           float scale, const int32_t* row_ptr, const int32_t* col_idx, int64_t nnz, void* o,
                           float* lse, void* o_lo, void* ws, size_t ws_bytes, void* stream);

/*
 * a7 — block-sparse attention backward (Prism trains natively with the
 * sparse attention, README "Overview"), selection held fixed:
 * D_i = sum_c dO_ic O_ic; P_ij = exp(scale q_i.k_j - lse_i) on the selected
 * blocks; dV_j = sum_i P_ij dO_i; dS_ij = P_ij (dO_i . v_j - D_i);
 * dQ_i = scale sum_j dS_ij k_j; dK_j = scale sum_i dS_ij q_i.
 * Arguments as prism_bsa_fwd; o, o_lo (or NULL) and lse are the forward's
 * outputs (with o_lo, D_i = dO_i . (O_i + O_lo_i)); dout is device
 * [N, heads, head_dim]; dq, dk, dv are device outs like q. nnz =
 * row_ptr[heads*n_blocks] (for workspace sizing; checked against ws_bytes).
 * With at most 32 selected key blocks per row on average the passes gather
 * their streamed blocks straight from the inputs and the block-major copies
 * below go unused; the result is the same.
 * ws: at least prism_workspace_size(PRISM_OP_BSA_BWD, ...) bytes: D and the
 *       LSE in block order, the CSC of the selection (4 bytes per selected
 *       pair), two block-major operand copies (2 * heads * n_blocks *
 *       head_dim * 128 bytes; K and V for the dQ pass, then Q and dO for the
 *       dK/dV pass) and, for fp32 inputs, bf16 copies of Q, K, V and dO.
 */
PRISM_API prism_status prism_bsa_bwd(const prism_geometry* geo, const int32_t* zone_shape, const void* q, const void* k,
                           const void* v, const void* o, const void* o_lo, const float* lse, const void* dout,
                           prism_dtype dtype,
                           int32_t heads, int32_t head_dim, int64_t tok_stride, float scale, const int32_t* row_ptr,
                           const int32_t* col_idx, int64_t nnz, void* dq, void* dk, void* dv, void* ws,
                           size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H_ */
