/*
 * vdm.h -- C ABI of the B200 vecset SDF decoder ("lightning vecset decoder").
 *
 * A vecset is an unordered set of N latent tokens of width C that encodes one
 * shape; its decoder is a cross-attention from 3D query points to the token
 * set followed by the signed distance (SDF) at each point (FlashVDM,
 * "Unleashing Vecset Diffusion Model for Fast Shape Generation", aipaper.cc
 * summary, section 3 "foundational concepts: decoder").  Decoding a volume
 * means running that cross-attention for millions of grid points, which the
 * pages name the dominant cost of shape generation (section 2; techwalker
 * article, section 1: VAE decoding is 75.8% of end-to-end time).  The three
 * accelerations of section 4.1 are exposed here:
 *   1. hierarchical volume decoding (coarse pass, sign-change + near-surface
 *      marking, one dilation, refinement of the marked voxels only);
 *   2. adaptive KV selection (per sub-volume probe queries rank the tokens,
 *      the rest of the sub-volume attends to the Top-K tokens only);
 *   3. the efficient (slim) decoder: any width C = 64 H, MLP width F, and the
 *      query-side LayerNorms optional (query_ln = 0).
 *
 * Decoder network, per query point p (W[out][in] row-major, y = x W^T + b):
 *   pe  = [p, sin(2^k pi p_a), cos(2^k pi p_a)]  k = 0..7; lane 3+8a+k = sin,
 *         lane 27+8a+k = cos, lanes 51..63 = 0 (64 lanes)
 *   q   = Wq pe + bq                                        Wq: [C][64]
 *   K,V = LN_kv(z) Wk^T + bk, LN_kv(z) Wv^T + bv, split into H heads of 64
 *   a_h = softmax(q_h K_h^T / 8) V_h  (dense, or over a token subset)
 *   x1  = q + Wo a + bo
 *   x2  = x1 + W2 GELU(W1 LN1(x1) + b1) + b2                (LN1 iff query_ln)
 *   dec = w_head . LN2(x2) + b_head                         (LN2 iff query_ln)
 * LayerNorm: biased variance, eps 1e-5.  GELU: exact erf form.
 * Optional analytic term (synthetic shapes): field = min_s(|p - c_s| - r_s)
 *   + dec_scale * tanh(dec); without it the output is dec itself.
 * Grid: voxel (i,j,k) of an R^3 grid sits at -1 + (2i+1)/R per axis; linear
 *   index (i R + j) R + k (x slowest).  Children of a voxel at 2R: (2i+di, ...).
 *
 * Conventions for every entry point:
 *   - Pointers named d_* / documented "device" are CUDA device memory owned by
 *     the caller; the library never allocates device memory.  Host pointers
 *     are documented as such.
 *   - Work is ordered on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  vdm_precompute_kv returns without waiting.  The decode and
 *     selection calls synchronise `stream` before they return, so that the
 *     status of their device-side waits reaches the caller who made the call
 *     (vdm_decode_hierarchical also reads counts back once per level).
 *   - Errors are returned as vdm_status; nothing aborts, throws across the
 *     ABI or traps on the device.  vdm_last_error() gives a thread-local
 *     message for the last failing call.  Launch failures return VDM_ERR_CUDA;
 *     a tensor-core kernel whose bounded wait expired returns VDM_ERR_TIMEOUT
 *     from the call that launched it.
 *   - Shared device state: the device error word and, for C = 512 decoders on
 *     the tensor cores, a 20 MiB area that holds half of the residual stream
 *     while the MLP runs, are global to the library on each device.  Decode
 *     calls that overlap on the GPU (different streams or host threads, same
 *     device) race on them: issue decodes of one device on one stream.
 *   - Results are bit-identical run to run (no floating-point atomics).
 *   - Limits: head dim 64; C in {64, 128, 256, 512}; F a multiple of 64 and
 *     <= 4096; 1 <= N <= 8192; B >= 1.  Other shapes: VDM_ERR_UNSUPPORTED.
 */
#ifndef VDM_H
#define VDM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VDM_API __attribute__((visibility("default")))
#else
#define VDM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* vdm_stream; /* == cudaStream_t */

typedef enum {
    VDM_OK = 0,
    VDM_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, negative size ... */
    VDM_ERR_UNSUPPORTED = 2,   /* shape outside the limits above */
    VDM_ERR_WORKSPACE = 3,     /* workspace missing or too small */
    VDM_ERR_CUDA = 4,          /* a CUDA call or launch failed */
    VDM_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up */
    VDM_ERR_INTERNAL = 6
} vdm_status;

typedef enum { VDM_F32 = 0, VDM_BF16 = 1 } vdm_dtype;

#define VDM_HEAD_DIM 64
#define VDM_PE_LANES 64
#define VDM_MAX_LEVELS 6

/* Decoder parameters (all device pointers).  Matrices are stored in `dtype`
 * (float or bf16), row-major W[out][in]; vectors are float32.  Every matrix
 * and vector (except b_head) must be 16-byte aligned.  K and V produced by
 * vdm_precompute_kv are stored in `dtype` as well.                          */
typedef struct {
    int32_t C;          /* width, = 64 * H                                   */
    int32_t H;          /* heads                                             */
    int32_t F;          /* MLP hidden width                                  */
    int32_t query_ln;   /* 1: LayerNorm before the MLP and before the head   */
    vdm_dtype dtype;
    const void* Wq;     /* [C][64]; columns 51..63 meet zero embedding lanes */
    const void* Wk;     /* [C][C] */
    const void* Wv;     /* [C][C] */
    const void* Wo;     /* [C][C] */
    const void* W1;     /* [F][C] */
    const void* W2;     /* [C][F] */
    const float *bq, *bk, *bv, *bo, *b1, *b2;            /* [C] ([F] for b1) */
    const float *ln_kv_g, *ln_kv_b;                      /* [C]              */
    const float *ln1_g, *ln1_b, *ln2_g, *ln2_b;          /* [C]              */
    const float* w_head;                                 /* [C]              */
    const float* b_head;                                 /* [1]              */
    /* Optional truncated-SDF head (NULL: none): t = w_tsdf . LN2(x2) + b_tsdf,
     * a second linear output on the same final features (the pages' VAE is
     * trained to output a tSDF beside the SDF: aipaper.cc summary, section
     * 4.1 item 1, "key details" 1).  With it, hierarchical decoding takes
     * |tSDF| < vdm_hier_params.tsdf_threshold as its near-surface rule.      */
    const float* w_tsdf;                                 /* [C] or NULL      */
    const float* b_tsdf;                                 /* [1]              */
} vdm_decoder;

/* Analytic term of the synthetic field (optional).                         */
typedef struct {
    const float* spheres;  /* device [B][n_spheres][4] = (cx, cy, cz, r)     */
    int32_t n_spheres;     /* >= 1                                           */
    float dec_scale;       /* field = sphere SDF + dec_scale * tanh(dec)     */
    float tsdf_trunc;      /* with a tSDF head: tSDF = clip((sphere SDF +
                              dec_scale * tanh(t)) / tsdf_trunc, -1, 1); > 0 */
} vdm_analytic;

/* K/V projection of B vecsets (section 3: the vecset feeds the decoder's
 * cross-attention as keys and values).
 *   d_z     [B][N][C] float32 latents
 *   d_k_out [B][H][N][64] in dec->dtype  (keys)
 *   d_v_out [B][H][N][64] in dec->dtype  (values)
 * Errors: INVALID_ARG (null pointer, B/N < 1), UNSUPPORTED (limits).        */
VDM_API vdm_status vdm_precompute_kv(const vdm_decoder* dec, const float* d_z, int32_t B, int32_t N,
                             void* d_k_out, void* d_v_out, vdm_stream stream);

/* Dense decode: the decoder at M points per shape, full attention over all
 * N tokens (section 3; the plain "baseline" decoder of Table 3).
 *   d_k, d_v  [B][H][N][64] from vdm_precompute_kv
 *   d_xyz     [B][M][3] float32 points, or NULL: the points are the voxels of
 *             the grid_R^3 grid in linear order (then M must be grid_R^3)
 *   analytic  host pointer or NULL (raw decoder output)
 *   d_out     [B][M] float32
 * M = 0 is a no-op.  Returns after the decode has finished on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA, TIMEOUT.                          */
VDM_API vdm_status vdm_decode_dense(const vdm_decoder* dec, const void* d_k, const void* d_v,
                            int32_t B, int32_t N, const float* d_xyz, int64_t M, int32_t grid_R,
                            const vdm_analytic* analytic, float* d_out, vdm_stream stream);

/* Adaptive KV selection for T sub-volumes of one shape (section 4.1 item 2,
 * steps 2-4): the probe queries of sub-volume t are
 * d_probe_xyz[d_tile_off[t] .. d_tile_off[t+1]); every token gets the score
 * sum over probes and heads of its softmax weight, and the top_k tokens (ties
 * to the smaller index) are written in ascending index order.
 *   d_probe_xyz   [P][3] float32, P = d_tile_off[T]
 *   d_tile_off    [T+1] int32, non-decreasing, d_tile_off[0] = 0 (device)
 *   P_total       P (host value; must match d_tile_off[T])
 *   d_sel_out     [T][top_k] int32 (device)
 *   d_score_out   [T][N] float32 or NULL
 *   d_probe_dec_out [P] float32 or NULL: the raw decoder output at every
 *                 probe (full attention; the probes' values are final in the
 *                 adaptive procedure, section 4.1 item 2 step 3)
 * Sub-volumes with no probe select tokens 0..top_k-1.  top_k >= N selects
 * every token.
 * Kernels: with a bf16 decoder of width 128, 256 or 512 and at most 128
 * probes per sub-volume, the tensor-core kernels of vdm_decode_hierarchical's
 * adaptive levels (the probes are decoded with full attention, which gives
 * their per-head softmax maximum and sum, then scored and ranked in one
 * pass), so for the same probes, in the same order, the scores and the
 * selection are bit-identical to that path's; otherwise a CUDA-core kernel
 * (any dtype, width and probe count).  The tensor-core route takes a
 * stream-ordered temporary allocation (cudaMallocAsync / cudaFreeAsync on
 * `stream`) of about T * 128 * H * 8 + 4 P bytes.
 * Synchronisation: d_tile_off is copied to the host and checked first (one
 * round trip on `stream`); the call returns after the selection has finished.
 * Errors: INVALID_ARG (offsets not starting at 0, decreasing or not ending at
 * P_total), UNSUPPORTED (N, top_k > 8192), CUDA, TIMEOUT.                   */
VDM_API vdm_status vdm_select_kv(const vdm_decoder* dec, const void* d_k, const void* d_v, int32_t N,
                         const float* d_probe_xyz, const int32_t* d_tile_off, int32_t T,
                         int64_t P_total, int32_t top_k, int32_t* d_sel_out, float* d_score_out,
                         float* d_probe_dec_out, vdm_stream stream);

/* Hierarchical volume decoding parameters (section 4.1 items 1-2).        */
typedef struct {
    int32_t r0;          /* coarse resolution, multiple of 4                 */
    int32_t n_levels;    /* >= 1; final resolution r0 * 2^(n_levels-1)      */
    int32_t adaptive;    /* 1: adaptive KV selection on the fine levels      */
    int32_t tile;        /* sub-volume edge in fine voxels; must be 8        */
    int32_t n_probe;     /* probes per sub-volume, 1..512                    */
    int32_t top_k;       /* kept tokens per sub-volume                       */
    uint64_t seed;       /* probe sampler seed                               */
    float tsdf_threshold;/* with a tSDF head: near-surface voxels are those
                            with |tSDF| < tsdf_threshold (0.95 on the pages:
                            techwalker article, section 5), compared in
                            float32; without one: |f| < float32(4 / R)      */
} vdm_hier_params;

/* Per-shape, per-level counts written by vdm_decode_hierarchical (host).   */
typedef struct {
    int64_t resolution[VDM_MAX_LEVELS];
    int64_t decoded[VDM_MAX_LEVELS];        /* queries decoded at the level  */
    int64_t active_parents[VDM_MAX_LEVELS]; /* refined voxels of level l-1   */
    int64_t tiles[VDM_MAX_LEVELS];          /* non-empty sub-volumes         */
    int64_t selected_tiles[VDM_MAX_LEVELS]; /* sub-volumes with selection    */
    int64_t probes[VDM_MAX_LEVELS];         /* queries decoded over all N
                                               tokens: probes plus every query
                                               of sub-volumes with <= n_probe
                                               queries (adaptive levels)      */
} vdm_hier_stats;

/* Optional per-level copies for testing (all device pointers, nullable; a
 * NULL entry skips that copy).  Shapes are handled one after the other, so
 * each array holds shape b at offset b * (its per-shape size).  "Sub-volume i"
 * below is entry i of tile_ids: the i-th non-empty 8^3 sub-volume of the fine
 * level in ascending sub-volume order.  Entries for i >= max_tiles are not
 * written.                                                                  */
typedef struct {
    float* grid[VDM_MAX_LEVELS];        /* [B][R_l^3] dense field of level l */
    uint64_t* active[VDM_MAX_LEVELS];   /* [B][(R_l/4)^3] refine mask of level
                                           l (l < n_levels-1): word w = block
                                           (bi,bj,bk) of 4^3 voxels in linear
                                           block order, bit (di*4+dj)*4+dk   */
    float* dec[VDM_MAX_LEVELS];         /* [B][R_l^3] raw decoder output at the
                                           voxels decoded at level l; other
                                           voxels are left untouched         */
    int32_t* tile_ids[VDM_MAX_LEVELS];  /* [B][max_tiles] sub-volume ids (linear
                                           index of the 8^3 tile at level l)
                                           of the non-empty sub-volumes       */
    int32_t* sel[VDM_MAX_LEVELS];       /* [B][max_tiles][top_k] kept tokens of
                                           sub-volume i (rows of sub-volumes
                                           without a selection, those with at
                                           most n_probe queries: unspecified) */
    int64_t max_tiles;                  /* capacity of the per-sub-volume rows */
    int32_t* probes[VDM_MAX_LEVELS];    /* [B][max_tiles][n_probe] fine voxel
                                           indices of the probes of sub-volume
                                           i in rank order (all its queries if
                                           it has <= n_probe), -1 padded      */
    float* scores[VDM_MAX_LEVELS];      /* [B][max_tiles][N] token scores of
                                           sub-volume i (rows of sub-volumes
                                           without a selection: untouched)   */
    float* attn[VDM_MAX_LEVELS];        /* [B][ceil(R_l^3/attn_stride)][C]
                                           attention output a (heads
                                           concatenated, before Wo) at every
                                           decoded voxel v of level l with
                                           v % attn_stride == 0, in row
                                           v / attn_stride; other rows are
                                           left untouched                    */
    int64_t attn_stride;                /* >= 1 when any attn[l] is set       */
    float* tsdf[VDM_MAX_LEVELS];        /* [B][R_l^3] tSDF grid of level l
                                           (decoded or inherited), decoders
                                           with a tSDF head only             */
} vdm_hier_debug;

/* Workspace bytes needed by vdm_decode_hierarchical (host output).         */
VDM_API vdm_status vdm_hierarchical_workspace_size(const vdm_decoder* dec, const vdm_hier_params* p,
                                           int32_t N, size_t* bytes);

/* Hierarchical volume decoding of B shapes (section 4.1 item 1, with item 2
 * on the fine levels when p->adaptive):
 *   level 0: dense decode of the r0^3 grid;
 *   level l -> l+1: mark voxels with a sign change in their 3x3x3
 *   neighbourhood or |f| < 2h (h = 2/R_l, threshold float32(4/R_l); with a
 *   tSDF head: |tSDF| < p->tsdf_threshold instead), dilate
 *   once (3x3x3), decode the 8 children of every marked voxel at 2R_l, and let
 *   the other fine voxels inherit their parent's value.
 *   d_grid_out [B][Rf^3] float32 final field, Rf = r0 * 2^(n_levels-1)
 *   d_ws/ws_bytes  device workspace >= vdm_hierarchical_workspace_size
 *   stats    host, B entries, nullable;  debug  host, nullable
 * Synchronisation: after each level's marking the call copies two counts to
 * the host and synchronises `stream` (one round trip per level), and it
 * synchronises once more at the end to read the device error status.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA, TIMEOUT.              */
VDM_API vdm_status vdm_decode_hierarchical(const vdm_decoder* dec, const void* d_k, const void* d_v,
                                   int32_t B, int32_t N, const vdm_hier_params* p,
                                   const vdm_analytic* analytic, float* d_grid_out,
                                   void* d_ws, size_t ws_bytes, vdm_hier_stats* stats,
                                   const vdm_hier_debug* debug, vdm_stream stream);

/* Hierarchical decoding with no device allocation at all (no counterpart in
 * the paper; a deployment aid).  Same arguments and results as
 * vdm_decode_hierarchical, minus the workspace: the scratch space is a 32 MiB
 * array built into the library (held on every GPU that loads it until the
 * process exits).  For callers that may not call cudaMalloc: applications that
 * own all device memory themselves, and latency-critical code that avoids
 * cudaMalloc/cudaFree because they can synchronise the device.
 *   - Problems whose vdm_hierarchical_workspace_size exceeds 32 MiB return
 *     VDM_ERR_UNSUPPORTED (a 32 -> 64 -> 128 adaptive decode with 32 probes and
 *     top_k 512 needs about 27 MiB, with 64 probes and top_k 1024 about 44 MiB,
 *     which is rejected; 64 -> 128 -> 256 without adaptive KV about 18 MiB).
 *   - All calls on a device share that scratch: calls that overlap on the GPU
 *     race; issue them one after another on one stream.
 *   - Like vdm_decode_hierarchical, the call synchronises `stream` once per
 *     level and once at the end.
 *   - The first call on each device looks up the scratch address (no
 *     allocation); make that first call before any stream capture.          */
VDM_API vdm_status vdm_decode_hierarchical_noalloc(const vdm_decoder* dec, const void* d_k,
                                                   const void* d_v, int32_t B, int32_t N,
                                                   const vdm_hier_params* p,
                                                   const vdm_analytic* analytic, float* d_grid_out,
                                                   vdm_hier_stats* stats,
                                                   const vdm_hier_debug* debug, vdm_stream stream);

/* One level step of hierarchical volume decoding without the decoder
 * (section 4.1 item 1, steps 2-3, and the inherit fill), for callers that run
 * their own decoder on the refined voxels:
 *   mark: voxels with a sign change in their 3x3x3 neighbourhood or
 *   |f| < float32(4 / R); dilate once (3x3x3); compact the refined voxels;
 *   fill: every voxel of the (2R)^3 grid takes its parent's value (decoding
 *   the children of refined voxels then overwrites them).
 *   d_f        [R^3] float32 (device, 16-byte aligned), R % 4 == 0, R <= 512
 *   d_f_fine   [(2R)^3] float32 (device, 16-byte aligned) or NULL (no fill)
 *   d_mask     [(R/4)^3] uint64 blocked refine mask (layout of vdm_hier_debug)
 *   d_parents  [R^3] int32 or NULL: refined voxels' linear indices, grouped by
 *              4^3 block in block order, ascending bit order inside a block
 *   d_counts   [2] int32 (device): refined voxels, non-empty 4^3 blocks
 *   d_ws/ws_bytes  device workspace >= vdm_refine_workspace_size(R)
 * Asynchronous on `stream`.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
VDM_API vdm_status vdm_refine_workspace_size(int32_t R, size_t* bytes);
VDM_API vdm_status vdm_refine_level(const float* d_f, int32_t R, float* d_f_fine, uint64_t* d_mask,
                                    int32_t* d_parents, int32_t* d_counts, void* d_ws, size_t ws_bytes,
                                    vdm_stream stream);

/* Vecset encoding: a point cloud -> a vecset of N latent tokens by
 * cross-attention (aipaper.cc summary, section 3 "Foundational Concepts:
 * encoder").  The tokens sit at N query points (normally a subset of the
 * cloud); every point of the cloud is embedded with the decoder's Fourier
 * features and projected, u = W_in pe(p) + b_in; the block's LayerNorm and K/V
 * projections make keys and values of u (as vdm_precompute_kv does of
 * latents); each token runs the block from its query point (q = Wq pe(x) + bq,
 * attention over the cloud, x1 = q + Wo a + bo, x2 = x1 + MLP(LN1 x1)) and is
 * its block output x2.  The block uses the vdm_decoder layout; its head and
 * LN2 are not used.
 *   blk         block parameters (any supported C; dtype of W_in as well)
 *   d_W_in      [C][64] in blk->dtype (columns 51..63 meet zero lanes); d_b_in [C]
 *   d_points    [B][M][3] float32, 1 <= M <= 8192;  d_queries [B][N][3] float32
 *   d_z_out     [B][N][C] float32 vecsets (a decoder's vdm_precompute_kv input)
 *   d_ws/ws_bytes  device workspace >= vdm_encode_workspace_size(blk, M)
 * Returns after the encoding has finished on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA, TIMEOUT.               */
VDM_API vdm_status vdm_encode_workspace_size(const vdm_decoder* blk, int32_t M, size_t* bytes);
VDM_API vdm_status vdm_encode(const vdm_decoder* blk, const void* d_W_in, const float* d_b_in,
                              const float* d_points, int32_t B, int32_t M, const float* d_queries,
                              int32_t N, float* d_z_out, void* d_ws, size_t ws_bytes, vdm_stream stream);

/* Local (MSVS-style) decoder query on a multi-scale latent hierarchy (kwkr.cn
 * MSVS-VAE article, section 1.1 "AVS-Conv" and section 1.3 "multi-scale query
 * decoding"): per scale s the K anchors nearest to the query (squared
 * distances in float32, summed x, y then z, no fused multiply-adds; ties to
 * the smaller anchor index) are aggregated with per-channel dynamic weights
 * from a small MLP of the relative offsets plus a mean-pooling residual,
 *   f_s(x) = (1/K) sum_j (W2_s GELU(W1_s (a_j - x) + b1_s) + b2_s + 1) * F_j,
 * and the scales are fused into the SDF: wo . GELU(Wf [f_0, f_1, ...] + bf) + bo.
 * All arrays are float32 device memory; anchors anywhere (those outside
 * [-1, 1]^3 only make the neighbour search visit more cells).             */
#define VDM_LOCAL_MAX_SCALES 4
typedef struct {
    int32_t n_scales;                          /* 1..4                          */
    int32_t K;                                 /* neighbours per scale, 1..16   */
    int32_t hidden;                            /* dynamic-weight width, 1..32   */
    int32_t fuse_hidden;                       /* fusion width, 1..64           */
    int32_t n_anchors[VDM_LOCAL_MAX_SCALES];   /* host values, K..2^20          */
    int32_t channels[VDM_LOCAL_MAX_SCALES];    /* C_s, multiple of 4, <= 64;
                                                  sum over scales <= 128        */
    const float* anchors[VDM_LOCAL_MAX_SCALES];/* [n_s][3]                      */
    const float* feats[VDM_LOCAL_MAX_SCALES];  /* [n_s][C_s], 16-byte aligned   */
    const float* W1[VDM_LOCAL_MAX_SCALES];     /* [hidden][3]                   */
    const float* b1[VDM_LOCAL_MAX_SCALES];     /* [hidden]                      */
    const float* W2[VDM_LOCAL_MAX_SCALES];     /* [C_s][hidden]                 */
    const float* b2[VDM_LOCAL_MAX_SCALES];     /* [C_s]                         */
    const float* Wf;                           /* [fuse_hidden][sum C_s]        */
    const float* bf;                           /* [fuse_hidden]                 */
    const float* wo;                           /* [fuse_hidden]                 */
    const float* bo;                           /* [1]                           */
} vdm_local_decoder;

/* SDF of the local decoder at M points.
 *   d_xyz      [M][3] float32;  d_out [M] float32
 *   d_knn_out  [M][n_scales][K] int32 neighbour indices (nearest first) or NULL
 *   d_ws/ws_bytes  device workspace >= vdm_local_workspace_size (the anchors'
 *              grid binning, rebuilt at every call)
 * M = 0 is a no-op.  Returns after the decode has finished on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.                        */
VDM_API vdm_status vdm_local_workspace_size(const vdm_local_decoder* dec, size_t* bytes);
VDM_API vdm_status vdm_decode_local(const vdm_local_decoder* dec, const float* d_xyz, int64_t M, float* d_out,
                                    int32_t* d_knn_out, void* d_ws, size_t ws_bytes, vdm_stream stream);

/* Comparison of two fields sampled on the same grid, for accuracy reports
 * (aipaper.cc summary, section 5 "Evaluation Metrics": volume IoU of the
 * inside sets; Table 3 reports it for each acceleration of the decoder).
 * Inside means f < 0.  One pass over both arrays.
 *   d_a, d_b  [n] float32 (device)
 *   d_out     [5] uint64 (device, 8-byte aligned): number of voxels inside
 *             a, inside b, inside both, with the same sign in a and b, and
 *             the largest |a - b| as float32 bits in the low 32 bits
 * V-IoU = d_out[2] / (d_out[0] + d_out[1] - d_out[2]); sign agreement =
 * d_out[3] / n.  Counts are exact integers; asynchronous on `stream`.
 * Errors: INVALID_ARG, CUDA.                                                */
VDM_API vdm_status vdm_compare_volumes(const float* d_a, const float* d_b, int64_t n, uint64_t* d_out,
                                       vdm_stream stream);

/* Surface extraction (techwalker article, section 1: the pipeline's last
 * stage after VAE decoding): marching cubes on the samples of a decoded
 * R^3 volume (voxel centres, as above), visiting only the 8^3-cube blocks
 * near voxels with a 26-neighbour of the other sign; the mesh equals marching
 * cubes over every cube of the grid.  Inside is f < 0.
 *   d_f            [R^3] float32 (device, 16-byte aligned), R % 8 == 0, R <= 1024
 *   d_vertices     [max_vertices][3] float32 xyz (device)
 *   d_triangles    [max_triangles][3] int32 vertex indices (device); triangle
 *                  normals (right-hand rule) point to f > 0
 *   n_vertices, n_triangles  host outputs: the mesh's sizes (written even when
 *                  the capacity is too small, which returns VDM_ERR_WORKSPACE and
 *                  writes nothing else; capacities of 0 query the sizes)
 *   d_ws/ws_bytes  device workspace >= vdm_surface_workspace_size(R)
 * Case rules (no memorised table; the 256 cases are generated from them): a
 * face with two sign changes gets one segment; with four, two segments that
 * each cut off one inside corner; loops are fanned from their first vertex
 * (loop order from the smallest edge id) with no fan diagonal inside a face.
 * Edge e = 4 a + 2 u + v runs along axis a between the corners whose other
 * two coordinates are (u, v); corner c = 4 ci + 2 cj + ck.  Vertex on the
 * crossed edge from sample p0 to p0 + e_a: p0 + t h e_a, t = f0 / (f0 - f1),
 * h = 2 / R.  Order: samples (vertex owners, vertices in axis order) and cubes
 * (by minimum corner; triangles in loop and fan order) by 8^3 block in linear
 * block order, then linear order inside the block.
 * Synchronises `stream` twice (sizes, then the mesh).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA, INTERNAL.              */
VDM_API vdm_status vdm_surface_workspace_size(int32_t R, size_t* bytes);
VDM_API vdm_status vdm_extract_surface(const float* d_f, int32_t R, float* d_vertices, int64_t max_vertices,
                                       int32_t* d_triangles, int64_t max_triangles, int64_t* n_vertices,
                                       int64_t* n_triangles, void* d_ws, size_t ws_bytes, vdm_stream stream);
/* The generated case table (host outputs, for inspection and tests):
 * ntri[256] triangles per sign pattern (bit c = corner c inside) and
 * tri[256][5][3] their edge ids.                                            */
VDM_API vdm_status vdm_surface_case_table(uint8_t* ntri, uint8_t* tri);

/* Test hook for failure detection (not needed for decoding).  mode n >= 1
 * makes the n-th tensor-core decode launch from now on (1 = the next one)
 * withhold one completion signal, so its warps run into their bounded waits;
 * `timeout_cycles` (> 0) shortens those waits.  The call that made that
 * launch returns VDM_ERR_TIMEOUT (a hierarchical call checks after each
 * level's marking and at its end) and the CUDA context stays usable.  mode 0
 * restores normal operation.                                                */
VDM_API vdm_status vdm_debug_inject(int32_t mode, int64_t timeout_cycles);

/* Test hook for the decoder's softmax arithmetic (not needed for decoding):
 * d_y[i] = 2^d_x[i] (device float32 arrays of n elements, n >= 0) computed the
 * way the tensor-core decoder computes a quarter of its softmax exponentials:
 * x = m + f with m = round(x) and f in [-1/2, 1/2] (range reduction in the
 * manner of Cody and Waite), 2^f by a cubic fitted for this function (relative
 * error <= 7.5e-5 for -125 <= x <= 9), 2^m added to the exponent field.
 * Inputs below -125 (and -inf) give a result in [0, 2^-124] (not 0, and not
 * accurate once it leaves the normal range); NaN is not an input the decoder
 * produces and gives no meaningful result.
 * Asynchronous on `stream`.  Errors: INVALID_ARG, CUDA.                     */
VDM_API vdm_status vdm_debug_exp2(const float* d_x, float* d_y, int64_t n, vdm_stream stream);

/* Test hook for the decoder's GELU (not needed for decoding): for the n inputs
 * d_x (device float32), d_y[i] = the tensor-core decoder's GELU of x_i as it
 * feeds the MLP's second matrix (bf16, widened to float32; computed on pairs of
 * inputs), and d_y[n + i] = the same GELU in scalar float32 before rounding.
 * GELU(x) = x Phi(x), with erf by Abramowitz & Stegun formula 7.1.26 (absolute
 * error <= 1.5e-7).  d_y holds 2 n floats.  Asynchronous on `stream`.
 * Errors: INVALID_ARG, CUDA.                                                */
VDM_API vdm_status vdm_debug_gelu(const float* d_x, float* d_y, int64_t n, vdm_stream stream);

/* Tensor-core decoding on CTA pairs: with enable = 1, each 256-query MMA runs
 * on the two CTAs of a cluster (cta_group::2); each CTA holds 128 query rows
 * and loads half of every weight and key/value tile, which halves the bytes
 * each SM streams per query.  enable = 0 (the default) runs one CTA per
 * 128-query MMA.  Both give the same results up to the order of floating-point
 * sums.  Measured on B200: pairs are slightly faster when attention is short
 * (128 tokens), and slower for 3072-token attention and on the adaptive
 * hierarchical workload.  Takes effect for the launches that follow; not
 * thread-safe against concurrent decodes.                                     */
VDM_API vdm_status vdm_set_cta_pairs(int32_t enable);

/* Kernel timing for measurement (not needed for decoding).  Between
 * vdm_profile_begin() and vdm_profile_end() the calling thread's launches are
 * bracketed by CUDA events on their stream; vdm_profile_end() waits for those
 * events and returns, per kernel class, the launch count and the summed
 * device time.  Classes: 0 K/V projection, 1 decode, 2 probe scoring + Top-K,
 * 3 mark + dilate, 4 scan, 5 parent list / offsets, 6 inherit fill,
 * 7 probe ordering.                                                         */
#define VDM_PROF_CLASSES 8
typedef struct {
    int64_t launches[VDM_PROF_CLASSES];
    double ms[VDM_PROF_CLASSES];
} vdm_profile;
VDM_API vdm_status vdm_profile_begin(void);
VDM_API vdm_status vdm_profile_end(vdm_profile* out);

VDM_API const char* vdm_status_string(vdm_status s);
VDM_API const char* vdm_last_error(void);   /* thread-local message of the last error */
VDM_API int32_t vdm_abi_version(void);      /* 3                                      */

#ifdef __cplusplus
}
#endif
#endif /* VDM_H */
