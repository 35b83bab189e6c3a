/*
 * zb.h -- C ABI of the Zebra3D hybrid global-attention layer for NVIDIA B200
 * (sm_100a).  Library: linear_hybrid_attention_b200/libzb.so.
 *
 * The layer has two stage types.  A sensitive stage runs tile-sparse softmax
 * attention: every query tile keeps exact softmax over its top-k key tiles and
 * each omitted key tile is folded into one mean-key/mean-value landmark.  A
 * tolerant stage runs linear attention whose output is mapped by a per-head
 * affine (A, b) fitted in closed form to the dense output.  Sources (by page
 * title): "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D
 * Reconstruction" -- Abstract and Figure 1 (a) caption; "Zebra3D speeds up 3D
 * reconstruction by up to 7.1x on 1024 frames without training from scratch"
 * -- section "How Zebra3D works".
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are DEVICE pointers, row-major and contiguous.  Q, K, V, O are
 *    [heads][n_tokens][head_dim]; bf16 values are passed as their uint16_t bit
 *    patterns.  Every pointer must be 16-byte aligned.
 *  - The caller owns every buffer.  The library allocates no device memory,
 *    frees nothing it did not allocate, and keeps no reference after return.
 *  - Every compute call is asynchronous on `stream` (a cudaStream_t passed as
 *    void*; NULL = the legacy default stream).  Arguments are validated on the
 *    host before anything is launched: a bad argument returns an error code and
 *    launches nothing.  A failed launch returns ZB_ERR_CUDA.  No call aborts or
 *    exits the process.
 *  - Device-side problems (a bounded wait that ran out, an index list that is
 *    out of range or not strictly ascending, a singular fit) are recorded in a
 *    per-device status word that zb_last_device_status() reports.
 *  - head_dim must be 64; tile must be 64 or 128.  Batch > 1 is folded into
 *    heads.
 *  - Tiles are contiguous runs of `tile` tokens of the flattened
 *    [views x tokens] order; T = ceil(n_tokens / tile); the last tile holds
 *    n_tokens - (T-1)*tile tokens.
 */
#ifndef ZB_H
#define ZB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum zb_status {
    ZB_OK = 0,
    ZB_ERR_NULL = 1,        /* a required pointer is NULL                         */
    ZB_ERR_SHAPE = 2,       /* a size or count is out of range                    */
    ZB_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                   */
    ZB_ERR_UNSUPPORTED = 4, /* head_dim != 64, tile not 64/128, too many tiles    */
    ZB_ERR_WORKSPACE = 5,   /* workspace pointer NULL or smaller than required    */
    ZB_ERR_CUDA = 6,        /* a CUDA runtime call or a kernel launch failed      */
    ZB_ERR_TIMEOUT = 7,     /* a bounded device-side wait gave up (device status) */
    ZB_ERR_DEVICE = 8,      /* the current device is not an sm_100 GPU            */
    ZB_ERR_INDEX = 9,       /* an index list was out of range / not ascending     */
    ZB_ERR_SINGULAR = 10    /* a least-squares system was not positive definite   */
} zb_status;

typedef struct zb_shape {
    int32_t heads;    /* H >= 1                                   */
    int64_t n_tokens; /* N >= 1, views x tokens_per_view          */
    int32_t head_dim; /* d, must be 64                            */
    int32_t tile;     /* t, 64 or 128                             */
} zb_shape;

/* Version of this ABI (major * 100 + minor). */
int32_t zb_abi_version(void);

/* Human-readable name of a zb_status value (static string, never NULL). */
const char* zb_status_string(int32_t status);

/*
 * Landmarks: the per-tile means of Q, K and V.
 * Figure 1 (a) caption of "Zebra3D: Efficient Hybrid Foundation Models ...":
 * an omitted key tile is replaced by its mean key and mean value.  The mean
 * query of a tile is the pooled query used for tile scoring.
 *   in : Q, K, V      bf16 [H][N][d]
 *   out: Qbar, Kbar   fp64 [H][T][d]  means, summed in fp64 (exact for bf16
 *                     inputs unless a tile's values span > ~38 binades)
 *        Kbar_bf16, Vbar_bf16  bf16 [H][T][d]  the means rounded to nearest
 *                     even, in the layout zb_tile_sparse_attn reads
 *   Q and Qbar may both be NULL (no query pooling).
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED, ZB_ERR_CUDA.
 */
zb_status zb_landmark_build(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            zb_shape s, double* Qbar, double* Kbar,
                            uint16_t* Kbar_bf16, uint16_t* Vbar_bf16, void* stream);

/*
 * Tile selection: for every (head h, query tile i) the k key tiles j with the
 * largest score Qbar[h,i] . Kbar[h,j] (fp64 dot products), equal scores going
 * to the lower j; the kept set is written in ascending order.  The pages name
 * "selected tiles" (Figure 1 (a) caption) without the criterion; this is the
 * mean-pooled reading.  The budget k is the kept share of the key tiles (the
 * y in "xL/yS" of the Table 20 caption is the dropped share).
 * The selection is that of the fp64 scores, but most scores are never formed
 * in fp64: each row of Qbar and Kbar becomes three signed 8-bit digit planes of
 * a 21-bit fixed-point copy, int8 tensor-core products give every score to
 * within a proven bound, and only the key tiles whose approximate score lies
 * within that bound of the k-th largest are re-scored in fp64 (one FMA chain
 * over d in index order) to decide the boundary.
 *   in : Qbar, Kbar fp64 [H][T][d];  0 <= k <= T
 *   ws : scratch for one group of heads: digit planes, exponents and an fp32
 *        score matrix (T x T rounded up to 128 columns) per head.  Its size
 *        for one head is zb_tile_score_topk_workspace_bytes() of a one-head
 *        shape; a larger ws takes that many heads per pass (up to all H).  The
 *        default size (4 heads) is zb_tile_score_topk_workspace_bytes(s).
 *        16-byte aligned, owned by the caller, not shared with a call running
 *        at the same time.  Not needed (may be NULL) when k == 0 or k == T.
 *   out: idx int32 [H][T][k]
 * Non-finite values in Qbar or Kbar do not stop the call: the rows they reach
 * are ranked by the fp64 order keys of their scores alone (NaN keys above
 * +inf or below -inf by sign).
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED (T > 32768),
 * ZB_ERR_WORKSPACE, ZB_ERR_CUDA; ZB_ERR_TIMEOUT in the device status if a
 * bounded wait of the score GEMM gave up.
 */
size_t zb_tile_score_topk_workspace_bytes(zb_shape s);
zb_status zb_tile_score_topk(const double* Qbar, const double* Kbar, zb_shape s,
                             int32_t k, int32_t* idx, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * Tile-sparse softmax attention with landmarks (Figure 1 (a) caption; section
 * "How Zebra3D works").  For query row r of tile i, softmax runs over
 *   - every key of each selected tile j in idx[h][i] (logit scale * q.k), and
 *   - if use_landmarks != 0, one landmark per unselected tile j with logit
 *     scale * q.Kbar_bf16[h][j] + ln(n_j) and value Vbar_bf16[h][j];
 * O_r is the softmax-weighted sum of the matching values.  bf16 tensor-core
 * products, fp32 accumulation and softmax, O rounded to bf16.
 *   in : Q, K, V bf16 [H][N][d];  Kbar_bf16, Vbar_bf16 bf16 [H][T][d] (may be
 *        NULL when use_landmarks == 0);  idx int32 [H][T][k], each row strictly
 *        ascending in [0, T) (checked on the device: ZB_ERR_INDEX);  0 <= k <= T
 *        (k == 0 needs use_landmarks);  scale > 0 (usually 1/sqrt(d)).
 *   ws : NULL, or zb_tile_sparse_attn_workspace_bytes() bytes, 16-byte aligned,
 *        owned by the caller and not shared with a call running at the same
 *        time.  With a workspace the call zeroes a counter in it (in stream
 *        order) and launches cooperatively; the work items in flight on all SMs
 *        then start each round together, so their ascending sweeps over a
 *        head's selected K/V tiles stay close and share L2 (far less DRAM
 *        traffic at long sequences).  The result is bit-identical either way.
 *   out: O bf16 [H][N][d];  lse fp32 [H][N] natural-log log-sum-exp of each
 *        row's logits (may be NULL).
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED (T > 32768),
 * ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
size_t zb_tile_sparse_attn_workspace_bytes(void);
zb_status zb_tile_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                              const uint16_t* Kbar_bf16, const uint16_t* Vbar_bf16,
                              const int32_t* idx, int32_t k, int32_t use_landmarks,
                              float scale, zb_shape s, uint16_t* O, float* lse,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * Dense softmax attention softmax(scale * Q K^T) V: the unconverted layer the
 * pages compare against, and the target Y of the affine fit.  Same kernel as
 * zb_tile_sparse_attn with every key tile kept and no landmarks; queries and
 * keys may have different lengths.
 *   in : Q bf16 [H][n_q][d];  K, V bf16 [H][n_kv][d]
 *   out: O [H][n_q][d], bf16 (out_fp32 == 0) or fp32 (out_fp32 != 0);
 *        lse fp32 [H][n_q] (may be NULL)
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED, ZB_ERR_CUDA.
 */
zb_status zb_dense_attn(const uint16_t* Q, int64_t n_q, const uint16_t* K,
                        const uint16_t* V, int64_t n_kv, int32_t heads,
                        int32_t head_dim, float scale, void* O, int32_t out_fp32,
                        float* lse, void* stream);

/*
 * Dense softmax attention as zb_dense_attn, with the keys split into `splits`
 * equal parts so that a small query set (the affine fit's calibration rows:
 * "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D
 * Reconstruction", Abstract, closed-form fit against the dense layer) fills
 * the GPU.  The dense kernel runs over heads * splits virtual heads (virtual
 * head h * splits + p sees keys [p n_kv / splits, (p + 1) n_kv / splits) of
 * head h: the same [H][n_kv][d] memory viewed as [H * splits][n_kv / splits][d])
 * into fp32 partial outputs with their log-sum-exp, and a merge kernel forms
 *   O = sum_p e^(lse_p - M) O_p / sum_p e^(lse_p - M),  M = max_p lse_p,
 *   lse = M + ln sum_p e^(lse_p - M)  (natural log),
 * the softmax over all n_kv keys.  splits == 1 is zb_dense_attn itself.
 *   in : Q bf16 [H][n_q][d];  K, V bf16 [H][n_kv][d];  1 <= splits <= 16,
 *        n_kv a multiple of splits
 *   ws : zb_dense_attn_split_workspace_bytes() bytes (0 for splits == 1):
 *        query replicas, partial outputs and their lse; 16-byte aligned,
 *        owned by the caller, not shared with a call running at the same time
 *   out: O [H][n_q][d], bf16 (out_fp32 == 0) or fp32;  lse fp32 [H][n_q]
 *        (may be NULL)
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE (also n_kv not a multiple of splits),
 * ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED, ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
size_t zb_dense_attn_split_workspace_bytes(int64_t n_q, int32_t heads, int32_t head_dim, int32_t splits);
zb_status zb_dense_attn_split(const uint16_t* Q, int64_t n_q, const uint16_t* K, const uint16_t* V,
                              int64_t n_kv, int32_t heads, int32_t head_dim, float scale, int32_t splits,
                              void* O, int32_t out_fp32, float* lse, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * Linear-attention state (Abstract: linear attention for tolerant stages):
 *   S[h] = sum_r phi(k_r)^T v_r  (d x d),  z[h] = sum_r phi(k_r)  (d),
 * phi(x) = elu(x) + 1, non-causal over all N tokens.  phi(k) is rounded to
 * bf16 for the tensor-core product; sums are fp32 and the per-CTA partials are
 * added in a fixed order (deterministic).
 *   in : K, V bf16 [H][N][d];  ws of >= zb_linear_state_workspace_bytes() bytes
 *   out: S fp32 [H][d][d] (row index = feature of phi(k), column = value dim),
 *        z fp32 [H][d]
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED,
 * ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
size_t zb_linear_state_workspace_bytes(int32_t heads, int64_t n_tokens, int32_t head_dim);
zb_status zb_linear_state(const uint16_t* K, const uint16_t* V, int32_t heads,
                          int64_t n_tokens, int32_t head_dim, float* S, float* z,
                          void* ws, size_t ws_bytes, void* stream);

/*
 * Linear-attention output with the per-head affine map (section "How Zebra3D
 * works": the linear parts are corrected by a closed-form affine map):
 *   O_r = (phi(q_r) S / (phi(q_r) . z)) A + b      (row vectors)
 * computed around the centre c = 1^T S / 1^T z (the output for phi(q) = 1):
 *   O_r = phi(q_r) ((S - z c^T) A) / (phi(q_r) . z) + (c A + b),
 * an exact identity that keeps rounded intermediates small.
 *   out_fp32 == 0: bf16 O; (S - z c^T) A and z are rounded to bf16 for the
 *                  tensor-core product, the division and the bias are fp32.
 *   out_fp32 != 0: fp32 O computed on the CUDA cores in fp32 (meant for
 *                  calibration-sized row sets such as the affine fit's X).
 *   in : Q bf16 [H][n_q][d];  S fp32 [H][d][d];  z fp32 [H][d];
 *        A fp32 [H][d][d] or NULL (identity);  b fp32 [H][d] or NULL (zero)
 *   out: O [H][n_q][d] (bf16 or fp32, see above)
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED, ZB_ERR_CUDA.
 */
zb_status zb_linear_apply(const uint16_t* Q, int32_t heads, int64_t n_q,
                          int32_t head_dim, const float* S, const float* z,
                          const float* A, const float* b, void* O, int32_t out_fp32,
                          void* stream);

/*
 * The whole linear-attention stage in one call: zb_linear_state followed by
 * zb_linear_apply (bf16 output) on the same tokens, the state S, z kept in the
 * workspace (Abstract: linear attention for the tolerant stages; section "How
 * Zebra3D works": its output corrected by the per-head affine map).
 *   in : Q, K, V bf16 [H][N][d];  A fp32 [H][d][d] or NULL (identity);
 *        b fp32 [H][d] or NULL (zero);  ws of >= zb_linear_attn_workspace_bytes()
 *        bytes, 16-byte aligned, owned by the caller
 *   out: O bf16 [H][N][d]
 * Two kernel launches for the state, one for the output, all on `stream`.
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED,
 * ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
size_t zb_linear_attn_workspace_bytes(int32_t heads, int64_t n_tokens, int32_t head_dim);
zb_status zb_linear_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int32_t heads,
                         int64_t n_tokens, int32_t head_dim, const float* A, const float* b,
                         uint16_t* O, void* ws, size_t ws_bytes, void* stream);

/*
 * Mean key of each head over all tokens, mu_h = (1/N) sum_r k_r: the shift of
 * the linear-centered variant (Abstract of "Zebra3D: Efficient Hybrid
 * Foundation Models For Scalable 3D Reconstruction": linear-centered attention
 * for the tolerant stages; Table 3 (a): "Linear-centered + fit").  The pages
 * give no formula; the reading taken centres the keys only, by this mean.
 *   in : K bf16 [H][N][d];  ws of >= zb_key_mean_workspace_bytes() bytes,
 *        16-byte aligned, owned by the caller (per-chunk fp64 partial sums)
 *   out: mu fp32 [H][d]
 * Sums run in fp32 per thread over a few hundred rows, then fp64 in a fixed
 * order (the result does not depend on scheduling).  Two kernel launches.
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED
 * (H > 65535), ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
size_t zb_key_mean_workspace_bytes(int32_t heads, int64_t n_tokens, int32_t head_dim);
zb_status zb_key_mean(const uint16_t* K, int32_t heads, int64_t n_tokens, int32_t head_dim,
                      float* mu, void* ws, size_t ws_bytes, void* stream);

/*
 * Linear-attention state of the linear-centered variant: zb_linear_state with
 * every key shifted by its head's key_mean before the feature map,
 *   S = sum_r phi(k_r - mu_h)^T v_r,  z = sum_r phi(k_r - mu_h),
 * (k - mu in fp32, phi in fp32, rounded to bf16 for the tensor-core product
 * as in zb_linear_state).  The output is then zb_linear_apply on the same Q,
 * unchanged: only the keys are centred.  Softmax attention is unchanged by
 * such a shift, so the affine fit keeps the same dense target.
 *   in : K, V bf16 [H][N][d];  key_mean fp32 [H][d] (normally from
 *        zb_key_mean);  ws of >= zb_linear_state_workspace_bytes() bytes
 *   out: S fp32 [H][d][d], z fp32 [H][d]
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED,
 * ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
zb_status zb_linear_state_centered(const uint16_t* K, const uint16_t* V, const float* key_mean,
                                   int32_t heads, int64_t n_tokens, int32_t head_dim, float* S,
                                   float* z, void* ws, size_t ws_bytes, void* stream);

/*
 * Block-mass diagnostic (Figure 2 (b) and Figure 8 of "Zebra3D: Efficient
 * Hybrid Foundation Models For Scalable 3D Reconstruction": the attention mass
 * kept by the heaviest 20% of 64 x 64 token blocks, from a dense pass).
 *
 * zb_block_mass: M[h][a][b] = sum over query rows r of block a and keys c of
 * block b of p_rc = exp(scale q_r . k_c - lse[h][r]), the dense softmax
 * probabilities.  Blocks are runs of s.tile (64 or 128) tokens, the last one
 * ragged.  lse is each row's log-sum-exp in natural log, as zb_dense_attn
 * returns it for the same Q, K and scale.
 *   in : Q, K bf16 [H][N][d];  lse fp32 [H][N]
 *   out: M fp32 [H][Tb][Tb], Tb = ceil(N / s.tile)   (every entry written)
 * S = Q K^T is recomputed on the tensor cores; every entry of M is stored
 * once, summed in a fixed order.
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE (scale <= 0), ZB_ERR_ALIGN,
 * ZB_ERR_UNSUPPORTED (H > 65535, Tb > 49152), ZB_ERR_CUDA.
 *
 * zb_block_mass_top_fraction: per row of M [heads * n_blocks][n_blocks], the
 * sum of its m largest entries over the row sum (fp64 sums), 0 <= m <= n_blocks;
 * frac fp32 [heads * n_blocks].  Errors: ZB_ERR_NULL, ZB_ERR_SHAPE,
 * ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED (n_blocks > 49152), ZB_ERR_CUDA.
 *
 * zb_block_mass_selected_fraction: per row of M (masses at the tile size), the
 * mass in the k key tiles that idx [heads][n_blocks][k] lists for that row
 * (zb_tile_score_topk's selection) over the row sum.  Indices out of range
 * count nothing and set ZB_ERR_INDEX in the device status.  Errors:
 * ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_CUDA.
 */
zb_status zb_block_mass(const uint16_t* Q, const uint16_t* K, const float* lse, zb_shape s, float scale,
                        float* M, void* stream);
zb_status zb_block_mass_top_fraction(const float* M, int32_t heads, int32_t n_blocks, int32_t m, float* frac,
                                     void* stream);
zb_status zb_block_mass_selected_fraction(const float* M, int32_t heads, int32_t n_blocks, const int32_t* idx,
                                          int32_t k, float* frac, void* stream);

/*
 * Closed-form affine fit (Abstract: closed-form affine fitting makes the
 * conversion training-free; Table 3 (a) of "Zebra3D: Efficient Hybrid
 * Foundation Models ..." compares no fit with fitted variants): per head, the
 * least-squares solution of [X 1] [A; b] = Y over R calibration rows whose A
 * has minimum norm, computed with a vanishing ridge
 * lam = 1e-8 * max_i ((X - mean X)^T (X - mean X))_ii on A, so that calibration
 * outputs varying in fewer than d directions stay solvable (the linear stage's
 * outputs always do: each row satisfies O . (S^-1 z) = 1).
 * Solved in fp64: row means, centred Gram matrices, Cholesky factorisation.
 *   in : X fp32 [H][R][d] (unfitted linear output), Y fp32 [H][R][d] (dense
 *        output on the same rows);  R >= d + 1;  ws of >=
 *        zb_affine_fit_workspace_bytes() bytes
 *   out: A fp32 [H][d][d], b fp32 [H][d]
 * A system that is not positive definite sets ZB_ERR_SINGULAR in the device
 * status and writes NaN into that head's A and b.
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED,
 * ZB_ERR_WORKSPACE, ZB_ERR_CUDA.
 */
size_t zb_affine_fit_workspace_bytes(int32_t heads, int64_t rows, int32_t head_dim);
zb_status zb_affine_fit(const float* X, const float* Y, int32_t heads,
                        int64_t rows, int32_t head_dim, float* A, float* b,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * Linear-attention state without a workspace.  The method has no counterpart:
 * this is a service entry point of the library.  Same result as
 * zb_linear_state, for callers that cannot allocate device memory at call
 * time (a process whose device memory is reserved by another allocator, or a
 * latency-critical loop where an allocation and its implicit synchronisation
 * are not allowed).  The per-CTA partial states go to a fixed scratch array
 * inside the library (zb_linear_state_static_scratch_bytes() = 8 MiB), held
 * on every GPU that loads the library until the process exits.
 *   in : K, V bf16 [H][N][d]
 *   out: S fp32 [H][d][d], z fp32 [H][d]
 *   - Allocates nothing and needs no workspace.
 *   - The first call on a device looks up the scratch array's device address
 *     (with that device current); make that first call before any stream
 *     capture.
 *   - Every call shares the one scratch array: calls that overlap on the GPU
 *     (other streams, other threads) race and must be serialised by the
 *     caller.  A call overwrites all the scratch it reads, so the contents
 *     left by an earlier call do not matter.
 * Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED (also
 * when the partial states of the shape exceed the scratch: more than 504
 * heads), ZB_ERR_CUDA.
 */
size_t zb_linear_state_static_scratch_bytes(void);
zb_status zb_linear_state_static(const uint16_t* K, const uint16_t* V, int32_t heads,
                                 int64_t n_tokens, int32_t head_dim, float* S, float* z,
                                 void* stream);

/*
 * Copy whole tiles of a [H][N][d] bf16 tensor into a compact buffer (the
 * calibration rows of the affine fit are whole query tiles).
 *   in : X bf16 [H][N][d];  tiles int32 [n_tiles] DEVICE array, each in [0, T)
 *   out: out bf16 [H][n_tiles * tile][d]; tile m of the list lands in rows
 *        [m*tile, (m+1)*tile); rows past N of a ragged tile are zero.
 * An index out of range sets ZB_ERR_INDEX in the device status (its rows are
 * zero).  Errors: ZB_ERR_NULL, ZB_ERR_SHAPE, ZB_ERR_ALIGN, ZB_ERR_UNSUPPORTED,
 * ZB_ERR_CUDA.
 */
zb_status zb_gather_tiles(const uint16_t* X, zb_shape s, const int32_t* tiles,
                          int32_t n_tiles, uint16_t* out, void* stream);

/*
 * Spatial tiles (synopsis of "3D reconstruction drops dense attention layer by
 * layer: up to 5.6x end-to-end speedup at 1,024 views": exact softmax over
 * selected *spatial* tiles).  zb_spatial_order writes, on the HOST, a token
 * order that groups each view's patches into 2-D windows.  A view holds
 * `specials` camera/register tokens followed by grid x grid patch tokens in
 * row-major order; in the new order each view keeps its specials first, then
 * its patches window by window (win_rows x win_cols windows, row-major over the
 * window grid, row-major inside a window, edge windows smaller).  Running the
 * tile-sparse stage on tokens gathered into this order makes its contiguous
 * tiles cover compact 2-D regions; gathering the output with the inverse order
 * puts every row back.
 *   out: order   int32 [views * (specials + grid*grid)] HOST array: position p
 *                of the new sequence holds original token order[p]
 *        inverse int32 [same] HOST array or NULL: inverse[order[p]] = p
 * No device work.  Errors: ZB_ERR_SHAPE, ZB_ERR_NULL, ZB_ERR_UNSUPPORTED (more
 * than 2^31 - 1 tokens).
 */
zb_status zb_spatial_order(int32_t views, int32_t grid, int32_t specials, int32_t win_rows,
                           int32_t win_cols, int32_t* order, int32_t* inverse);

/*
 * Row gather of a bf16 [heads][n_in][head_dim] tensor: out[h][r] = X[h][rows[r]]
 * for r < n_out (the same row list for every head); moves tensors into and
 * out of a token order such as zb_spatial_order's.
 *   in : X bf16 [H][n_in][64];  rows int32 [n_out] DEVICE array
 *   out: out bf16 [H][n_out][64]
 * A row index outside [0, n_in) gives a zero row and sets ZB_ERR_INDEX in the
 * device status.  Errors: ZB_ERR_SHAPE, ZB_ERR_UNSUPPORTED, ZB_ERR_NULL,
 * ZB_ERR_ALIGN, ZB_ERR_CUDA.
 */
zb_status zb_gather_rows(const uint16_t* X, int32_t heads, int64_t n_in, int64_t n_out, int32_t head_dim,
                         const int32_t* rows, uint16_t* out, void* stream);

/*
 * Synchronise `stream`, then report and clear the current device's status
 * word: ZB_OK, or the first of ZB_ERR_TIMEOUT / ZB_ERR_INDEX / ZB_ERR_SINGULAR
 * recorded by a kernel since the last call.  ZB_ERR_CUDA if the stream or the
 * device reports an error.
 */
zb_status zb_last_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ZB_H */
