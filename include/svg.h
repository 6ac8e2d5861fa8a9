/*
 * svg.h — C ABI of the B200 (sm_100a) Sparse VideoGen attention step.
 *
 * The step, as the pages describe it (page title, section):
 *   1. QK-Norm (RMSNorm) and 3D RoPE on Q and K
 *        ("Sparse VideoGen" WeChat article, "其他优化方法";
 *         ICML 2025 report (机器之心), "Layout Transformation + Kernel 加速");
 *   2. online profiling: a few sampled query rows per head are attended densely,
 *      with the spatial mask and with the temporal mask; each head takes the mask
 *      with the smaller MSE against dense
 *        (article, "Online Profiling Strategy"; report, "动态自适应的稀疏策略" steps 1-3);
 *   3. frame-major -> token-major layout transform for temporal heads
 *        (article, "硬件高效的 Layout Transformation"; report, "Layout Transformation + Kernel 加速");
 *   4. per-head block-sparse attention over the kept key tiles
 *        (article, "Spatial Head" / "Temporal Head" / "其他优化方法"; report, "Sparse VideoGen 的核心设计");
 *   5. the inverse layout transform of the output.
 *
 * Conventions shared by every entry point
 *   - Tensors Q, K, V, O are bfloat16 (passed as uint16_t bit patterns), contiguous
 *     [B, H, L, d] with d in {64, 128}; L = F*Hs*Ws + text_len.  Video token
 *     i < F*Hs*Ws is frame f = i / (Hs*Ws), spatial index s = i % (Hs*Ws),
 *     grid position (s / Ws, s % Ws).  Text tokens follow the video tokens.
 *   - "device" pointers are CUDA device memory owned by the caller; every device
 *     pointer must be 16-byte aligned.  "host" pointers are ordinary host memory.
 *     The library never frees or keeps caller memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Kernels are
 *     enqueued on it; calls return without synchronising.
 *   - Argument errors are detected on the host before anything is enqueued and
 *     returned as a status; nothing is launched then.  A launch failure returns
 *     SVG_ERR_CUDA.  Errors found by the kernels themselves (a bounded wait that
 *     ran out, a block list larger than its capacity) are recorded in a per-device
 *     error word that svg_sync_status() reads and clears.
 *   - Outputs never alias inputs.
 */
#ifndef SVG_H
#define SVG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVG_OK = 0,
  SVG_ERR_INVALID_ARG = 1,   /* null pointer, bad flag, n out of range            */
  SVG_ERR_SHAPE = 2,         /* inconsistent shape (L != F*Hs*Ws + text_len, ...)  */
  SVG_ERR_UNSUPPORTED = 3,   /* valid but not implemented (d, tile sizes, split)    */
  SVG_ERR_ALIGNMENT = 4,     /* a device pointer is not 16-byte aligned             */
  SVG_ERR_CAPACITY = 5,      /* a caller buffer is too small                        */
  SVG_ERR_CUDA = 6,          /* a CUDA call or launch failed                        */
  SVG_ERR_TIMEOUT = 7        /* a kernel's bounded wait ran out (device error word) */
} svg_status;

typedef enum {
  SVG_HEAD_SPATIAL = 0,      /* keys whose frame is within +-spatial_frames        */
  SVG_HEAD_TEMPORAL = 1,     /* keys whose spatial index is within +-temporal_radius */
  SVG_HEAD_DENSE = 2         /* every key                                           */
} svg_head_kind;

typedef struct {
  int B, H;                  /* batch, heads                                         */
  int L;                     /* sequence length = F*Hs*Ws + text_len                 */
  int d;                     /* head dimension: 64 or 128                            */
  int F, Hs, Ws;             /* latent frames and per-frame spatial grid             */
  int text_len;              /* text tokens after the video tokens (always kept)     */
} svg_shape;

typedef struct {
  int spatial_frames;        /* w: spatial head keeps |frame_q - frame_k| <= w        */
  int temporal_radius;       /* r: temporal head keeps |s_q - s_k| <= r               */
  int block_q;               /* query tile rows of the block list: 64 or 128          */
  int block_k;               /* key tile columns of the block list: 64               */
  float eps;                 /* RMSNorm epsilon                                      */
  float rope_base;           /* RoPE base (e.g. 10000)                               */
  int rope_split[3];         /* RoPE widths of the t, h, w sections; even; sum = d    */
  float softmax_scale;       /* 0 -> 1/sqrt(d)                                        */
} svg_params;

enum { SVG_NORM_ROPE = 1, SVG_LAYOUT = 2 };

/* ------------------------------------------------------------------------ */
/* Stage 1 (+3): QK-Norm + 3D RoPE and/or the layout transform.
 *   flags & SVG_NORM_ROPE: q_out/k_out rows = RMSNorm(row) * gamma, then, on video
 *     rows only, RoPE: in section a (t, h, w; widths rope_split, laid out from d=0)
 *     the pair (2j, 2j+1) is rotated by p_a * rope_base^(-2j/n_a), p_a = (f, y, x).
 *     Arithmetic in fp32; results rounded to nearest-even bf16.
 *   flags & SVG_LAYOUT: rows are written in the head's layout: for heads whose
 *     head_kind is TEMPORAL, video row f*S+s goes to s*F+f (S = Hs*Ws); text rows and
 *     other heads stay in place.  v (required with LAYOUT) is moved the same way
 *     without normalisation.
 * q, k, v, q_out, k_out, v_out: device bf16 [B,H,L,d].  Each tensor comes with its
 *   output or is NULL with it (q or k must be given); v is given only with SVG_LAYOUT,
 *   which requires it.
 * gamma_q, gamma_k: device fp32 [d].  With SVG_NORM_ROPE, q (k) is normalised iff
 *   gamma_q (gamma_k) is given; at least one must be.  With SVG_LAYOUT a tensor
 *   without its gamma is only moved, so {q raw, k already normalised, v} with only
 *   gamma_q gives the step's single fused pass; without SVG_LAYOUT every given
 *   tensor must be normalised (e.g. k alone).
 * rope_table: device fp32 table of svg_rope_table_size() floats written on the host
 *   by svg_rope_table_fill() and copied by the caller; required with SVG_NORM_ROPE.
 * head_kind: device uint8 [B*H]; required with SVG_LAYOUT. */
svg_status svg_qknorm_rope_layout(const svg_shape* shape, const svg_params* params, int flags,
                                  const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const float* gamma_q, const float* gamma_k, const float* rope_table,
                                  const uint8_t* head_kind,
                                  uint16_t* q_out, uint16_t* k_out, uint16_t* v_out, void* stream);

/* Stage 2: online profiling.
 * For every (b, h) and each of the n sampled video tokens sample_idx[0..n) (device
 * int32, the same rows for every head, 1 <= n <= 64): the dense, the spatial-masked and
 * the temporal-masked attention outputs of that query row (fp32 softmax; P rounded to
 * bf16 for the tensor-core P.V, and the row sums taken from the same rounded values,
 * so each output stays a weighted average).  Per head
 *   MSE_m = mean over the n rows and d columns of (O_m - O_dense)^2,  m in {spatial, temporal}
 * and head_kind_out[b*H+h] = SPATIAL if MSE_spatial <= MSE_temporal else TEMPORAL.
 * qn, kn: device bf16 [B,H,L,d] after stage 1, frame-major order; v: device bf16.
 * workspace: device scratch of at least svg_profile_workspace_size(shape, n) bytes.
 * mse_out: device fp32 [B*H*2] (spatial, temporal) or NULL.
 * head_kind_out: device uint8 [B*H]. */
svg_status svg_profile_heads(const svg_shape* shape, const svg_params* params,
                             const uint16_t* qn, const uint16_t* kn, const uint16_t* v,
                             const int32_t* sample_idx, int n, void* workspace, size_t workspace_bytes,
                             float* mse_out, uint8_t* head_kind_out, void* stream);

/* Stage 2 on raw Q: as svg_profile_heads, but q is the un-normalised Q (model order)
 * and each sampled row gets QK-Norm + RoPE inside the kernel, with the same device
 * routine (same lane split and operation order) as svg_qknorm_rope_layout, so the
 * rows are bit-identical to that stage's output.  This lets a step normalise Q in
 * the same pass that moves it into the heads' layouts.
 * gamma_q: device fp32 [d]; rope_table: as for svg_qknorm_rope_layout; kn: K after
 * QK-Norm + RoPE.  Other arguments and errors as for svg_profile_heads. */
svg_status svg_profile_heads_raw_q(const svg_shape* shape, const svg_params* params,
                                   const uint16_t* q, const float* gamma_q, const float* rope_table,
                                   const uint16_t* kn, const uint16_t* v,
                                   const int32_t* sample_idx, int n, void* workspace, size_t workspace_bytes,
                                   float* mse_out, uint8_t* head_kind_out, void* stream);

/* Stage 2 without a caller-provided workspace.  The paper has no counterpart:
 * this entry point exists for callers that can hand the library only their
 * inputs and outputs and cannot allocate device memory themselves -- for
 * example a plugin running inside a host runtime that owns all device memory
 * and exposes no allocator, or a serving process that reserved its whole
 * memory pool at start-up and must not call cudaMalloc while serving.
 * It takes the same arguments as svg_profile_heads minus the workspace and
 * allocates nothing: its scratch is a fixed 16 MiB device array inside the
 * library, which every GPU that loads the library holds until the process
 * exits.  Its results are those of svg_profile_heads up to the order in which
 * the key chunks are merged: when fewer chunks fit in the scratch than the
 * workspace entry point uses, the MSEs may differ in their last bits (and a
 * head whose two MSEs are that close may be given the other kind); with the
 * same chunk count the results are bit-identical.
 *   - Size limit: one key chunk of partial results takes B*H*128*(3+2d)*4 bytes
 *     and the per-row error sums B*H*64*2*8 bytes; if together they exceed
 *     16 MiB (B*H > 125 at d=128, > 246 at d=64) the call returns
 *     SVG_ERR_CAPACITY and launches nothing.  Otherwise it splits the
 *     keys into as many chunks as fit (at most as many as svg_profile_heads).
 *   - Set-up: the first call on each device looks up the scratch's device
 *     address (cudaGetSymbolAddress, with that device current) and caches it
 *     for the life of the process; make that first call before any stream
 *     capture.  The cache is never refreshed: after cudaDeviceReset on a
 *     device the cached address is stale, so do not call this entry point on
 *     that device again in the same process.
 *   - Sharing: every call uses the same scratch and leaves its contents behind.
 *     Each call writes every scratch entry it later reads, so nothing needs to
 *     start at zero; but two calls whose kernels overlap on the GPU (different
 *     streams, or different host threads) race on the scratch and corrupt each
 *     other's results.  Serialise them.
 * Errors are reported as for svg_profile_heads (SVG_ERR_CUDA if the set-up
 * lookup fails). */
svg_status svg_profile_heads_noalloc(const svg_shape* shape, const svg_params* params,
                                     const uint16_t* qn, const uint16_t* kn, const uint16_t* v,
                                     const int32_t* sample_idx, int n,
                                     float* mse_out, uint8_t* head_kind_out, void* stream);

/* Block index (not on the pages; the block-sparse kernel they describe needs it).
 * In each head's layout, the tile (q-block qb: rows [qb*block_q, +block_q),
 * k-block kb: keys [kb*block_k, +block_k), rows/keys >= L excluded) is listed iff at
 * least one (query, key) pair in it is kept by the head's mask; full[e] = 1 iff every
 * pair is kept.  CSR over (b, h, qb) in that order, kb ascending:
 *   row_ptr: device int32 [B*H*nqb + 1], col: device int32 [capacity],
 *   full: device uint8 [capacity].
 * If the list needs more than `capacity` entries, nothing past capacity is written
 * and svg_sync_status() reports SVG_ERR_CAPACITY.  svg_block_index_capacity() is
 * always enough. */
svg_status svg_build_block_index(const svg_shape* shape, const svg_params* params,
                                 const uint8_t* head_kind, int32_t* row_ptr, int32_t* col,
                                 uint8_t* full, int64_t capacity, void* stream);

/* Stage 4: block-sparse attention, tcgen05/TMEM tile loop fed by TMA.
 *   out[b,h,i,:] = sum_k softmax_k(scale * q_i . k_k | kept) v_k
 * over the keys of the tiles listed for the query's q-block, with the head's
 * token-level mask applied inside partial tiles (full = 0) and to keys >= L.
 * Online softmax in fp32; P rounded to bf16 for the P.V product.
 * q, k, v: device bf16 [B,H,L,d] in the head's layout (stage 3 output).
 * head_kind: device uint8 [B*H].  row_ptr/col/full: the block index above.
 * out: device bf16 [B,H,L,d] in the head's layout.
 * lse_out: device fp32 [B,H,L] natural-log sum of exp of the kept scaled logits, or NULL.
 * Requires block_k = 64 and block_q in {64, 128}. */
svg_status svg_block_sparse_attn(const svg_shape* shape, const svg_params* params,
                                 const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 const uint8_t* head_kind, const int32_t* row_ptr,
                                 const int32_t* col, const uint8_t* full,
                                 uint16_t* out, float* lse_out, void* stream);

/* Stage 4 with stage 5 fused into its epilogue: as svg_block_sparse_attn, but
 * every output row (and LSE entry) is stored at its model-order position --
 * rows of temporal heads go from s*F+f back to f*S+s, all other rows stay -- so
 * the separate inverse-layout pass and its read and write of O disappear.
 * The pages describe the inverse transform as a step of its own ("Sparse
 * VideoGen" WeChat article, "硬件高效的 Layout Transformation"); fusing it is
 * this library's choice.  out: device bf16 [B,H,L,d] in model order;
 * lse_out: device fp32 [B,H,L] in model order, or NULL.  Other arguments and
 * errors as for svg_block_sparse_attn. */
svg_status svg_block_sparse_attn_model_order(const svg_shape* shape, const svg_params* params,
                                             const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                             const uint8_t* head_kind, const int32_t* row_ptr,
                                             const int32_t* col, const uint8_t* full,
                                             uint16_t* out, float* lse_out, void* stream);

/* Stage 5: inverse of the layout transform (temporal heads: row s*F+f -> f*S+s).
 * src, dst: device bf16 [B,H,L,d]; head_kind: device uint8 [B*H]. */
svg_status svg_inverse_layout(const svg_shape* shape, const uint8_t* head_kind,
                              const uint16_t* src, uint16_t* dst, void* stream);

/* The whole step on one stream, in five passes:
 *   1. QK-Norm + RoPE of K into kn (frame-major);
 *   2. profiling (svg_profile_heads_raw_q: the sampled Q rows are normalised in
 *      the kernel) -- skipped when head_kind_in != NULL, whose kinds are used;
 *   3. the block index;
 *   4. one pass that normalises Q and writes Q, kn and V in the heads' layouts
 *      (qp, kp, vp);
 *   5. block-sparse attention; with op = NULL it writes `out` in model order
 *      directly (svg_block_sparse_attn_model_order), otherwise it writes op in the
 *      heads' layout and svg_inverse_layout produces `out`.
 * Every output equals running the stages one by one with svg_qknorm_rope_layout
 * (NORM_ROPE), svg_profile_heads, svg_build_block_index, svg_qknorm_rope_layout
 * (LAYOUT) and svg_block_sparse_attn + svg_inverse_layout: the norm routine is
 * the same in every pass.  All buffers are device memory owned by the caller:
 *   kn, qp, kp, vp: bf16 [B,H,L,d] intermediates; op: bf16 [B,H,L,d] or NULL;
 *   out: bf16 [B,H,L,d] final output in model order;
 *   head_kind_out: uint8 [B*H]; mse_out: fp32 [B*H*2] or NULL;
 *   row_ptr/col/full: block index with `capacity` entries;
 *   workspace: svg_profile_workspace_size(shape, n) bytes. */
svg_status svg_attention_step(const svg_shape* shape, const svg_params* params,
                              const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const float* gamma_q, const float* gamma_k, const float* rope_table,
                              const int32_t* sample_idx, int n, const uint8_t* head_kind_in,
                              uint16_t* kn, uint16_t* qp, uint16_t* kp, uint16_t* vp,
                              uint16_t* op, uint16_t* out, uint8_t* head_kind_out, float* mse_out,
                              int32_t* row_ptr, int32_t* col, uint8_t* full, int64_t capacity,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The whole step on HOST buffers (the end-to-end call of a caller whose tensors
 * live in host memory).  The B*H heads are split into `groups` head groups
 * (sizes differ by at most one): group g+1's Q, K and V are copied to the
 * device while group g runs the five passes of svg_attention_step, and each
 * group's output is copied back while the next group runs, on three streams
 * the library creates once per device.  Every stage is per head, so the
 * output equals svg_attention_step on the whole problem (head kinds and
 * attention rows alike).
 *   q_host, k_host, v_host: host bf16 [B,H,L,d] (model order);
 *   gamma_q_host, gamma_k_host: host fp32 [d]; sample_idx_host: host int32 [n];
 *   out_host: host bf16 [B,H,L,d], the output in model order;
 *   head_kind_out_host: host uint8 [B*H] (the profiled kinds) or NULL;
 *   1 <= groups <= B*H;
 *   workspace: device scratch of svg_attention_step_host_workspace_size()
 *     bytes, 16-byte aligned, owned by the caller: full-size device copies of
 *     Q, K, V and O plus one head group's intermediates.
 * The work starts after the caller's earlier work on `stream`, and `stream`
 * waits for the last copy: synchronise it before reading out_host.  The host
 * buffers should be pinned (cudaHostAlloc / cudaHostRegister); with pageable
 * memory the copies still happen but do not overlap the passes.  Calls that
 * share a workspace must be ordered on the GPU (the same stream, or
 * synchronised).  The RoPE table is built on the host into a pinned staging
 * buffer the library keeps per device.  Errors as for svg_attention_step, plus
 * SVG_ERR_CAPACITY for a workspace below the size required. */
size_t svg_attention_step_host_workspace_size(const svg_shape* shape, const svg_params* params, int n,
                                              int groups);
svg_status svg_attention_step_host(const svg_shape* shape, const svg_params* params,
                                   const uint16_t* q_host, const uint16_t* k_host, const uint16_t* v_host,
                                   const float* gamma_q_host, const float* gamma_k_host,
                                   const int32_t* sample_idx_host, int n, uint16_t* out_host,
                                   uint8_t* head_kind_out_host, int groups, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* ------------------------------ semantic-aware permutation ("Sparse VideoGen2") */
/* The second workload ("Sparse VideoGen2" explainer, "A. 语义感知排列" and
 * "B. 基于质心的 Top-p 选择"): per head, the video rows of Q and of K are
 * clustered by k-means, each tensor is sorted so that every cluster is
 * contiguous, every query cluster attends the top-p key clusters estimated
 * from size-weighted centroid scores, and text tokens stay at the end, kept by
 * every query and keeping every key.  Cluster counts are 1..64 (a query
 * cluster's key set is one 64-bit mask).  Decisions taken from floating point
 * follow a fixed operation order (stated with each call), so they do not
 * depend on scheduling. */

/* Bytes of device scratch svg2_kmeans needs: B*H*C*d*8. */
size_t svg2_kmeans_workspace_size(const svg_shape* shape, int C);

/* k-means of the F*Hs*Ws video rows of every head of x (device bf16 [B,H,L,d]):
 * with init != 0 the centroids start at video rows floor(c*Lv/C); otherwise
 * `cent` holds the starting centroids (e.g. the previous denoising step's: the
 * pages' centroid cache).  `iters` rounds of (assign every row to its nearest
 * centroid; move each centroid to the mean of its rows, an empty cluster keeps
 * its centroid), then a final assignment.  The nearest centroid minimises
 * |c|^2 - 2 x.c (the squared distance less |x|^2): both sums in float with
 * fused multiply-add in the order i = 0..d-1, then |c|^2 - 2 (x.c) rounded
 * once; the lowest index wins a tie.  This equals the fp64 nearest centroid
 * except where the two nearest squared distances differ by less than about
 * 1e-5 of |x|^2 + |c1|^2 + |c2|^2.  Sums in 64-bit fixed point (x * 2^40
 * truncated); mean ((double)sum / 2^40) / count rounded to float.  The sums
 * are exact for |x| < min(2^23 / Lv, 2^12); a value outside that range (or
 * inf / NaN) is left out of its sum and reported as SVG_ERR_INVALID_ARG by
 * svg_sync_status.
 * cent: device float [B*H][C][d] (in/out); assign: device uint8 [B*H][Lv];
 * counts: device int32 [B*H][C], the sizes of the final assignment. */
svg_status svg2_kmeans(const svg_shape* shape, const uint16_t* x, int C, int iters, int init, float* cent,
                       uint8_t* assign, int32_t* counts, void* workspace, size_t workspace_bytes, void* stream);

/* Stable counting sort of each head's video rows by cluster: perm (device int32
 * [B*H][Lv]) = the row placed at each position, off (device int32 [B*H][C+1]) =
 * the first position of each cluster (off[C] = Lv).  An assignment outside
 * [0, C) is left out and reported as SVG_ERR_INVALID_ARG by svg_sync_status. */
svg_status svg2_permutation(const svg_shape* shape, const uint8_t* assign, int C, int32_t* perm, int32_t* off,
                            void* stream);

/* Top-p key clusters of every query cluster: s_ij = scale * (cq_i . ck_j) in
 * double (multiply and add in the order of the d components), weights
 * w_ij = n_j * exp(s_ij - max over non-empty j), key clusters in decreasing
 * weight (lower index first on a tie), and the shortest prefix whose running sum
 * reaches top_p times the sum of all weights (summed in index order).
 * cq, ck: device float [B*H][Cq|Ck][d]; counts_k: device int32 [B*H][Ck];
 * sel: device uint64 [B*H][Cq], bit j = key cluster j.  scale = softmax_scale or
 * 1/sqrt(d) in double.  0 < top_p <= 1. */
svg_status svg2_select(const svg_shape* shape, const svg_params* params, const float* cq, const float* ck,
                       const int32_t* counts_k, int Cq, int Ck, double top_p, uint64_t* sel, void* stream);

/* Q, K, V into cluster order: video position p of q_out takes row perm_q[p];
 * k_out and v_out take row perm_k[p]; text rows are copied in place.  An entry
 * outside [0, Lv) copies row p instead and is reported as SVG_ERR_INVALID_ARG
 * by svg_sync_status. */
svg_status svg2_permute(const svg_shape* shape, const int32_t* perm_q, const int32_t* perm_k, const uint16_t* q,
                        const uint16_t* k, const uint16_t* v, uint16_t* q_out, uint16_t* k_out, uint16_t* v_out,
                        void* stream);

/* Block index over the cluster order (same CSR format and `full` meaning as
 * svg_build_block_index): tile (qb, kb) is listed iff one of its pairs is kept. */
svg_status svg2_build_block_index(const svg_shape* shape, const svg_params* params, int Cq, int Ck,
                                  const int32_t* qoff, const int32_t* koff, const uint64_t* sel, int32_t* row_ptr,
                                  int32_t* col, uint8_t* full, int64_t capacity, void* stream);

/* Block-sparse attention in cluster order (q, k, v from svg2_permute) with the
 * cluster mask, written back in model order: video position p goes to row
 * perm_q[p] of out (and of lse_out, if given).  Requires block_q = 128.
 * perm_q, qoff, koff and sel must not be NULL (SVG_ERR_INVALID_ARG before any
 * launch).  A perm_q entry outside [0, Lv) leaves its row unwritten and is
 * reported as SVG_ERR_INVALID_ARG by svg_sync_status. */
svg_status svg2_attention(const svg_shape* shape, const svg_params* params, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, int Cq, int Ck, const int32_t* qoff, const int32_t* koff,
                          const uint64_t* sel, const int32_t* perm_q, const int32_t* row_ptr, const int32_t* col,
                          const uint8_t* full, uint16_t* out, float* lse_out, void* stream);

/* --------------------------------------------- AdaSpa blockified search --
 * "AdaSpa" abstract: a blockified sparse pattern, found by a "Fused
 * LSE-Cached Search" and used by "Head-adaptive Hierarchical Block Sparse
 * Attention"; the pattern and each row's log-sum-exp stay the same across
 * denoising steps.  The search is exact given the cached LSE: the weight of a
 * pair is exp(scale * q.k - lse_q), so one pass over Q K^T gives the mass of
 * every (query tile, key tile) block.  The kept blocks then run through
 * svg_block_sparse_attn with every head SVG_HEAD_DENSE (each listed block is
 * computed whole).  Model order throughout; block_q = 128, block_k = 64. */

/* Block masses.  q, k: device bf16 [B,H,L,d] (after QK-Norm + RoPE); lse:
 * device float [B*H][L], the rows' natural log-sum-exp from an earlier step
 * (e.g. the lse_out of a dense step of svg_block_sparse_attn); mass: device
 * float [B*H][nqb][nkb]: mass[bh][qb][kb] = sum over rows q < L of tile qb and
 * keys k < L of tile kb of exp(scale * q.k - lse[q]) (scores in fp32 on the
 * tensor cores, 2^x by the hardware approximation, per-row sums in fp32, the
 * tile's 128 rows added in a fixed order).  Requires block_q = 128, block_k = 64
 * (SVG_ERR_UNSUPPORTED otherwise). */
svg_status svg_adaspa_block_mass(const svg_shape* shape, const svg_params* params, const uint16_t* q,
                                 const uint16_t* k, const float* lse, float* mass, void* stream);

/* The kept key tiles of every (head, query tile), as CSR (same format as
 * svg_build_block_index; every entry full = 1).  Video key tiles (no key in
 * [Lv, L)) are ranked by mass, heavier first and the lower index on a tie; the
 * shortest prefix whose running sum reaches top_p times their total is kept,
 * at least one tile.  Sums are in 32-bit fixed point (mass * 2^32 truncated,
 * exact in any order; the goal is top_p * total in double).  Key tiles holding
 * text keys are always kept, and query tiles holding text rows keep every key
 * tile.  mass: device float [B*H][nqb][nkb]; 0 < top_p <= 1; at most 4096 key
 * tiles per query tile.  Capacity overflow is reported by svg_sync_status. */
svg_status svg_adaspa_select(const svg_shape* shape, const svg_params* params, const float* mass, double top_p,
                             int32_t* row_ptr, int32_t* col, uint8_t* full, int64_t capacity, void* stream);

/* ----------------------------------------------------------- host helpers */

/* n distinct video-token indices in [0, Lv) into host_out[0..n): the first n slots of
 * a partial Fisher-Yates shuffle driven by SplitMix64(seed) (slot i swaps with
 * i + x mod (Lv - i)).  Host only; needs no GPU. */
svg_status svg_sample_queries(uint64_t seed, int64_t Lv, int n, int32_t* host_out);

/* Number of fp32 values of the RoPE table, and its contents (host memory):
 * for section a, position p in [0, F | Hs | Ws), pair j < n_a/2: (cos, sin) of
 * p * base^(-2j/n_a), computed in double and rounded to float. */
size_t svg_rope_table_size(const svg_shape* shape, const svg_params* params);
svg_status svg_rope_table_fill(const svg_shape* shape, const svg_params* params, float* host_out);

/* What one layer's attention does at denoising step `step` of `total_steps`
 * ("Sparse VideoGen" WeChat article, "其他优化方法": the first 25% of the
 * generation steps run dense attention, the other 75% sparse; "Online Profiling
 * Strategy": the best pattern changes from step to step, so it is profiled
 * online).  *mode_out is
 *   SVG_STEP_DENSE   if step < dense_fraction * total_steps (all heads DENSE;
 *                    pass head_kind_in = all SVG_HEAD_DENSE to svg_attention_step),
 *   SVG_STEP_PROFILE on the first sparse step and then every `reprofile_every`
 *                    sparse steps (head_kind_in = NULL: profile, use the result),
 *   SVG_STEP_REUSE   otherwise (head_kind_in = the last profiled kinds).
 * reprofile_every = 1 profiles every sparse step, as the pages do; larger values
 * are this library's option, not the pages'.
 * SVG_ERR_INVALID_ARG for step outside [0, total_steps), total_steps < 1,
 * dense_fraction outside [0, 1] or reprofile_every < 1.  Host only. */
typedef enum { SVG_STEP_DENSE = 0, SVG_STEP_PROFILE = 1, SVG_STEP_REUSE = 2 } svg_step_mode;
svg_status svg_step_policy(int step, int total_steps, float dense_fraction, int reprofile_every,
                           int* mode_out);

/* Entries that always suffice for svg_build_block_index: B*H*nqb*nkb. */
int64_t svg_block_index_capacity(const svg_shape* shape, const svg_params* params);

/* Device scratch bytes svg_profile_heads needs for n sampled rows. */
size_t svg_profile_workspace_size(const svg_shape* shape, int n);

/* (Not on the pages: a sizing helper of this library's boundary.)
 * Device scratch bytes that every entry point taking a caller workspace needs
 * for this shape and parameters: svg_profile_heads and svg_profile_heads_raw_q
 * with any n from 1 to 64 (the scratch does not grow with n).  0 for a null
 * pointer, a shape the library rejects, negative window parameters, or tiles
 * other than block_k = 64 and block_q in {64, 128}. */
size_t svg_workspace_size(const svg_shape* shape, const svg_params* params);

/* (Not on the pages: resource management of this library.)
 * Releases the library's cached state: on every device that has run
 * svg_attention_step_host, it waits for the library's own three streams to
 * finish, then destroys them and their events and frees the pinned staging
 * buffer of the RoPE table.  Nothing else is cached (the fixed scratch of
 * svg_profile_heads_noalloc is a device array that lives as long as the
 * library).  The next svg_attention_step_host creates them again.  Call it
 * from one thread, with no call of the library in flight on another.
 * Restores the calling thread's current device.  Returns SVG_OK, or
 * SVG_ERR_CUDA if a synchronisation or a release failed (the state is
 * dropped all the same).  Touches no GPU when nothing is cached. */
svg_status svg_release(void);

/* Synchronises `stream`, then reads and clears this device's error word:
 * SVG_OK, SVG_ERR_TIMEOUT or SVG_ERR_CAPACITY (or SVG_ERR_CUDA if the
 * synchronisation itself failed). */
svg_status svg_sync_status(void* stream);

/* Failure-path self-test (not on the pages): launches one warp that waits on a
 * barrier nothing completes.  The wait gives up after its limit (about a
 * second), records SVG_ERR_TIMEOUT in the error word and returns, exactly as a
 * stalled pipeline in any kernel of this library would; the context stays
 * usable.  svg_sync_status(stream) then reports SVG_ERR_TIMEOUT and clears it. */
svg_status svg_selftest_wait_timeout(void* stream);

const char* svg_status_string(svg_status status);
const char* svg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVG_H */
