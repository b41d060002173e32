/*
 * dynrad.h -- C ABI of the DynamicRad block-sparse attention hot path on
 * NVIDIA B200 (sm_100a).
 *
 * Source of the method: "DynamicRad: Content-Adaptive Sparse Attention for
 * Long Video Diffusion" (arXiv 2604.20470).  Three stages:
 *
 *   1. dynrad_build_candidates -- the radial candidate block set of Sec. 3.1
 *      (Eqs. 1-7, "Density control within blocks"; Algorithm 1, candidate construction and block aggregation).
 *   2. dynrad_select_blocks    -- per query block, mean-pooled block scores
 *      (the 1/sqrt(d) logit scale of Eq. 9) and one of the two selection modes
 *      of Sec. 3.2: static-ratio (top rho fraction, k rule of Eq. 8) or
 *      dynamic-threshold (smallest prefix whose softmax block mass reaches
 *      tau).  Output: CSR block indices.
 *   3. dynrad_sparse_attn      -- block-sparse softmax attention over the kept
 *      blocks, Eqs. 12-13 with epsilon -> 0, returning O and the log-sum-exp.
 *      dynrad_attn_backward is its gradient (dQ, dK, dV) under the same mask.
 *
 * Conventions shared by every call
 *   - Pointers named q, k, v, o, lse, *_row_ptr, *_col*, forced_*, scores_out,
 *     workspace are DEVICE pointers owned by the caller.  Geometry structs and
 *     *_out scalars are HOST pointers.
 *   - Q, K, V, O are bf16, layout [B, H, N, D] contiguous (D fastest), base
 *     address 16-byte aligned.  LSE is fp32 [B, H, N].
 *   - Token t of a head sits at frame t / (height*width), in-frame index
 *     t % (height*width) (row-major h * width + w).  Blocks are contiguous runs
 *     of `block` tokens; the last block may be partial (padded keys are never
 *     attended, padded query rows are never written).  Nb = ceil(N / block).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) unless stated.  The library allocates no memory and frees none of
 *     the caller's (dynrad_host_path creates, and releases, three streams and
 *     a few events per call).
 *   - Every call returns a dynrad_status.  Argument errors are found on the
 *     host before any launch.  Errors found by a kernel (capacity exceeded, a
 *     bounded wait that ran out) are recorded in a device status word read by
 *     dynrad_device_status().
 */
#ifndef DYNRAD_H
#define DYNRAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dynrad_stream_t; /* same type as cudaStream_t */

typedef enum dynrad_status {
  DYNRAD_OK = 0,
  DYNRAD_ERR_INVALID_ARG = 1, /* null pointer, bad size, parameter out of range */
  DYNRAD_ERR_UNSUPPORTED = 2, /* head dim / block size / size limit not built */
  DYNRAD_ERR_CAPACITY = 3,    /* an output or workspace buffer is too small */
  DYNRAD_ERR_CUDA = 4,        /* a CUDA runtime or launch error */
  DYNRAD_ERR_DEVICE = 5       /* a kernel-side check or bounded wait failed */
} dynrad_status;

typedef enum dynrad_mode {
  DYNRAD_STATIC_RATIO = 0,     /* Sec. 3.2 "Static-ratio mode" (block-pooled top rho) */
  DYNRAD_DYNAMIC_THRESHOLD = 1 /* Sec. 3.2 "Dynamic-threshold mode" (softmax mass tau) */
} dynrad_mode;

/* Latent grid and radial parameters (Sec. 3.1; parameter list of Table 4). */
typedef struct dynrad_geom {
  int32_t frames;  /* N_f */
  int32_t height;  /* latent grid rows per frame */
  int32_t width;   /* latent grid columns per frame; N_t = height * width */
  int32_t block;   /* B_s, tokens per block: 32, 64 or 128 for attention; any >= 1 here */
  double gamma;    /* decay factor of Eq. 2, > 0 */
  double lambda;   /* long-range factor of Eq. 4, > 0 */
  double theta_c;  /* column density threshold, [0, 1] (0 = any linked query) */
  double theta_m;  /* block activation threshold, [0, 1] (0 = any active column) */
  double eps;      /* epsilon of Eq. 5, >= 0 (1e-6 in this library's workloads) */
  int32_t force_t; /* frame distances <= force_t (0 or 1) are always kept */
} dynrad_geom;

/* Number of blocks Nb = ceil(frames*height*width / block); 0 on a bad geometry. */
int64_t dynrad_num_blocks(const dynrad_geom *geom);

/*
 * Stage 1: radial candidate set (Eqs. 1-7 and the (theta_c, theta_m) block
 * aggregation of Sec. 3.1), plus each row's always-kept range.
 *
 * For query block I the candidates are the blocks J for which the token pairs
 * (q in I, k in J) that lie in P(frame(q), frame(k)) of Eq. 7 -- the frame pair
 * retained by the split rule of Eq. 6 and |u - v| <= w of Eq. 3 -- pass the
 * aggregation: more than theta_c * n_I linked query tokens makes a key token
 * active, more than theta_m * n_J active key tokens makes J a candidate.  To
 * that set is added the forced range [forced_lo[I], forced_hi[I]]: the blocks
 * holding a token whose frame is within force_t of a frame of I (over frame
 * pairs the split rule retains).  It always contains I itself.
 *
 *   cand_row_ptr  device int32 [Nb + 1]  CSR row offsets (written in both modes)
 *   cand_col      device int32 [cand_cap] ascending block indices per row, or
 *                 NULL for the size query
 *   forced_lo/hi  device int32 [Nb] each (written in both modes)
 *   nnz_out       host; if non-NULL receives the total candidate count and the
 *                 call SYNCHRONIZES the stream.  Required when cand_col == NULL.
 *   max_row_out   host, optional; receives the longest row (same sync).
 * Size query: cand_col == NULL.  Fill: cand_col != NULL; if the total exceeds
 * cand_cap, nothing past cand_cap is written and the device status becomes
 * DYNRAD_ERR_CAPACITY (or the call returns it when nnz_out is given).
 * The candidate set depends only on the geometry, not on Q/K: it can be built
 * once and reused, as the paper caches static masks (App. D).
 */
int dynrad_build_candidates(const dynrad_geom *geom, int32_t *cand_row_ptr,
                            int32_t *cand_col, int64_t cand_cap,
                            int32_t *forced_lo, int32_t *forced_hi,
                            int64_t *nnz_out, int64_t *max_row_out,
                            dynrad_stream_t stream);

/* Workspace bytes dynrad_select_blocks needs (pooled means, scoring plan,
 * per-call counters). */
size_t dynrad_select_workspace_bytes(int32_t B, int32_t H, int32_t N, int32_t D,
                                     const dynrad_geom *geom, int64_t cand_nnz);

/*
 * Stage 2: block pooling, scoring and selection (Sec. 3.2, the selection
 * steps of Algorithm 1, in the block-pooled form).
 *
 * For every (b, h) and query block I: qbar_I, kbar_J = fp32 means of Q and K
 * over the valid tokens of each block; s_IJ = qbar_I . kbar_J * (1/sqrt(D))
 * in fp32 for every candidate J.  F_I = the forced range, N_I = the other
 * candidates, ranked by (s descending, J ascending).
 *   mode DYNRAD_STATIC_RATIO, value rho in (0, 1]: keep F_I and the first
 *     k = max(1, floor(rho * |N_I| + 1e-9)) of N_I (k = 0 if N_I is empty).
 *   mode DYNRAD_DYNAMIC_THRESHOLD, value tau in (0, 1]: with
 *     e_J = exp(s_J - max s) (fp64 from the fp32 scores) and Z their sum over
 *     the candidates, keep F_I and the shortest prefix of N_I such that
 *     sum_{F_I} e + sum_{prefix} e >= tau * Z.  tau = 1 keeps every candidate.
 * Kept blocks are written ascending.
 *
 *   q, k          device bf16 [B, H, N, D]; N must equal frames*height*width
 *   D             64 or 128
 *   cand_*, forced_*   stage-1 output for the same geometry; cand_nnz its total
 *   cand_max_row  longest candidate row (stage 1's max_row_out), or 0 for the
 *                 bound Nb; it sizes the shared-memory score arrays of the
 *                 selection (8 rows per CTA).
 *                 Rows of up to 1024 candidates are supported (a larger bound
 *                 returns DYNRAD_ERR_UNSUPPORTED); a row longer than the bound
 *                 is an error (device status DYNRAD_ERR_CAPACITY, row left empty)
 *   row_ptr       device int32 [B*H*Nb + 1]; row (b*H + h)*Nb + I
 *   col_idx       device int32 [col_cap]; col_cap >= B*H*cand_nnz always suffices
 *   scores_out    device fp32 [B*H*cand_nnz] or NULL: the fp32 scores in
 *                 candidate order, row (b, h, I) at (b*H+h)*cand_nnz + cand_row_ptr[I]
 *   workspace     device, >= dynrad_select_workspace_bytes(...) bytes, 256-byte aligned
 * If the kept total exceeds col_cap the device status becomes DYNRAD_ERR_CAPACITY
 * and col_idx is left partial.
 */
int dynrad_select_blocks(const void *q, const void *k, int32_t B, int32_t H,
                         int32_t N, int32_t D, const dynrad_geom *geom,
                         const int32_t *cand_row_ptr, const int32_t *cand_col,
                         int64_t cand_nnz, int64_t cand_max_row,
                         const int32_t *forced_lo,
                         const int32_t *forced_hi, int32_t mode,
                         double rho_or_tau, int32_t *row_ptr, int32_t *col_idx,
                         int64_t col_cap, float *scores_out, void *workspace,
                         size_t workspace_bytes, dynrad_stream_t stream);

/*
 * Stage 2 for callers that cannot allocate device memory (no counterpart in the
 * paper).  A host library that runs inside an application whose own caching
 * allocator owns the device's memory, or that must not risk the device-wide
 * synchronisation cudaMalloc / cudaFree can cause, has no way to provide the
 * workspace dynrad_select_blocks wants.  This call is dynrad_select_blocks with
 * the workspace taken from a device array built into the library:
 * dynrad_static_scratch_bytes() bytes (32 MiB) on every GPU that loads the
 * library, held until the process exits.  The caller still provides every input
 * and output buffer; the call allocates nothing and calls no allocating routine.
 *
 *   Arguments, layouts and results: as dynrad_select_blocks, without
 *   workspace / workspace_bytes.
 *   Errors: DYNRAD_ERR_CAPACITY when dynrad_select_workspace_bytes(...) exceeds
 *   dynrad_static_scratch_bytes() (e.g. B=1, H=12, 32,760 tokens, block 64 fits;
 *   H=40 at 75,600 tokens does not); DYNRAD_ERR_INVALID_ARG for arguments the
 *   workspace size cannot be computed for; otherwise as dynrad_select_blocks.
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.  The
 *   address is looked up again when the calling thread's context on the device
 *   is not the one it was found in (after cudaDeviceReset, or in a context the
 *   caller created), so such a first call in the new context also belongs
 *   before any capture.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents: calls that overlap on the GPU (other streams, other host threads)
 *   race and corrupt each other's results.  Serialise them.
 */
size_t dynrad_static_scratch_bytes(void);
int dynrad_select_blocks_static_scratch(
    const void *q, const void *k, int32_t B, int32_t H, int32_t N, int32_t D,
    const dynrad_geom *geom, const int32_t *cand_row_ptr,
    const int32_t *cand_col, int64_t cand_nnz, int64_t cand_max_row,
    const int32_t *forced_lo, const int32_t *forced_hi, int32_t mode,
    double rho_or_tau, int32_t *row_ptr, int32_t *col_idx, int64_t col_cap,
    float *scores_out, dynrad_stream_t stream);

/*
 * Stage 3: block-sparse attention forward (Eq. 13 with epsilon -> 0).
 *
 * For every (b, h) and query token q of block I:
 *   o_q   = sum_{J in kept(I)} sum_{valid k in J} softmax_k(scale * q.k) v_k
 *   lse_q = ln sum_{same keys} exp(scale * q.k)
 * Tensor cores (tcgen05, bf16 operands, fp32 accumulation in TMEM) compute
 * Q K^T and P V; the softmax runs in fp32.  Rows with no kept block get
 * o = 0 and lse = -inf.
 *
 *   q, k, v       device bf16 [B, H, N, D], D = 64 or 128
 *   block         32, 64 or 128 (the CSR's block size)
 *   row_ptr       device int32 [B*H*Nb + 1]; col_idx device int32, strictly
 *                 ascending block indices in [0, Nb) per row (entries outside
 *                 the range are skipped and flagged in the device status)
 *   scale         logit scale; 0 means 1/sqrt(D)
 *   o             device bf16 [B, H, N, D]; lse device fp32 [B, H, N]
 */
int dynrad_sparse_attn(const void *q, const void *k, const void *v, int32_t B,
                       int32_t H, int32_t N, int32_t D, int32_t block,
                       const int32_t *row_ptr, const int32_t *col_idx,
                       float scale, void *o, float *lse,
                       dynrad_stream_t stream);

/*
 * Paper-exact static-ratio mode (Sec. 3.2 "Static-ratio mode", Eq. 8): a
 * content-free, seeded block mask, the same for every (batch, head).
 *
 * For each ordered frame pair (i, j) at distance t = |i - j| >= 2 that the
 * split rule (Eq. 6) keeps, k = max(1, floor(|P(i,j)| * rho)) token pairs of
 * the candidate set P(i,j) of Eq. 7 are sampled, rho = rho1 when
 * L(t) >= block (near field) and rho2 when L(t) < block (far field); pairs at
 * t <= 1 are all kept (rho = 1).  The sample is the k pairs with the smallest
 * keys, the key of pair (u, v) being output c + 1 of the SplitMix64 generator
 * seeded with `seed`, c = ((i*F + j)*N_t + u)*N_t + v (keys never tie).  The
 * sampled token links are aggregated to blocks with (theta_c, theta_m) as for
 * the candidate set (Sec. 3.1) and united with each row's forced range.  The
 * mask is a subset of the candidate set; building it costs one pass over all
 * candidate token pairs, which pools the keys near each frame pair's expected
 * k-th key, then a radix select per frame pair over its pooled keys (cache the
 * mask: it depends only on the geometry, rho1, rho2 and seed).  T(i, j) is
 * exact whatever the pool size: a frame pair whose pool slots do not fit in
 * the workspace, or whose k-th key falls outside its pooled range, is
 * selected by radix passes that recompute all of its keys (one CTA per pair,
 * much slower).
 *
 *   geom, cand_*, forced_*  the geometry and its candidate set / forced ranges
 *                 from dynrad_build_candidates (DEVICE)
 *   rho1, rho2    in (0, 1]
 *   replicas      number of copies of the Nb-row mask written one after the
 *                 other (B*H, so the result feeds dynrad_sparse_attn directly)
 *   row_ptr       DEVICE int32 [replicas*Nb + 1]
 *   col_idx       DEVICE int32, capacity col_cap >= replicas * (kept blocks);
 *                 replicas * cand_nnz always suffices
 *   thresholds_out  nullable DEVICE uint64 [F*F]: T(i, j), the largest sampled
 *                 key of frame pair (i, j) (row-major i*F + j); UINT64_MAX
 *                 where no sampling happens (t <= 1, pairs the split rule
 *                 drops)
 *   workspace     DEVICE, 256-byte aligned, workspace_bytes long:
 *                 dynrad_sampled_mask_workspace_bytes(geom, cand_nnz) bytes
 *                 give every frame pair its pool; any size down to
 *                 dynrad_sampled_mask_workspace_min_bytes(geom, cand_nnz) is
 *                 accepted (the same result; frame pairs left without pool
 *                 slots take the slow exact path)
 * Errors: DYNRAD_ERR_INVALID_ARG (null pointer, rho out of range, replicas <
 * 1, misaligned workspace), DYNRAD_ERR_UNSUPPORTED (block not 32/64/128, size
 * limits), DYNRAD_ERR_CAPACITY (workspace) -- before any launch; a col_idx
 * capacity exceeded on the device is recorded in the device status.
 */
size_t dynrad_sampled_mask_workspace_bytes(const dynrad_geom *geom,
                                           int64_t cand_nnz);
size_t dynrad_sampled_mask_workspace_min_bytes(const dynrad_geom *geom,
                                               int64_t cand_nnz);
int dynrad_build_sampled_mask(const dynrad_geom *geom, double rho1, double rho2,
                              uint64_t seed, const int32_t *cand_row_ptr,
                              const int32_t *cand_col, int64_t cand_nnz,
                              const int32_t *forced_lo,
                              const int32_t *forced_hi, int32_t replicas,
                              int32_t *row_ptr, int32_t *col_idx,
                              int64_t col_cap, uint64_t *thresholds_out,
                              void *workspace, size_t workspace_bytes,
                              dynrad_stream_t stream);

/*
 * Paper-exact dynamic-threshold mode (Sec. 3.2 "Dynamic-threshold mode",
 * Eqs. 9-11; the fused-head proxy of Eq. 19): a block mask per batch element,
 * shared by its heads, from token-level proxy logits.
 *
 * For every candidate token pair (u, v) of an ordered frame pair (i, j) at
 * t >= 2 kept by the split rule: s = (1/hf) sum_{h < hf} q_u^h . k_v^h /
 * sqrt(D) over the FIRST hf heads (bf16 tensor-core products, fp32
 * accumulation in a fixed order); per frame pair, mu and the population sigma
 * of s over P(i, j) (fp32 partial sums of at most 16 logits, added in fp64);
 * the pair is kept
 * when (s - mu) / (sigma + 1e-6) > tau, tau = tau1 when L(t) >= block, tau2
 * otherwise; if none passes, the pair with the largest s (smallest u*N_t + v
 * among equals) is kept.  Pairs at t <= 1 are all kept.  Kept links are
 * aggregated with (theta_c, theta_m) and united with the forced range.
 *
 *   q, k          DEVICE bf16 [B, H, N, D], 16-byte aligned; D = 64 or 128;
 *                 hf in [1, min(H, 4)]
 *   tau1, tau2    finite z-score thresholds (near / far field)
 *   cand_*, forced_*  from dynrad_build_candidates for geom (DEVICE)
 *   row_ptr       DEVICE int32 [B*H*Nb + 1], rows (b, h, I); every head of a
 *                 batch element gets that element's mask
 *   col_idx       DEVICE int32, capacity col_cap (B*H*cand_nnz always suffices)
 *   stats_out     nullable DEVICE double [B][F*F][3]: mu, sigma and the score
 *                 threshold mu + tau (sigma + 1e-6) per (batch, frame pair);
 *                 zeros / -inf where nothing is thresholded (t <= 1, dropped)
 *   workspace     DEVICE, 256-byte aligned, dynrad_token_mask_workspace_bytes
 *                 (B, N, geom, cand_nnz) bytes (holds a B x Nb x N counter
 *                 array: ~360 MB per batch element at 75,600 tokens, block 64)
 * Errors: DYNRAD_ERR_INVALID_ARG / UNSUPPORTED / CAPACITY before any launch
 * (null pointer, hf out of range, non-finite tau, D, block, N_t > 65535,
 * 5 * frames + Nb > 49,136);
 * a col_idx capacity exceeded on the device is recorded in the device status.
 */
size_t dynrad_token_mask_workspace_bytes(int32_t B, int32_t N,
                                         const dynrad_geom *geom,
                                         int64_t cand_nnz);
int dynrad_build_token_mask(const void *q, const void *k, int32_t B, int32_t H,
                            int32_t N, int32_t D, int32_t hf,
                            const dynrad_geom *geom, double tau1, double tau2,
                            const int32_t *cand_row_ptr,
                            const int32_t *cand_col, int64_t cand_nnz,
                            const int32_t *forced_lo, const int32_t *forced_hi,
                            int32_t *row_ptr, int32_t *col_idx,
                            int64_t col_cap, double *stats_out,
                            void *workspace, size_t workspace_bytes,
                            dynrad_stream_t stream);

/*
 * Stages 2 and 3 from and to HOST memory (no counterpart in the paper: a
 * runtime convenience for callers whose Q, K, V live on the host).
 *
 * For each of n_runs selection settings ("runs": geometry, candidate set,
 * mode, rho or tau) over one layer's Q, K, V, computes the kept-block CSR
 * (as dynrad_select_blocks) and the attention output (as dynrad_sparse_attn)
 * and writes the run's O and LSE to host memory.  The B*H (batch, head) rows
 * go through in chunks of chunk_bh rows: the copy-in of later chunks, the
 * kernels of the current (chunk, run) items and the copy-out of finished
 * items run concurrently on three streams the call creates and on `stream`
 * (items alternate between `stream` and one created compute stream, so one
 * item's kernels start while the previous item's attention drains).
 * Results are bit-identical to the device-resident calls (every stage is
 * independent per (batch, head) row).
 *
 *   q_host, k_host, v_host  HOST bf16 [B, H, N, D]; pinned (page-locked)
 *                 memory for the copies to overlap (pageable memory works but
 *                 serialises)
 *   runs[r].geom, cand_*, forced_*  as for dynrad_select_blocks (candidate
 *                 CSR from dynrad_build_candidates for that geometry; DEVICE)
 *   runs[r].mode, rho_or_tau  as for dynrad_select_blocks
 *   runs[r].o_host, lse_host  HOST bf16 [B, H, N, D] and fp32 [B, H, N]
 *                 (pinned for overlap)
 *   n_runs        1 .. 16
 *   chunk_bh      rows per chunk (>= 1; the last chunk may be shorter; with
 *                 room for it, chunks of 1 and 2 rows open and close the
 *                 schedule to shorten the copies that cannot overlap).
 *                 Chunks of a whole number of waves of the attention kernel
 *                 keep it efficient (e.g. 4 heads of 75,600 tokens = 1,184
 *                 CTAs = 8 x 148 SMs).
 *   scale         as for dynrad_sparse_attn (0 means 1/sqrt(D))
 *   workspace     DEVICE, 256-byte aligned, at least
 *                 dynrad_host_path_workspace_bytes(...) bytes: it holds Q, K, V,
 *                 every run's O and LSE, and per compute stream one chunk's
 *                 kept CSR and selection workspace
 *
 * Ordering: the call's device work starts after the work already queued on
 * `stream` and `stream` continues only after the last copy-out, so back-to-
 * back calls on one stream never overlap.  The host buffers must stay valid
 * and unchanged until `stream` has passed the call.
 * Errors: DYNRAD_ERR_INVALID_ARG (null pointer, n_runs or chunk_bh out of
 * range, a geometry that does not match N, misaligned workspace),
 * DYNRAD_ERR_CAPACITY (workspace too small) -- both before any device work;
 * otherwise the errors of dynrad_select_blocks / dynrad_sparse_attn, and
 * DYNRAD_ERR_CUDA when a copy, stream or event call fails.  Such an error can
 * come after copies of earlier chunks were queued; the call still makes
 * `stream` wait for every copy it queued before it returns, so the rule above
 * holds on every return: the host buffers are in use until `stream` has
 * passed the call (their contents are then undefined for the failed run).
 * dynrad_host_path_workspace_bytes returns 0 for arguments it cannot size.
 */
typedef struct dynrad_host_run {
  dynrad_geom geom;
  const int32_t *cand_row_ptr;
  const int32_t *cand_col;
  int64_t cand_nnz;
  int64_t cand_max_row;
  const int32_t *forced_lo;
  const int32_t *forced_hi;
  int32_t mode;
  double rho_or_tau;
  void *o_host;
  float *lse_host;
} dynrad_host_run;

size_t dynrad_host_path_workspace_bytes(int32_t B, int32_t H, int32_t N,
                                        int32_t D, const dynrad_host_run *runs,
                                        int32_t n_runs, int32_t chunk_bh);
int dynrad_host_path(const void *q_host, const void *k_host,
                     const void *v_host, int32_t B, int32_t H, int32_t N,
                     int32_t D, const dynrad_host_run *runs, int32_t n_runs,
                     int32_t chunk_bh, float scale, void *workspace,
                     size_t workspace_bytes, dynrad_stream_t stream);

/*
 * Objective of the offline parameter search (Appendix C.4, Eq. 22; no
 * counterpart on the hot path): from the log-sum-exps of dynrad_sparse_attn
 * run with a full CSR and with a mask, each at logit scale c and 2c, writes
 * out[0] = ||A_dense - A_masked||_F^2 and out[1] = ||A_dense||_F^2 over the n
 * query rows, A the row-softmax matrices (the masked one renormalized over its
 * kept keys; a row with no kept key is all zero).  Uses, per row,
 * sum_j a_j^2 = exp(lse(2c) - 2 lse(c)) and kept mass exp(lse_kept - lse_dense).
 *
 *   lse_dense, lse_kept, lse2_dense, lse2_kept  DEVICE fp32 [n]
 *   out           DEVICE double [2] (overwritten)
 */
int dynrad_proxy_error(const float *lse_dense, const float *lse_kept,
                       const float *lse2_dense, const float *lse2_kept,
                       int64_t n, double *out, dynrad_stream_t stream);

/*
 * Backward of stage 3 (the gradient that the mask-aware fine-tuning of
 * Sec. 3.3 trains through): given dO, the forward's O and LSE and the SAME
 * kept-block CSR, computes for every (b, h)
 *   P_qk  = exp(scale * q.k - lse_q) on the kept blocks' valid keys, else 0
 *   D_q   = sum_d dO_qd O_qd
 *   dV_k  = sum_q P_qk dO_q
 *   dS_qk = P_qk (dO_q . v_k - D_q)
 *   dQ_q  = scale * sum_k dS_qk k_k,   dK_k = scale * sum_q dS_qk q_q
 * (the exact gradient of the forward's output; keys of unkept blocks get
 * dK = dV = 0, rows with no kept block get dQ = 0).  Tensor cores (tcgen05,
 * bf16 operands -- P and dS are rounded to bf16 -- fp32 accumulation in
 * TMEM); no atomics, deterministic: one CTA owns each 128-row tile of dK/dV
 * and of dQ, so S and dP are computed twice (once per side).  The workspace
 * holds -lse log2(e) and -D_q per query row and the transposed CSR.
 *
 *   q, k, v, o, dout  device bf16 [B, H, N, D], D = 64 or 128
 *   lse           device fp32 [B, H, N] (the forward's, natural log)
 *   block         32, 64 or 128 (at 32 each 64-row step of the tensor-core
 *                 tiles holds one block, half the tile)
 *   row_ptr, col_idx  the forward's CSR (device int32, B*H*Nb rows, strictly
 *                 ascending block indices in [0, Nb) per row)
 *   col_cap       capacity of the transposed CSR: >= row_ptr[B*H*Nb]
 *                 (overflow is flagged in the device status)
 *   scale         logit scale; 0 means 1/sqrt(D)
 *   dq, dk, dv    device bf16 [B, H, N, D] (overwritten)
 *   workspace     device, 256-byte aligned, workspace_bytes >=
 *                 dynrad_attn_backward_workspace_bytes(B, H, N, block, col_cap)
 *   B * H <= 65535.
 */
size_t dynrad_attn_backward_workspace_bytes(int32_t B, int32_t H, int32_t N,
                                            int32_t block, int64_t col_cap);
int dynrad_attn_backward(const void *q, const void *k, const void *v,
                         const void *o, const void *dout, const float *lse,
                         int32_t B, int32_t H, int32_t N, int32_t D,
                         int32_t block, const int32_t *row_ptr,
                         const int32_t *col_idx, int64_t col_cap, float scale,
                         void *dq, void *dk, void *dv, void *workspace,
                         size_t workspace_bytes, dynrad_stream_t stream);

/*
 * Reads the device status word (the first error a kernel recorded since the
 * last clear) into *status_out; clears it when clear != 0.  SYNCHRONIZES the
 * stream.  Returns DYNRAD_ERR_CUDA if the stream itself reports an error.
 */
int dynrad_device_status(int32_t *status_out, int32_t clear,
                         dynrad_stream_t stream);

/*
 * Diagnostic: evaluates, for n device floats x, the FMA-pipe approximation of
 * 2^x that the attention kernel's softmax uses for part of its exponentials
 * (poly_out) and CUDA's exp2f (ref_out), so the approximation can be checked
 * against CUDA's own results.  Valid range of the approximation: x <= 64
 * (inputs below -125 give 2^-125).  Device pointers; asynchronous.
 */
int dynrad_debug_exp2(const float *x, float *poly_out, float *ref_out,
                      int64_t n, dynrad_stream_t stream);

/*
 * Test hook for the attention forward's failure path (no counterpart in the
 * paper), for launches made after the call:
 *   wait_ns     limit, in nanoseconds of the GPU's global timer, of the
 *               kernel's pipeline waits; 0 restores the built-in limit (2 s)
 *   stall_step  >= 0: at that step of its walk the MMA warp of every CTA waits
 *               for a barrier that nothing completes, so that wait runs out
 *               after wait_ns; -1 (the default) never
 * A wait that runs out records DYNRAD_ERR_DEVICE in the device status; every
 * warp of the CTA unwinds, copies and tensor-core products already in flight
 * finish (those waits always keep the full limit), tensor memory is freed and
 * the kernel returns; the outputs of that launch are undefined.  Restore with
 * (0, -1).  Process-wide and not synchronised with launches on other host
 * threads: for tests only.  Errors: DYNRAD_ERR_INVALID_ARG for stall_step < -1.
 */
int dynrad_debug_attn_stall(uint64_t wait_ns, int32_t stall_step);

/* Static string for a status code ("ok", "invalid argument", ...). */
const char *dynrad_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* DYNRAD_H */
