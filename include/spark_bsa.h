/*
 * spark_bsa.h - C ABI of the B200 (sm_100a) two-branch block-sparse attention forward.
 *
 * The operation is the Spark-Attn forward described in the blog "Spark-H3: Adaptive Block
 * Sparse Attention for MiniMax-H3":
 *
 *   - section "Spark-Reblock": tokens are permuted into blocks (token ids track membership)
 *     and, per query block A,  BSA(Q_A) = Softmax(Q_A K~_A^T / sqrt(d)) V~_A,  where K~_A,
 *     V~_A hold the exact rows of every selected key block B in S_A and one summary per
 *     unselected block; a single row-wise softmax covers both branches; S_A is a fixed
 *     Top-K budget ("top 10%" of key blocks);
 *   - section "Discussion": blocks are scored from block-level means;
 *   - section "Spark-Reweight": each key block is scored once with a representative query
 *     (the mean of the head's queries); the scores give weighted key/value summaries and a
 *     log-mass bias so that exp(effective logit) equals E[exp(q.k)] instead of exp(E[q.k]).
 *
 * Definitions used by every entry point (sigma = 1/sqrt(d)):
 *   Qp[h,i] = Q[h, q_perm[h,i]],  Kp[h,j] = K[h, k_perm[h,j]],  Vp[h,j] = V[h, k_perm[h,j]]
 *   qbar[h]       = mean over all N queries of head h                    (the anchor)
 *   qbar_A[h,A]   = mean of Qp rows of query block A;  kbar[h,B] = mean of Kp rows of block B
 *   s_j           = sigma * qbar . Kp_j;  w = softmax of s over the rows j of block B
 *   k~_B = sum_j w_j Kp_j,  v~_B = sum_j w_j Vp_j
 *   c_B  = log(mean_j exp s_j) - sigma * qbar . k~_B + log|B|   (bias b plus log|B|)
 *   S[h,A,B]      = sigma * qbar_A . kbar_B;  sel[h,A,:] = the k largest (ties: smaller B),
 *                   stored ascending,  k = clamp(ceil(topk_ratio*nkb - 1e-9), 1, nkb)
 *   out[h, q_perm[h,i]] = softmax over { sigma q_i.k_j : j in selected blocks } union
 *                         { sigma q_i.k~_B + c_B : B unselected } applied to {v_j} U {v~_B}
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise; every buffer is
 *     owned by the caller; the library allocates nothing and keeps no state between calls
 *     (a per-process cache of the driver entry point used to encode TMA descriptors aside).
 *   - Tensors are contiguous, row-major: Q/K/V/out [H,N,d]; perms [H,N] int32 (row i of the
 *     reblocked layout holds original token perm[i]; one permutation per head); block
 *     offsets [nb+1] int32, shared by all heads, 0 = off[0] < off[1] < ... < off[nb] = N,
 *     every block 1..128 tokens.  q_perm == k_perm with equal offsets is legal (the pages'
 *     reblock_layout=q_reuse_k).
 *   - d must be 64 or 128.  bf16 inputs give bf16 out; fp32 inputs are rounded to bf16
 *     (round-to-nearest-even) on entry and give fp32 out.  Internally: bf16 tensor-core
 *     operands, fp32 accumulation, fp32 softmax, fp32 means, summaries' bias and scores.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are asynchronous
 *     on that stream; no entry point synchronises except spark_bsa_read_error.
 *   - Host-checkable problems return a status before anything is launched.  Problems only
 *     visible in device data (a permutation entry outside [0,N), bad offsets, a selected
 *     id outside [0,nkb)) never cause out-of-bounds accesses: the kernels skip the access
 *     and set bits in the device error word, which spark_bsa_read_error returns.
 */
#ifndef SPARK_BSA_H_
#define SPARK_BSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPARK_API __attribute__((visibility("default")))
#else
#define SPARK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARK_OK = 0,
  SPARK_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, ratio outside (0,1] ... */
  SPARK_ERR_UNSUPPORTED = 2,   /* d not in {64,128}, a size beyond the library's limits   */
  SPARK_ERR_WORKSPACE = 3,     /* workspace too small or misaligned                       */
  SPARK_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed           */
  SPARK_ERR_DEVICE_CHECK = 5   /* the device error word is non-zero                       */
} spark_status;

typedef enum { SPARK_BF16 = 0, SPARK_F32 = 1 } spark_dtype;

/* Bits of the device error word. */
#define SPARK_DEVERR_PERM 0x1u     /* a permutation entry outside [0, N)                      */
#define SPARK_DEVERR_OFFSETS 0x2u  /* a block outside [1,128] tokens or offsets not 0..N     */
#define SPARK_DEVERR_SEL 0x4u      /* a selected block id outside [0, nkb)                    */
#define SPARK_DEVERR_TIMEOUT 0x8u  /* a bounded in-kernel wait expired (kernel bug)          */

/* Library limits (SPARK_ERR_UNSUPPORTED beyond them). */
#define SPARK_MAX_BLOCK 128        /* tokens per block                                        */
#define SPARK_MAX_NKB 12800        /* key blocks per head                                     */
#define SPARK_MAX_NC (1 << 20)     /* context tokens per head                                 */

/* Human-readable name of a status code; never NULL. */
SPARK_API const char* spark_status_string(int status);

/* Limit of every bounded wait inside the library's kernels, in nanoseconds of the GPU's
 * global timer (no counterpart in the pages: a safety bound of this implementation).  The
 * kernels that wait on barriers (the attention, the partitioner's tensor-core kernels) take
 * the value current at their launch as a parameter; default 4e9 (4 s).  When a wait runs out
 * the kernel sets SPARK_DEVERR_TIMEOUT in the device error word, stops every CTA of the
 * launch, waits (with the default limit) for its own copies and MMAs in flight, frees its
 * tensor memory and returns, so the context stays usable and the error is read with
 * spark_bsa_read_error.  0 makes every wait expire at once, without looking at its barrier
 * (a deterministic test of that path).  Process-wide (all devices and threads); atomic. */
SPARK_API void spark_bsa_set_wait_limit_ns(uint64_t limit_ns);
SPARK_API uint64_t spark_bsa_get_wait_limit_ns(void);

/* k = clamp(ceil(topk_ratio * nkb - 1e-9), 1, nkb) - the blog's "top ratio" budget with
 * a guard against binary rounding of the ratio.  Returns -1 if nkb < 1 or the ratio is
 * outside (0, 1]. */
SPARK_API int spark_bsa_topk_count(int nkb, double topk_ratio);

/* Byte offsets of the intermediates inside a spark_bsa_forward workspace.  Each offset is
 * 256-byte aligned; `total` is the workspace size in bytes. */
typedef struct {
  size_t Qp, Kp, Vp;          /* bf16 [H,N,d] reblocked Q, K, V                          */
  size_t qbar_blocks;         /* fp32 [H,nqb,d] query-block means                        */
  size_t qbar;                /* fp32 [H,d] per-head anchor                              */
  size_t kbar;                /* fp32 [H,d,nkb] key-block means, d-major                 */
  size_t k_tilde, v_tilde;    /* bf16 [H,nkb,d] weighted summaries                       */
  size_t cbias;               /* fp32 [H,nkb] summary offsets c_B = b_B + log|B|        */
  size_t sel;                 /* int32 [H,nqb,k] selected key blocks, ascending          */
  size_t err;                 /* uint32 device error word                                */
  size_t total;
  int k;                      /* the Top-K count                                         */
} spark_bsa_layout;

/* Fills *layout for the given sizes.  Pure host arithmetic. */
SPARK_API spark_status spark_bsa_workspace_layout(int H, int N, int d, int nqb, int nkb,
                                        double topk_ratio, spark_bsa_layout* layout);

/* Workspace bytes spark_bsa_forward needs (0 if the arguments are invalid). */
SPARK_API size_t spark_bsa_workspace_size(int H, int N, int d, int nqb, int nkb, double topk_ratio);

/* The whole forward pass: gather + query-block means, anchor, key/value gather fused with
 * the key-block means and Spark-Reweight summaries, block scoring + Top-K, and the
 * two-branch tcgen05 attention.  `workspace` (device, 256-byte aligned, at least
 * spark_bsa_workspace_size bytes) receives the intermediates at the offsets of
 * spark_bsa_workspace_layout, so callers may inspect them after the call; its error word is
 * cleared by the call.  `out` is [H,N,d] of `dtype`, in the ORIGINAL token order. */
SPARK_API spark_status spark_bsa_forward(const void* Q, const void* K, const void* V, int dtype, int H,
                               int N, int d, const int32_t* q_perm, const int32_t* k_perm,
                               const int32_t* q_block_offsets, int nqb,
                               const int32_t* k_block_offsets, int nkb, double topk_ratio,
                               void* out, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Synchronises `stream`, then copies the device error word at `err_word` (device pointer,
 * e.g. workspace + layout.err) into *flags (host).  Returns SPARK_ERR_DEVICE_CHECK when it
 * is non-zero. */
SPARK_API spark_status spark_bsa_read_error(const uint32_t* err_word, void* stream, uint32_t* flags);

/* ---- The steps of the forward pass, one kernel each, on caller buffers. ----
 * `err` is a device uint32 error word (may be NULL: bad device data is then skipped
 * silently).  Bits are OR-ed in; the word is never cleared by these calls. */

/* Step 1 (queries; blog "Spark-Reblock" token permutation, "Discussion" block means):
 * Qp[h,i,:] = bf16(Q[h,q_perm[h,i],:]);  qbar_blocks[h,A,:] = mean of block A's Qp rows. */
SPARK_API spark_status spark_bsa_gather_q(const void* Q, int dtype, int H, int N, int d,
                                const int32_t* q_perm, const int32_t* q_block_offsets, int nqb,
                                void* Qp, float* qbar_blocks, uint32_t* err, void* stream);

/* Step 2 (blog "Spark-Reweight": the representative query; one anchor per head):
 * qbar[h,:] = (sum_A |A| * qbar_blocks[h,A,:]) / N. */
SPARK_API spark_status spark_bsa_anchor(const float* qbar_blocks, const int32_t* q_block_offsets, int H,
                              int N, int d, int nqb, float* qbar, void* stream);

/* Steps 1+3 fused (keys/values; blog "Spark-Reweight" weighted summaries and log-mass bias):
 * Kp, Vp (bf16 [H,N,d]) gathered by k_perm; kbar (fp32 [H,d,nkb], d-major: kbar[h][e][B] is
 * dimension e of block B's mean) block means;
 * k_tilde, v_tilde (bf16 [H,nkb,d]) and cbias (fp32 [H,nkb]) as defined above, with
 * c_B computed against the bf16-rounded k~_B that the attention step consumes. */
SPARK_API spark_status spark_bsa_gather_kv_summarize(const void* K, const void* V, int dtype, int H,
                                           int N, int d, const int32_t* k_perm,
                                           const int32_t* k_block_offsets, int nkb,
                                           const float* qbar, void* Kp, void* Vp, float* kbar,
                                           void* k_tilde, void* v_tilde, float* cbias,
                                           uint32_t* err, void* stream);

/* Step 1+3 with the baseline BSA compressed branch instead of Spark-Reweight's, as the
 * comparator of the blog's ablations (section "Spark-Reblock", BSA equations: an unselected
 * block repeats its uniform mean key and value |B| times): the same Kp, Vp and kbar as
 * spark_bsa_gather_kv_summarize, with k_tilde = bf16(mean key), v_tilde = bf16(mean value)
 * and cbias = log|B| (the |B| copies as one row).  No anchor is used.  The attention step
 * then takes these in place of the weighted summaries. */
SPARK_API spark_status spark_bsa_gather_kv_meanpool(const void* K, const void* V, int dtype, int H,
                                                    int N, int d, const int32_t* k_perm,
                                                    const int32_t* k_block_offsets, int nkb,
                                                    void* Kp, void* Vp, float* kbar,
                                                    void* k_tilde, void* v_tilde, float* cbias,
                                                    uint32_t* err, void* stream);

/* Step 4 (blog "Discussion": block-mean scoring; "Spark-Reblock": fixed Top-K budget):
 * fp32 scores sigma*qbar_A.kbar_B (qbar_blocks [H,nqb,d], kbar d-major [H,d,nkb] as written by
 * spark_bsa_gather_kv_summarize), the k largest per (h,A) with ties to the smaller B,
 * written ascending to sel [H,nqb,k].  1 <= k <= nkb <= SPARK_MAX_NKB. */
SPARK_API spark_status spark_bsa_route(const float* qbar_blocks, const float* kbar, int H, int nqb,
                             int nkb, int d, int k, int32_t* sel, uint32_t* err, void* stream);

/* Step 4 as Sol-Attn's content-adaptive routing, the comparator the blog's "Discussion"
 * describes (block logits taken as roughly Gaussian; blocks above mu + tau*sigma are exact).
 * Readings: mu and sigma are the mean and population standard deviation of the query block's
 * nkb scores (fp32); "above" is strict; at most kcap blocks are kept (the largest, ties to the
 * smaller B).  Writes the selection ascending to the first count[h,A] entries of row (h,A) of
 * sel [H,nqb,kcap] (the rest of the row is untouched) and count [H,nqb] (0..kcap).
 * kbar is d-major as written by spark_bsa_gather_kv_summarize. */
SPARK_API spark_status spark_bsa_route_threshold(const float* qbar_blocks, const float* kbar,
                                                 int H, int nqb, int nkb, int d, double tau,
                                                 int kcap, int32_t* sel, int32_t* count,
                                                 uint32_t* err, void* stream);

/* Step 5 with a per-query-block selection count (as spark_bsa_route_threshold writes): sel
 * rows are kcap apart and row (h,A) holds count[h,A] ascending block ids; the other blocks
 * enter the compressed branch.  Otherwise as spark_bsa_attend. */
SPARK_API spark_status spark_bsa_attend_var(const void* Qp, const void* Kp, const void* Vp,
                                            const void* k_tilde, const void* v_tilde,
                                            const float* cbias, const int32_t* sel, int kcap,
                                            const int32_t* count, const int32_t* q_perm,
                                            const int32_t* q_block_offsets, int nqb,
                                            const int32_t* k_block_offsets, int nkb, int H,
                                            int N, int d, void* out, int out_dtype,
                                            uint32_t* err, void* stream);

/* Step 5 (blog "Spark-Reblock" BSA equations with the Spark-Reweight summaries): the
 * two-branch attention of every (h, A), one row-wise softmax over the exact rows of the
 * selected blocks and the summary rows (logit sigma q.k~_B + c_B) of the others, written to
 * out[h, q_perm[h,i], :] (out dtype `out_dtype`).  Qp/Kp/Vp/k_tilde/v_tilde are bf16 and
 * must be 16-byte aligned; sel [H,nqb,k] ascending, distinct. */
SPARK_API spark_status spark_bsa_attend(const void* Qp, const void* Kp, const void* Vp,
                              const void* k_tilde, const void* v_tilde, const float* cbias,
                              const int32_t* sel, int k, const int32_t* q_perm,
                              const int32_t* q_block_offsets, int nqb,
                              const int32_t* k_block_offsets, int nkb, int H, int N, int d,
                              void* out, int out_dtype, uint32_t* err, void* stream);

/* ---- Context (sink) tokens ----
 * Spark-H3 blog, section "Spark-Reblock", after the BSA equations: context/sink tokens stay
 * exact and are not counted against the video-block Top-K budget.  Reading taken here: each
 * head has nc context tokens with keys Kc[h] and values Vc[h] ([H,nc,d], row-major, same dtype
 * as Q/K/V).  Every video query attends to all of them exactly, in the same row-wise softmax
 * as the exact and compressed branches (logit sigma q.kc_j).  They form no block and take no
 * part in the anchor, the block means, the summaries or the routing; k is still taken over the
 * nkb video blocks.  Context queries are not part of this operation (the caller attends them
 * densely).  0 <= nc <= SPARK_MAX_NC; nc == 0 is exactly the call without context. */

/* Workspace bytes spark_bsa_forward_ctx needs: spark_bsa_workspace_size plus two bf16
 * [H,nc,d] regions (each rounded up to 256 bytes) that receive the converted context rows at
 * offsets layout.total and layout.total + round256(H*nc*d*2).  0 if the arguments are
 * invalid. */
SPARK_API size_t spark_bsa_workspace_size_ctx(int H, int N, int d, int nqb, int nkb,
                                              double topk_ratio, int nc);

/* spark_bsa_forward with context tokens.  Kc, Vc: device, 16-byte aligned, [H,nc,d] of
 * `dtype` (may be NULL when nc == 0).  bf16 context rows are read in place; fp32 ones are
 * first converted to bf16 into the workspace (after the intermediates of
 * spark_bsa_workspace_layout).  They are attended as extra exact key tiles.  Errors as spark_bsa_forward; SPARK_ERR_INVALID_ARG for nc outside
 * [0, SPARK_MAX_NC] or missing/misaligned context pointers. */
SPARK_API spark_status spark_bsa_forward_ctx(const void* Q, const void* K, const void* V,
                                             const void* Kc, const void* Vc, int nc, int dtype,
                                             int H, int N, int d, const int32_t* q_perm,
                                             const int32_t* k_perm,
                                             const int32_t* q_block_offsets, int nqb,
                                             const int32_t* k_block_offsets, int nkb,
                                             double topk_ratio, void* out, void* workspace,
                                             size_t workspace_bytes, void* stream);

/* Step of the context path: Kc_bf16[i] = bf16(Kc[i]), Vc_bf16[i] = bf16(Vc[i]) (round to
 * nearest even; a copy for bf16 input), [H,nc,d].  All pointers device, 16-byte aligned. */
SPARK_API spark_status spark_bsa_context_bf16(const void* Kc, const void* Vc, int dtype, int H,
                                              int nc, int d, void* Kc_bf16, void* Vc_bf16,
                                              void* stream);

/* spark_bsa_attend with context rows: Kc, Vc are bf16 [H,nc,d] (16-byte aligned; NULL allowed
 * when nc == 0).  The tiles of a query block are the selected video blocks, then ceil(nc/128)
 * context tiles, then the summary tiles. */
SPARK_API spark_status spark_bsa_attend_ctx(const void* Qp, const void* Kp, const void* Vp,
                                            const void* k_tilde, const void* v_tilde,
                                            const float* cbias, const int32_t* sel, int k,
                                            const void* Kc, const void* Vc, int nc,
                                            const int32_t* q_perm,
                                            const int32_t* q_block_offsets, int nqb,
                                            const int32_t* k_block_offsets, int nkb, int H,
                                            int N, int d, void* out, int out_dtype,
                                            uint32_t* err, void* stream);

/* ---- FP8 logits ----
 * Spark-H3 blog, section "Benchmark Results": Spark-H3's attention is also timed in FP8; the
 * scheme is not given.  Readings taken here:
 *   - only the logit product is FP8: the queries Qp, the exact keys Kp, the summary keys k~
 *     and the context keys enter it as e4m3 (OCP E4M3FN: largest finite 448, round to
 *     nearest even, saturating); routing, anchor, summaries, values and probabilities are
 *     those of the bf16 path;
 *   - one power-of-two scale 2^e per group of rows: each query block, each key block, each
 *     128-row tile of the summary rows and of the context rows, e the smallest integer with
 *     max|x| <= 448 * 2^e (at least -126; 0 for an all-zero group); the code of x is
 *     e4m3(x * 2^-e), which is exact before the rounding;
 *   - the logit of query i (block A) and key j (group G) is sigma * sA * sG * (qcode . kcode),
 *     plus c_B for a summary row.
 * d must be 128 (one 128-byte row of codes per token). */

/* Codes of bf16 rows src [H,R,d] (device, 16-byte aligned) into dst [H,R,d] (one byte per
 * value) and scales [H,ngroups] (fp32, 2^e).  Groups are the blocks of `group_offsets`
 * ([ngroups+1] device int32, shared by all heads, non-decreasing within 0..R), or, when it is
 * NULL, the 128-row tiles (ngroups must then be ceil(R/128)).  Bad offsets set
 * SPARK_DEVERR_OFFSETS and leave that group unwritten (scale 1). */
SPARK_API spark_status spark_bsa_quantize_fp8(const void* src, int H, int R, int d,
                                              const int32_t* group_offsets, int ngroups,
                                              void* dst, float* scales, uint32_t* err,
                                              void* stream);

/* Step 5 with FP8 logits: as spark_bsa_attend_ctx, with Qp8 [H,N,d] / q_scale [H,nqb] (per
 * query block), Kp8 [H,N,d] / k_scale [H,nkb] (per key block), kt8 [H,nkb,d] / kt_scale
 * [H,ceil(nkb/128)] and Kc8 [H,nc,d] / kc_scale [H,ceil(nc/128)] (per 128-row tile; Kc8,
 * kc_scale and Vc may be NULL when nc == 0), as written by spark_bsa_quantize_fp8; Vp,
 * v_tilde and Vc stay bf16.  d must be 128 (SPARK_ERR_UNSUPPORTED otherwise). */
SPARK_API spark_status spark_bsa_attend_fp8(const void* Qp8, const float* q_scale,
                                            const void* Kp8, const float* k_scale,
                                            const void* Vp, const void* kt8,
                                            const float* kt_scale, const void* v_tilde,
                                            const float* cbias, const int32_t* sel, int k,
                                            const void* Kc8, const float* kc_scale,
                                            const void* Vc, int nc, const int32_t* q_perm,
                                            const int32_t* q_block_offsets, int nqb,
                                            const int32_t* k_block_offsets, int nkb, int H,
                                            int N, int d, void* out, int out_dtype,
                                            uint32_t* err, void* stream);

/* Workspace bytes of spark_bsa_forward_fp8: spark_bsa_workspace_size_ctx plus the codes and
 * scales; 0 when d != 128 or the sizes are invalid. */
SPARK_API size_t spark_bsa_workspace_size_fp8(int H, int N, int d, int nqb, int nkb,
                                              double topk_ratio, int nc);

/* The forward pass of spark_bsa_forward_ctx (nc may be 0, Kc/Vc then NULL) with FP8 logits:
 * after the routing, Qp, Kp, k~ and the context keys are quantised in the workspace and the
 * attention runs on the codes.  The bf16 layout (spark_bsa_workspace_layout) stays at the
 * start of the workspace. */
SPARK_API spark_status spark_bsa_forward_fp8(const void* Q, const void* K, const void* V,
                                             const void* Kc, const void* Vc, int nc, int dtype,
                                             int H, int N, int d, const int32_t* q_perm,
                                             const int32_t* k_perm,
                                             const int32_t* q_block_offsets, int nqb,
                                             const int32_t* k_block_offsets, int nkb,
                                             double topk_ratio, void* out, void* workspace,
                                             size_t workspace_bytes, void* stream);

/* ---- Host buffers, pipelined by head chunks ----
 * No counterpart in the pages: the forward pass for inputs and output in host memory.  The
 * heads are processed in chunks of `heads_per_chunk`; the copies of chunk c+1 in and of
 * chunk c-1 out run on `h2d_stream` / `d2h_stream` while chunk c is computed on
 * `compute_stream`, through two device staging slots.  The result equals spark_bsa_forward
 * on the same inputs bit for bit (heads are independent).
 *   - Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister); pageable memory
 *     works but the copies then do not overlap the computation.
 *   - `staging`: device, 256-byte aligned, spark_bsa_host_staging_size bytes;
 *     `workspace`: device, 256-byte aligned, spark_bsa_workspace_size(min(heads_per_chunk, H),
 *     ...) bytes, reused by every chunk.
 *   - The call only enqueues work; `compute_stream` completes after the last copy back, so
 *     synchronising it is enough.  The three streams must be distinct.
 *   - The workspace's error word describes the last chunk only.
 *   - The copy streams first wait for the work already queued on `compute_stream`, so
 *     back-to-back calls sharing staging buffers are ordered.
 *   - The call creates and releases seven CUDA events; it allocates no device memory. */
SPARK_API size_t spark_bsa_host_staging_size(int H, int N, int d, int dtype, int nqb, int nkb,
                                             int heads_per_chunk);

SPARK_API spark_status spark_bsa_forward_host(const void* Q, const void* K, const void* V,
                                              int dtype, int H, int N, int d,
                                              const int32_t* q_perm, const int32_t* k_perm,
                                              const int32_t* q_block_offsets, int nqb,
                                              const int32_t* k_block_offsets, int nkb,
                                              double topk_ratio, void* out, int heads_per_chunk,
                                              void* staging, size_t staging_bytes,
                                              void* workspace, size_t workspace_bytes,
                                              void* compute_stream, void* h2d_stream,
                                              void* d2h_stream);

/* The same host-buffer pipeline for the other variants: nc context (sink) rows per head
 * (Kc, Vc: HOST [H,nc,d] of `dtype`, copied per chunk with the chunk's heads; NULL when nc is
 * 0; the semantics of spark_bsa_forward_ctx), and FP8 logits when fp8_logits is non-zero (the
 * semantics of spark_bsa_forward_fp8; d = 128).  The result equals the device-buffer call of
 * the same variant bit for bit.
 *   - `staging`: spark_bsa_host_staging_size_ex bytes (it includes the context rows);
 *     `workspace`: spark_bsa_workspace_size_fp8(min(heads_per_chunk, H), ..., nc) bytes with
 *     FP8 logits, else spark_bsa_workspace_size_ctx(min(heads_per_chunk, H), ..., nc).
 *   - Everything else as for spark_bsa_forward_host, which is this call with nc = 0 and no
 *     FP8. */
SPARK_API size_t spark_bsa_host_staging_size_ex(int H, int N, int d, int dtype, int nqb, int nkb,
                                                int heads_per_chunk, int nc);

SPARK_API spark_status spark_bsa_forward_host_ex(const void* Q, const void* K, const void* V,
                                                 const void* Kc, const void* Vc, int nc,
                                                 int fp8_logits, int dtype, int H, int N, int d,
                                                 const int32_t* q_perm, const int32_t* k_perm,
                                                 const int32_t* q_block_offsets, int nqb,
                                                 const int32_t* k_block_offsets, int nkb,
                                                 double topk_ratio, void* out,
                                                 int heads_per_chunk, void* staging,
                                                 size_t staging_bytes, void* workspace,
                                                 size_t workspace_bytes, void* compute_stream,
                                                 void* h2d_stream, void* d2h_stream);

/* ---- Spark-Reblock token partitioner ----
 * Spark-H3 blog, section "Spark-Reblock": queries are grouped under the Mahalanobis cosine
 * distance d_Q(q_i,q_j) = 1 - cos(M_K^{1/2} q_i, M_K^{1/2} q_j), M_K = E[k k^T] (keys
 * symmetrically with M_Q), by a hierarchical partitioner that splits every group level by
 * level into children of assigned capacities until every leaf is one block.  The blog does
 * not spell out the split; the reading implemented here:
 *   - fixed-size blocks of `block` tokens (the last takes the remainder), offsets shared by
 *     all heads; a binary tree over the block range, the left child of an m-block node
 *     holding ceil(m/2) blocks; a child's capacity is the tokens of its blocks;
 *   - unit vectors x_i = W q_i / |W q_i| with W = M_K^{1/2} (symmetric square root; computed
 *     by a fixed number of Newton-Schulz iterations in fp32; x stored as bf16);
 *   - a node splits along its principal direction (4 power iterations of the node covariance
 *     from (1,...,1)/sqrt(d)): its capacity-largest projections go left, equal projections to
 *     the token earlier in the node's current order, both children keep the current order;
 *   - the root order is 0..N-1; leaves in block order give the permutation.
 * Mode SPARK_REBLOCK_Q_REUSE_K: keys reuse the query partition (the pages' released
 * reblock_layout=q_reuse_k); SPARK_REBLOCK_SEPARATE: keys are partitioned the same way with
 * Q and K swapped.  Deterministic (fixed-order sums, integer histograms). */
#define SPARK_REBLOCK_Q_REUSE_K 0
#define SPARK_REBLOCK_SEPARATE 1

/* Workspace regions a caller may inspect after spark_reblock_whiten (byte offsets):
 * M fp32 [H,d,d] second moment of the other side, W fp32 [H,d,d] = M^{1/2},
 * X bf16 [H,N,d] unit rows; `levels` = depth of the block tree; `nb` = number of blocks. */
typedef struct {
  size_t M, W, X, total;
  int levels, nb;
} spark_reblock_layout;

/* Fills *layout (pure host arithmetic).  1 <= block <= SPARK_MAX_BLOCK, d in {64,128},
 * ceil(N/block) <= SPARK_MAX_NKB. */
SPARK_API spark_status spark_reblock_workspace_layout(int H, int N, int d, int block,
                                                      spark_reblock_layout* layout);
SPARK_API size_t spark_reblock_workspace_size(int H, int N, int d, int block);
/* Depth of the block tree (levels of splits) for N tokens, or -1 for invalid arguments. */
SPARK_API int spark_reblock_levels(int N, int block);

/* The partitioner.  Q, K: device [H,N,d] of `dtype`, 16-byte aligned.  Outputs (device):
 * q_perm, k_perm [H,N] int32 (reblocked row i of head h is token perm[h,i]) and offsets
 * [nb+1] int32 (fixed-size blocks), ready for spark_bsa_forward.  `workspace`: device,
 * 256-byte aligned, spark_reblock_workspace_size bytes.  Asynchronous on `stream`. */
SPARK_API spark_status spark_reblock(const void* Q, const void* K, int dtype, int H, int N, int d,
                                     int block, int mode, int32_t* q_perm, int32_t* k_perm,
                                     int32_t* offsets, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* Step: M = second moment of Y's rows, W = M^{1/2}, X = unit rows of W x_i into the
 * workspace (offsets of spark_reblock_layout). */
SPARK_API spark_status spark_reblock_whiten(const void* X, const void* Y, int dtype, int H, int N,
                                            int d, int block, void* workspace,
                                            size_t workspace_bytes, void* stream);

/* Step: the splits of tree level `level` (0 = root) of the workspace's X rows: perm_in ->
 * perm_out ([H,N] int32 device, distinct buffers; tokens of nodes that do not split at this
 * level are copied). */
SPARK_API spark_status spark_reblock_level(int H, int N, int d, int block, int level,
                                           const int32_t* perm_in, int32_t* perm_out,
                                           void* workspace, size_t workspace_bytes, void* stream);

/* ---- Routing inside the attention kernel ----
 * Spark-H3 blog, "Related Works" (Sol-Attn joins dynamic routing, sparse computation and the
 * approximation correction in one online-softmax pass) and "Discussion" (block-mean scoring,
 * fixed Top-K budget): the same forward pass as spark_bsa_forward with the block scoring and
 * Top-K selection moved into the attention kernel.  One persistent CTA per SM walks the query
 * blocks head-major; while it attends one query block, its K-tile producer warp scores the
 * next one against every key-block mean and selects the Top-K in shared memory, so there is no
 * routing launch and the selection is never read back from global memory.  The arithmetic is
 * the routing kernel's (sequential fp32 FMA over d, exact radix select, ties to the smaller
 * block), so selections and outputs equal spark_bsa_forward's bit for bit.
 *   - bf16 attention operands, d = 128, Top-K with k < nkb, and a problem small enough for
 *     two selections, two bias rows and the routing keys to fit in shared memory next to the
 *     tiles: spark_bsa_fused_supported(d, nkb, ratio) says whether it does (nkb <= 2468 at
 *     ratio 0.1, <= 2180 at 0.3); otherwise these calls return SPARK_ERR_UNSUPPORTED.
 *   - spark_bsa_forward_fused: arguments, workspace and outputs of spark_bsa_forward; the
 *     workspace's sel region receives a copy of every selection (for inspection).
 *   - spark_bsa_attend_fused: the attention step on caller buffers with the block means of
 *     steps 1 and 2 (qbar_blocks fp32 [H,nqb,d], kbar fp32 [H,d,nkb]) instead of a selection;
 *     `sel_out` (int32 [H,nqb,k], may be NULL) receives the selections. */
SPARK_API int spark_bsa_fused_supported(int d, int nkb, double topk_ratio);

SPARK_API spark_status spark_bsa_forward_fused(const void* Q, const void* K, const void* V,
                                               int dtype, int H, int N, int d,
                                               const int32_t* q_perm, const int32_t* k_perm,
                                               const int32_t* q_block_offsets, int nqb,
                                               const int32_t* k_block_offsets, int nkb,
                                               double topk_ratio, void* out, void* workspace,
                                               size_t workspace_bytes, void* stream);

SPARK_API spark_status spark_bsa_attend_fused(const void* Qp, const void* Kp, const void* Vp,
                                              const void* k_tilde, const void* v_tilde,
                                              const float* cbias, const float* qbar_blocks,
                                              const float* kbar, int k, const int32_t* q_perm,
                                              const int32_t* q_block_offsets, int nqb,
                                              const int32_t* k_block_offsets, int nkb, int H,
                                              int N, int d, void* out, int out_dtype,
                                              int32_t* sel_out, uint32_t* err, void* stream);

/* ---- Forward pass without any allocation ----
 * No counterpart in the pages: this entry point exists for callers that cannot allocate
 * device memory while they run (a memory budget owned by a host framework, work recorded into
 * a CUDA stream capture, a real-time path where an allocation may block or fail).  It is
 * spark_bsa_forward with its workspace taken from a static device array of
 * SPARK_NOALLOC_SCRATCH_BYTES bytes inside the library instead of from the caller; it calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *   - Problems whose spark_bsa_workspace_size exceeds SPARK_NOALLOC_SCRATCH_BYTES are rejected
 *     with SPARK_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device (with that device current) resolves the array's device
 *     address; make that first call before any stream capture.
 *   - The array is reserved on a device when the library's module is loaded there: on the
 *     first use of the library on that device under CUDA's lazy module loading (the default),
 *     at context creation under eager loading (CUDA_MODULE_LOADING=EAGER).  It is held until
 *     the process exits.
 *   - The device address is resolved once per device and cached.  A device reset
 *     (cudaDeviceReset) or any other teardown of the device's context makes the cached address
 *     stale; calling this entry point after one is not supported.
 *   - All calls share the one array and it keeps the last call's contents; the call clears
 *     the error word itself.  Calls that overlap on the GPU (two streams, or two host threads)
 *     race on the array: serialise them.
 *   - The device error word lives in the array and is not returned; bad device data is still
 *     skipped by the kernels. */
#define SPARK_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

SPARK_API spark_status spark_bsa_forward_noalloc(const void* Q, const void* K, const void* V,
                                                 int dtype, int H, int N, int d,
                                                 const int32_t* q_perm, const int32_t* k_perm,
                                                 const int32_t* q_block_offsets, int nqb,
                                                 const int32_t* k_block_offsets, int nkb,
                                                 double topk_ratio, void* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARK_BSA_H_ */
