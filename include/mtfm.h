/*
 * mtfm.h -- C ABI of the B200 (sm_100a) library for MTFM's hybrid masked
 * attention: HSTU-style pointwise-SiLU attention over jagged user-level
 * samples [H | R | T] with the dynamic H/R/T mask, in Full-Attention layers
 * (every token queries) and Target-Attention layers (only T tokens query),
 * with grouped-query attention and the GLN gate.
 *
 * Sources (web pages on MTFM):
 *   [DY] "美团推荐大模型 MTFM 深度硬核解析" (dingyadong.top), §4.1 Full Attention
 *        layer equations, §4.1.1 and §8.2 dynamic mask, §4.2 Target Attention.
 *   [MT] "MTFM：美团统一推荐基座大模型在外卖多业务场景的落地实践" (Meituan tech
 *        blog), §3.2 mask rules, §3.3 hybrid architecture and V2 target
 *        scale-up, §6.1 kernels (1-D jagged mask, SiLU fusion, GLN [G, D]).
 *
 * What every attention call computes, for user u with N_u = L_H + L_R + L_T
 * tokens, query row i, query head h and KV group g = h / (hq / hkv):
 *
 *     A[i, h] = (1 / N_u) * sum_{j visible from i} SiLU(alpha * q[i,h] . k[j,g]) * v[j,g]
 *     Y[i]    = GLN_type(i)(A[i]) (*) U[i]      (GLN over the whole row of hq*head_dim)
 *
 * Visibility ([MT] §3.2): H keys are visible to every query; R keys are causal
 * within R (self included) and visible to a T query only when the R action's
 * timestamp is strictly earlier than that target's exposure; a T key is
 * visible only to itself (V2: to the sub-tokens of its own target).  H rows
 * see only H.  Since SiLU(0) = 0, masking the scores before phi_2 ([DY] §4.1)
 * is the same as dropping invisible keys.
 *
 * Conventions for every call below:
 *   - Pointers named d_* are DEVICE pointers; all memory is owned by the
 *     caller.  The library never allocates, frees or synchronises, except
 *     mtfm_pack_check(), which synchronises the given stream on purpose.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *     Every call is asynchronous on that stream.
 *   - bf16 tensors are passed as uint16_t bit patterns.  Activation layout is
 *     jagged row-major: the rows of user 0, then user 1, ...; within a user
 *     the H rows, then R rows, then T rows.  Q/U/Y/A of a Full layer are
 *     [sum N, hq*head_dim]; of a Target layer [sum L_T, hq*head_dim] (T rows
 *     only, same user order); K/V are always [sum N, hkv*head_dim].  Head h
 *     occupies columns [h*head_dim, (h+1)*head_dim).
 *   - Host-side argument checks run before any launch; a call that returns
 *     an error launched nothing.  Errors found on the device (lengths that do
 *     not add up to the totals, unsorted timestamps) are recorded in the
 *     metadata block; every later kernel that reads that block does nothing,
 *     and mtfm_pack_check() reports them.
 *   - The metadata block is read-only for every call but mtfm_pack, except
 *     for a work counter in its header: the persistent Full-layer forward
 *     attention kernel draws its work from it and sets it back to zero when it
 *     finishes.  Hence two Full-layer forward calls on one metadata block must
 *     be ordered (same stream, or an event); other calls may overlap.
 *   - Supported: head_dim in {32, 64, 128, 256}; hq % hkv == 0; hq/hkv <= 8;
 *     hq*head_dim <= 1024 and a multiple of 32; v2_subtokens in {1, 4}.
 *   - Outputs are fp32 (bf16 inputs, fp32 accumulation throughout).
 *   - No exceptions cross this boundary; no global state is kept (the one
 *     exception is the fixed scratch array of mtfm_attn_target_bwd_static).
 *     tcgen05/TMEM kernels run: the Full-layer forward at head_dim 64 with
 *     hq/hkv in {1, 2, 4} and at head_dim 32 with hq/hkv in {1, 2, 4, 8}; the
 *     Target-layer forward at head_dim 64 and 32 with hq/hkv in {1, 2, 4, 8};
 *     both forwards at head_dim 256; the backward at head_dim 64 and 32.  The
 *     other shapes (head_dim 128; hq/hkv of 3, 5, 6, 7; hq/hkv 8 in the Full
 *     forward at head_dim 64; the backward at head_dim 128 and 256) run the
 *     portable mma.sync kernels.  The choice depends on the shape only (no
 *     run-time switch).
 */
#ifndef MTFM_H_
#define MTFM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MTFM_OK = 0,
  MTFM_ERR_INVALID_ARG = 1,         /* null pointer, negative size, hq % hkv != 0, ... */
  MTFM_ERR_UNSORTED_TS = 2,         /* R timestamps of some user not ascending (device check) */
  MTFM_ERR_UNSUPPORTED = 3,         /* valid but unsupported shape (head_dim, widths) */
  MTFM_ERR_WORKSPACE_TOO_SMALL = 4, /* meta or workspace buffer smaller than the size query */
  MTFM_ERR_CUDA = 5,                /* a CUDA runtime call failed (launch error etc.) */
  MTFM_ERR_TIMEOUT = 6,             /* a bounded device wait gave up (kernel returned early) */
  MTFM_ERR_BAD_LENGTHS = 7,         /* device lengths negative, not summing to the totals, or
                                       L_T not a multiple of v2_subtokens */
  MTFM_ERR_BOUNDS = 8               /* bounds-checked build only: a kernel found a TMA coordinate
                                       or a global index out of bounds and skipped the access */
} mtfm_status;

/* Problem description shared by all calls (host memory, read only). */
typedef struct {
  int32_t batch;          /* B: number of users (jagged samples) */
  int32_t total_tokens;   /* sum over users of N_u = L_H + L_R + L_T */
  int32_t total_r;        /* sum of L_R */
  int32_t total_t;        /* sum of L_T */
  int32_t hq;             /* query heads H */
  int32_t hkv;            /* KV heads G (GQA groups); r = hq / hkv query heads share one */
  int32_t head_dim;       /* per-head width */
  int32_t v2_subtokens;   /* 1: one token per target; 4: V2 target scale-up ([MT] §3.3.2) */
  float alpha;            /* score scale inside SiLU; <= 0 selects 1/sqrt(head_dim) */
  float gln_eps;          /* GLN epsilon; <= 0 selects 1e-5 */
} mtfm_cfg;

/* Human-readable text of a status (static string, never NULL). */
const char* mtfm_status_string(mtfm_status s);

/* ---------------------------------------------------------------------------
 * Jagged pack + mask metadata ("1-D jagged mask" of [MT] §6.1; mask rules of
 * [MT] §3.2).  Builds, in the caller's d_meta block: per-user offsets, per-row
 * token type and prefix end kv_end (H row: L_H; R row a: L_H + a + 1; T row:
 * L_H + #{R : ts < exposure}), and the work lists of 128-row query tiles with
 * their key bounds, users ordered longest first.  Fully masked key blocks are
 * never visited by the attention kernels: they read only keys below the
 * tile's largest kv_end plus the T tile's own sibling block.
 *
 *   d_lh, d_lr, d_lt : int32 [batch] device arrays of per-user lengths.
 *   d_r_ts           : int64 [total_r] R-token timestamps, ascending per user.
 *   d_t_exp          : int64 [total_t] exposure time of every T token (V2:
 *                      the 4 sub-tokens of one target carry the same value).
 *   d_meta           : device block of at least mtfm_meta_bytes(cfg) bytes,
 *                      256-byte aligned; fully rewritten by this call.
 * ------------------------------------------------------------------------- */
size_t mtfm_meta_bytes(const mtfm_cfg* cfg);
mtfm_status mtfm_pack(const mtfm_cfg* cfg, const int32_t* d_lh, const int32_t* d_lr,
                      const int32_t* d_lt, const int64_t* d_r_ts, const int64_t* d_t_exp,
                      void* d_meta, size_t meta_bytes, void* stream);

/* Synchronises `stream` and returns the device-side verdict of the last
 * mtfm_pack on d_meta (MTFM_OK, MTFM_ERR_BAD_LENGTHS, MTFM_ERR_UNSORTED_TS),
 * MTFM_ERR_BOUNDS if a kernel of the bounds-checked build found an access out
 * of bounds, or MTFM_ERR_TIMEOUT if a kernel recorded a timeout there.
 * Optional: the hot path never needs it. */
mtfm_status mtfm_pack_check(const void* d_meta, void* stream);

/* Bounds-checked build (compiled with -DMTFM_DEBUG_BOUNDS; no counterpart on the
 * pages: it stands in for a device memory checker).  Its kernels test every TMA
 * coordinate and the global row indices they compute before use; a failed test
 * records MTFM_ERR_BOUNDS in d_meta's header (see mtfm_pack_check) with its site,
 * and skips the access.  mtfm_debug_bounds_build returns 1 in that build, else 0.
 * mtfm_debug_site synchronises `stream` and writes to *site (host) the first failed
 * test's site, file id * 100000 + source line, or 0; d_meta as for mtfm_pack_check. */
int32_t mtfm_debug_bounds_build(void);
mtfm_status mtfm_debug_site(const void* d_meta, int32_t* site, void* stream);

/* Copies the metadata block's arrays into caller host buffers (synchronous;
 * any pointer may be NULL).  seq_off/r_off/t_off are int32 [batch+1],
 * kv_end int32 [total_tokens], row_type uint8 [total_tokens] (0 H, 1 R, 2 T).
 * items_full / items_target receive the work lists as int32 [n][4] rows
 * (user, tile, kv_min, kv_max) and must hold mtfm_max_items(cfg, 0 / 1) rows.
 * For tests and debugging. */
mtfm_status mtfm_meta_read(const mtfm_cfg* cfg, const void* d_meta, int32_t* seq_off,
                           int32_t* r_off, int32_t* t_off, int32_t* kv_end, uint8_t* row_type,
                           int32_t* n_items_full, int32_t* n_items_target, int32_t* items_full,
                           int32_t* items_target, void* stream);

/* Capacity of the Full (is_target = 0) or Target (1) work list: the upper bound
 * sum(ceil(rows_u / 128)) <= ceil(rows / 128) + batch. */
int32_t mtfm_max_items(const mtfm_cfg* cfg, int is_target);

/* ---------------------------------------------------------------------------
 * Full-Attention layer forward ([DY] §4.1): every token of every user is a query.
 *   d_q, d_u : bf16 [total_tokens, hq*head_dim];   d_k, d_v : bf16 [total_tokens, hkv*head_dim]
 *   d_gamma, d_beta : fp32 [3, hq*head_dim] GLN affine rows for H, R, T tokens
 *                     ([MT] §6.1, one [G, D] matrix indexed by token type), or
 *                     both NULL for the plain gate Y = A (*) U.
 *   d_y       : fp32 [total_tokens, hq*head_dim] output Y.
 *   d_a       : fp32 [total_tokens, hq*head_dim] output A (attention before the
 *               gate; saved for the backward pass).  Required.
 *   d_stats   : fp32 [total_tokens, 2] output (mean, rstd) of each row's GLN;
 *               ignored (may be NULL) when d_gamma is NULL.
 * ------------------------------------------------------------------------- */
mtfm_status mtfm_attn_full_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                               const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                               const float* d_gamma, const float* d_beta, float* d_y, float* d_a,
                               float* d_stats, void* stream);

/* Target-Attention layer forward ([DY] §4.2): only T rows query; K/V span the
 * whole sequence of each user.  As mtfm_attn_full_fwd except that d_q, d_u,
 * d_y, d_a are [total_t, hq*head_dim] and d_stats is [total_t, 2]; all rows use
 * the T row of gamma/beta.  H/R rows are not touched (the shortcut of [DY] §4.2). */
mtfm_status mtfm_attn_target_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                 const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                 const float* d_gamma, const float* d_beta, float* d_y,
                                 float* d_a, float* d_stats, void* stream);

/* The same two layer forwards with Y = GLN(A) (*) U ([DY] §4.1, §4.2) stored as bf16
 * (uint16 bit patterns, [rows, hq*head_dim], 16-byte aligned): each element is the
 * fp32 value the fp32 entry point computes, rounded to nearest even.  For a caller whose
 * next step takes Y as a bf16 operand (the output projection f2), at half the bytes; A
 * and d_stats stay fp32 (the backward's saved inputs).  Same arguments, checks and
 * errors as mtfm_attn_full_fwd / mtfm_attn_target_fwd otherwise.  (Storing Y in bf16
 * adds up to half a bf16 ulp per element: against an exact reference, max-abs
 * errors then track the largest |Y| of the batch.) */
mtfm_status mtfm_attn_full_fwd_bf16y(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                     const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                     const float* d_gamma, const float* d_beta, uint16_t* d_y, float* d_a,
                                     float* d_stats, void* stream);
mtfm_status mtfm_attn_target_fwd_bf16y(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                       const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                       const float* d_gamma, const float* d_beta, uint16_t* d_y,
                                       float* d_a, float* d_stats, void* stream);

/* The two halves of a layer forward, for callers that schedule them apart
 * (the layer calls above are exactly attention followed by the gate).
 *   mtfm_attn_full / mtfm_attn_target : writes A only (fp32, shapes as above).
 *   mtfm_gate_fwd : Y = GLN(A) (*) U (plain A (*) U when d_gamma is NULL) for the
 *                   Full (is_target = 0, GLN row picked by token type) or Target
 *                   (is_target = 1, T row of gamma/beta) layout; writes d_y and,
 *                   with GLN, d_stats.  [DY] §4.1 gate; [MT] §6.1 GLN kernel. */
mtfm_status mtfm_attn_full(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                           const uint16_t* d_k, const uint16_t* d_v, float* d_a, void* stream);
mtfm_status mtfm_attn_target(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                             const uint16_t* d_k, const uint16_t* d_v, float* d_a, void* stream);
mtfm_status mtfm_gate_fwd(const mtfm_cfg* cfg, const void* d_meta, int is_target, const float* d_a,
                          const uint16_t* d_u, const float* d_gamma, const float* d_beta,
                          float* d_y, float* d_stats, void* stream);

/* ---------------------------------------------------------------------------
 * Target-Attention forward over a cached key/value prefix: request-level
 * inference where each user's H and R keys/values were computed once and are
 * shared by the candidates (T rows) of later requests ([DY] §5.2.3: M-Falcon
 * micro-batching with a shared KV cache).  The result is exactly the Target layer of mtfm_attn_target_fwd
 * on the sequence [prefix; candidates] of each user (same metadata from mtfm_pack
 * with the prefix's L_H, L_R and the request's L_T = candidates, exposures in
 * t_exp); only the K/V layout differs:
 *   d_k_prefix, d_v_prefix : bf16 [total_tokens - total_t, hkv*head_dim], the H and
 *                            R rows of every user, users back to back in batch order
 *                            (user u's rows start at seq_off[u] - t_off[u]);
 *   d_k_cand, d_v_cand     : bf16 [total_t, hkv*head_dim], the candidates' own keys
 *                            and values (row t_off[u] + t for candidate t of user u);
 *   d_q, d_u, d_y, d_a, d_stats, d_gamma, d_beta : as mtfm_attn_target_fwd.
 * Supported where the tensor-core Target kernel runs (head_dim 64 or 32, hq / hkv
 * in {1, 2, 4, 8}); other shapes return MTFM_ERR_UNSUPPORTED.  mtfm_attn_target_cached
 * writes A only.
 * ------------------------------------------------------------------------- */
mtfm_status mtfm_attn_target_cached_fwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                        const uint16_t* d_k_prefix, const uint16_t* d_v_prefix,
                                        const uint16_t* d_k_cand, const uint16_t* d_v_cand,
                                        const uint16_t* d_u, const float* d_gamma, const float* d_beta,
                                        float* d_y, float* d_a, float* d_stats, void* stream);
mtfm_status mtfm_attn_target_cached(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                    const uint16_t* d_k_prefix, const uint16_t* d_v_prefix,
                                    const uint16_t* d_k_cand, const uint16_t* d_v_cand, float* d_a,
                                    void* stream);

/* ---------------------------------------------------------------------------
 * Backward passes (training step): gradients of the Full-Attention layer
 * ([DY] §4.1) and Target-Attention layer ([DY] §4.2) forward above, the
 * backward half of the Full/Target attention kernels the Meituan tech blog
 * describes in §6.1 (its FA2-derived kernels cover training, forward and
 * backward, with the dynamic mask read and SiLU fused).  With x = alpha q.k,
 * sigma = sigmoid(x) and P = SiLU(x) / N_u on visible pairs:
 *   dU = GLN(A) (*) dY;  dA = GLN backward of dY (*) U;  dgamma, dbeta per type;
 *   dV_j += sum_i P_ij dA_i;  dS_ij = (dA_i . v_j) sigma (1 + x (1 - sigma)) / N_u;
 *   dQ_i = alpha sum_j dS_ij k_j;  dK_j = alpha sum_i dS_ij q_i  (over the r heads
 *   of a KV group for dK, dV).
 * Inputs are the forward's inputs, its saved
 * A (d_a) and stats, and the upstream gradient d_dy (bf16, same shape as Y).
 * Outputs (fp32, fully overwritten):
 *   d_dq, d_du : same rows as Q/U;   d_dk, d_dv : [total_tokens, hkv*head_dim]
 *   d_dgamma, d_dbeta : [3, hq*head_dim] (NULL iff d_gamma is NULL)
 * d_ws is scratch of at least mtfm_bwd_workspace_bytes(cfg, is_target) bytes.
 * ------------------------------------------------------------------------- */
size_t mtfm_bwd_workspace_bytes(const mtfm_cfg* cfg, int is_target);
mtfm_status mtfm_attn_full_bwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                               const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                               const float* d_gamma, const float* d_beta, const float* d_a,
                               const float* d_stats, const uint16_t* d_dy, float* d_dq,
                               float* d_dk, float* d_dv, float* d_du, float* d_dgamma,
                               float* d_dbeta, void* d_ws, size_t ws_bytes, void* stream);
mtfm_status mtfm_attn_target_bwd(const mtfm_cfg* cfg, const void* d_meta, const uint16_t* d_q,
                                 const uint16_t* d_k, const uint16_t* d_v, const uint16_t* d_u,
                                 const float* d_gamma, const float* d_beta, const float* d_a,
                                 const float* d_stats, const uint16_t* d_dy, float* d_dq,
                                 float* d_dk, float* d_dv, float* d_du, float* d_dgamma,
                                 float* d_dbeta, void* d_ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Allocation-free Target-layer backward.  No passage of the pages corresponds
 * to this call: it exists for callers that cannot allocate device memory (code
 * running inside someone else's memory pool or allocator, or a process that
 * reserved all of its device memory up front) and so cannot provide the
 * scratch block mtfm_attn_target_bwd asks for.
 *
 * Same arguments and results as mtfm_attn_target_bwd, minus d_ws / ws_bytes:
 * the scratch is a fixed 24 MiB array inside the library, held on every GPU
 * that loads the library until the process exits.  Returns
 * MTFM_ERR_WORKSPACE_TOO_SMALL, launching nothing, when the problem needs
 * more scratch than that (mtfm_bwd_workspace_bytes(cfg, 1) > 24 MiB; at
 * hq * head_dim = 512 that is about 10,000 T rows).
 *
 * Device memory: the array is committed when the library's module holding it
 * is loaded on a device.  Under CUDA's lazy module loading (the default) that
 * happens during the first call of this entry point on that device, so a
 * caller that reserves the rest of its device memory, or starts a stream
 * capture, afterwards should make one call first; every later call allocates
 * nothing.  Each call looks up the array's device address on the current
 * device, which must be the device of `stream` (MTFM_ERR_INVALID_ARG
 * otherwise).  All calls share the one array: calls whose GPU work can overlap
 * (other streams, or unordered host threads) race on it and must be serialised
 * by the caller.  Its contents are left over from the previous call; none of
 * them is read before this call rewrites it.
 * ------------------------------------------------------------------------- */
mtfm_status mtfm_attn_target_bwd_static(const mtfm_cfg* cfg, const void* d_meta,
                                        const uint16_t* d_q, const uint16_t* d_k,
                                        const uint16_t* d_v, const uint16_t* d_u,
                                        const float* d_gamma, const float* d_beta,
                                        const float* d_a, const float* d_stats,
                                        const uint16_t* d_dy, float* d_dq, float* d_dk,
                                        float* d_dv, float* d_du, float* d_dgamma,
                                        float* d_dbeta, void* stream);

/* ---------------------------------------------------------------------------
 * Backbone stack forward ([DY] §4.1 and §4.2; blocks of one Full-Attention
 * layer followed by Target-Attention layers, [DY] §4.1 and [MT] §3.3).
 * Each layer, on the token matrix X (fp32 [total_tokens, d_model], updated in
 * place):
 *   X~ = RMSNorm(X) * rms_w (eps 1e-6; the pages leave the pre-norm unnamed),
 *   Full  : [U Q K V] = SiLU(X~ W_in^T)            (phi_1 = SiLU, no biases)
 *   Target: [U Q]_T = SiLU(X~_T W_in^T), [K V] = SiLU(X~ W_kv^T)
 *   A = masked SiLU attention (as mtfm_attn_full / mtfm_attn_target),
 *   Y = GLN(A) (*) U (plain A (*) U when gamma is NULL),
 *   Full  : X <- X + Y W_o^T;  Target: X_T <- X_T + Y_T W_o^T, H/R rows unchanged.
 * Precision: X~, U, Q, K, V and Y are rounded to bf16 (round to nearest) as
 * the tensor-core operands; accumulation and X are fp32.
 *
 * mtfm_layer_weights holds device pointers (the struct itself is host memory):
 *   rms_w : fp32 [d_model] RMSNorm weight
 *   w_in  : bf16 [out, d_model] ("out x in", like a linear layer's weight);
 *           Full: out = 2*hq*head_dim + 2*hkv*head_dim, rows ordered U, Q, K, V
 *           (heads contiguous inside each part); Target: out = 2*hq*head_dim (U, Q)
 *   w_kv  : Target only (NULL for Full): bf16 [2*hkv*head_dim, d_model] (K, V)
 *   w_o   : bf16 [d_model, hq*head_dim]
 *   gamma, beta : fp32 [3, hq*head_dim] GLN rows for H, R, T tokens, or both NULL.
 * Shapes: d_model a multiple of 64 and <= 1024; hq*head_dim a multiple of 64.
 * d_ws: scratch of at least mtfm_stack_workspace_bytes(cfg, d_model) bytes,
 * 256-byte aligned, owned by the caller (reused by every layer; its contents
 * are not needed between calls).  mtfm_stack_workspace_bytes returns 0 for an
 * unsupported configuration.
 * mtfm_stack_fwd runs n_layers layers; kinds[l] is 'F' (Full) or 'T' (Target).
 * All layers' arguments are checked before the first launch.
 * ------------------------------------------------------------------------- */
typedef struct mtfm_layer_weights {
  const float* rms_w;
  const uint16_t* w_in;
  const uint16_t* w_kv;
  const uint16_t* w_o;
  const float* gamma;
  const float* beta;
} mtfm_layer_weights;

size_t mtfm_stack_workspace_bytes(const mtfm_cfg* cfg, int32_t d_model);
mtfm_status mtfm_layer_fwd(const mtfm_cfg* cfg, const void* d_meta, int32_t d_model, int is_target,
                           const mtfm_layer_weights* weights, float* d_x, void* d_ws,
                           size_t ws_bytes, void* stream);
mtfm_status mtfm_stack_fwd(const mtfm_cfg* cfg, const void* d_meta, int32_t d_model,
                           int32_t n_layers, const char* kinds, const mtfm_layer_weights* layers,
                           float* d_x, void* d_ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * V2 Target Scale-Up layer forward (Meituan tech blog §3.3.2: each target is 4
 * sub-tokens, items 2-4).  Requires cfg->v2_subtokens = 4 (every user's L_T a
 * multiple of 4; the 4 sub-tokens of a target are consecutive T rows, position
 * s = (T row within the user) mod 4).  On X (fp32 [total_tokens, d_model],
 * updated in place), with X~ = RMSNorm(X) * rms_w (eps 1e-6):
 *   [U Q]_t = SiLU(X~_t W_uq[s]^T)   for each T row t at sub-token position s
 *             (item 2: a Q projection per sub-token position; U comes from the
 *             same query-side projection),
 *   [K V]   = SiLU(X~ W_kv^T)        on all rows,
 *   A       = masked SiLU attention of the Target layer with the V2 mask (the 4
 *             sub-tokens of a target see each other and their shared prefix),
 *   X_T    <- X_T + (GLN(A) (*) U) W_o^T,
 *   X_T    <- Mix(X_T): per target, new sub-token h = [part h of sub-token 0 |
 *             part h of sub-token 1 | ... | part h of sub-token 3], each part
 *             d_model / 4 wide (item 4: the zero-parameter mixing of RankMixer),
 *   X_T    <- X_T + SwiGLU_s(RMSNorm(X_T) * rms_w2) for each T row at position s
 *             (item 2: a SwiGLU FFN per sub-token position):
 *             SwiGLU_s(z) = (SiLU(z W_gate[s]^T) * (z W_up[s]^T)) W_down[s]^T.
 * H / R rows are not touched.  The attention block's parameters are this layer's
 * own, separate from any Full (self-attention) layer's (item 3).
 * Weights (device pointers; the struct is host memory): rms_w, rms_w2 fp32 [d_model];
 * w_uq[s] bf16 [2*hq*head_dim, d_model] (U rows, then Q rows); w_kv bf16
 * [2*hkv*head_dim, d_model]; w_o bf16 [d_model, hq*head_dim]; gamma, beta fp32
 * [3, hq*head_dim] or both NULL; w_gate[s], w_up[s] bf16 [d_ff, d_model];
 * w_down[s] bf16 [d_model, d_ff].
 * Shapes: d_model a multiple of 64, <= 1024; hq*head_dim a multiple of 64; d_ff a
 * multiple of 64.  d_ws: scratch of at least mtfm_v2_workspace_bytes bytes,
 * 256-byte aligned (0 for an unsupported configuration).  Precision as the stack:
 * bf16 tensor-core operands, fp32 accumulation, X fp32.
 * ------------------------------------------------------------------------- */
typedef struct mtfm_v2_layer_weights {
  const float* rms_w;
  const uint16_t* w_uq[4];
  const uint16_t* w_kv;
  const uint16_t* w_o;
  const float* gamma;
  const float* beta;
  const float* rms_w2;
  const uint16_t* w_gate[4];
  const uint16_t* w_up[4];
  const uint16_t* w_down[4];
} mtfm_v2_layer_weights;

size_t mtfm_v2_workspace_bytes(const mtfm_cfg* cfg, int32_t d_model, int32_t d_ff);
mtfm_status mtfm_v2_target_layer_fwd(const mtfm_cfg* cfg, const void* d_meta, int32_t d_model, int32_t d_ff,
                                     const mtfm_v2_layer_weights* weights, float* d_x, void* d_ws,
                                     size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Self-test of failure detection (no counterpart on the pages).  Launches one
 * CTA that waits, with the bounded mbarrier wait every tensor-core kernel of
 * this library uses, on a barrier nothing arrives on; after limit_cycles SM
 * clock cycles (1 .. 4e9; ~1.9e9 per second) it gives up and sets the timeout
 * bit in d_meta's header, as an aborting kernel does.  mtfm_pack_check then
 * returns MTFM_ERR_TIMEOUT and every later kernel on d_meta does nothing until
 * the next mtfm_pack.  Nothing is left in flight; the context stays usable.
 * d_meta: a metadata block written by mtfm_pack (256-byte aligned).
 * ------------------------------------------------------------------------- */
mtfm_status mtfm_selftest_wait_timeout(void* d_meta, int64_t limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MTFM_H_ */
