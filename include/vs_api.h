/*
 * vs_api.h -- C ABI of the B200 (sm_100a) vocabulary-scoring library libvs.so.
 *
 * Per-row scoring of language-model logits over the full vocabulary and over
 * a sampling support, following these pages:
 *
 *  [SkyRL]  SkyRL PR #2004 "perf(sample-support): reuse replay scores for
 *           entropy", section "Implementation": logprobs, optional entropy and
 *           valid-row metadata returned together; entropy conditioned on the
 *           recorded support; a singleton support has exactly zero entropy
 *           and zero entropy gradient; rows without recorded support fall
 *           back to the full-vocabulary logprob and leave the entropy
 *           reduction; entropy computation and gradient tracking are separate
 *           controls; dense support representation.
 *  [xorl]   xorl issue #71 "Consolidate the exact and generic scoring paths;
 *           implement top-k/top-p/min-p", section 3: the transform program
 *           (temperature, then stable token-id top-k, then inclusive top-p,
 *           then min-p relative to the original row max; top_p == 1 is the
 *           identity) and section 1: chunked projection, fixed-order LSE,
 *           support, selected logprob and VJP.
 *  [DSpark] DeepSpec PR #87 "[Perf] Reuse DSpark probability distance across
 *           loss and metrics", section "Purpose": per-token L1 distance
 *           between softmax(draft) and softmax(target), accept_rate =
 *           clamp(1 - 0.5 L1, 0, 1), weighted L1 loss.
 *
 * Notation: row i has logits l[i, 0..V-1] and temperature T_i; z = l / T_i;
 * p = softmax(z) over the vocabulary; S = support; q = softmax(z on S).
 *
 * Conventions for every entry point
 *  - All array pointers are DEVICE pointers owned by the caller.  The library
 *    allocates no device memory; where scratch is needed the caller passes a
 *    workspace sized by the matching *_workspace_size query.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous: they enqueue kernels and return.
 *  - Every call returns a vs_status.  Argument errors are detected on the
 *    host before anything is enqueued (VS_ERR_INVALID_ARG /
 *    VS_ERR_UNSUPPORTED / VS_ERR_WORKSPACE); a failed launch returns
 *    VS_ERR_CUDA.  vs_last_error() then describes the failure (thread-local
 *    string, valid until the next call on the same thread).  Nothing is
 *    thrown across the ABI and nothing traps on the device.
 *  - Problems in the data of one row (bad target, bad support id, non-finite
 *    logits) never fail the call: they are reported in that row's status word
 *    (VS_ROW_* bits) and the row's outputs follow the rules stated below.
 *  - Logits are row-major [rows, ld] with ld >= vocab.  The logits pointer
 *    must be 16-byte aligned and ld * sizeof(element) a multiple of 16
 *    (elements beyond `vocab` in each row are never used).
 */
#ifndef VS_API_H
#define VS_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t vs_status;
#define VS_OK 0
#define VS_ERR_INVALID_ARG 1
#define VS_ERR_UNSUPPORTED 2
#define VS_ERR_WORKSPACE 3
#define VS_ERR_CUDA 4

typedef int32_t vs_dtype;
#define VS_F32 0
#define VS_BF16 1

/* vs_score_args.flags */
#define VS_WANT_ENTROPY (1u << 0)      /* write entropy_full / entropy_support */
#define VS_WANT_SUPPORT_MASK (1u << 1) /* write the support_mask bitset */
#define VS_WANT_GRAD (1u << 2)         /* write ctx for vs_score_bwd */
#define VS_WANT_SAMPLE (1u << 3)       /* write sampled: a seeded Gumbel-max token from S */

/* per-row status bits (vs_score_out.status) */
#define VS_ROW_TARGET_OUT_OF_RANGE (1u << 0)   /* target outside [0, vocab): logprobs NaN */
#define VS_ROW_TARGET_NOT_IN_SUPPORT (1u << 1) /* non-empty S without y: lp_S = -inf */
#define VS_ROW_BAD_SUPPORT_ID (1u << 2)        /* a recorded id < -1 or >= vocab: ignored */
#define VS_ROW_DUP_SUPPORT_ID (1u << 3)        /* a recorded id repeated: counted once */
#define VS_ROW_NONFINITE_INPUT (1u << 4)       /* NaN/inf logit: outputs NaN, valid 0 */
#define VS_ROW_DEVICE_TIMEOUT (1u << 5)        /* a bounded device wait gave up: outputs unreliable */
#define VS_ROW_EMPTY_SUPPORT (1u << 6)         /* vs_support_lmhead_score: no kept id, lp_S NaN */

/* bytes of saved state per row written when VS_WANT_GRAD is set */
#define VS_CTX_BYTES_PER_ROW 64

/* maximum recorded-support width and fused-head top-k */
#define VS_MAX_SUPPORT_WIDTH 1024
#define VS_MAX_FUSED_TOPK 64

/* Arguments shared by vs_score_fwd and vs_score_bwd. */
typedef struct vs_score_args {
  int32_t rows;        /* R >= 0 */
  int32_t vocab;       /* V >= 1 */
  int64_t ld;          /* row stride of logits, in elements, >= V */
  vs_dtype dtype;      /* VS_BF16 or VS_F32 */
  const void* logits;  /* [R, ld] */
  /* per-row temperature [R] (> 0, finite), or NULL to use temperature_scalar */
  const float* temperature;
  float temperature_scalar;
  const int32_t* targets; /* [R] selected token ids y_i */
  /* computed support ([xorl] section 3); per-row arrays or NULL + scalar.
   * A filter is disabled by top_k <= 0 or >= V, top_p >= 1, min_p <= 0.
   * top_p must lie in (0, 1], min_p in [0, 1). */
  const int32_t* top_k;
  int32_t top_k_scalar;
  const float* top_p;
  float top_p_scalar;
  const float* min_p;
  float min_p_scalar;
  /* recorded support ([SkyRL]): [R, support_ld] int32 ids, the first
   * support_width of each row used, -1 = padding anywhere in the row.
   * NULL selects the computed support.  Giving a recorded support together
   * with an active filter is VS_ERR_INVALID_ARG. */
  const int32_t* support_ids;
  int32_t support_width; /* 0 .. VS_MAX_SUPPORT_WIDTH */
  int64_t support_ld;    /* >= support_width */
  uint32_t flags;        /* VS_WANT_* */
  /* seed of the Gumbel noise (VS_WANT_SAMPLE): row i of a call draws from
   * the Philox4x64-10 stream keyed by (sample_seed, i) */
  uint64_t sample_seed;
} vs_score_args;

/* Outputs of vs_score_fwd.  Every pointer may be NULL (that output is not
 * written) unless a flag requires it. */
typedef struct vs_score_out {
  float* logprob_full;    /* [R] lp_V = z_y - logsumexp(z) */
  float* logprob_support; /* [R] lp_S = z_y - logsumexp(z on S); lp_V if S is empty;
                             -inf if y is not in a non-empty S */
  float* entropy_full;    /* [R] H_V (needs VS_WANT_ENTROPY) */
  float* entropy_support; /* [R] H_S, 0 for an empty S (needs VS_WANT_ENTROPY) */
  uint8_t* valid;         /* [R] 1 iff S is non-empty and the row is finite */
  uint32_t* status;       /* [R] VS_ROW_* bits */
  int32_t* support_size;  /* [R] |S| */
  uint32_t* support_mask; /* [R, ceil(V/32)] bit j%32 of word j/32 set iff j in S
                             (needs VS_WANT_SUPPORT_MASK) */
  void* ctx;              /* [R, VS_CTX_BYTES_PER_ROW] saved state (needs VS_WANT_GRAD),
                             16-byte aligned; opaque, pass unchanged to vs_score_bwd */
  double* entropy_sum;    /* [1] sum over valid rows of H_S (needs VS_WANT_ENTROPY) */
  int32_t* valid_count;   /* [1] number of valid rows */
  /* [R] (needs VS_WANT_SAMPLE; [xorl] section 3, the program's final
   * "seeded gumbel" step, here): argmax over j in S of fl32(l_j / T) + G_j,
   * the smallest j on equal scores, -1 for an empty S or a non-finite row.
   * G_j = -log(-log U_j), U_j = (bits 63..40 of r + 1/2) 2^-24, r = word
   * (j mod 4) of Philox4x64-10(counter = (floor(j / 4), 0, 0, 0),
   * key = (sample_seed, i)); every step one IEEE fp32 round-to-nearest
   * operation (the logarithm by a fixed reduction and series), so the
   * token is reproducible bit for bit. */
  int32_t* sampled;
} vs_score_out;

/* Forward scoring ([SkyRL] Implementation; [xorl] sections 1 and 3).
 *
 * Computed support (support_ids == NULL): S = min-p(top-p(top-k(row))) in
 * the total order (z descending, token id ascending): top-k keeps the first
 * k; top-p keeps the shortest prefix of that set whose probability, renormalised
 * over the top-k set, is >= top_p (the crossing token is kept); min-p keeps
 * tokens with p_j >= min_p * max_j p_j.  With no active filter S is the whole
 * vocabulary.  Full-vocabulary statistics are always computed.
 *
 * Recorded support: S = the distinct ids >= 0 among the first support_width
 * entries of the row.  Full-vocabulary statistics (and hence a full read of
 * the row) are computed for every row when logprob_full or entropy_full is
 * requested, else only for rows whose S is empty (the lp_V fallback).
 *
 * Workspace: none for computed supports and for recorded lists wider than
 * 64 ids (pass NULL, 0).  Recorded lists of up to 64 ids need
 * vs_score_fwd_workspace_size(args) bytes, 16-byte aligned, owned by the
 * caller and not shared by calls that may run at the same time: it holds
 * the list of rows that need full-vocabulary statistics and one partial
 * per (row, chunk) of them (4,096 ids for bf16, 2,048 for fp32), so that
 * those rows' reads spread over every SM.  VS_ERR_WORKSPACE when it is
 * missing, misaligned or too small.
 *
 * Returns VS_ERR_INVALID_ARG for NULL required pointers, R < 0, V < 1,
 * ld < V, bad alignment, a non-positive or non-finite temperature_scalar,
 * top_p_scalar outside (0, 1], min_p_scalar outside [0, 1), a flag whose
 * output pointer is NULL; VS_ERR_UNSUPPORTED for V beyond the resident-row
 * limit (vs_score_max_vocab) or support_width > VS_MAX_SUPPORT_WIDTH.
 * Per-row arrays (temperature, top_k, top_p, min_p) are not range-checked on
 * the host; out-of-range entries behave as documented for the scalars' edges
 * (top_p >= 1 disables, min_p <= 0 disables, a temperature <= 0 gives NaN). */
vs_status vs_score_fwd(const vs_score_args* args, const vs_score_out* out, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Workspace bytes vs_score_fwd needs for these arguments: 0 for computed
 * supports and recorded lists wider than 64 ids; for narrower recorded
 * lists 16 + 2 r16(4 rows) + r16(20 rows ceil(vocab / chunk)), chunk =
 * 4,096 (bf16) or 2,048 (fp32), r16 rounding up to a multiple of 16. */
size_t vs_score_fwd_workspace_size(const vs_score_args* args);

/* Largest vocabulary vs_score_fwd accepts for a dtype. */
int32_t vs_score_max_vocab(vs_dtype dtype);

/* dlogits modes for vs_score_bwd */
#define VS_GRAD_DENSE 0      /* dlogits [R, V] (row stride grad_ld) overwritten */
#define VS_GRAD_ACCUMULATE 1 /* dlogits [R, V] += gradient */
#define VS_GRAD_SPARSE 2     /* recorded support only: dlogits [R, support_width] fp32,
                                the gradient at each listed id (0 at pads, bad ids and
                                repeats); valid only when no full-vocabulary term
                                (g_lp_full, g_h_full, or an empty-support row's g_lp_support)
                                is non-zero */

/* Backward of the forward outputs ([xorl] section 1 "selected logprob + VJP";
 * [SkyRL] Implementation).  With g_* the upstream gradients of lp_V, lp_S,
 * H_V, H_S (each [R] fp32 or NULL = 0), and 1_S the support indicator:
 *
 *   dl_j = (1/T) * ( g_lpV ([j==y] - p_j) + g_lpS 1_S(j) ([j==y] - q_j)
 *                   - g_HV p_j (log p_j + H_V) - g_HS 1_S(j) q_j (log q_j + H_S) )
 *
 * Empty S: lp_S is lp_V, so g_lpS joins the full-vocabulary term; H_S has no
 * gradient.  y outside a non-empty S, an out-of-range y, or a non-finite row:
 * no logprob gradient (and no gradient at all for a non-finite row).
 * `args` must be the arguments of the forward call and `ctx` its saved state.
 * dlogits has dtype dl_dtype (VS_F32 or VS_BF16, rounded to nearest even),
 * row stride grad_ld elements (>= V in the dense modes, >= support_width in
 * the sparse mode), 16-byte aligned with grad_ld * sizeof a multiple of 16. */
vs_status vs_score_bwd(const vs_score_args* args, const void* ctx, const float* g_lp_full,
                       const float* g_lp_support, const float* g_h_full,
                       const float* g_h_support, void* dlogits, vs_dtype dl_dtype,
                       int64_t grad_ld, int32_t mode, void* stream);

/* Draft/target probability distance ([DSpark] Purpose).  Per row i:
 *   p = softmax(draft_i), q = softmax(target_i)          (no temperature)
 *   l1[i] = sum_j |p_j - q_j|
 *   accept_rate[i] = clamp(1 - 0.5 * l1[i], 0, 1)
 *   loss_num_den_loss[0..2] = { sum_i w_i l1_i, sum_i w_i, num / den (0 if den == 0) }
 * with w = row_weight (NULL = all ones).  When grad_draft is non-NULL it
 * receives d loss / d draft (target detached):
 *   (w_i / sum w) p_j (s_j - sum_k p_k s_k),  s = sign(p - q), sign(0) = 0.
 * Any of l1, accept_rate, loss_num_den_loss, grad_draft may be NULL.
 * draft and target are [rows, ld] of `dtype`; grad_draft is [rows, grad_ld]
 * of grad_dtype.  Needs a workspace of vs_l1_distance_workspace_size(rows)
 * bytes (16-byte aligned) when loss_num_den_loss or grad_draft is requested. */
vs_status vs_l1_distance(int32_t rows, int32_t vocab, int64_t ld, vs_dtype dtype,
                         const void* draft, const void* target, const float* row_weight,
                         float* l1, float* accept_rate, float* loss_num_den_loss,
                         void* grad_draft, vs_dtype grad_dtype, int64_t grad_ld,
                         void* workspace, size_t workspace_bytes, void* stream);

size_t vs_l1_distance_workspace_size(int32_t rows);

/* vs_l1_distance for a batch whose rows are split across ranks (data
 * parallelism; [DSpark] Purpose keeps the distributed normalisation of the
 * weighted loss: loss = sum over all ranks of w_i L1_i / sum over all ranks
 * of w_i).  global_weight_sum is a DEVICE pointer to one double: the sum of
 * the row weights over every rank (for example the all-reduce of each
 * rank's weight sum; rows with row_weight NULL weigh 1).  Outputs as in
 * vs_l1_distance, except:
 *  - grad_draft uses the global denominator:
 *      (w_i / global_weight_sum) p_j (s_j - sum_k p_k s_k);
 *  - loss_num_den_loss = { this call's sum w_i L1_i, this call's sum w_i,
 *      this call's sum w_i L1_i / global_weight_sum } (0 if the global sum is
 *      0), so the third entries of all ranks add up to the batch loss and the
 *      first two all-reduce to its numerator and denominator.
 * The same workspace rules as vs_l1_distance apply.  VS_ERR_INVALID_ARG when
 * global_weight_sum is NULL or not 8-byte aligned.  The library performs no
 * collective: the caller reduces the scalars. */
/* Sum of this shard's row weights in fp64, accumulated in a fixed order,
 * written to the DEVICE double *out (rows with row_weight NULL weigh 1, so
 * the sum is rows).  The first step of the row-sharded loss: all-reduce it
 * over the ranks and pass the result to vs_l1_distance_sharded.
 * VS_ERR_INVALID_ARG when rows < 0 or out is NULL or not 8-byte aligned. */
vs_status vs_l1_weight_sum(int32_t rows, const float* row_weight, double* out, void* stream);

vs_status vs_l1_distance_sharded(int32_t rows, int32_t vocab, int64_t ld, vs_dtype dtype,
                                 const void* draft, const void* target, const float* row_weight,
                                 const double* global_weight_sum, float* l1, float* accept_rate,
                                 float* loss_num_den_loss, void* grad_draft, vs_dtype grad_dtype,
                                 int64_t grad_ld, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* vs_l1_distance without a caller workspace.  The pages have no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc -- for
 * example a plugin inside a host application whose device memory pool it
 * cannot reach, or a serving loop that must not allocate after start-up
 * because cudaMalloc may synchronise the device.  Arguments and results are
 * those of vs_l1_distance; the scratch comes from a file-scope device array
 * of VS_L1_STATIC_SCRATCH_BYTES inside libvs.so, which every GPU that loads
 * the library holds until the process exits.  Nothing is allocated.
 *  - rows above VS_L1_STATIC_MAX_ROWS: VS_ERR_UNSUPPORTED, nothing enqueued.
 *  - The first call on a device, with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress) and caches it; make that
 *    first call before any stream capture.  The cached address belongs to
 *    the device's context at that time and does not survive a
 *    cudaDeviceReset of that device (the module is unloaded and the array
 *    may sit elsewhere once it is loaded again): a caller that resets a
 *    device must not call this entry point on it afterwards in the same
 *    process.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents (each call overwrites what it reads), so calls that overlap on
 *    the GPU (concurrent streams, or threads without ordering) race. */
#define VS_L1_STATIC_MAX_ROWS 65536
#define VS_L1_STATIC_SCRATCH_BYTES (16 + 8 * VS_L1_STATIC_MAX_ROWS)
vs_status vs_l1_distance_static(int32_t rows, int32_t vocab, int64_t ld, vs_dtype dtype,
                                const void* draft, const void* target, const float* row_weight,
                                float* l1, float* accept_rate, float* loss_num_den_loss,
                                void* grad_draft, vs_dtype grad_dtype, int64_t grad_ld,
                                void* stream);

/* Fused LM-head scoring ([xorl] section 1: chunked projection -> fixed-order
 * LSE -> support -> selected logprob; [SkyRL] Performance: the full logits
 * are never materialised).
 *   z[i, v] = (sum_k hidden[i, k] * weight[v, k]) / T_i
 * computed on tcgen05 tensor cores (bf16 inputs, fp32 accumulation) tile by
 * tile; each tile updates per-row online (max, sum exp, sum z exp) and a
 * per-row top-k candidate list; a merge step then forms S = min-p(top-p(
 * top-k)) over the k candidates and writes lp_V, lp_S, H_V, H_S (entropy
 * outputs need VS_WANT_ENTROPY), valid, status, support_size, and, when
 * non-NULL, topk_ids [rows, top_k] (the top-k token ids in the total order)
 * and topk_logprob [rows, top_k] (their full-vocabulary logprobs).
 * hidden [rows, hidden_dim] and weight [vocab, hidden_dim] are bf16, K-major,
 * row strides ldh/ldw elements (multiples of 8), 16-byte aligned; hidden_dim
 * a multiple of 64.  top_k in [1, VS_MAX_FUSED_TOPK] (top-p without top-k is
 * not offered here).  out->support_mask and sampled must be NULL (and
 * VS_WANT_SAMPLE unset).  With VS_WANT_GRAD, out->ctx receives
 * [rows, VS_CTX_BYTES_PER_ROW] bytes of saved state (16-byte aligned) for
 * vs_fused_lmhead_bwd, which also needs topk_ids (the support is its first
 * support_size entries); VS_WANT_GRAD and ctx go together and need topk_ids.
 * Needs vs_fused_lmhead_workspace_size(...) bytes. */
vs_status vs_fused_lmhead_score(int32_t rows, int32_t vocab, int32_t hidden_dim,
                                const void* hidden, int64_t ldh, const void* weight,
                                int64_t ldw, const float* temperature,
                                float temperature_scalar, const int32_t* targets,
                                int32_t top_k, float top_p, float min_p, uint32_t flags,
                                const vs_score_out* out, int32_t* topk_ids,
                                float* topk_logprob, void* workspace, size_t workspace_bytes,
                                void* stream);

size_t vs_fused_lmhead_workspace_size(int32_t rows, int32_t vocab, int32_t hidden_dim,
                                      int32_t top_k);

/* Backward of vs_fused_lmhead_score ([xorl] section 1: "selected logprob +
 * VJP"; the logits are recomputed, never stored whole).  With x = H W^T,
 * z = x / T and the upstream gradients g_* of lp_V, lp_S, H_V, H_S ([R] fp32
 * each, NULL = 0), the logit gradient is
 *   dx_j = (1/T) ( g_lpV ([j==y] - p_j) + g_lpS 1_S(j) ([j==y] - q_j)
 *                 - g_HV p_j (log p_j + H_V) - g_HS 1_S(j) q_j (log q_j + H_S) )
 * (the rules of vs_score_bwd for empty supports, targets outside S or
 * outside [0, V), and non-finite rows), and
 *   d_hidden [rows, hidden_dim] = dx W        (fp32, row stride ld_dh),
 *   d_weight [vocab, hidden_dim] = dx^T H     (fp32, row stride ld_dw);
 * either may be NULL (not computed).  Both are overwritten.  The logit tiles
 * are recomputed on the tensor cores chunk by chunk of the vocabulary, dx is
 * formed in the GEMM epilogue and rounded to bf16 (the support and target
 * entries are recomputed and written whole), and the two products run as
 * plain bf16 GEMMs with fp32 accumulation (cuBLASLt, inside the caller's
 * workspace).  hidden, weight, targets and top_k are those of the forward
 * call; ctx and topk_ids its outputs (VS_WANT_GRAD).  Output pointers 16-byte
 * aligned, ld_dh / ld_dw >= hidden_dim and multiples of 4.  Needs
 * vs_fused_lmhead_bwd_workspace_size(rows, vocab, hidden_dim) bytes (a bf16
 * [rows, 32768] gradient chunk plus 32 MiB).  Errors as for
 * vs_fused_lmhead_score. */
vs_status vs_fused_lmhead_bwd(int32_t rows, int32_t vocab, int32_t hidden_dim, const void* hidden,
                              int64_t ldh, const void* weight, int64_t ldw,
                              const int32_t* targets, int32_t top_k, const void* ctx,
                              const int32_t* topk_ids, const float* g_lp_full,
                              const float* g_lp_support, const float* g_h_full,
                              const float* g_h_support, float* d_hidden, int64_t ld_dh,
                              float* d_weight, int64_t ld_dw, void* workspace,
                              size_t workspace_bytes, void* stream);

size_t vs_fused_lmhead_bwd_workspace_size(int32_t rows, int32_t vocab, int32_t hidden_dim);

/* Vocabulary-parallel fused head (tensor parallelism over the vocabulary:
 * [SkyRL] Implementation shares the tensor-parallel reduction of the replay
 * logprob; [xorl] section 3 names a vocabulary-sharded LM-head group).  Each
 * rank holds weight rows [vocab_begin, vocab_begin + vocab_count) of a
 * vocab_total-row head and the full hidden states.
 *
 * Step 1, vs_fused_lmhead_partial: this shard's projection with the scoring
 * epilogue, reduced to ONE partial record per row in `partial` (16-byte
 * aligned, vs_fused_lmhead_partial_bytes(rows, top_k) bytes; the layout is
 * opaque and the same on every rank): the shard's online statistics
 * (max, count of max, sum 2^(u - max), sum (u - max) 2^(u - max) in base-2
 * units u = z log2 e), its top_k (logit, vocabulary id) candidates in the
 * total order, the target's logit when the shard holds the target (else 0),
 * and a timeout flag.  Needs vs_fused_lmhead_partial_workspace_size(rows,
 * vocab_count, hidden_dim, top_k) bytes of workspace.
 *
 * The exchange (the caller's): gather every rank's block into one buffer of
 * n_shards consecutive blocks, in the order of the shards' vocab_begin (an
 * all-gather of the bytes).
 *
 * Step 2, vs_fused_lmhead_merge: merges the n_shards blocks (statistics in
 * shard order, k-way merge of the candidate lists, the target logit) and
 * writes exactly the outputs of vs_fused_lmhead_score for the whole
 * vocabulary (top-k, then inclusive top-p on the top-k mass, then min-p
 * against the row max): lp_V, lp_S, H_V, H_S, valid, status, support_size,
 * topk_ids, topk_logprob.  Every rank that merges gets the same outputs.
 * out->support_mask, ctx and sampled must be NULL.  The full logits are
 * never materialised and only (16 + 8 top_k + 4) bytes per row cross the
 * ranks.  Errors as for vs_fused_lmhead_score; n_shards in [1, 64]. */
size_t vs_fused_lmhead_partial_bytes(int32_t rows, int32_t top_k);
size_t vs_fused_lmhead_partial_workspace_size(int32_t rows, int32_t vocab_count,
                                              int32_t hidden_dim, int32_t top_k);
vs_status vs_fused_lmhead_partial(int32_t rows, int32_t vocab_total, int32_t vocab_begin,
                                  int32_t vocab_count, int32_t hidden_dim, const void* hidden,
                                  int64_t ldh, const void* weight_shard, int64_t ldw,
                                  const float* temperature, float temperature_scalar,
                                  const int32_t* targets, int32_t top_k, void* partial,
                                  void* workspace, size_t workspace_bytes, void* stream);
vs_status vs_fused_lmhead_merge(int32_t rows, int32_t vocab_total, int32_t n_shards,
                                const void* partials, const float* temperature,
                                float temperature_scalar, const int32_t* targets, int32_t top_k,
                                float top_p, float min_p, uint32_t flags,
                                const vs_score_out* out, int32_t* topk_ids, float* topk_logprob,
                                void* stream);

/* Support-only fused projection ([SkyRL] Performance: with a fused LM head
 * the replay path projects only the selected hidden-state / weight pairs and
 * never materialises vocabulary logits; Implementation: dense -1-padded
 * support lists).  For row i and each kept id s of support_ids[i, :width]
 * (0 <= s < vocab, first occurrence; -1 pads anywhere are skipped, other
 * out-of-range ids set VS_ROW_BAD_SUPPORT_ID, repeats VS_ROW_DUP_SUPPORT_ID):
 *   z[i, s] = (sum_k hidden[i, k] * weight[s, k]) / T_i
 * (bf16 inputs, fp32 accumulation), then over the kept set S_i:
 * logprob_support = z_y - log sum_S exp z (-inf and
 * VS_ROW_TARGET_NOT_IN_SUPPORT when y is not kept), entropy_support =
 * -sum_S q log q (exactly 0 for a singleton; needs VS_WANT_ENTROPY), valid,
 * status and support_size, as vs_score_fwd gives them for a recorded
 * support.  The work scales with the support width, not with vocab.
 * A row with no kept id has no full-vocabulary fallback here (it needs the
 * full projection, vs_fused_lmhead_score): logprob_support NaN, entropy 0,
 * valid 0, status VS_ROW_EMPTY_SUPPORT.  Non-finite projections: outputs NaN,
 * valid 0, VS_ROW_NONFINITE_INPUT.
 * hidden [rows, hidden_dim] (row stride ldh) and weight [vocab, hidden_dim]
 * (row stride ldw) are bf16, 16-byte aligned, strides multiples of 8;
 * hidden_dim a multiple of 8, at most 16384.  support_ids [rows, support_ld]
 * int32, width in [0, VS_MAX_SUPPORT_WIDTH].  out->logprob_full,
 * entropy_full, support_mask, ctx and sampled must be NULL
 * (VS_ERR_INVALID_ARG).  When
 * support_logits is non-NULL it receives [rows, logits_ld] fp32: z[i, s] at
 * each kept slot, -inf at pads, bad and repeated ids.  No workspace. */
vs_status vs_support_lmhead_score(int32_t rows, int32_t vocab, int32_t hidden_dim,
                                  const void* hidden, int64_t ldh, const void* weight,
                                  int64_t ldw, const float* temperature, float temperature_scalar,
                                  const int32_t* targets, const int32_t* support_ids,
                                  int32_t support_width, int64_t support_ld, uint32_t flags,
                                  const vs_score_out* out, float* support_logits,
                                  int64_t logits_ld, void* stream);

/* Message describing the last failed call on this thread ("" after success). */
const char* vs_last_error(void);

/* Library version, e.g. "0.1.0". */
const char* vs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VS_API_H */
