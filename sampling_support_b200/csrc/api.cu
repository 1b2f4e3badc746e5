// C ABI of libvs.so: argument validation, launch configuration, error text.
// Every check runs on the host before anything is enqueued; nothing here
// allocates device memory.

#include <cmath>
#include <cstdio>
#include <string>

#include "internal.h"

namespace vs {
size_t l1_workspace_bytes(int rows);
int l1_max_vocab(vs_dtype dtype);
cudaError_t launch_l1(int rows, int vocab, int64_t ld, vs_dtype dtype, const void* draft,
                      const void* target, const float* row_weight, float* l1, float* accept,
                      float* loss3, void* grad, vs_dtype gdtype, int64_t grad_ld, void* ws,
                      const double* global_wsum, cudaStream_t s);
cudaError_t launch_l1_weight_sum(int rows, const float* row_weight, double* out, cudaStream_t s);
size_t lmhead_workspace_bytes(int rows, int vocab, int hidden, int top_k);
vs_status lmhead_run(int rows, int vocab, int hidden, const void* H, int64_t ldh, const void* W,
                     int64_t ldw, const float* temperature, float temperature_scalar,
                     const int32_t* targets, int top_k, float top_p, float min_p,
                     uint32_t flags, const vs_score_out* out, int32_t* topk_ids,
                     float* topk_logprob, void* ws, size_t ws_bytes, cudaStream_t s,
                     std::string* err);
size_t lmhead_bwd_workspace_bytes(int rows, int vocab, int hidden);
size_t lmhead_partial_bytes(int rows, int top_k);
vs_status lmhead_partial_run(int rows, int vocab_total, int vocab_begin, int vocab_count,
                             int hidden, const void* H, int64_t ldh, const void* W, int64_t ldw,
                             const float* temperature, float temperature_scalar,
                             const int32_t* targets, int top_k, void* partial, void* ws,
                             size_t ws_bytes, cudaStream_t s, std::string* err);
vs_status lmhead_merge_run(int rows, int vocab_total, int n_shards, const void* partials,
                           const float* temperature, float temperature_scalar,
                           const int32_t* targets, int top_k, float top_p, float min_p,
                           uint32_t flags, const vs_score_out* out, int32_t* topk_ids,
                           float* topk_logprob, cudaStream_t s, std::string* err);
vs_status lmhead_bwd_run(int rows, int vocab, int hidden, const void* H, int64_t ldh,
                         const void* W, int64_t ldw, const int32_t* targets, int top_k,
                         const void* ctx, const int32_t* topk_ids, const float* g_lp_full,
                         const float* g_lp_support, const float* g_h_full,
                         const float* g_h_support, float* d_hidden, int64_t ld_dh,
                         float* d_weight, int64_t ld_dw, void* ws, size_t ws_bytes,
                         cudaStream_t s, std::string* err);
vs_status support_head_run(int rows, int vocab, int hidden, const void* H, int64_t ldh,
                           const void* W, int64_t ldw, const float* temperature,
                           float temperature_scalar, const int32_t* targets,
                           const int32_t* support_ids, int width, int64_t support_ld,
                           uint32_t flags, const vs_score_out* out, float* support_logits,
                           int64_t logits_ld, cudaStream_t s, std::string* err);
}  // namespace vs

namespace {

thread_local std::string g_err;

vs_status fail(vs_status code, const std::string& msg) {
  g_err = msg;
  return code;
}

vs_status ok() {
  g_err.clear();
  return VS_OK;
}

vs_status cuda_fail(cudaError_t e, const char* where) {
  return fail(VS_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t esize(vs_dtype d) { return d == VS_BF16 ? 2 : 4; }

bool filters_active(const vs_score_args* a) {
  if (a->top_k || a->top_p || a->min_p) return true;
  if (a->top_k_scalar > 0 && a->top_k_scalar < a->vocab) return true;
  if (a->top_p_scalar < 1.f) return true;
  if (a->min_p_scalar > 0.f) return true;
  return false;
}

// Checks shared by the forward and backward calls.
vs_status check_args(const vs_score_args* a) {
  if (!a) return fail(VS_ERR_INVALID_ARG, "args is NULL");
  if (a->rows < 0) return fail(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (a->vocab < 1) return fail(VS_ERR_INVALID_ARG, "vocab must be >= 1");
  if (a->ld < a->vocab) return fail(VS_ERR_INVALID_ARG, "ld must be >= vocab");
  if (a->dtype != VS_BF16 && a->dtype != VS_F32)
    return fail(VS_ERR_INVALID_ARG, "dtype must be VS_BF16 or VS_F32");
  if (a->rows == 0) return VS_OK;
  if (!a->logits) return fail(VS_ERR_INVALID_ARG, "logits is NULL");
  if (!aligned16(a->logits)) return fail(VS_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  if ((static_cast<uint64_t>(a->ld) * esize(a->dtype)) % 16 != 0)
    return fail(VS_ERR_INVALID_ARG, "ld * sizeof(element) must be a multiple of 16 bytes");
  if (!a->targets) return fail(VS_ERR_INVALID_ARG, "targets is NULL");
  if (!a->temperature &&
      !(std::isfinite(a->temperature_scalar) && a->temperature_scalar > 0.f))
    return fail(VS_ERR_INVALID_ARG, "temperature_scalar must be finite and > 0");
  if (!a->top_p && !(a->top_p_scalar > 0.f && a->top_p_scalar <= 1.f))
    return fail(VS_ERR_INVALID_ARG, "top_p_scalar must lie in (0, 1]");
  if (!a->min_p && !(a->min_p_scalar >= 0.f && a->min_p_scalar < 1.f))
    return fail(VS_ERR_INVALID_ARG, "min_p_scalar must lie in [0, 1)");
  if (a->support_ids) {
    if (a->support_width < 0 || a->support_width > VS_MAX_SUPPORT_WIDTH)
      return fail(VS_ERR_UNSUPPORTED, "support_width must lie in [0, VS_MAX_SUPPORT_WIDTH]");
    if (a->support_ld < a->support_width)
      return fail(VS_ERR_INVALID_ARG, "support_ld must be >= support_width");
    if (filters_active(a))
      return fail(VS_ERR_INVALID_ARG,
                  "a recorded support cannot be combined with top-k/top-p/min-p filters");
  }
  return VS_OK;
}

}  // namespace

namespace vs {
// Record the outcome of a C-ABI call made from another translation unit.
vs_status set_last_error(vs_status code, const char* msg) {
  if (code == VS_OK)
    g_err.clear();
  else
    g_err = msg;
  return code;
}
}  // namespace vs

extern "C" {

const char* vs_last_error(void) { return g_err.c_str(); }

const char* vs_version(void) { return "0.1.0"; }

int32_t vs_score_max_vocab(vs_dtype dtype) {
  if (dtype != VS_BF16 && dtype != VS_F32) return 0;
  return vs::score_max_vocab(dtype);
}

size_t vs_score_fwd_workspace_size(const vs_score_args* args) {
  if (!args || !args->support_ids || args->rows <= 0 || args->vocab <= 0) return 0;
  return vs::score_recorded_workspace_bytes(args->rows, args->vocab, args->support_width, args->dtype);
}

vs_status vs_score_fwd(const vs_score_args* a, const vs_score_out* o, void* workspace,
                       size_t workspace_bytes, void* stream) {
  vs_status st = check_args(a);
  if (st != VS_OK) return st;
  if (!o) return fail(VS_ERR_INVALID_ARG, "out is NULL");
  if (a->rows == 0) return ok();
  const bool want_entropy = a->flags & VS_WANT_ENTROPY;
  if ((a->flags & VS_WANT_SUPPORT_MASK) && !o->support_mask)
    return fail(VS_ERR_INVALID_ARG, "VS_WANT_SUPPORT_MASK needs support_mask");
  if ((a->flags & VS_WANT_GRAD) && !o->ctx)
    return fail(VS_ERR_INVALID_ARG, "VS_WANT_GRAD needs ctx");
  if (((a->flags & VS_WANT_SAMPLE) != 0) != (o->sampled != nullptr))
    return fail(VS_ERR_INVALID_ARG, "VS_WANT_SAMPLE and sampled go together");
  if (o->ctx && !aligned16(o->ctx)) return fail(VS_ERR_INVALID_ARG, "ctx must be 16-byte aligned");
  if (want_entropy && !o->entropy_full && !o->entropy_support)
    return fail(VS_ERR_INVALID_ARG, "VS_WANT_ENTROPY needs entropy_full or entropy_support");
  if (!want_entropy && (o->entropy_full || o->entropy_support || o->entropy_sum))
    return fail(VS_ERR_INVALID_ARG, "entropy outputs need VS_WANT_ENTROPY");
  if (o->entropy_sum && !o->entropy_support)
    return fail(VS_ERR_INVALID_ARG, "entropy_sum needs entropy_support");
  if ((o->entropy_sum || o->valid_count) && !o->valid)
    return fail(VS_ERR_INVALID_ARG, "entropy_sum / valid_count need valid");
  const bool recorded = a->support_ids != nullptr;
  if (!recorded && a->vocab > vs::score_max_vocab(a->dtype))
    return fail(VS_ERR_UNSUPPORTED, "vocab exceeds vs_score_max_vocab for this dtype");
  if (recorded) {
    const size_t need = vs::score_recorded_workspace_bytes(a->rows, a->vocab, a->support_width, a->dtype);
    if (need && (!workspace || !aligned16(workspace) || workspace_bytes < need))
      return fail(VS_ERR_WORKSPACE,
                  "workspace missing, misaligned or smaller than vs_score_fwd_workspace_size");
  }

  vs::ScoreParams p{};
  p.rows = a->rows;
  p.vocab = a->vocab;
  p.ld = a->ld;
  p.logits = a->logits;
  p.temperature = a->temperature;
  p.temperature_scalar = a->temperature_scalar;
  p.targets = a->targets;
  p.top_k = a->top_k;
  p.top_k_scalar = a->top_k_scalar;
  p.top_p = a->top_p;
  p.top_p_scalar = a->top_p_scalar;
  p.min_p = a->min_p;
  p.min_p_scalar = a->min_p_scalar;
  p.support_ids = a->support_ids;
  p.support_width = a->support_width;
  p.support_ld = a->support_ld;
  p.lp_full = o->logprob_full;
  p.lp_support = o->logprob_support;
  p.h_full = want_entropy ? o->entropy_full : nullptr;
  p.h_support = want_entropy ? o->entropy_support : nullptr;
  p.valid = o->valid;
  p.status = o->status;
  p.support_size = o->support_size;
  p.support_mask = (a->flags & VS_WANT_SUPPORT_MASK) ? o->support_mask : nullptr;
  p.ctx = static_cast<vs::RowCtx*>((a->flags & VS_WANT_GRAD) ? o->ctx : nullptr);
  p.want_entropy = want_entropy ? 1 : 0;
  p.full_stats = (o->logprob_full || (want_entropy && o->entropy_full)) ? 1 : 0;
  p.sampled = (a->flags & VS_WANT_SAMPLE) ? o->sampled : nullptr;
  p.sample_seed = a->sample_seed;
  p.row_base = 0;
  // fixed-point scale: vocab * 2^shift <= 2^63
  int bits = 0;
  while ((1ll << bits) <= static_cast<long long>(a->vocab)) ++bits;
  p.fx_shift = 63 - bits;
  if (p.fx_shift > 60) p.fx_shift = 60;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (recorded)
    e = vs::launch_score_recorded(p, a->dtype, workspace, s);
  else
    e = vs::launch_score_computed(p, a->dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "vs_score_fwd launch");
  if (o->entropy_sum || o->valid_count) {
    e = vs::launch_score_reduce(p.h_support, o->valid, a->rows, o->entropy_sum, o->valid_count, s);
    if (e != cudaSuccess) return cuda_fail(e, "vs_score_fwd reduction launch");
  }
  return ok();
}

vs_status vs_score_bwd(const vs_score_args* a, const void* ctx, const float* g_lp_full,
                       const float* g_lp_support, const float* g_h_full,
                       const float* g_h_support, void* dlogits, vs_dtype dl_dtype,
                       int64_t grad_ld, int32_t mode, void* stream) {
  vs_status st = check_args(a);
  if (st != VS_OK) return st;
  if (mode != VS_GRAD_DENSE && mode != VS_GRAD_ACCUMULATE && mode != VS_GRAD_SPARSE)
    return fail(VS_ERR_INVALID_ARG, "mode must be VS_GRAD_DENSE, VS_GRAD_ACCUMULATE or VS_GRAD_SPARSE");
  if (dl_dtype != VS_BF16 && dl_dtype != VS_F32)
    return fail(VS_ERR_INVALID_ARG, "dl_dtype must be VS_BF16 or VS_F32");
  if (a->rows == 0) return ok();
  if (!ctx || !aligned16(ctx)) return fail(VS_ERR_INVALID_ARG, "ctx must be non-NULL and 16-byte aligned");
  if (!dlogits || !aligned16(dlogits))
    return fail(VS_ERR_INVALID_ARG, "dlogits must be non-NULL and 16-byte aligned");
  const bool recorded = a->support_ids != nullptr;
  if (mode == VS_GRAD_SPARSE) {
    if (!recorded) return fail(VS_ERR_INVALID_ARG, "VS_GRAD_SPARSE needs a recorded support");
    if (dl_dtype != VS_F32) return fail(VS_ERR_INVALID_ARG, "VS_GRAD_SPARSE writes fp32");
    if (grad_ld < a->support_width) return fail(VS_ERR_INVALID_ARG, "grad_ld must be >= support_width");
    if (g_lp_full || g_h_full)
      return fail(VS_ERR_INVALID_ARG, "VS_GRAD_SPARSE cannot hold full-vocabulary gradient terms");
  } else {
    if (grad_ld < a->vocab) return fail(VS_ERR_INVALID_ARG, "grad_ld must be >= vocab");
    if ((static_cast<uint64_t>(grad_ld) * esize(dl_dtype)) % 16 != 0)
      return fail(VS_ERR_INVALID_ARG, "grad_ld * sizeof(element) must be a multiple of 16 bytes");
  }
  vs::BwdParams p{};
  p.rows = a->rows;
  p.vocab = a->vocab;
  p.ld = a->ld;
  p.logits = a->logits;
  p.targets = a->targets;
  p.support_ids = a->support_ids;
  p.support_width = a->support_width;
  p.support_ld = a->support_ld;
  p.ctx = static_cast<const vs::RowCtx*>(ctx);
  p.g_lp_full = g_lp_full;
  p.g_lp_support = g_lp_support;
  p.g_h_full = g_h_full;
  p.g_h_support = g_h_support;
  p.dlogits = dlogits;
  p.grad_ld = grad_ld;
  // enough CTAs to cover the GPU several times over; slices of >= 2048 elements
  int nchunks = 1;
  const int want_ctas = 4 * 148;
  if (a->rows < want_ctas) {
    nchunks = (want_ctas + a->rows - 1) / a->rows;
    const int max_chunks = (a->vocab + 2047) / 2048;
    if (nchunks > max_chunks) nchunks = max_chunks;
    if (nchunks < 1) nchunks = 1;
  }
  int chunk = (a->vocab + nchunks - 1) / nchunks;
  chunk = (chunk + 31) & ~31;
  nchunks = (a->vocab + chunk - 1) / chunk;
  p.chunk = chunk;
  cudaError_t e = vs::launch_score_bwd(p, a->dtype, dl_dtype, mode, nchunks == 1, nchunks,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vs_score_bwd launch");
  return ok();
}

size_t vs_l1_distance_workspace_size(int32_t rows) { return vs::l1_workspace_bytes(rows); }

}  // extern "C"

namespace {

vs_status l1_call(int32_t rows, int32_t vocab, int64_t ld, vs_dtype dtype, const void* draft,
                  const void* target, const float* row_weight, float* l1, float* accept_rate,
                  float* loss_num_den_loss, void* grad_draft, vs_dtype grad_dtype,
                  int64_t grad_ld, const double* global_weight_sum, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (rows < 0) return fail(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (vocab < 1) return fail(VS_ERR_INVALID_ARG, "vocab must be >= 1");
  if (ld < vocab) return fail(VS_ERR_INVALID_ARG, "ld must be >= vocab");
  if (dtype != VS_BF16 && dtype != VS_F32)
    return fail(VS_ERR_INVALID_ARG, "dtype must be VS_BF16 or VS_F32");
  if (vocab > vs::l1_max_vocab(dtype))
    return fail(VS_ERR_UNSUPPORTED, "vocab exceeds the resident-row limit of vs_l1_distance");
  if (grad_draft) {
    if (grad_dtype != VS_BF16 && grad_dtype != VS_F32)
      return fail(VS_ERR_INVALID_ARG, "grad_dtype must be VS_BF16 or VS_F32");
    if (grad_ld < vocab) return fail(VS_ERR_INVALID_ARG, "grad_ld must be >= vocab");
    if (!aligned16(grad_draft) || (static_cast<uint64_t>(grad_ld) * esize(grad_dtype)) % 16 != 0)
      return fail(VS_ERR_INVALID_ARG, "grad_draft must be 16-byte aligned with 16-byte rows");
  }
  if (rows == 0) {
    if (loss_num_den_loss) return fail(VS_ERR_INVALID_ARG, "rows == 0 has no loss to write");
    return ok();
  }
  if (!draft || !target) return fail(VS_ERR_INVALID_ARG, "draft and target must be non-NULL");
  if (!aligned16(draft) || !aligned16(target) ||
      (static_cast<uint64_t>(ld) * esize(dtype)) % 16 != 0)
    return fail(VS_ERR_INVALID_ARG, "draft/target must be 16-byte aligned with 16-byte rows");
  if (loss_num_den_loss || grad_draft) {
    if (!workspace || !aligned16(workspace) || workspace_bytes < vs::l1_workspace_bytes(rows))
      return fail(VS_ERR_WORKSPACE, "workspace missing, misaligned or smaller than vs_l1_distance_workspace_size(rows)");
  }
  cudaError_t e = vs::launch_l1(rows, vocab, ld, dtype, draft, target, row_weight, l1, accept_rate,
                                loss_num_den_loss, grad_draft, grad_dtype, grad_ld, workspace,
                                global_weight_sum, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vs_l1_distance launch");
  return ok();
}

}  // namespace

extern "C" {

vs_status vs_l1_distance(int32_t rows, int32_t vocab, int64_t ld, vs_dtype dtype,
                         const void* draft, const void* target, const float* row_weight,
                         float* l1, float* accept_rate, float* loss_num_den_loss,
                         void* grad_draft, vs_dtype grad_dtype, int64_t grad_ld,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return l1_call(rows, vocab, ld, dtype, draft, target, row_weight, l1, accept_rate,
                 loss_num_den_loss, grad_draft, grad_dtype, grad_ld, nullptr, workspace,
                 workspace_bytes, stream);
}

vs_status vs_l1_weight_sum(int32_t rows, const float* row_weight, double* out, void* stream) {
  if (rows < 0) return fail(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (!out || reinterpret_cast<uintptr_t>(out) % 8 != 0)
    return fail(VS_ERR_INVALID_ARG, "out must be a non-NULL, 8-byte aligned device pointer");
  cudaError_t e = vs::launch_l1_weight_sum(rows, row_weight, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vs_l1_weight_sum launch");
  return ok();
}

vs_status vs_l1_distance_sharded(int32_t rows, int32_t vocab, int64_t ld, vs_dtype dtype,
                                 const void* draft, const void* target, const float* row_weight,
                                 const double* global_weight_sum, float* l1, float* accept_rate,
                                 float* loss_num_den_loss, void* grad_draft, vs_dtype grad_dtype,
                                 int64_t grad_ld, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!global_weight_sum) return fail(VS_ERR_INVALID_ARG, "global_weight_sum must be non-NULL");
  if (reinterpret_cast<uintptr_t>(global_weight_sum) % 8 != 0)
    return fail(VS_ERR_INVALID_ARG, "global_weight_sum must be 8-byte aligned");
  return l1_call(rows, vocab, ld, dtype, draft, target, row_weight, l1, accept_rate,
                 loss_num_den_loss, grad_draft, grad_dtype, grad_ld, global_weight_sum,
                 workspace, workspace_bytes, stream);
}

size_t vs_fused_lmhead_partial_bytes(int32_t rows, int32_t top_k) {
  return vs::lmhead_partial_bytes(rows, top_k);
}

size_t vs_fused_lmhead_partial_workspace_size(int32_t rows, int32_t vocab_count,
                                              int32_t hidden_dim, int32_t top_k) {
  return vs::lmhead_workspace_bytes(rows, vocab_count, hidden_dim, top_k);
}

vs_status vs_fused_lmhead_partial(int32_t rows, int32_t vocab_total, int32_t vocab_begin,
                                  int32_t vocab_count, int32_t hidden_dim, const void* hidden,
                                  int64_t ldh, const void* weight_shard, int64_t ldw,
                                  const float* temperature, float temperature_scalar,
                                  const int32_t* targets, int32_t top_k, void* partial,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  std::string err;
  const vs_status st = vs::lmhead_partial_run(
      rows, vocab_total, vocab_begin, vocab_count, hidden_dim, hidden, ldh, weight_shard, ldw,
      temperature, temperature_scalar, targets, top_k, partial, workspace, workspace_bytes,
      static_cast<cudaStream_t>(stream), &err);
  if (st != VS_OK) return fail(st, err);
  return ok();
}

vs_status vs_fused_lmhead_merge(int32_t rows, int32_t vocab_total, int32_t n_shards,
                                const void* partials, const float* temperature,
                                float temperature_scalar, const int32_t* targets, int32_t top_k,
                                float top_p, float min_p, uint32_t flags,
                                const vs_score_out* out, int32_t* topk_ids, float* topk_logprob,
                                void* stream) {
  std::string err;
  const vs_status st = vs::lmhead_merge_run(rows, vocab_total, n_shards, partials, temperature,
                                            temperature_scalar, targets, top_k, top_p, min_p,
                                            flags, out, topk_ids, topk_logprob,
                                            static_cast<cudaStream_t>(stream), &err);
  if (st != VS_OK) return fail(st, err);
  return ok();
}

size_t vs_fused_lmhead_bwd_workspace_size(int32_t rows, int32_t vocab, int32_t hidden_dim) {
  return vs::lmhead_bwd_workspace_bytes(rows, vocab, hidden_dim);
}

vs_status vs_fused_lmhead_bwd(int32_t rows, int32_t vocab, int32_t hidden_dim, const void* hidden,
                              int64_t ldh, const void* weight, int64_t ldw,
                              const int32_t* targets, int32_t top_k, const void* ctx,
                              const int32_t* topk_ids, const float* g_lp_full,
                              const float* g_lp_support, const float* g_h_full,
                              const float* g_h_support, float* d_hidden, int64_t ld_dh,
                              float* d_weight, int64_t ld_dw, void* workspace,
                              size_t workspace_bytes, void* stream) {
  std::string err;
  const vs_status st = vs::lmhead_bwd_run(
      rows, vocab, hidden_dim, hidden, ldh, weight, ldw, targets, top_k, ctx, topk_ids, g_lp_full,
      g_lp_support, g_h_full, g_h_support, d_hidden, ld_dh, d_weight, ld_dw, workspace,
      workspace_bytes, static_cast<cudaStream_t>(stream), &err);
  if (st != VS_OK) return fail(st, err);
  return ok();
}

size_t vs_fused_lmhead_workspace_size(int32_t rows, int32_t vocab, int32_t hidden_dim,
                                      int32_t top_k) {
  return vs::lmhead_workspace_bytes(rows, vocab, hidden_dim, top_k);
}

vs_status vs_fused_lmhead_score(int32_t rows, int32_t vocab, int32_t hidden_dim,
                                const void* hidden, int64_t ldh, const void* weight,
                                int64_t ldw, const float* temperature,
                                float temperature_scalar, const int32_t* targets,
                                int32_t top_k, float top_p, float min_p, uint32_t flags,
                                const vs_score_out* out, int32_t* topk_ids,
                                float* topk_logprob, void* workspace, size_t workspace_bytes,
                                void* stream) {
  std::string err;
  vs_status st = vs::lmhead_run(rows, vocab, hidden_dim, hidden, ldh, weight, ldw, temperature,
                                temperature_scalar, targets, top_k, top_p, min_p, flags, out,
                                topk_ids, topk_logprob, workspace, workspace_bytes,
                                static_cast<cudaStream_t>(stream), &err);
  if (st != VS_OK) return fail(st, err);
  return ok();
}

vs_status vs_support_lmhead_score(int32_t rows, int32_t vocab, int32_t hidden_dim,
                                  const void* hidden, int64_t ldh, const void* weight,
                                  int64_t ldw, const float* temperature, float temperature_scalar,
                                  const int32_t* targets, const int32_t* support_ids,
                                  int32_t support_width, int64_t support_ld, uint32_t flags,
                                  const vs_score_out* out, float* support_logits,
                                  int64_t logits_ld, void* stream) {
  std::string err;
  vs_status st = vs::support_head_run(rows, vocab, hidden_dim, hidden, ldh, weight, ldw,
                                      temperature, temperature_scalar, targets, support_ids,
                                      support_width, support_ld, flags, out, support_logits,
                                      logits_ld, static_cast<cudaStream_t>(stream), &err);
  if (st != VS_OK) return fail(st, err);
  return ok();
}

}  // extern "C"
