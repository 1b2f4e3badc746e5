// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vs_api.h"

namespace vs {

// Saved per-row state written by the forward pass for the backward pass
// (VS_CTX_BYTES_PER_ROW bytes).  Base-2 units: u = l * c, c = log2(e) / T.
struct alignas(16) RowCtx {
  float m2;         // max_j u_j over the vocabulary (NaN if not computed)
  float log2z;      // log2 sum_j 2^(u_j - m2)          (NaN if not computed)
  float msup;       // reference for q: u-offset of the support sums
  float log2zs;     // log2 sum_{j in S} 2^(u_j - msup)
  float h_full;     // H_V (nat)
  float h_support;  // H_S (nat)
  float c;          // log2(e) / T
  uint32_t tkey;    // computed support: threshold key
  int32_t tie_cut;  // computed support: largest id kept among keys == tkey
  uint32_t flags;   // kCtx*
  int32_t n_support;
  uint32_t status;
  // split normalisers (see Stats): Z = c0 + zr, for 1 - p_y when y is a max
  float c0_full, zr_full;
  float c0_sup, zr_sup;
};
static_assert(sizeof(RowCtx) == VS_CTX_BYTES_PER_ROW, "ctx layout");

enum : uint32_t {
  kCtxFullStats = 1u << 0,   // m2 / log2z / h_full valid
  kCtxAllVocab = 1u << 1,    // S is the whole vocabulary
  kCtxThreshold = 1u << 2,   // S = {key > tkey} + {key == tkey, id <= tie_cut}
  kCtxRecorded = 1u << 3,    // S from the recorded id list
  kCtxEmpty = 1u << 4,       // S is empty
  kCtxTargetOk = 1u << 5,    // 0 <= y < V
  kCtxTargetInS = 1u << 6,   // y in S
  kCtxNonFinite = 1u << 7,   // row had a non-finite logit
};

// Device-side view of a scoring call.
struct ScoreParams {
  int32_t rows, vocab;
  int64_t ld;
  const void* logits;
  const float* temperature;
  float temperature_scalar;
  const int32_t* targets;
  const int32_t* top_k;
  int32_t top_k_scalar;
  const float* top_p;
  float top_p_scalar;
  const float* min_p;
  float min_p_scalar;
  const int32_t* support_ids;
  int32_t support_width;
  int64_t support_ld;
  float* lp_full;
  float* lp_support;
  float* h_full;
  float* h_support;
  uint8_t* valid;
  uint32_t* status;
  int32_t* support_size;
  uint32_t* support_mask;
  RowCtx* ctx;
  int32_t want_entropy;
  int32_t full_stats;  // recorded support: compute full-vocabulary stats for every row
  int32_t fx_shift;    // fixed-point scale of mass histograms: 2^fx_shift
  int32_t* sampled;    // [R] seeded Gumbel-max token, or nullptr
  uint64_t sample_seed;
  int32_t row_base;    // index of row 0 of this launch within the call (noise key)
};

struct BwdParams {
  int32_t rows, vocab;
  int64_t ld;
  const void* logits;
  const int32_t* targets;
  const int32_t* support_ids;
  int32_t support_width;
  int64_t support_ld;
  const RowCtx* ctx;
  const float* g_lp_full;
  const float* g_lp_support;
  const float* g_h_full;
  const float* g_h_support;
  void* dlogits;
  int64_t grad_ld;
  int32_t chunk;  // elements per CTA (multiple of 32); == padded vocab when whole rows
};

// launchers (return a cudaError_t from the launch)
cudaError_t launch_score_computed(const ScoreParams& p, vs_dtype dtype, cudaStream_t s);
// Recorded supports.  Lists of up to 64 ids need a workspace of
// score_recorded_workspace_bytes (16-byte aligned); wider lists none.
size_t score_recorded_workspace_bytes(int rows, int vocab, int width, vs_dtype dtype);
cudaError_t launch_score_recorded(const ScoreParams& p, vs_dtype dtype, void* ws, cudaStream_t s);
cudaError_t launch_score_reduce(const float* h_support, const uint8_t* valid, int rows,
                                double* entropy_sum, int32_t* valid_count, cudaStream_t s);
cudaError_t launch_score_bwd(const BwdParams& p, vs_dtype dtype, vs_dtype gdtype, int mode,
                             bool whole_rows, int nchunks, cudaStream_t s);

int score_max_vocab(vs_dtype dtype);

}  // namespace vs
