// Fused LM-head scoring (placeholder until the tensor-core kernel lands).
#include <string>

#include "internal.h"

namespace vs {

size_t lmhead_workspace_bytes(int rows, int vocab, int hidden, int top_k) {
  (void)rows; (void)vocab; (void)hidden; (void)top_k;
  return 0;
}

vs_status lmhead_run(int rows, int vocab, int hidden, const void* H, int64_t ldh, const void* W,
                     int64_t ldw, const float* temperature, float temperature_scalar,
                     const int32_t* targets, int top_k, float top_p, float min_p,
                     uint32_t flags, const vs_score_out* out, int32_t* topk_ids,
                     float* topk_logprob, void* ws, size_t ws_bytes, cudaStream_t s,
                     std::string* err) {
  *err = "vs_fused_lmhead_score is not available in this build";
  return VS_ERR_UNSUPPORTED;
}

}  // namespace vs
