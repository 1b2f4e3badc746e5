// Support-only fused projection (SkyRL PR #2004, "Performance": with a fused
// LM head the replay path uses the selected hidden-state / weight
// projections and never materialises vocabulary logits; "Implementation":
// the recorded support is a dense -1-padded id list).  For row i and each
// kept support id s (0 <= s < vocab, first occurrence in the row's list):
//
//   a[i, s] = sum_k hidden[i, k] * weight[s, k]      (bf16 inputs, fp32 sums)
//   z[i, s] = a[i, s] / T_i
//
// then the support-conditioned log-probability of the target and the
// support entropy, as for a recorded support.  The work scales with the
// support width, not the vocabulary: one 128-thread CTA per row stages the
// hidden state in shared memory, and its warps each stream whole weight rows
// (coalesced 16-byte loads, eight in flight per lane; one mixed-precision
// bf16 x bf16 + fp32 FMA per element) into one dot product per kept id.
// Weight rows that several rows' supports share are read from L2.

#include <cmath>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace vs {

static_assert(kRowDeviceTimeout == VS_ROW_DEVICE_TIMEOUT, "status bit of a device timeout");

namespace {

constexpr int kSHThreads = 128;
constexpr int kSHWarps = kSHThreads / 32;
constexpr int kSHUnroll = 8;         // 16-byte weight loads in flight per lane
constexpr int kSHMaxHidden = 16384;  // hidden state staged in shared memory (32 KB)

struct SupportHeadParams {
  int32_t rows, vocab, hidden;
  const uint16_t* H;
  int64_t ldh;
  const uint16_t* W;
  int64_t ldw;
  const float* temperature;
  float temperature_scalar;
  const int32_t* targets;
  const int32_t* support_ids;
  int32_t width;
  int64_t support_ld;
  float* lp_support;
  float* h_support;
  uint8_t* valid;
  uint32_t* status;
  int32_t* support_size;
  float* logits;  // [rows, width] support logits, or nullptr
  int64_t logits_ld;
};

// lo += h.lo * w.lo, hi += h.hi * w.hi for the bf16 pairs of two words: one
// mixed-precision FMA per element (bf16 operands widen exactly, one fp32
// rounding), so no separate conversion instructions.
__device__ __forceinline__ void fma_bf16x2(uint32_t h, uint32_t w, float& lo, float& hi) {
  asm("{\n .reg .b16 hl, hh, wl, wh;\n mov.b32 {hl, hh}, %2;\n mov.b32 {wl, wh}, %3;\n"
      " fma.rn.f32.bf16 %0, hl, wl, %0;\n fma.rn.f32.bf16 %1, hh, wh, %1;\n}\n"
      : "+f"(lo), "+f"(hi)
      : "r"(h), "r"(w));
}

// Dot product of the staged hidden state with weight row w (the warp's
// lanes take 8 consecutive elements per 256-element step); every lane
// returns the warp's sum, reduced in a fixed order.
__device__ __forceinline__ float warp_dot(const uint4* hs4, const uint4* w4, int nvec) {
  const int lane = threadIdx.x & 31;
  // four accumulators: elements 0,4 / 1,5 / 2,6 / 3,7 of each 8-element vector
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  auto fma8 = [&](const uint4& h, const uint4& w) {
    fma_bf16x2(h.x, w.x, s0, s1);
    fma_bf16x2(h.y, w.y, s2, s3);
    fma_bf16x2(h.z, w.z, s0, s1);
    fma_bf16x2(h.w, w.w, s2, s3);
  };
  int v = lane;
  for (; v + (kSHUnroll - 1) * 32 < nvec; v += kSHUnroll * 32) {
    uint4 w[kSHUnroll];
#pragma unroll
    for (int u = 0; u < kSHUnroll; ++u) w[u] = __ldg(w4 + v + u * 32);
#pragma unroll
    for (int u = 0; u < kSHUnroll; ++u) fma8(hs4[v + u * 32], w[u]);
  }
  for (; v < nvec; v += 32) fma8(hs4[v], __ldg(w4 + v));
  float s = (s0 + s1) + (s2 + s3);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

__global__ void __launch_bounds__(kSHThreads) support_head_kernel(SupportHeadParams P) {
  extern __shared__ __align__(16) uint4 hs4[];  // the row's hidden state
  __shared__ int32_t ids[VS_MAX_SUPPORT_WIDTH];
  __shared__ float acc[VS_MAX_SUPPORT_WIDTH];      // a[i, s] of kept slots
  __shared__ uint8_t kept[VS_MAX_SUPPORT_WIDTH];   // slot holds a kept id
  __shared__ int16_t kslot[VS_MAX_SUPPORT_WIDTH];  // kept slots, in claim order
  __shared__ uint32_t nkeep_sh, flags_sh;
  __shared__ int32_t yslot;
  __shared__ float fred[kSHWarps];
  __shared__ uint32_t ured[kSHWarps];

  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int V = P.vocab, Wd = P.width;
  const int nvec = P.hidden / 8;
  const int32_t* srow = P.support_ids + static_cast<int64_t>(row) * P.support_ld;
  const uint4* h4 = reinterpret_cast<const uint4*>(P.H + static_cast<int64_t>(row) * P.ldh);
  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const float c = kLog2e / T;
  const int y = P.targets[row];
  const bool target_ok = y >= 0 && y < V;

  if (tid == 0) {
    nkeep_sh = 0;
    flags_sh = 0;
    yslot = -1;
  }
  for (int w = tid; w < Wd; w += kSHThreads) ids[w] = srow[w];
  for (int v = tid; v < nvec; v += kSHThreads) hs4[v] = __ldg(h4 + v);
  cta_sync();

  // kept slots: a valid id at its first occurrence.  Each warp takes groups
  // of 32 consecutive slots: repeats within a group by a match mask, repeats
  // of an earlier group's id by a scan of those slots with no early exit
  // (independent loads)
  uint32_t local_flags = 0;
  for (int base = warp * 32; base < Wd; base += kSHThreads) {
    const int w = base + lane;
    const int32_t id = w < Wd ? ids[w] : -1;
    bool dup = (__match_any_sync(0xffffffffu, id) & ((1u << lane) - 1u)) != 0u;
    for (int w2 = 0; w2 < base; ++w2) dup |= ids[w2] == id;
    if (w >= Wd) continue;
    kept[w] = 0;
    if (id == -1) continue;
    if (id < -1 || id >= V) {
      local_flags |= VS_ROW_BAD_SUPPORT_ID;
      continue;
    }
    if (dup) {
      local_flags |= VS_ROW_DUP_SUPPORT_ID;
      continue;
    }
    kept[w] = 1;
    kslot[atomicAdd(&nkeep_sh, 1u)] = static_cast<int16_t>(w);
    if (id == y) yslot = w;
  }
  if (local_flags) atomicOr(&flags_sh, local_flags);
  cta_sync();
  const int nkeep = static_cast<int>(nkeep_sh);

  // one dot product per kept id, warps taking the kept slots in turn
  for (int j = warp; j < nkeep; j += kSHWarps) {
    const int w = kslot[j];
    const uint4* w4 = reinterpret_cast<const uint4*>(P.W + static_cast<int64_t>(ids[w]) * P.ldw);
    const float a = warp_dot(hs4, w4, nvec);
    if (lane == 0) acc[w] = a;
  }
  cta_sync();

  if (P.logits) {
    float* lrow = P.logits + static_cast<int64_t>(row) * P.logits_ld;
    for (int w = tid; w < Wd; w += kSHThreads) {
      lrow[w] = kept[w] ? __fdiv_rn(acc[w], T) : -kInf;
    }
  }
  if (warp != 0) return;

  // support statistics over the kept slots, relative to the support maximum:
  // warp 0 alone (lane l takes slots l, l + 32, ...; shuffle trees)
  float amax = -kInf;
  bool nonfinite = false;
  for (int w = lane; w < Wd; w += 32) {
    if (!kept[w]) continue;
    const float a = acc[w];
    if (!isfinite(a)) nonfinite = true;  // a NaN or inf among the inputs
    amax = fmaxf(amax, a);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const bool any_nf = __any_sync(0xffffffffu, nonfinite);
  Stats s{amax, 0.f, 0.f, 0.f};
  for (int w = lane; w < Wd; w += 32) {
    if (!kept[w]) continue;
    const float d = (acc[w] - amax) * c;
    const float e = ex2(d);
    if (d == 0.f)
      s.c0 += 1.f;
    else
      s.zr += e;
    s.a = fmaf(d, e, s.a);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s.c0 += __shfl_xor_sync(0xffffffffu, s.c0, o);
    s.zr += __shfl_xor_sync(0xffffffffu, s.zr, o);
    s.a += __shfl_xor_sync(0xffffffffu, s.a, o);
  }

  if (tid == 0) {
    const float nan = __int_as_float(0x7fc00000);
    const bool empty = nkeep == 0;
    const bool nf = any_nf && !empty;
    uint32_t status = flags_sh;
    float lp_s = nan;
    const float log2zs = empty ? nan : stats_log2z(s);
    const float h_sup = empty ? 0.f : kLn2 * (log2zs - s.a / stats_z(s));
    if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
    if (empty) status |= VS_ROW_EMPTY_SUPPORT;
    if (nf) {
      status |= VS_ROW_NONFINITE_INPUT;
    } else if (target_ok && !empty) {
      if (yslot >= 0) {
        lp_s = kLn2 * ((acc[yslot] - amax) * c - log2zs);
      } else {
        lp_s = -kInf;
        status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
      }
    }
    if (P.lp_support) P.lp_support[row] = lp_s;
    if (P.h_support) P.h_support[row] = nf ? nan : h_sup;
    if (P.valid) P.valid[row] = (nf || empty) ? 0 : 1;
    if (P.status) P.status[row] = status;
    if (P.support_size) P.support_size[row] = nf ? 0 : nkeep;
  }
}

}  // namespace

vs_status support_head_run(int rows, int vocab, int hidden, const void* H, int64_t ldh,
                           const void* W, int64_t ldw, const float* temperature,
                           float temperature_scalar, const int32_t* targets,
                           const int32_t* support_ids, int width, int64_t support_ld,
                           uint32_t flags, const vs_score_out* out, float* support_logits,
                           int64_t logits_ld, cudaStream_t s, std::string* err) {
  auto bad = [&](vs_status code, const char* msg) {
    *err = msg;
    return code;
  };
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (rows < 0) return bad(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (vocab < 1) return bad(VS_ERR_INVALID_ARG, "vocab must be >= 1");
  if (hidden < 8 || hidden % 8 != 0 || hidden > kSHMaxHidden)
    return bad(VS_ERR_UNSUPPORTED, "hidden_dim must be a positive multiple of 8, at most 16384");
  if (width < 0 || width > VS_MAX_SUPPORT_WIDTH)
    return bad(VS_ERR_UNSUPPORTED, "support_width must lie in [0, VS_MAX_SUPPORT_WIDTH]");
  if (support_ld < width) return bad(VS_ERR_INVALID_ARG, "support_ld must be >= support_width");
  if (!temperature && !(std::isfinite(temperature_scalar) && temperature_scalar > 0.f))
    return bad(VS_ERR_INVALID_ARG, "temperature_scalar must be finite and > 0");
  if (!out) return bad(VS_ERR_INVALID_ARG, "out is NULL");
  if (out->logprob_full || out->entropy_full || out->support_mask || out->ctx || out->sampled)
    return bad(VS_ERR_INVALID_ARG,
               "logprob_full, entropy_full, support_mask, ctx and sampled are not offered by "
               "the support-only projection: pass NULL");
  const bool want_entropy = flags & VS_WANT_ENTROPY;
  if (flags & ~static_cast<uint32_t>(VS_WANT_ENTROPY))
    return bad(VS_ERR_INVALID_ARG, "flags other than VS_WANT_ENTROPY are not offered here");
  if (!want_entropy && out->entropy_support)
    return bad(VS_ERR_INVALID_ARG, "entropy outputs need VS_WANT_ENTROPY");
  if (support_logits && logits_ld < width)
    return bad(VS_ERR_INVALID_ARG, "logits_ld must be >= support_width");
  if (rows == 0) return VS_OK;
  if (!H || !W || !targets || (width > 0 && !support_ids))
    return bad(VS_ERR_INVALID_ARG, "hidden, weight, targets and support_ids must be non-NULL");
  if (!a16(H) || !a16(W) || ldh % 8 != 0 || ldw % 8 != 0 || ldh < hidden || ldw < hidden)
    return bad(VS_ERR_INVALID_ARG, "hidden/weight must be 16-byte aligned with ld >= hidden_dim, ld % 8 == 0");

  static int32_t no_ids[1] = {0};
  SupportHeadParams P{};
  P.rows = rows;
  P.vocab = vocab;
  P.hidden = hidden;
  P.H = static_cast<const uint16_t*>(H);
  P.ldh = ldh;
  P.W = static_cast<const uint16_t*>(W);
  P.ldw = ldw;
  P.temperature = temperature;
  P.temperature_scalar = temperature_scalar;
  P.targets = targets;
  P.support_ids = width > 0 ? support_ids : no_ids;  // never read when width is 0
  P.width = width;
  P.support_ld = support_ld;
  P.lp_support = out->logprob_support;
  P.h_support = want_entropy ? out->entropy_support : nullptr;
  P.valid = out->valid;
  P.status = out->status;
  P.support_size = out->support_size;
  P.logits = support_logits;
  P.logits_ld = logits_ld;
  const size_t smem = static_cast<size_t>(hidden) * 2;
  support_head_kernel<<<rows, kSHThreads, smem, s>>>(P);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));
  return VS_OK;
}

}  // namespace vs
