// Oracle for per-row vocabulary scoring: a plain, slow, fp64 CPU restatement
// of what the scoring path computes.
//
// TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
// the test suite, the smoke check and the benchmark's CPU-baseline leg may load
// it.  It shares no code, header, table or constant with the CUDA library in
// sampling_support_b200/csrc, and it does not include or link that library.
//
// Sources (web pages this restates; no code is taken from them):
//  [SkyRL]  "perf(sample-support): reuse replay scores for entropy", SkyRL PR
//           #2004 -- sections "Implementation" and the paragraph after it:
//           support-renormalised logprob, support-conditioned entropy, the
//           valid-row metadata, singleton support => zero entropy and zero
//           entropy gradient, empty support => full-vocabulary logprob
//           fallback and exclusion from the entropy reduction, dense padded
//           support representation.
//  [xorl]   "Consolidate the exact and generic scoring paths; implement
//           top-k/top-p/min-p", xorl issue #71 -- section 3 (the program
//           temperature -> stable token-id top-k -> inclusive top-p -> min-p
//           relative to the original row max; the top_p == 1.0 identity) and
//           section 1 (chunked projection -> fixed-order LSE -> support ->
//           selected logprob + VJP).
//  [DSpark] "[Perf] Reuse DSpark probability distance across loss and
//           metrics", DeepSpec PR #87 -- section "Purpose": per-token L1
//           distance between softmax(draft) and softmax(target), accept_rate =
//           clamp(1 - 0.5 * L1, 0, 1), weighted L1 loss.
//
// Readings where the pages are silent (each is also listed in the design
// notes): top-p is taken on the mass renormalised over the top-k set; min-p is
// inclusive (p_j >= min_p * p_max) with p_max the unfiltered row maximum;
// ties in the order are broken by ascending token id; top_k <= 0 or >= V,
// top_p >= 1 and min_p <= 0 disable a filter; a target outside a non-empty
// support gets lp_S = -inf and no lp_S gradient; sign(0) = 0 in the L1
// gradient; the weighted L1 loss is sum(w * L1) / sum(w), 0 when sum(w) == 0.
//
// Every quantity is computed in double precision from the exact input values
// (bf16 and fp32 inputs are widened exactly).  No blocking, fusion or
// reordering beyond the definitions: sort by the total order, take prefixes,
// sum.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

namespace {

constexpr double kInf = std::numeric_limits<double>::infinity();
constexpr double kNaN = std::numeric_limits<double>::quiet_NaN();

// Input element types understood by the oracle.
enum OracleDtype : int { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

// Per-row status bits.  The values are the oracle's own; the test suite maps
// them onto the library's status word by name.
enum : uint32_t {
  ORC_TARGET_OUT_OF_RANGE = 1u << 0,
  ORC_TARGET_NOT_IN_SUPPORT = 1u << 1,
  ORC_BAD_SUPPORT_ID = 1u << 2,
  ORC_DUP_SUPPORT_ID = 1u << 3,
  ORC_NONFINITE_INPUT = 1u << 4,
};

// Widen one input element to double, exactly.
double load_value(const void* base, int dtype, int64_t index) {
  if (dtype == ORC_F64) return static_cast<const double*>(base)[index];
  if (dtype == ORC_F32) return static_cast<double>(static_cast<const float*>(base)[index]);
  // bf16: the upper 16 bits of an IEEE binary32.
  uint16_t h = static_cast<const uint16_t*>(base)[index];
  uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

// log sum_j exp(z_j - m) over the selected entries, with m their maximum,
// evaluated as log(#{z_j == m}) + log1p(sum_{z_j < m} exp(z_j - m) / #{z_j == m}):
// the same sum, split so that a row dominated by one token (sum = 1 + tiny)
// keeps its relative precision.
double log_sum_exp_shifted(const std::vector<double>& z, const std::vector<uint8_t>* sel,
                           double m) {
  double top = 0.0, rest = 0.0;
  for (size_t j = 0; j < z.size(); ++j) {
    if (sel && !(*sel)[j]) continue;
    if (z[j] == m)
      top += 1.0;
    else
      rest += std::exp(z[j] - m);
  }
  return std::log(top) + std::log1p(rest / top);
}

// Everything the oracle knows about one scored row.
struct RowResult {
  double lse_full = kNaN;      // log sum_j exp(z_j)
  double lp_full = kNaN;       // z_y - lse_full
  double lp_support = kNaN;    // z_y - log sum_{j in S} exp(z_j)
  double h_full = kNaN;        // -sum_j p_j log p_j
  double h_support = 0.0;      // -sum_{j in S} q_j log q_j
  double lse_support = kNaN;
  double m_full = kNaN, lz_full = kNaN;        // lse_full = m_full + lz_full
  double m_support = kNaN, lz_support = kNaN;  // lse_support = m_support + lz_support
  uint8_t valid = 0;
  uint32_t status = 0;
  int32_t support_size = 0;
  double topp_margin = kInf;   // distance of the inclusive top-p crossing from p
  double minp_margin = kInf;   // relative distance of the min-p boundary from min_p
  double topk_gap = kInf;      // z(k-th) - z(k+1-th) in the total order
  std::vector<double> z;       // tempered logits
  std::vector<uint8_t> in_support;
};

// Score one row.  z_j = l_j / T  ([xorl] section 3: temperature first).
RowResult score_row(const void* logits, int dtype, int64_t row_offset, int vocab,
                    double temperature, int32_t target, int32_t top_k, double top_p,
                    double min_p, const int32_t* support_row, int width, bool keep_z) {
  RowResult r;
  r.z.resize(vocab);
  bool finite = true;
  for (int j = 0; j < vocab; ++j) {
    double l = load_value(logits, dtype, row_offset + j);
    if (!std::isfinite(l)) finite = false;
    r.z[j] = l / temperature;
  }
  const bool target_ok = target >= 0 && target < vocab;
  if (!target_ok) r.status |= ORC_TARGET_OUT_OF_RANGE;
  if (!finite) {
    // Non-finite logits: nothing is scored; the row is flagged and invalid.
    r.status |= ORC_NONFINITE_INPUT;
    r.in_support.assign(vocab, 0);
    r.lp_full = r.lp_support = r.h_full = r.h_support = kNaN;
    r.valid = 0;
    return r;
  }

  // Full-vocabulary log-sum-exp, logprob and entropy; log p_j = (z_j - m) - log sum exp(z - m).
  const double m = *std::max_element(r.z.begin(), r.z.end());
  const double lz = log_sum_exp_shifted(r.z, nullptr, m);
  r.m_full = m;
  r.lz_full = lz;
  r.lse_full = m + lz;
  double h = 0.0;
  for (int j = 0; j < vocab; ++j) {
    double logp = (r.z[j] - m) - lz;
    h -= std::exp(logp) * logp;
  }
  r.h_full = h;
  r.lp_full = target_ok ? (r.z[target] - m) - lz : kNaN;

  // Support S.
  r.in_support.assign(vocab, 0);
  if (support_row != nullptr) {
    // Recorded support ([SkyRL]: dense id list; pads are -1 wherever they sit).
    for (int w = 0; w < width; ++w) {
      int32_t id = support_row[w];
      if (id == -1) continue;
      if (id < -1 || id >= vocab) {
        r.status |= ORC_BAD_SUPPORT_ID;
        continue;
      }
      if (r.in_support[id]) {
        r.status |= ORC_DUP_SUPPORT_ID;
        continue;
      }
      r.in_support[id] = 1;
    }
  } else {
    // Computed support ([xorl] section 3): stable token-id top-k, then
    // inclusive top-p on the top-k set, then min-p against the original max.
    const bool use_k = top_k > 0 && top_k < vocab;
    const bool use_p = top_p < 1.0;
    const bool use_minp = min_p > 0.0;
    if (!use_k && !use_p && !use_minp) {
      r.in_support.assign(vocab, 1);
    } else {
      // Total order: z descending, token id ascending on equal z.
      std::vector<int32_t> order(vocab);
      std::iota(order.begin(), order.end(), 0);
      std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
        if (r.z[a] != r.z[b]) return r.z[a] > r.z[b];
        return a < b;
      });
      // top-k: the first k of the order.
      int n1 = use_k ? top_k : vocab;
      if (use_k) r.topk_gap = r.z[order[n1 - 1]] - r.z[order[n1]];
      // top-p on r_j = p_j / sum_{S1} p: smallest prefix whose mass >= p.
      int n2 = n1;
      if (use_p) {
        double mass1 = 0.0;
        for (int i = 0; i < n1; ++i) mass1 += std::exp(r.z[order[i]] - m);
        double cum = 0.0;
        n2 = n1;
        for (int i = 0; i < n1; ++i) {
          double before = cum / mass1;
          cum += std::exp(r.z[order[i]] - m);
          double after = cum / mass1;
          if (after >= top_p) {
            n2 = i + 1;
            r.topp_margin = std::min(after - top_p, top_p - before);
            break;
          }
        }
      }
      // min-p: keep j in S2 with p_j >= min_p * max_j p_j, i.e. exp(z_j - m) >= min_p.
      int n3 = n2;
      if (use_minp) {
        n3 = 0;
        for (int i = 0; i < n2; ++i) {
          double ratio = std::exp(r.z[order[i]] - m);
          if (ratio >= min_p) n3 = i + 1;
        }
        double mg = std::fabs(std::exp(r.z[order[n3 - 1]] - m) - min_p) / min_p;
        if (n3 < n2) mg = std::min(mg, std::fabs(std::exp(r.z[order[n3]] - m) - min_p) / min_p);
        r.minp_margin = mg;
      }
      for (int i = 0; i < n3; ++i) r.in_support[order[i]] = 1;
    }
  }

  int count = 0;
  for (int j = 0; j < vocab; ++j) count += r.in_support[j];
  r.support_size = count;

  if (count == 0) {
    // Empty support ([SkyRL]): full-vocabulary logprob fallback; the row is
    // excluded from the entropy reduction (valid = 0, H_S written as 0).
    r.valid = 0;
    r.lp_support = r.lp_full;
    r.h_support = 0.0;
    r.lse_support = kNaN;
    return r;
  }
  r.valid = 1;
  // Support-renormalised distribution q = softmax(z restricted to S).
  double ms = -kInf;
  for (int j = 0; j < vocab; ++j)
    if (r.in_support[j]) ms = std::max(ms, r.z[j]);
  const double lzs = log_sum_exp_shifted(r.z, &r.in_support, ms);
  r.m_support = ms;
  r.lz_support = lzs;
  r.lse_support = ms + lzs;
  double hs = 0.0;
  for (int j = 0; j < vocab; ++j) {
    if (!r.in_support[j]) continue;
    double logq = (r.z[j] - ms) - lzs;
    hs -= std::exp(logq) * logq;
  }
  r.h_support = hs;
  if (!target_ok) {
    r.lp_support = kNaN;
  } else if (r.in_support[target]) {
    r.lp_support = (r.z[target] - ms) - lzs;
  } else {
    r.status |= ORC_TARGET_NOT_IN_SUPPORT;
    r.lp_support = -kInf;
  }
  if (!keep_z) r.z.clear();
  return r;
}

template <typename T>
T pick(const T* arr, int i, T fallback) {
  return arr ? arr[i] : fallback;
}

}  // namespace

extern "C" {

// Score `rows` rows.  Per-row parameter arrays may be null (then the scalar
// after them is used).  `support_ids` (row stride `sld`, `width` entries) may
// be null, which selects the computed support.  `mask` ([rows, vocab] bytes),
// and the margin arrays may be null.
int vso_score(int rows, int vocab, int64_t ld, int dtype, const void* logits,
              const double* temperature, double temperature_scalar, const int32_t* targets,
              const int32_t* top_k, int32_t top_k_scalar, const double* top_p,
              double top_p_scalar, const double* min_p, double min_p_scalar,
              const int32_t* support_ids, int width, int64_t sld, double* lp_full,
              double* lp_support, double* h_full, double* h_support, uint8_t* valid,
              uint32_t* status, int32_t* support_size, uint8_t* mask, double* topp_margin,
              double* minp_margin, double* topk_gap, double* lse_full) {
  if (rows < 0 || vocab <= 0 || ld < vocab || !logits || !targets) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < rows; ++i) {
    RowResult r = score_row(logits, dtype, static_cast<int64_t>(i) * ld, vocab,
                            pick(temperature, i, temperature_scalar), targets[i],
                            pick(top_k, i, top_k_scalar), pick(top_p, i, top_p_scalar),
                            pick(min_p, i, min_p_scalar),
                            support_ids ? support_ids + static_cast<int64_t>(i) * sld : nullptr,
                            width, false);
    if (lp_full) lp_full[i] = r.lp_full;
    if (lp_support) lp_support[i] = r.lp_support;
    if (h_full) h_full[i] = r.h_full;
    if (h_support) h_support[i] = r.h_support;
    if (valid) valid[i] = r.valid;
    if (status) status[i] = r.status;
    if (support_size) support_size[i] = r.support_size;
    if (topp_margin) topp_margin[i] = r.topp_margin;
    if (minp_margin) minp_margin[i] = r.minp_margin;
    if (topk_gap) topk_gap[i] = r.topk_gap;
    if (lse_full) lse_full[i] = r.lse_full;
    if (mask) std::memcpy(mask + static_cast<int64_t>(i) * vocab, r.in_support.data(), vocab);
  }
  return 0;
}

// Prefix facts of the computed-support order, for checking a support whose
// top-p or min-p decision sits within rounding of its threshold.  For row i
// and a prefix length n = prefix_len[i] of the total order (z descending,
// token id ascending; [xorl] section 3), with m the row maximum and the
// top-p mass renormalised over the top-k set (k = top_k when 0 < top_k <
// vocab, else vocab):
//   ids[i, 0 .. n-1]  the first n ids (n <= max_ids),
//   mass_n[i]         sum_{first n} exp(z - m) / sum_{first k} exp(z - m),
//   mass_prev[i]      the same over the first n - 1 (0 when n == 0),
//   ratio_n[i]        exp(z - m) of the n-th entry (1 when n == 0),
//   ratio_next[i]     exp(z - m) of the (n+1)-th entry (0 when n == vocab),
//   nk[i]             k.
// Any output array may be null.  Returns 1 on bad arguments.
int vso_prefix(int rows, int vocab, int64_t ld, int dtype, const void* logits,
               const double* temperature, double temperature_scalar, const int32_t* top_k,
               int32_t top_k_scalar, const int32_t* prefix_len, int32_t* ids, int max_ids,
               double* mass_n, double* mass_prev, double* ratio_n, double* ratio_next,
               int32_t* nk) {
  if (rows < 0 || vocab <= 0 || ld < vocab || !logits || !prefix_len) return 1;
  for (int i = 0; i < rows; ++i)
    if (prefix_len[i] < 0 || prefix_len[i] > vocab || (ids && prefix_len[i] > max_ids)) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < rows; ++i) {
    const double t = pick(temperature, i, temperature_scalar);
    std::vector<double> z(vocab);
    for (int j = 0; j < vocab; ++j)
      z[j] = load_value(logits, dtype, static_cast<int64_t>(i) * ld + j) / t;
    std::vector<int32_t> order(vocab);
    std::iota(order.begin(), order.end(), 0);
    std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
      if (z[a] != z[b]) return z[a] > z[b];
      return a < b;
    });
    const double m = z[order[0]];
    const int32_t k = pick(top_k, i, top_k_scalar);
    const int n1 = (k > 0 && k < vocab) ? k : vocab;
    const int n = prefix_len[i];
    double mass1 = 0.0, cum = 0.0, prev = 0.0;
    for (int r = 0; r < n1; ++r) mass1 += std::exp(z[order[r]] - m);
    for (int r = 0; r < n; ++r) {
      prev = cum;
      cum += std::exp(z[order[r]] - m);
    }
    if (ids)
      for (int r = 0; r < n; ++r) ids[static_cast<int64_t>(i) * max_ids + r] = order[r];
    if (mass_n) mass_n[i] = cum / mass1;
    if (mass_prev) mass_prev[i] = n > 0 ? prev / mass1 : 0.0;
    if (ratio_n) ratio_n[i] = n > 0 ? std::exp(z[order[n - 1]] - m) : 1.0;
    if (ratio_next) ratio_next[i] = n < vocab ? std::exp(z[order[n]] - m) : 0.0;
    if (nk) nk[i] = n1;
  }
  return 0;
}

// Gradient of  g_lpV*lp_V + g_lpS*lp_S + g_hV*H_V + g_hS*H_S  with respect to
// the input logits l (dl = dz / T), by the closed forms
//   d lp / dz_j = [j == y] - p_j                      (softmax over the set)
//   d H  / dz_j = -p_j (log p_j + H)
// applied once over the full vocabulary (p) and once over S (q, zero off S).
// Empty support: lp_S is lp_V, so g_lpS flows through the full-vocabulary
// term and H_S (a constant 0) has no gradient.  Target outside a non-empty S:
// lp_S = -inf carries no gradient.  Out-of-range targets and non-finite rows
// get no logprob gradient.  ([SkyRL] Implementation; [xorl] section 1 "VJP".)
int vso_score_grad(int rows, int vocab, int64_t ld, int dtype, const void* logits,
                   const double* temperature, double temperature_scalar,
                   const int32_t* targets, const int32_t* top_k, int32_t top_k_scalar,
                   const double* top_p, double top_p_scalar, const double* min_p,
                   double min_p_scalar, const int32_t* support_ids, int width, int64_t sld,
                   const double* g_lp_full, const double* g_lp_support, const double* g_h_full,
                   const double* g_h_support, double* dlogits) {
  if (rows < 0 || vocab <= 0 || ld < vocab || !logits || !targets || !dlogits) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < rows; ++i) {
    const double T = pick(temperature, i, temperature_scalar);
    RowResult r = score_row(logits, dtype, static_cast<int64_t>(i) * ld, vocab, T, targets[i],
                            pick(top_k, i, top_k_scalar), pick(top_p, i, top_p_scalar),
                            pick(min_p, i, min_p_scalar),
                            support_ids ? support_ids + static_cast<int64_t>(i) * sld : nullptr,
                            width, true);
    double* out = dlogits + static_cast<int64_t>(i) * vocab;
    std::fill(out, out + vocab, 0.0);
    if (r.status & ORC_NONFINITE_INPUT) continue;
    const double glv = g_lp_full ? g_lp_full[i] : 0.0;
    const double gls = g_lp_support ? g_lp_support[i] : 0.0;
    const double ghv = g_h_full ? g_h_full[i] : 0.0;
    const double ghs = g_h_support ? g_h_support[i] : 0.0;
    const int32_t y = targets[i];
    const bool target_ok = !(r.status & ORC_TARGET_OUT_OF_RANGE);
    // Coefficient on the full-vocabulary logprob term.
    double g_full_lp = target_ok ? glv : 0.0;
    double g_supp_lp = 0.0;
    if (target_ok) {
      if (r.support_size == 0)
        g_full_lp += gls;  // lp_S falls back to lp_V
      else if (r.in_support[y])
        g_supp_lp = gls;
    }
    for (int j = 0; j < vocab; ++j) {
      const double logp = (r.z[j] - r.m_full) - r.lz_full;
      const double p = std::exp(logp);
      double dz = g_full_lp * ((j == y ? 1.0 : 0.0) - p) + ghv * (-p * (logp + r.h_full));
      if (r.support_size > 0 && r.in_support[j]) {
        const double logq = (r.z[j] - r.m_support) - r.lz_support;
        const double q = std::exp(logq);
        dz += g_supp_lp * ((j == y ? 1.0 : 0.0) - q) + ghs * (-q * (logq + r.h_support));
      }
      out[j] = dz / T;
    }
  }
  return 0;
}

// Draft/target probability distance ([DSpark] Purpose):
//   p = softmax(draft), q = softmax(target) per row,
//   L1 = sum_j |p_j - q_j|, accept = clamp(1 - 0.5 L1, 0, 1),
//   loss = sum_i w_i L1_i / sum_i w_i  (w = 1 when row_weight is null).
// Gradient with respect to the draft logits only (the target is detached):
//   dloss/dd_j = (w_i / sum w) p_j (s_j - sum_k p_k s_k),  s = sign(p - q),
// which is the softmax Jacobian applied to d|p - q|/dp = s.
// `near_ties` (may be null) counts, per row, elements with |p - q| < tie_eps,
// where a sign decision at lower precision may differ.
//
// Row-sharded batches ([DSpark] Purpose keeps the distributed normalisation
// of the loss): when global_wsum is non-null it is the weight sum over all
// shards, and the loss denominator of the gradient and of loss_num_den[2];
// loss_num_den[0..1] stay this call's numerator and weight sum.
int vso_l1(int rows, int vocab, int64_t ld, int dtype, const void* draft, const void* target,
           const double* row_weight, double* l1, double* accept, double* loss_num_den,
           double* grad, double tie_eps, int32_t* near_ties, const double* global_wsum) {
  if (rows < 0 || vocab <= 0 || ld < vocab || !draft || !target) return 1;
  double local_wsum = 0.0;
  for (int i = 0; i < rows; ++i) local_wsum += row_weight ? row_weight[i] : 1.0;
  const double wsum = global_wsum ? *global_wsum : local_wsum;
  std::vector<double> l1v(rows);
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < rows; ++i) {
    const int64_t off = static_cast<int64_t>(i) * ld;
    std::vector<double> p(vocab), q(vocab);
    double md = -kInf, mt = -kInf;
    for (int j = 0; j < vocab; ++j) {
      p[j] = load_value(draft, dtype, off + j);
      q[j] = load_value(target, dtype, off + j);
      md = std::max(md, p[j]);
      mt = std::max(mt, q[j]);
    }
    double sd = 0.0, st = 0.0;
    for (int j = 0; j < vocab; ++j) {
      p[j] = std::exp(p[j] - md);
      sd += p[j];
      q[j] = std::exp(q[j] - mt);
      st += q[j];
    }
    double dist = 0.0, ps = 0.0;
    int ties = 0;
    for (int j = 0; j < vocab; ++j) {
      p[j] /= sd;
      q[j] /= st;
      const double d = p[j] - q[j];
      dist += std::fabs(d);
      const double s = d > 0 ? 1.0 : (d < 0 ? -1.0 : 0.0);
      ps += p[j] * s;
      if (std::fabs(d) < tie_eps) ++ties;
    }
    l1v[i] = dist;
    if (l1) l1[i] = dist;
    if (accept) accept[i] = std::min(1.0, std::max(0.0, 1.0 - 0.5 * dist));
    if (near_ties) near_ties[i] = ties;
    if (grad) {
      double* g = grad + static_cast<int64_t>(i) * vocab;
      const double w = row_weight ? row_weight[i] : 1.0;
      const double coef = wsum > 0.0 ? w / wsum : 0.0;
      for (int j = 0; j < vocab; ++j) {
        const double d = p[j] - q[j];
        const double s = d > 0 ? 1.0 : (d < 0 ? -1.0 : 0.0);
        g[j] = coef * p[j] * (s - ps);
      }
    }
  }
  if (loss_num_den) {
    double num = 0.0;
    for (int i = 0; i < rows; ++i) num += (row_weight ? row_weight[i] : 1.0) * l1v[i];
    loss_num_den[0] = num;
    loss_num_den[1] = local_wsum;
    loss_num_den[2] = wsum > 0.0 ? num / wsum : 0.0;
  }
  return 0;
}

// Materialise tempered LM-head logits for selected rows:
//   out[r, v] = (sum_k H[rows_sel[r], k] * W[v, k]) / T   in fp64,
// H [*, hidden] bf16 (row stride ldh), W [vocab, hidden] bf16 (row stride ldw).
// The scoring program on these logits is then vso_score with T = 1
// ([xorl] section 1: projection, then the scoring op on its output).
int vso_lmhead_logits(int nsel, const int32_t* rows_sel, int vocab, int hidden,
                      const uint16_t* H, int64_t ldh, const uint16_t* W, int64_t ldw,
                      double temperature, double* out) {
  if (nsel < 0 || vocab <= 0 || hidden <= 0 || !H || !W || !out) return 1;
  std::vector<double> hsel(static_cast<size_t>(nsel) * hidden);
  for (int r = 0; r < nsel; ++r)
    for (int k = 0; k < hidden; ++k)
      hsel[static_cast<size_t>(r) * hidden + k] =
          load_value(H, ORC_BF16, static_cast<int64_t>(rows_sel[r]) * ldh + k);
#pragma omp parallel for schedule(static)
  for (int v = 0; v < vocab; ++v) {
    std::vector<double> w(hidden);
    for (int k = 0; k < hidden; ++k) w[k] = load_value(W, ORC_BF16, static_cast<int64_t>(v) * ldw + k);
    for (int r = 0; r < nsel; ++r) {
      const double* h = hsel.data() + static_cast<size_t>(r) * hidden;
      double acc = 0.0;
      for (int k = 0; k < hidden; ++k) acc += h[k] * w[k];
      out[static_cast<int64_t>(r) * vocab + v] = acc / temperature;
    }
  }
  return 0;
}

}  // extern "C"

namespace {

// ---------------------------------------------------------------------------
// Seeded Gumbel-max sampling over the support ([xorl] section 3: the
// program ends in a "seeded gumbel" step; the pages fix neither the
// generator nor the noise recipe, so this is the project's reading):
//
//   score_j = fl32(l_j / T) + G_j,   G_j = -log(-log U_j)      (fp32)
//   y       = argmax over j in S of score_j, the smallest j among equal scores
//   U_j     = (bits 63..40 of r_j + 1/2) * 2^-24,  r_j = word (j mod 4) of
//             Philox4x64-10(counter = (floor(j / 4), 0, 0, 0), key = (seed, row))
//
// The decision is taken in fp32 with one fixed sequence of IEEE operations
// (each rounded separately, no fused multiply-add), so any implementation
// that follows the same sequence reaches the same token.

uint64_t mulhilo64(uint64_t a, uint64_t b, uint64_t* hi) {
  const unsigned __int128 p = static_cast<unsigned __int128>(a) * b;
  *hi = static_cast<uint64_t>(p >> 64);
  return static_cast<uint64_t>(p);
}

// Philox4x64 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011): each round multiplies words 0 and
// 2 by the two Philox-4x64 multipliers, swaps and xors the halves with the
// round key; the key advances by the two Weyl constants between rounds.
void philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
  uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint64_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    uint64_t hi0, hi1;
    const uint64_t lo0 = mulhilo64(M0, x0, &hi0);
    const uint64_t lo1 = mulhilo64(M1, x2, &hi1);
    const uint64_t y0 = hi1 ^ x1 ^ k0, y2 = hi0 ^ x3 ^ k1;
    x0 = y0;
    x1 = lo1;
    x2 = y2;
    x3 = lo0;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

// Natural logarithm of a positive normal fp32 value: x = m 2^e with m in
// [sqrt(1/2), sqrt(2)), log m = 2 atanh(s), s = (m - 1) / (m + 1), by the
// series 2 (s + s^3/3 + s^5/5 + s^7/7 + s^9/9) (|s| < 0.172, so the next
// term is below 2^-29 of the sum), and e ln 2 with ln 2 split into a head
// exact in fp32 products and a tail (Cody and Waite's reduction).
float log_f32(float x) {
  uint32_t b;
  std::memcpy(&b, &x, 4);
  int e = static_cast<int>(b >> 23) - 127;
  uint32_t mb = (b & 0x007FFFFFu) | 0x3F800000u;
  float m;
  std::memcpy(&m, &mb, 4);
  if (m > 1.41421356f) {
    m = m * 0.5f;
    e += 1;
  }
  const float f = m - 1.0f;
  const float s = f / (f + 2.0f);
  const float z = s * s;
  float t = 1.0f / 9.0f;
  t = t * z;
  t = t + 1.0f / 7.0f;
  t = t * z;
  t = t + 1.0f / 5.0f;
  t = t * z;
  t = t + 1.0f / 3.0f;
  const float s2 = s * 2.0f;
  const float zt = z * t;
  const float lm = s2 + s2 * zt;
  const float ef = static_cast<float>(e);
  const float ln2_hi = 0.693145751953125f;       // 0x3F317200
  const float ln2_lo = 1.42860677e-06f;          // fl32(ln 2 - ln2_hi)
  const float tail = ef * ln2_lo + lm;
  return ef * ln2_hi + tail;
}

// U_j and G_j of the recipe above.
float gumbel_f32(uint64_t seed, int row, int64_t j) {
  const uint64_t ctr[4] = {static_cast<uint64_t>(j) >> 2, 0, 0, 0};
  const uint64_t key[2] = {seed, static_cast<uint64_t>(row)};
  uint64_t w[4];
  philox4x64_10(ctr, key, w);
  const uint64_t r = w[j & 3];
  const float u = (static_cast<float>(r >> 40) + 0.5f) * 5.9604644775390625e-08f;  // 2^-24
  return -log_f32(-log_f32(u));
}

}  // namespace

extern "C" {

// One Philox4x64-10 block (for the tests that pin the generator).
void vso_philox4x64_10(const uint64_t* ctr, const uint64_t* key, uint64_t* out) {
  philox4x64_10(ctr, key, out);
}

float vso_log_f32(float x) { return log_f32(x); }

float vso_gumbel_f32(uint64_t seed, int row, int64_t j) { return gumbel_f32(seed, row, j); }

// Sample one token per row from the support given as a byte mask
// ([rows, vocab], 1 = in S): y = argmax_{j in S} fl32(l_j / T) + G_j, the
// smallest j on equal scores; -1 when the row's support is empty.
// temperature (fp32 per row) may be null, then temperature_scalar.
int vso_gumbel_sample(int rows, int vocab, int64_t ld, int dtype, const void* logits,
                      const float* temperature, float temperature_scalar, const uint8_t* mask,
                      uint64_t seed, int32_t* out) {
  if (rows < 0 || vocab <= 0 || ld < vocab || !logits || !mask || !out) return 1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < rows; ++i) {
    const float T = temperature ? temperature[i] : temperature_scalar;
    int32_t best = -1;
    float best_score = 0.f;
    for (int j = 0; j < vocab; ++j) {
      if (!mask[static_cast<int64_t>(i) * vocab + j]) continue;
      const float l = static_cast<float>(load_value(logits, dtype, static_cast<int64_t>(i) * ld + j));
      const float score = l / T + gumbel_f32(seed, i, j);
      if (best < 0 || score > best_score) {
        best = j;
        best_score = score;
      }
    }
    out[i] = best;
  }
  return 0;
}

}  // extern "C"
