// Forward scoring kernels.
//
//  (The computed-support kernel lives in score_row.cu.)
//  * score_recorded_kernel: recorded support (SkyRL PR #2004,
//    "Implementation": dense -1-padded id list).  One CTA per row gathers the
//    support logits; rows with an empty support (full-vocabulary fallback),
//    or every row when full statistics are requested, also stream the whole
//    row once with 16-byte loads.  A requested sample is the seeded
//    Gumbel-max token over the kept ids (noise recipe in gumbel.cuh).

#include <climits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "gumbel.cuh"
#include "internal.h"

namespace vs {

namespace {

// ---------------------------------------------------------------------------
// recorded support

constexpr int kRecThreads = 256;
constexpr int kRecUnroll = 8;  // 16-byte loads in flight per thread on a full-row stream

template <typename Raw>
__global__ void __launch_bounds__(kRecThreads) score_recorded_kernel(ScoreParams P) {
  constexpr int VEC = 16 / sizeof(Raw);
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int V = P.vocab;
  const int W = P.support_width;
  __shared__ int32_t ids[VS_MAX_SUPPORT_WIDTH];
  __shared__ float vals[VS_MAX_SUPPORT_WIDTH];  // kept support values, NaN elsewhere
  __shared__ Stats red[kRecThreads / 32];
  __shared__ uint32_t ured[kRecThreads / 32];
  __shared__ float fred[kRecThreads / 32];
  __shared__ uint32_t flags_sh;
  __shared__ int32_t target_hit;
  __shared__ unsigned long long kred[kRecThreads / 32];

  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  const int32_t* srow = P.support_ids + static_cast<int64_t>(row) * P.support_ld;
  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const float c = kLog2e / T;
  const int y = P.targets[row];
  const bool target_ok = y >= 0 && y < V;

  if (tid == 0) {
    flags_sh = 0;
    target_hit = 0;
  }
  for (int w = tid; w < W; w += blockDim.x) ids[w] = srow[w];
  __syncthreads();

  // kept: id valid and first occurrence; gather the kept values
  uint32_t local_flags = 0;
  uint32_t nkeep = 0;
  bool nonfinite_sup = false;
  float lmax = -kInf;
  for (int w = tid; w < W; w += blockDim.x) {
    const int32_t id = ids[w];
    vals[w] = __int_as_float(0x7fc00000);
    if (id == -1) continue;
    if (id < -1 || id >= V) {
      local_flags |= VS_ROW_BAD_SUPPORT_ID;
      continue;
    }
    bool dup = false;
    for (int w2 = 0; w2 < w; ++w2)
      if (ids[w2] == id) {
        dup = true;
        break;
      }
    if (dup) {
      local_flags |= VS_ROW_DUP_SUPPORT_ID;
      continue;
    }
    ++nkeep;
    const float x = value_of(grow[id]);
    if (!isfinite(x)) nonfinite_sup = true;
    vals[w] = x;
    lmax = fmaxf(lmax, x);
    if (id == y) target_hit = 1;
  }
  if (local_flags) atomicOr(&flags_sh, local_flags);
  nkeep = block_sum(nkeep, ured);
  const uint32_t any_nf = block_sum(static_cast<uint32_t>(nonfinite_sup), ured);
  const bool empty = nkeep == 0;
  // support statistics relative to the support maximum (value domain)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if ((tid & 31) == 0) fred[tid >> 5] = lmax;
  __syncthreads();
  float vsmax = -kInf;
  for (int i = 0; i < kRecThreads / 32; ++i) vsmax = fmaxf(vsmax, fred[i]);
  __syncthreads();
  Stats s{vsmax, 0.f, 0.f, 0.f};
  for (int w = tid; w < W; w += blockDim.x) {
    const float x = vals[w];
    if (x != x) continue;  // not kept
    const float d = (x - vsmax) * c;
    const float e = ex2(d);
    if (d == 0.f)
      s.c0 += 1.f;
    else
      s.zr += e;
    s.a = fmaf(d, e, s.a);
  }
  s.c0 = block_sum(s.c0, fred);
  s.zr = block_sum(s.zr, fred);
  s.a = block_sum(s.a, fred);

  // full-vocabulary statistics: for empty rows (fallback) or on request
  const bool need_full = empty || P.full_stats;
  Stats f = stats_empty();
  float fvmax = -kInf;  // value-domain maximum of the row
  if (need_full) {
    const int nfull = V / VEC;
    const uint4* g4 = reinterpret_cast<const uint4*>(grow);
    int v = tid;
    if constexpr (sizeof(Raw) == 2) {
      // packed statistics, four chains, kRecUnroll vectors in flight; the
      // block maximum of every thread's first round seeds the chains'
      // running maximum, so that later vectors rarely raise it
      Stats f4[4] = {stats_empty(), stats_empty(), stats_empty(), stats_empty()};
      const f32x2 c2 = pack2(c, c);
      uint4 q[kRecUnroll];
      uint32_t mx = 0xFF80FF80u;  // (-inf, -inf)
#pragma unroll
      for (int k = 0; k < kRecUnroll; ++k) {
        const int vk = v + k * kRecThreads;
        q[k] = vk < nfull ? __ldcs(g4 + vk) : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
        mx = bmax2(mx, bmax2(bmax2(q[k].x, q[k].y), bmax2(q[k].z, q[k].w)));
      }
      float m1 = fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xFFFF0000u));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      if ((tid & 31) == 0) fred[tid >> 5] = m1;
      __syncthreads();
      m1 = -kInf;
      for (int i = 0; i < kRecThreads / 32; ++i) m1 = fmaxf(m1, fred[i]);
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 4; ++k) f4[k].m = __fmul_rn(m1, c);
      for (;;) {
#pragma unroll
        for (int k = 0; k < kRecUnroll; ++k)
          if (v + k * kRecThreads < nfull) stats_vec_bf16(q[k], c, c2, f4[k & 3], fvmax);
        v += kRecUnroll * kRecThreads;
        if (v >= nfull) break;
#pragma unroll
        for (int k = 0; k < kRecUnroll; ++k) {
          const int vk = v + k * kRecThreads;
          q[k] = vk < nfull ? __ldcs(g4 + vk) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      f = f4[0];
      stats_merge(f, f4[1]);
      stats_merge(f, f4[2]);
      stats_merge(f, f4[3]);
    } else {
      for (; v + 3 * kRecThreads < nfull; v += 4 * kRecThreads) {
        uint4 q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __ldcs(g4 + v + k * kRecThreads);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          Raw r[VEC];
          unpack(q[k], r);
          float u[VEC];
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            const float x = value_of(r[i]);
            fvmax = fmaxf(fvmax, x);
            u[i] = __fmul_rn(x, c);
          }
          stats_add(f, u);
        }
      }
      for (; v < nfull; v += kRecThreads) {
        Raw r[VEC];
        unpack(__ldcs(g4 + v), r);
        float u[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          const float x = value_of(r[i]);
          fvmax = fmaxf(fvmax, x);
          u[i] = __fmul_rn(x, c);
        }
        stats_add(f, u);
      }
    }
    for (int j = nfull * VEC + tid; j < V; j += kRecThreads) {
      const float x = value_of(grow[j]);
      fvmax = fmaxf(fvmax, x);
      float u[1] = {__fmul_rn(x, c)};
      stats_add(f, u);
    }
    f = block_reduce(f, red);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) fvmax = fmaxf(fvmax, __shfl_xor_sync(0xffffffffu, fvmax, o));
    if ((tid & 31) == 0) fred[tid >> 5] = fvmax;
    __syncthreads();
    fvmax = -kInf;
    for (int i = 0; i < kRecThreads / 32; ++i) fvmax = fmaxf(fvmax, fred[i]);
  }

  if (tid == 0) {
    const float nan = __int_as_float(0x7fc00000);
    uint32_t status = flags_sh;
    bool nonfinite = any_nf != 0;
    float m2 = nan, log2z = nan, h_full = nan;
    if (need_full) {
      if (!stats_finite(f)) nonfinite = true;
      m2 = f.m;
      log2z = stats_log2z(f);
      h_full = kLn2 * (log2z - f.a / stats_z(f));
    }
    const float msup = vsmax;
    const float log2zs = empty ? nan : stats_log2z(s);
    const float h_sup = empty ? 0.f : kLn2 * (log2zs - s.a / stats_z(s));
    float lp_v = nan, lp_s = nan;
    bool in_s = false;
    if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
    if (nonfinite) {
      status |= VS_ROW_NONFINITE_INPUT;
    } else if (target_ok) {
      const float uy = __fmul_rn(value_of(grow[y]), c);
      if (need_full) lp_v = kLn2 * (uy - m2 - log2z);
      in_s = target_hit != 0;
      if (empty) {
        lp_s = lp_v;
      } else if (in_s) {
        lp_s = kLn2 * ((value_of(grow[y]) - msup) * c - log2zs);
      } else {
        lp_s = -kInf;
        status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
      }
    }
    const bool valid = !nonfinite && !empty;
    if (P.lp_full) P.lp_full[row] = lp_v;
    if (P.lp_support) P.lp_support[row] = lp_s;
    if (P.want_entropy) {
      if (P.h_full) P.h_full[row] = nonfinite ? nan : h_full;
      if (P.h_support) P.h_support[row] = nonfinite ? nan : h_sup;
    }
    if (P.valid) P.valid[row] = valid ? 1 : 0;
    if (P.status) P.status[row] = status;
    if (P.support_size) P.support_size[row] = nonfinite ? 0 : static_cast<int32_t>(nkeep);
    if (P.ctx) {
      RowCtx cx{};
      cx.m2 = fvmax;  // value domain (the stream's sums are relative to fl(fvmax c))
      cx.log2z = log2z;
      cx.msup = msup;
      cx.log2zs = log2zs;
      cx.h_full = h_full;
      cx.h_support = h_sup;
      cx.c = c;
      cx.tkey = 0;
      cx.tie_cut = 0;
      uint32_t fl = kCtxRecorded;
      if (need_full) fl |= kCtxFullStats;
      if (nonfinite) fl |= kCtxNonFinite;
      if (empty || nonfinite) fl |= kCtxEmpty;
      if (target_ok) fl |= kCtxTargetOk;
      if (in_s) fl |= kCtxTargetInS;
      cx.flags = fl;
      cx.n_support = nonfinite ? 0 : static_cast<int32_t>(nkeep);
      cx.status = status;
      cx.c0_full = f.c0;
      cx.zr_full = f.zr;
      cx.c0_sup = s.c0;
      cx.zr_sup = s.zr;
      P.ctx[row] = cx;
    }
  }
  // seeded Gumbel-max token over the kept ids
  if (P.sampled) {
    unsigned long long best = 0ull;
    // a non-finite row (its support, or the whole row when its statistics
    // were taken) samples nothing
    if (!empty && any_nf == 0 && !(need_full && !stats_finite(f))) {
      for (int w = tid; w < W; w += blockDim.x) {
        const float x = vals[w];
        if (x != x) continue;  // not kept
        const int32_t id = ids[w];
        float g[4];
        gumbel4(P.sample_seed, static_cast<uint32_t>(P.row_base + row), static_cast<uint64_t>(id) >> 2, g);
        const unsigned long long k = gumbel_key(gumbel_score(x, T, g[id & 3]), id);
        best = k > best ? k : best;
      }
    }
    best = block_max_key(best, kred);
    if (tid == 0) P.sampled[row] = gumbel_key_id(best);
  }

  // support bitmask: clear the row, then set the kept ids
  if (P.support_mask) {
    const int64_t wstride = (V + 31) / 32;
    uint32_t* mrow = P.support_mask + static_cast<int64_t>(row) * wstride;
    for (int64_t w = tid; w < wstride; w += blockDim.x) mrow[w] = 0u;
    __syncthreads();
    if (any_nf == 0) {
      for (int w = tid; w < W; w += blockDim.x) {
        const int32_t id = ids[w];
        if (id < 0 || id >= V) continue;
        atomicOr(&mrow[id >> 5], 1u << (id & 31));
      }
    }
  }
}

// Deterministic reduction of the entropy sum and valid count over rows.
__global__ void score_reduce_kernel(const float* h_support, const uint8_t* valid, int rows,
                                    double* entropy_sum, int32_t* valid_count) {
  __shared__ double dred[32];
  __shared__ int ired[32];
  double s = 0.0;
  int cnt = 0;
  for (int i = threadIdx.x; i < rows; i += blockDim.x) {
    if (valid[i]) {
      ++cnt;
      if (h_support) s += static_cast<double>(h_support[i]);
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  }
  if (lane == 0) {
    dred[warp] = s;
    ired[warp] = cnt;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    int tc = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
      t += dred[w];
      tc += ired[w];
    }
    if (entropy_sum) *entropy_sum = t;
    if (valid_count) *valid_count = tc;
  }
}

}  // namespace

// Rows are streamed through one CTA each, so the vocabulary is bounded only
// by the index types (kept below 2^26).
int score_max_vocab(vs_dtype dtype) {
  (void)dtype;
  return 1 << 26;
}

cudaError_t launch_score_recorded(const ScoreParams& p, vs_dtype dtype, cudaStream_t s) {
  if (dtype == VS_BF16)
    score_recorded_kernel<uint16_t><<<p.rows, kRecThreads, 0, s>>>(p);
  else
    score_recorded_kernel<uint32_t><<<p.rows, kRecThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_score_reduce(const float* h_support, const uint8_t* valid, int rows,
                                double* entropy_sum, int32_t* valid_count, cudaStream_t s) {
  score_reduce_kernel<<<1, 1024, 0, s>>>(h_support, valid, rows, entropy_sum, valid_count);
  return cudaGetLastError();
}

}  // namespace vs
