// Backward of the forward scores by the closed forms (xorl issue #71,
// section 1 "selected logprob + VJP"; SkyRL PR #2004, "Implementation"):
//
//   dl_j = (1/T) ( g_lpV ([j==y] - p_j) + g_lpS 1_S(j) ([j==y] - q_j)
//                - g_HV p_j (log p_j + H_V) - g_HS 1_S(j) q_j (log q_j + H_S) )
//
// The dense kernel is a pure stream: one 16-byte load of logits and one
// 16-byte (bf16) or 32-byte (fp32) store of gradients per 8 elements, with
// the per-row constants taken from the forward's saved state.  Computed
// supports are tested per element by their threshold key and tie cut;
// recorded supports by a per-CTA bitmap built in shared memory from the id
// list.

#include <climits>

#include "common.cuh"
#include "internal.h"

namespace vs {

namespace {

constexpr int kThreads = 256;

template <typename G>
struct GradStore;
template <>
struct GradStore<float> {
  __device__ static float load(const float* p) { return *p; }
  __device__ static void store(float* p, float v) { *p = v; }
};
template <>
struct GradStore<uint16_t> {
  __device__ static float load(const uint16_t* p) {
    return __uint_as_float(static_cast<uint32_t>(*p) << 16);
  }
  __device__ static void store(uint16_t* p, float v) {
    *p = static_cast<uint16_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
  }
};

// Coefficients of one row.
struct RowCoef {
  float gv, gs, ghv, ghs;  // effective upstream gradients
  float m2, log2z, msup, log2zs, h_full, h_sup, c, scale;
  float omp_full, omp_sup;  // 1 - p_y and 1 - q_y when y holds the maximum
  uint32_t tkey;
  int32_t tie_cut;
  uint32_t flags;
  int32_t y;
  bool need_full, need_sup, zero;
};

__device__ __forceinline__ RowCoef row_coef(const BwdParams& P, int row) {
  const RowCtx cx = P.ctx[row];
  RowCoef k;
  const bool tok = cx.flags & kCtxTargetOk;
  const bool empty = cx.flags & kCtxEmpty;
  const float glv = P.g_lp_full ? P.g_lp_full[row] : 0.f;
  const float gls = P.g_lp_support ? P.g_lp_support[row] : 0.f;
  k.ghv = P.g_h_full ? P.g_h_full[row] : 0.f;
  k.ghs = (P.g_h_support && !empty) ? P.g_h_support[row] : 0.f;
  k.gv = tok ? glv + (empty ? gls : 0.f) : 0.f;
  k.gs = (tok && !empty && (cx.flags & kCtxTargetInS)) ? gls : 0.f;
  k.m2 = cx.m2;
  k.log2z = cx.log2z;
  k.msup = cx.msup;
  k.log2zs = cx.log2zs;
  k.h_full = cx.h_full;
  k.h_sup = cx.h_support;
  k.c = cx.c;
  k.scale = cx.c * kLn2;  // 1 / T
  k.tkey = cx.tkey;
  k.tie_cut = cx.tie_cut;
  k.flags = cx.flags;
  k.y = P.targets[row];
  k.zero = (cx.flags & kCtxNonFinite) != 0;
  k.omp_full = (cx.c0_full - 1.f + cx.zr_full) / (cx.c0_full + cx.zr_full);
  k.omp_sup = (cx.c0_sup - 1.f + cx.zr_sup) / (cx.c0_sup + cx.zr_sup);
  k.need_full = !k.zero && (k.gv != 0.f || k.ghv != 0.f);
  k.need_sup = !k.zero && !empty && (k.gs != 0.f || k.ghs != 0.f);
  return k;
}

// [j == y] - p_j, with 1 - p_y taken from the split normaliser when y holds
// the maximum (there 1 - p_y = (c0 - 1 + zr) / (c0 + zr) without cancellation).
__device__ __forceinline__ float ind_minus(float p, bool is_y, bool is_max, float omp) {
  if (!is_y) return -p;
  return is_max ? omp : 1.f - p;
}

// u is the raw logit value; row maxima in the saved state are raw values too.
__device__ __forceinline__ float grad_elem(const RowCoef& k, float u, int j, bool in_s) {
  float dz = 0.f;
  const bool is_y = j == k.y;
  if (k.need_full) {
    const float d = (u - k.m2) * k.c;
    const float lp2 = d - k.log2z;
    const float p = ex2(lp2);
    dz += k.gv * ind_minus(p, is_y, d == 0.f, k.omp_full) - k.ghv * p * fmaf(lp2, kLn2, k.h_full);
  }
  if (in_s && k.need_sup) {
    const float d = (u - k.msup) * k.c;
    const float lq2 = d - k.log2zs;
    const float q = ex2(lq2);
    dz += k.gs * ind_minus(q, is_y, d == 0.f, k.omp_sup) - k.ghs * q * fmaf(lq2, kLn2, k.h_sup);
  }
  return dz * k.scale;
}

template <typename Raw, typename G, bool ACC>
__global__ void __launch_bounds__(kThreads) score_bwd_kernel(BwdParams P, int nchunks) {
  constexpr int VEC = 16 / sizeof(Raw);
  extern __shared__ __align__(16) uint32_t bitmap[];  // recorded support bits of this slice
  __shared__ float fred[kThreads / 32];
  const int row = blockIdx.x / nchunks;
  const int part = blockIdx.x % nchunks;
  const int V = P.vocab;
  const int c0 = part * P.chunk;
  const int c1 = min(V, c0 + P.chunk);
  const int n = max(0, c1 - c0);
  RowCoef k = row_coef(P, row);
  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  G* gout = static_cast<G*>(P.dlogits) + static_cast<int64_t>(row) * P.grad_ld;
  const bool recorded = k.flags & kCtxRecorded;
  const bool all_vocab = k.flags & kCtxAllVocab;

  // full-vocabulary statistics missing from the forward (recorded support
  // without full statistics): this launch covers whole rows, compute them.
  if (k.need_full && !(k.flags & kCtxFullStats)) {
    // maximum, then sums relative to it (value domain, as the forward)
    const int nfull = V / VEC;
    const uint4* g4 = reinterpret_cast<const uint4*>(grow);
    float vm = -kInf;
    for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
      Raw r[VEC];
      unpack(g4[v], r);
#pragma unroll
      for (int i = 0; i < VEC; ++i) vm = fmaxf(vm, value_of(r[i]));
    }
    for (int j = nfull * VEC + threadIdx.x; j < V; j += blockDim.x) vm = fmaxf(vm, value_of(grow[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
    if ((threadIdx.x & 31) == 0) fred[threadIdx.x >> 5] = vm;
    cta_sync();
    vm = -kInf;
    for (int i = 0; i < kThreads / 32; ++i) vm = fmaxf(vm, fred[i]);
    cta_sync();
    float c0 = 0.f, zr = 0.f, a = 0.f;
    for (int j = threadIdx.x; j < V; j += blockDim.x) {
      const float d = (value_of(grow[j]) - vm) * k.c;
      const float e = ex2(d);
      if (d == 0.f)
        c0 += 1.f;
      else
        zr += e;
      a = fmaf(d, e, a);
    }
    c0 = block_sum(c0, fred);
    zr = block_sum(zr, fred);
    a = block_sum(a, fred);
    const Stats s{vm, c0, zr, a};
    k.m2 = vm;
    k.log2z = stats_log2z(s);
    k.h_full = kLn2 * (k.log2z - s.a / stats_z(s));
    k.omp_full = (s.c0 - 1.f + s.zr) / (s.c0 + s.zr);
  }

  if (recorded && k.need_sup) {
    const int words = (n + 31) / 32;
    for (int w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0u;
    cta_sync();
    const int32_t* srow = P.support_ids + static_cast<int64_t>(row) * P.support_ld;
    for (int w = threadIdx.x; w < P.support_width; w += blockDim.x) {
      const int32_t id = srow[w];
      if (id >= c0 && id < c1) atomicOr(&bitmap[(id - c0) >> 5], 1u << ((id - c0) & 31));
    }
    cta_sync();
  }

  auto in_support = [&](int jl, Raw raw) -> bool {
    if (!k.need_sup) return false;
    if (all_vocab) return true;
    if (recorded) return (bitmap[jl >> 5] >> (jl & 31)) & 1u;
    const uint32_t key = key_of(raw);
    return key > k.tkey || (key == k.tkey && (c0 + jl) <= k.tie_cut);
  };

  const int nfull = n / VEC;
  const uint4* g4 = reinterpret_cast<const uint4*>(grow + c0);
  for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
    float out[VEC];
    // off-support elements of a recorded support carry no gradient unless a
    // full-vocabulary term is active: such groups are written as zeros (or
    // left alone when accumulating) without reading their logits
    bool load = k.need_full || k.need_sup;
    if (load && recorded && !k.need_full) {
      const int j0 = v * VEC;
      load = ((bitmap[j0 >> 5] >> (j0 & 31)) & ((1u << VEC) - 1u)) != 0u;
    }
    if (ACC && !load) continue;
    if (load) {
      Raw r[VEC];
      unpack(__ldcs(g4 + v), r);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const int jl = v * VEC + i;
        out[i] = grad_elem(k, value_of(r[i]), c0 + jl, in_support(jl, r[i]));
      }
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) out[i] = 0.f;
    }
    G* dst = gout + c0 + v * VEC;
    if (ACC) {
#pragma unroll
      for (int i = 0; i < VEC; ++i) out[i] += GradStore<G>::load(dst + i);
    }
    if constexpr (sizeof(G) == 2) {
      uint32_t w[VEC / 2];
#pragma unroll
      for (int i = 0; i < VEC / 2; ++i) {
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(out[2 * i]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(out[2 * i + 1]));
        w[i] = lo | (hi << 16);
      }
      if constexpr (VEC == 8) {
        __stcs(reinterpret_cast<uint4*>(dst), make_uint4(w[0], w[1], w[2], w[3]));
      } else {
        __stcs(reinterpret_cast<uint2*>(dst), make_uint2(w[0], w[1]));
      }
    } else {
#pragma unroll
      for (int i = 0; i < VEC; i += 4)
        __stcs(reinterpret_cast<float4*>(dst + i), make_float4(out[i], out[i + 1], out[i + 2], out[i + 3]));
    }
  }
  for (int jl = nfull * VEC + threadIdx.x; jl < n; jl += blockDim.x) {
    const Raw raw = grow[c0 + jl];
    float g = 0.f;
    if (k.need_full || k.need_sup)
      g = grad_elem(k, value_of(raw), c0 + jl, in_support(jl, raw));
    G* dst = gout + c0 + jl;
    if (ACC) g += GradStore<G>::load(dst);
    GradStore<G>::store(dst, g);
  }
}

// Sparse gradient for a recorded support: out[row, w] for each listed id.
template <typename Raw>
__global__ void __launch_bounds__(kThreads) score_bwd_sparse_kernel(BwdParams P) {
  const int row = blockIdx.x;
  const RowCoef k = row_coef(P, row);
  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  const int32_t* srow = P.support_ids + static_cast<int64_t>(row) * P.support_ld;
  float* gout = static_cast<float*>(P.dlogits) + static_cast<int64_t>(row) * P.grad_ld;
  for (int w = threadIdx.x; w < P.support_width; w += blockDim.x) {
    const int32_t id = srow[w];
    float g = 0.f;
    if (id >= 0 && id < P.vocab && k.need_sup) {
      bool dup = false;
      for (int w2 = 0; w2 < w; ++w2)
        if (srow[w2] == id) {
          dup = true;
          break;
        }
      if (!dup) {
        RowCoef ks = k;
        ks.need_full = false;  // full-vocabulary terms are not representable here
        g = grad_elem(ks, value_of(grow[id]), id, true);
      }
    }
    gout[w] = g;
  }
}

template <typename Raw, typename G>
cudaError_t launch_dense(const BwdParams& p, int mode, int nchunks, cudaStream_t s) {
  const size_t smem = static_cast<size_t>((p.chunk + 31) / 32) * sizeof(uint32_t);
  const unsigned grid = static_cast<unsigned>(p.rows) * static_cast<unsigned>(nchunks);
  if (mode == VS_GRAD_ACCUMULATE) {
    cudaFuncSetAttribute(score_bwd_kernel<Raw, G, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    score_bwd_kernel<Raw, G, true><<<grid, kThreads, smem, s>>>(p, nchunks);
  } else {
    cudaFuncSetAttribute(score_bwd_kernel<Raw, G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    score_bwd_kernel<Raw, G, false><<<grid, kThreads, smem, s>>>(p, nchunks);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_bwd(const BwdParams& p, vs_dtype dtype, vs_dtype gdtype, int mode,
                             bool whole_rows, int nchunks, cudaStream_t s) {
  (void)whole_rows;
  if (mode == VS_GRAD_SPARSE) {
    if (dtype == VS_BF16)
      score_bwd_sparse_kernel<uint16_t><<<p.rows, kThreads, 0, s>>>(p);
    else
      score_bwd_sparse_kernel<uint32_t><<<p.rows, kThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  if (dtype == VS_BF16) {
    if (gdtype == VS_BF16) return launch_dense<uint16_t, uint16_t>(p, mode, nchunks, s);
    return launch_dense<uint16_t, float>(p, mode, nchunks, s);
  }
  if (gdtype == VS_BF16) return launch_dense<uint32_t, uint16_t>(p, mode, nchunks, s);
  return launch_dense<uint32_t, float>(p, mode, nchunks, s);
}

}  // namespace vs
