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
  cta_sync();

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
  cta_sync();
  float vsmax = -kInf;
  for (int i = 0; i < kRecThreads / 32; ++i) vsmax = fmaxf(vsmax, fred[i]);
  cta_sync();
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
      Chain f4[4] = {chain_empty(), chain_empty(), chain_empty(), chain_empty()};
      uint32_t vm2 = 0xFF80FF80u;
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
      cta_sync();
      m1 = -kInf;
      for (int i = 0; i < kRecThreads / 32; ++i) m1 = fmaxf(m1, fred[i]);
      cta_sync();
#pragma unroll
      for (int k = 0; k < 4; ++k) chain_seed(f4[k], m1, c);
      for (;;) {
#pragma unroll
        for (int k = 0; k < kRecUnroll; ++k)
          if (v + k * kRecThreads < nfull) chain_vec(q[k], c, c2, f4[k & 3], vm2);
        v += kRecUnroll * kRecThreads;
        if (v >= nfull) break;
#pragma unroll
        for (int k = 0; k < kRecUnroll; ++k) {
          const int vk = v + k * kRecThreads;
          q[k] = vk < nfull ? __ldcs(g4 + vk) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      f = f4[0].s;
      stats_merge(f, f4[1].s);
      stats_merge(f, f4[2].s);
      stats_merge(f, f4[3].s);
      fvmax = fmaxf(fvmax, vmax_of(vm2));
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
    cta_sync();
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
    cta_sync();
    if (any_nf == 0) {
      for (int w = tid; w < W; w += blockDim.x) {
        const int32_t id = ids[w];
        if (id < 0 || id >= V) continue;
        atomicOr(&mrow[id >> 5], 1u << (id & 31));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// full-vocabulary statistics of the rows that need them (an empty recorded
// support, or every row when they are requested), spread over the whole GPU:
// a list of those rows, then (row, chunk) work items of one warp's 32 x
// kFsVecs 16-byte vectors taken by a persistent grid of warps, each writing
// one partial; the warp-per-row kernel merges a row's partials.

constexpr int kFsVecs = 16;        // 16-byte vectors per lane of one work item
constexpr int kFsThreads = 256;

// One work item's statistics and maximum (20 bytes).
struct FsPart {
  Stats s;
  float vmax;
};

// Elements of one work item: one warp's 32 x kFsVecs vectors.
__host__ __device__ inline int fs_chunk(int esize) { return 32 * kFsVecs * (16 / esize); }

// Workspace of the narrow-list recorded path: [count | slot[rows] | list[rows]
// | parts[rows][nch]], 16-byte aligned pieces.
struct FsLayout {
  size_t slot, list, parts, bytes;
  int nch;
};
__host__ __device__ inline FsLayout fs_layout(int rows, int vocab, int esize) {
  FsLayout l;
  const int ch = fs_chunk(esize);
  l.nch = (vocab + ch - 1) / ch;
  l.slot = 16;
  l.list = l.slot + ((static_cast<size_t>(rows) * 4 + 15) & ~size_t(15));
  l.parts = l.list + ((static_cast<size_t>(rows) * 4 + 15) & ~size_t(15));
  l.bytes = l.parts + ((static_cast<size_t>(rows) * l.nch * sizeof(FsPart) + 15) & ~size_t(15));
  return l;
}

__device__ __forceinline__ void fs_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void fs_pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// One warp per row: does the row need full-vocabulary statistics?  Those
// rows are appended to the list (any order: each row's result does not
// depend on its place) and their list index kept in slot[row] (-1: none).
__global__ void __launch_bounds__(256) fs_list_kernel(ScoreParams P, int32_t* count, int32_t* slot,
                                                       int32_t* list) {
  fs_pdl_wait();
  fs_pdl_launch();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= P.rows) return;
  const int32_t* srow = P.support_ids + static_cast<int64_t>(row) * P.support_ld;
  bool any = false;
  for (int w = lane; w < P.support_width; w += 32) {
    const int32_t id = srow[w];
    any |= id >= 0 && id < P.vocab;
  }
  const bool need = P.full_stats || !__any_sync(0xffffffffu, any);
  if (lane == 0) {
    int32_t idx = -1;
    if (need) {
      idx = atomicAdd(count, 1);
      list[idx] = row;
    }
    slot[row] = idx;
  }
}

// Persistent grid of warps over the work items (list index, chunk): each
// warp takes every W-th item (W = the grid's warps), loads its 32 x kFsVecs
// vectors at once and writes one partial, with no block barrier.
template <typename Raw>
__global__ void __launch_bounds__(kFsThreads) fs_chunk_kernel(ScoreParams P, const int32_t* count,
                                                              const int32_t* list, FsPart* parts,
                                                              int nch) {
  constexpr int VEC = 16 / sizeof(Raw);
  constexpr int CH = 32 * kFsVecs * VEC;
  fs_pdl_wait();
  fs_pdl_launch();
  const int items = *count * nch;
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (kFsThreads / 32);
  for (int it = blockIdx.x * (kFsThreads / 32) + (threadIdx.x >> 5); it < items; it += nw) {
    const int row = list[it / nch];
    const int j0 = (it % nch) * CH, j1 = min(P.vocab, j0 + CH);
    const Raw* g = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld + j0;
    const uint4* g4 = reinterpret_cast<const uint4*>(g);
    const int nv = (j1 - j0) / VEC;
    uint4 q[kFsVecs];
#pragma unroll
    for (int k = 0; k < kFsVecs; ++k) {
      const int v = lane + 32 * k;
      q[k] = v < nv ? __ldcs(g4 + v) : make_uint4(0u, 0u, 0u, 0u);
    }
    const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
    const float c = kLog2e / T;
    Stats s = stats_empty();
    float vmax = -kInf;
    if constexpr (sizeof(Raw) == 2) {
      // the chains start at the warp's largest value, so that only the
      // vectors holding it take the scalar path
      uint32_t vm2 = 0xFF80FF80u;
#pragma unroll
      for (int k = 0; k < kFsVecs; ++k)
        if (lane + 32 * k < nv) vm2 = bmax2(vm2, bmax2(bmax2(q[k].x, q[k].y), bmax2(q[k].z, q[k].w)));
      float seed = vmax_of(vm2);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) seed = fmaxf(seed, __shfl_xor_sync(0xffffffffu, seed, o));
      Chain ch[2];
      chain_seed(ch[0], seed, c);
      chain_seed(ch[1], seed, c);
      const f32x2 c2 = pack2(c, c);
#pragma unroll
      for (int k = 0; k < kFsVecs; ++k)
        if (lane + 32 * k < nv) chain_vec(q[k], c, c2, ch[k & 1], vm2);
      s = ch[0].s;
      stats_merge(s, ch[1].s);
      vmax = vmax_of(vm2);
    } else {
#pragma unroll
      for (int k = 0; k < kFsVecs; ++k) {
        if (lane + 32 * k >= nv) continue;
        Raw r[VEC];
        unpack(q[k], r);
        float u[VEC];
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          const float x = value_of(r[i]);
          vmax = fmaxf(vmax, x);
          u[i] = __fmul_rn(x, c);
        }
        stats_add(s, u);
      }
    }
    for (int j = nv * VEC + lane; j < j1 - j0; j += 32) {
      const float x = value_of(g[j]);
      vmax = fmaxf(vmax, x);
      float u[1] = {__fmul_rn(x, c)};
      stats_add(s, u);
    }
    // warp merge: the warp maximum, each lane rebased onto it once, sums
    const float m = [&] {
      float t = s.m;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
      return t;
    }();
    if (s.c0 != 0.f || s.zr != 0.f) stats_rebase(s, m);
    float c0 = s.c0, zr = s.zr, a = s.a;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c0 += __shfl_xor_sync(0xffffffffu, c0, o);
      zr += __shfl_xor_sync(0xffffffffu, zr, o);
      a += __shfl_xor_sync(0xffffffffu, a, o);
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    if (lane == 0) parts[it] = FsPart{Stats{m, c0, zr, a}, vmax};
  }
}

// ---------------------------------------------------------------------------
// recorded support, narrow lists (width <= 64): one warp per row for the
// gather and the support statistics, 16 rows per 512-thread CTA; the
// full-vocabulary statistics that a row needs (an empty support, or all
// rows when they are requested) come merged from fs_chunk_kernel's partials.

constexpr int kWarpRows = 16;           // rows per CTA, one per warp
constexpr int kWarpRowThreads = 512;
constexpr int kWarpRowMaxWidth = 64;    // two list slots per lane

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename Raw>
__global__ void __launch_bounds__(kWarpRowThreads) score_recorded_warp_kernel(
    ScoreParams P, const int32_t* slot, const FsPart* parts, int nch) {
  // Phase A reads only the call's inputs and the list kernel's slots, both
  // complete before this grid is launched (the statistics grid launches it
  // only after its own wait on the list grid, which waited on whatever
  // produced the inputs); the wait on the statistics grid comes just before
  // its partials are read, so phase A overlaps that grid's tail.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarpRows + warp;
  const bool row_ok = row < P.rows;
  const int V = P.vocab;
  const int W = P.support_width;
  const uint32_t lt = (1u << lane) - 1u;

  // ---- phase A (warp per row): ids, dedup, gather, support statistics
  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row_ok ? row : 0) * P.ld;
  const int32_t* srow = P.support_ids + static_cast<int64_t>(row_ok ? row : 0) * P.support_ld;
  const float T = row_ok ? (P.temperature ? P.temperature[row] : P.temperature_scalar) : 1.f;
  const float c = kLog2e / T;
  const int y = row_ok ? P.targets[row] : -1;
  const bool target_ok = y >= 0 && y < V;
  int32_t id0 = -1, id1 = -1;
  if (row_ok && lane < W) id0 = srow[lane];
  if (row_ok && lane + 32 < W) id1 = srow[lane + 32];
  const bool bad0 = id0 < -1 || id0 >= V, bad1 = id1 < -1 || id1 >= V;
  bool dup0 = (__match_any_sync(0xffffffffu, id0) & lt) != 0u;
  bool dup1 = (__match_any_sync(0xffffffffu, id1) & lt) != 0u;
  if (W > 32) {
    // a second-slot id repeats any first-slot id (an earlier slot)
    for (int l = 0; l < 32; ++l) dup1 |= __shfl_sync(0xffffffffu, id0, l) == id1;
  }
  const bool keep0 = id0 >= 0 && !bad0 && !dup0, keep1 = id1 >= 0 && !bad1 && !dup1;
  uint32_t flags = 0;
  if (__any_sync(0xffffffffu, bad0 || bad1)) flags |= VS_ROW_BAD_SUPPORT_ID;
  if (__any_sync(0xffffffffu, (dup0 && id0 >= 0 && !bad0) || (dup1 && id1 >= 0 && !bad1)))
    flags |= VS_ROW_DUP_SUPPORT_ID;
  const float nanf_ = __int_as_float(0x7fc00000);
  const float x0 = keep0 ? value_of(grow[id0]) : nanf_;
  const float x1 = keep1 ? value_of(grow[id1]) : nanf_;
  const uint32_t nkeep = __popc(__ballot_sync(0xffffffffu, keep0)) + __popc(__ballot_sync(0xffffffffu, keep1));
  const bool any_nf = __any_sync(0xffffffffu, (keep0 && !isfinite(x0)) || (keep1 && !isfinite(x1)));
  const bool hit = __any_sync(0xffffffffu, (keep0 && id0 == y) || (keep1 && id1 == y));
  const bool empty = nkeep == 0;
  // support statistics relative to the support maximum (value domain)
  const float vsmax = warp_max(fmaxf(keep0 ? x0 : -kInf, keep1 ? x1 : -kInf));
  Stats s{vsmax, 0.f, 0.f, 0.f};
  {
    float c0 = 0.f, zr = 0.f, a = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const bool kp = k == 0 ? keep0 : keep1;
      if (!kp) continue;
      const float x = k == 0 ? x0 : x1;
      const float d = (x - vsmax) * c;
      const float e = ex2(d);
      if (d == 0.f)
        c0 += 1.f;
      else
        zr += e;
      a = fmaf(d, e, a);
    }
    s.c0 = warp_sum(c0);
    s.zr = warp_sum(zr);
    s.a = warp_sum(a);
  }
  const bool need = row_ok && (empty || P.full_stats);
  if (!row_ok) return;
  fs_pdl_wait();

  // ---- full-vocabulary statistics (need): this row's chunk partials,
  // merged in a fixed order (lane l takes chunks l, l + 32, ... in order,
  // then a shuffle tree; the merge is commutative, so every lane gets the
  // same result)
  Stats f = stats_empty();
  float fvmax = -kInf;
  if (need && slot[row] >= 0) {
    const FsPart* pr = parts + static_cast<int64_t>(slot[row]) * nch;
    for (int k = lane; k < nch; k += 32) {
      const FsPart pt = pr[k];
      stats_merge(f, pt.s);
      fvmax = fmaxf(fvmax, pt.vmax);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      stats_merge(f, shfl_xor(f, o));
      fvmax = fmaxf(fvmax, __shfl_xor_sync(0xffffffffu, fvmax, o));
    }
  }

  // ---- phase C (warp per row): outputs
  const float nan = __int_as_float(0x7fc00000);
  if (lane == 0) {
    uint32_t status = flags;
    bool nonfinite = any_nf;
    float m2 = nan, log2z = nan, h_full = nan;
    if (need) {
      if (!stats_finite(f)) nonfinite = true;
      m2 = f.m;
      log2z = stats_log2z(f);
      h_full = kLn2 * (log2z - f.a / stats_z(f));
    }
    const float log2zs = empty ? nan : stats_log2z(s);
    const float h_sup = empty ? 0.f : kLn2 * (log2zs - s.a / stats_z(s));
    float lp_v = nan, lp_s = nan;
    bool in_s = false;
    if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
    if (nonfinite) {
      status |= VS_ROW_NONFINITE_INPUT;
    } else if (target_ok) {
      const float xy = value_of(grow[y]);
      const float uy = __fmul_rn(xy, c);
      if (need) lp_v = kLn2 * (uy - m2 - log2z);
      in_s = hit;
      if (empty) {
        lp_s = lp_v;
      } else if (in_s) {
        lp_s = kLn2 * ((xy - vsmax) * c - log2zs);
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
      cx.msup = vsmax;
      cx.log2zs = log2zs;
      cx.h_full = h_full;
      cx.h_support = h_sup;
      cx.c = c;
      cx.tkey = 0;
      cx.tie_cut = 0;
      uint32_t fl = kCtxRecorded;
      if (need) fl |= kCtxFullStats;
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
    if (!empty && !any_nf && !(need && !stats_finite(f))) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const bool kp = k == 0 ? keep0 : keep1;
        if (!kp) continue;
        const int32_t id = k == 0 ? id0 : id1;
        float gg[4];
        gumbel4(P.sample_seed, static_cast<uint32_t>(P.row_base + row), static_cast<uint64_t>(id) >> 2, gg);
        const unsigned long long key = gumbel_key(gumbel_score(k == 0 ? x0 : x1, T, gg[id & 3]), id);
        best = key > best ? key : best;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, best, o);
      best = ob > best ? ob : best;
    }
    if (lane == 0) P.sampled[row] = gumbel_key_id(best);
  }
  // support bitmask: clear the row, then set the kept ids
  if (P.support_mask) {
    const int64_t wstride = (V + 31) / 32;
    uint32_t* mrow = P.support_mask + static_cast<int64_t>(row) * wstride;
    for (int64_t w = lane; w < wstride; w += 32) mrow[w] = 0u;
    __syncwarp();
    if (!any_nf) {
      if (keep0) atomicOr(&mrow[id0 >> 5], 1u << (id0 & 31));
      if (keep1) atomicOr(&mrow[id1 >> 5], 1u << (id1 & 31));
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
  cta_sync();
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

size_t score_recorded_workspace_bytes(int rows, int vocab, int width, vs_dtype dtype) {
  return width <= kWarpRowMaxWidth ? fs_layout(rows, vocab, dtype == VS_BF16 ? 2 : 4).bytes : 0;
}

cudaError_t launch_score_recorded(const ScoreParams& p, vs_dtype dtype, void* ws, cudaStream_t s) {
  if (p.support_width <= kWarpRowMaxWidth) {
    if (!ws) return cudaErrorInvalidValue;
    const FsLayout L = fs_layout(p.rows, p.vocab, dtype == VS_BF16 ? 2 : 4);
    char* base = static_cast<char*>(ws);
    int32_t* count = reinterpret_cast<int32_t*>(base);
    int32_t* slot = reinterpret_cast<int32_t*>(base + L.slot);
    int32_t* list = reinterpret_cast<int32_t*>(base + L.list);
    FsPart* parts = reinterpret_cast<FsPart*>(base + L.parts);
    cudaError_t e = cudaMemsetAsync(count, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    fs_list_kernel<<<static_cast<unsigned>((p.rows + 7) / 8), 256, 0, s>>>(p, count, slot, list);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // persistent grid: every resident CTA of the chunk kernel, once
    static int grid_of[64][2] = {};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int which = dtype == VS_BF16 ? 0 : 1;
    int grid = 148;
    if (dev >= 0 && dev < 64 && grid_of[dev][which] > 0) {
      grid = grid_of[dev][which];
    } else {
      int sms = 0, per = 0;
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      e = dtype == VS_BF16
              ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fs_chunk_kernel<uint16_t>, kFsThreads, 0)
              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fs_chunk_kernel<uint32_t>, kFsThreads, 0);
      if (e != cudaSuccess) return e;
      grid = sms * (per > 0 ? per : 1);
      if (dev >= 0 && dev < 64) grid_of[dev][which] = grid;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kFsThreads);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = dtype == VS_BF16
            ? cudaLaunchKernelEx(&cfg, fs_chunk_kernel<uint16_t>, p, static_cast<const int32_t*>(count),
                                 static_cast<const int32_t*>(list), parts, L.nch)
            : cudaLaunchKernelEx(&cfg, fs_chunk_kernel<uint32_t>, p, static_cast<const int32_t*>(count),
                                 static_cast<const int32_t*>(list), parts, L.nch);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(static_cast<unsigned>((p.rows + kWarpRows - 1) / kWarpRows));
    cfg.blockDim = dim3(kWarpRowThreads);
    e = dtype == VS_BF16
            ? cudaLaunchKernelEx(&cfg, score_recorded_warp_kernel<uint16_t>, p,
                                 static_cast<const int32_t*>(slot), static_cast<const FsPart*>(parts), L.nch)
            : cudaLaunchKernelEx(&cfg, score_recorded_warp_kernel<uint32_t>, p,
                                 static_cast<const int32_t*>(slot), static_cast<const FsPart*>(parts), L.nch);
    if (e != cudaSuccess) return e;
  } else if (dtype == VS_BF16) {
    score_recorded_kernel<uint16_t><<<p.rows, kRecThreads, 0, s>>>(p);
  } else {
    score_recorded_kernel<uint32_t><<<p.rows, kRecThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_score_reduce(const float* h_support, const uint8_t* valid, int rows,
                                double* entropy_sum, int32_t* valid_count, cudaStream_t s) {
  score_reduce_kernel<<<1, 1024, 0, s>>>(h_support, valid, rows, entropy_sum, valid_count);
  return cudaGetLastError();
}

}  // namespace vs
