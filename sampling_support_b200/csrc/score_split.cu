// Computed-support forward scoring of bf16 rows, each row split into S
// contiguous chunks (temperature -> stable token-id top-k -> inclusive top-p
// -> min-p against the original row max; xorl issue #71, section 3).
//
// Kernel 1, one CTA per (row, chunk):
//   pass a (HBM)  online statistics of the chunk: running max, count of
//                 max-valued elements, sum 2^(u - m), sum (u - m) 2^(u - m)
//                 (u = z log2 e), rebased whenever a vector raises the max;
//   pass b (L2)   only for filtered rows: a histogram of the EXACT 16-bit keys
//                 in the 4,096 keys at and below the chunk max, skipping
//                 elements that provably cannot enter the support, and the
//                 number of elements tied with the target's value that
//                 precede it;
//   then a 32-byte record and the histogram (16-bit counts) are written.
// Kernel 2, one 512-thread CTA per row (programmatic dependent launch, so its
// launch overlaps kernel 1): the row max is the largest chunk max, the
// statistics are rebased onto it, and the chunk histograms are added at their
// offsets into the row's window of 4,096 keys below the row max (every chunk
// window reaches at least as low as the row window, so the merged window is
// exact).  Each bin holds one value, so its mass is count x 2^(u - m); block
// scans over the bins give the k-th element and the top-p crossing, and the
// support sums.  A crossing below the window falls back to an 8-bit radix
// descent over the row (rows whose support reaches far below the max).
// Kernel 3 (only when the bitmask is requested) writes the support bitmask.
//
// The tie cut (which of the elements equal to the threshold value are kept:
// the lowest ids) is resolved to an id only for the saved state or the
// bitmask; the target's own membership comes from the count of its earlier
// ties.

#include <climits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace vs {

namespace {

constexpr int kCT = 128;          // threads per chunk CTA
constexpr int kMT = 512;          // threads per merge CTA
constexpr int kMW = kMT / 32;     // warps per merge CTA
constexpr int kUnroll = 8;        // 16-byte loads in flight per thread
constexpr int kMaxChunks = 256;   // chunks per row
constexpr int kChunkAlign = 256;  // chunk length granularity (elements)
constexpr int kMaxChunk = 65280;  // 16-bit histogram counts
constexpr int kHistWords = kSelWin / 2;  // one chunk histogram, u16 pairs
constexpr size_t kSplitWsCap = size_t(64) << 20;

// Per (row, chunk) record.
struct alignas(16) ChunkRec {
  float vmax;       // chunk maximum (value)
  float c0, zr, a;  // statistics relative to fl(vmax c)
  uint32_t nb;      // histogram bins written (bins >= nb hold nothing)
  uint32_t ylt;     // chunk holding the target: its earlier ties (else 0)
  uint32_t pad0, pad1;
};
static_assert(sizeof(ChunkRec) == 32, "record layout");

// Per-row support decision, for the bitmask kernel.
struct alignas(16) RowDecision {
  uint32_t tkey;
  int32_t tie_cut;
  uint32_t mode;  // 0 empty (non-finite row), 1 whole vocabulary, 2 threshold
  uint32_t pad;
};

struct ChunkShared {
  Stats wst[kCT / 32];
  float fred[kCT / 32];
  uint32_t ured[kCT / 32];
};

// Support sums: counts above the threshold, of its tie group and of the
// max-valued elements; mass and (u - m)-weighted mass of the others.
struct SupSums {
  uint32_t ngt, neq, ntp;
  float smass, sa;
};

struct MergeShared {
  SelShared<kMW> sel;
  SupSums sums[kMW];
  Stats wst[kMW];
  float fred[kMW];
  uint32_t ured[kMW];
  u64 ulred[kMW];
  int32_t coff[kMaxChunks];  // row bin of each chunk's bin 0 (negative: none)
  uint32_t cnb[kMaxChunks];  // bins each chunk wrote
  int32_t tie_cut;
  int32_t found_chunk;
  int32_t found_need;
};

struct SplitArgs {
  int S;              // chunks per row
  int chunk;          // elements per chunk (multiple of kChunkAlign)
  ChunkRec* recs;     // [rows * S]
  uint32_t* hists;    // [rows * S * kHistWords]
  RowDecision* dec;   // [rows]
};

__device__ __forceinline__ uint32_t bf16_key(uint32_t r) { return key_of(static_cast<uint16_t>(r)); }

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  const __nv_bfloat162 r = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                   *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Programmatic dependent launch (PTX griddepcontrol): the dependent grid may
// be scheduled once every CTA of this grid has signalled; it waits for this
// grid's completion (and memory) before reading what this grid wrote.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float block_max(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = -kInf;
  const int nw = blockDim.x >> 5;
  for (int w = 0; w < nw; ++w) t = fmaxf(t, scratch[w]);
  __syncthreads();
  return t;
}

__device__ __forceinline__ uint32_t block_max_u(uint32_t v, uint32_t* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t t = 0;
  const int nw = blockDim.x >> 5;
  for (int w = 0; w < nw; ++w) t = max(t, scratch[w]);
  __syncthreads();
  return t;
}

__device__ __forceinline__ SupSums block_sum_sup(SupSums v, MergeShared& sh);

// f(raw, id) for every element of g[j0, j1) (j0 a multiple of 8), the
// block's NT threads striding 16-byte vectors read through L2.
template <int NT, typename F>
__device__ __forceinline__ void for_each_elem(const uint16_t* g, int j0, int j1, F&& f) {
  const int nv = (j1 - j0) / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(g + j0);
#pragma unroll 4
  for (int v = threadIdx.x; v < nv; v += NT) {
    const uint4 q = __ldcg(v4 + v);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f(w[i] & 0xFFFFu, j0 + v * 8 + 2 * i);
      f(w[i] >> 16, j0 + v * 8 + 2 * i + 1);
    }
  }
  for (int j = j0 + nv * 8 + threadIdx.x; j < j1; j += NT) f(static_cast<uint32_t>(g[j]), j);
}

// 8-bit radix descent over the keys of the whole row: the key where the
// cumulative count (by_mass false) or mass reaches target.  target 0 with
// by_mass asks for the top-p target of the full mass (p).
template <int NT>
__device__ Desc descend_row(const uint16_t* g, int V, float c, float m, float fxs, bool by_mass,
                            bool need_mass, u64 target, float p, MergeShared& sh,
                            RadixArrays& ra) {
  uint32_t prefix = 0;
  u64 above_cnt = 0, above_mass = 0;
  Desc out{};
  for (int shift = 8; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < kSelBins; b += NT) {
      ra.cnt[b] = 0;
      ra.mass[b] = 0;
    }
    __syncthreads();
    const int pshift = shift + 8;
    const uint32_t pre = prefix;
    for_each_elem<NT>(g, 0, V, [&](uint32_t raw, int) {
      const uint32_t key = bf16_key(raw);
      if (pshift >= 16 || (key >> pshift) == pre) {
        const uint32_t digit = (key >> shift) & 255u;
        atomicAdd(&ra.cnt[digit], 1u);
        if (need_mass) {
          const u64 fx = __float2ull_rn(ex2(__fmul_rn(value_of(static_cast<uint16_t>(raw)), c) - m) * fxs);
          if (fx) atomicAdd(&ra.mass[digit], fx);
        }
      }
    });
    __syncthreads();
    if (threadIdx.x < 32) {
      u64 tgt = target;
      if (tgt == 0) {
        u64 tot = 0;
        for (int i = threadIdx.x; i < kSelBins; i += 32) tot += ra.mass[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        tgt = topp_target(p, static_cast<double>(tot));
      }
      const u64 have = by_mass ? above_mass : above_cnt;
      const u64 need = tgt > have ? tgt - have : 1;
      uint32_t digit;
      u64 ac, am;
      scan_bins(ra.cnt, ra.mass, by_mass, need, digit, ac, am);
      if (threadIdx.x == 0) {
        sh.sel.b_above_cnt = ac;
        sh.sel.b_above_mass = am;
        sh.sel.b_key = digit;
        sh.sel.b_at_cnt = ra.cnt[digit];
        sh.sel.b_at_mass = ra.mass[digit];
        sh.ulred[0] = tgt;
      }
    }
    __syncthreads();
    target = sh.ulred[0];
    above_cnt += sh.sel.b_above_cnt;
    above_mass += sh.sel.b_above_mass;
    prefix = (prefix << 8) | sh.sel.b_key;
    out.at_cnt = sh.sel.b_at_cnt;
    out.at_mass = sh.sel.b_at_mass;
    __syncthreads();
  }
  out.key = prefix;
  out.above_cnt = above_cnt;
  out.above_mass = above_mass;
  if (threadIdx.x == 0) sh.ulred[1] = target;  // the resolved target (implicit top-p case)
  __syncthreads();
  return out;
}

// Id of the need-th (1-based) element of g[j0, j1) whose key is t, in id
// order; INT_MAX when there are fewer.  Thread t owns a contiguous run of
// every segment, so a block scan of the runs' counts orders them.
template <int NT>
__device__ int32_t tie_scan(const uint16_t* g, int j0, int j1, uint32_t t, int need,
                            MergeShared& sh) {
  constexpr int kRun = 256;  // elements per thread and segment (multiple of 8)
  if (threadIdx.x == 0) sh.tie_cut = INT_MAX;
  __syncthreads();
  int seen = 0;
  for (int s0 = j0; s0 < j1 && seen < need; s0 += NT * kRun) {
    const int a = min(j1, s0 + threadIdx.x * kRun), b = min(j1, a + kRun);
    int mine = 0;
    int j = a;
    for (; j + 8 <= b; j += 8) {
      const uint4 q = __ldcg(reinterpret_cast<const uint4*>(g + j));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) mine += (bf16_key(w[i] & 0xFFFFu) == t) + (bf16_key(w[i] >> 16) == t);
    }
    for (; j < b; ++j) mine += bf16_key(g[j]) == t;
    int total;
    const int excl = seen + block_excl_int<NT>(mine, total, sh.sel);
    if (excl < need && need <= excl + mine) {
      int cn = excl;
      for (int jj = a; jj < b; ++jj)
        if (bf16_key(g[jj]) == t && ++cn == need) {
          sh.tie_cut = jj;
          break;
        }
    }
    seen += total;
  }
  __syncthreads();
  const int32_t r = sh.tie_cut;
  __syncthreads();
  return r;
}

__device__ __forceinline__ SupSums block_sum_sup(SupSums v, MergeShared& sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.ngt += __shfl_xor_sync(0xffffffffu, v.ngt, o);
    v.neq += __shfl_xor_sync(0xffffffffu, v.neq, o);
    v.ntp += __shfl_xor_sync(0xffffffffu, v.ntp, o);
    v.smass += __shfl_xor_sync(0xffffffffu, v.smass, o);
    v.sa += __shfl_xor_sync(0xffffffffu, v.sa, o);
  }
  if ((threadIdx.x & 31) == 0) sh.sums[threadIdx.x >> 5] = v;
  __syncthreads();
  SupSums t{0u, 0u, 0u, 0.f, 0.f};
  for (int w = 0; w < kMW; ++w) {
    t.ngt += sh.sums[w].ngt;
    t.neq += sh.sums[w].neq;
    t.ntp += sh.sums[w].ntp;
    t.smass += sh.sums[w].smass;
    t.sa += sh.sums[w].sa;
  }
  __syncthreads();
  return t;
}

// Pass b of a chunk: count each element whose bin b = kmax - key lies below
// nbw.  MODE 1 (every kept key is a positive non-zero value): b = rmax - r;
// MODE 2 (the chunk max is negative): b = r - rmax; MODE 0: the key map.
// Out-of-window raw values wrap to huge bins in modes 1 and 2.  CNTY also
// counts the elements tied with key ky whose id is below y.
template <int MODE, bool CNTY>
__device__ __forceinline__ uint32_t hist_pass(const uint4* v4, int nv, int j0, uint32_t kmax,
                                              uint32_t rmax, uint32_t nbw, uint32_t ky, int y,
                                              uint32_t* hist) {
  uint32_t ylt = 0;
  auto one = [&](uint32_t r, int id) {
    uint32_t b;
    if constexpr (MODE == 1)
      b = rmax - r;
    else if constexpr (MODE == 2)
      b = r - rmax;
    else
      b = kmax - bf16_key(r);
    if (b < nbw) atomicAdd(&hist[b], 1u);
    if constexpr (CNTY) ylt += static_cast<uint32_t>(bf16_key(r) == ky) & static_cast<uint32_t>(id < y);
  };
  auto vec = [&](const uint4& q, int vi) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    const int id = j0 + vi * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      one(w[i] & 0xFFFFu, id + 2 * i);
      one(w[i] >> 16, id + 2 * i + 1);
    }
  };
  int v = threadIdx.x;
  for (; v + (kUnroll - 1) * kCT < nv; v += kUnroll * kCT) {
    uint4 q[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) q[k] = __ldcg(v4 + v + k * kCT);
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) vec(q[k], v + k * kCT);
  }
  for (; v < nv; v += kCT) vec(__ldcg(v4 + v), v);
  return ylt;
}

__global__ void __launch_bounds__(kCT, 8) score_chunk_kernel(ScoreParams P, SplitArgs Q) {
  __shared__ __align__(16) uint32_t hist[kSelWin];
  __shared__ ChunkShared sh;
  pdl_launch_dependents();

  const int row = blockIdx.x / Q.S;
  const int cs = blockIdx.x - row * Q.S;
  const int tid = threadIdx.x;
  const int V = P.vocab;
  const uint16_t* grow = static_cast<const uint16_t*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  const int j0 = cs * Q.chunk, j1 = min(V, j0 + Q.chunk);
  const int nv = (j1 - j0) / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(grow + j0);

  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const float c = kLog2e / T;
  const int kk = P.top_k ? P.top_k[row] : P.top_k_scalar;
  const float pp = P.top_p ? P.top_p[row] : P.top_p_scalar;
  const float mp = P.min_p ? P.min_p[row] : P.min_p_scalar;
  const bool use_k = kk > 0 && kk < V;
  const bool use_p = pp < 1.f;
  const bool use_minp = mp > 0.f;
  const bool any_filter = use_k || use_p || use_minp;

  if (any_filter)
    for (int b = tid; b < kSelWin; b += kCT) hist[b] = 0u;

  // ---- pass a (HBM): online statistics.  Each thread keeps the running max
  // (value vr, u-units mr), the count of max-valued elements c0 and packed
  // sums of 2^(u - mr) and (u - mr) 2^(u - mr) over the others.
  float vr = -kInf, mr = -kInf;
  uint32_t c0 = 0;
  f32x2 z2 = pack2(0.f, 0.f), a2 = pack2(0.f, 0.f);
  const f32x2 c2 = pack2(c, c);
  auto stats_vec = [&](const uint4& q) {
    const uint32_t mv = bmax2(bmax2(q.x, q.y), bmax2(q.z, q.w));
    const float vm = fmaxf(__uint_as_float(mv << 16), __uint_as_float(mv & 0xFFFF0000u));
    if (vm > vr) {  // rare after the first few vectors
      const float mn = __fmul_rn(vm, c);
      if (vr != -kInf) {
        // rebase onto the new max: the old max-valued elements join the rest
        float z0, z1, a0, a1;
        unpack2(z2, z0, z1);
        unpack2(a2, a0, a1);
        const float f = ex2(mr - mn);
        const float z = static_cast<float>(c0) + z0 + z1;
        z2 = pack2(f * z, 0.f);
        a2 = pack2(f * fmaf(mr - mn, z, a0 + a1), 0.f);
      }
      c0 = 0;
      vr = vm;
      mr = mn;
    }
    const f32x2 m2 = pack2(mr, mr);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x0 = __uint_as_float(w[i] << 16), x1 = __uint_as_float(w[i] & 0xFFFF0000u);
      const f32x2 d2 = sub2(mul2(pack2(x0, x1), c2), m2);
      float d0, d1;
      unpack2(d2, d0, d1);
      // max-valued elements are counted apart (compared by value: the packed
      // product need not round like the scalar one that made mr)
      const bool t0 = x0 == vr, t1 = x1 == vr;
      c0 += static_cast<uint32_t>(t0) + static_cast<uint32_t>(t1);
      const f32x2 e2 = pack2(t0 ? 0.f : ex2(d0), t1 ? 0.f : ex2(d1));
      z2 = add2(z2, e2);
      a2 = fma2(d2, e2, a2);
    }
  };
  int v = tid;
  for (; v + (kUnroll - 1) * kCT < nv; v += kUnroll * kCT) {
    uint4 q[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) q[k] = __ldg(v4 + v + k * kCT);
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) stats_vec(q[k]);
  }
  for (; v < nv; v += kCT) stats_vec(__ldg(v4 + v));
  Stats st;
  {
    float z0, z1, a0, a1;
    unpack2(z2, z0, z1);
    unpack2(a2, a0, a1);
    st = Stats{mr, static_cast<float>(c0), z0 + z1, a0 + a1};
  }
  // ragged tail (the last chunk of a row whose length is not a multiple of 8)
  for (int j = j0 + nv * 8 + tid; j < j1; j += kCT) {
    float u[1] = {__fmul_rn(value_of(grow[j]), c)};
    vr = fmaxf(vr, value_of(grow[j]));
    stats_add(st, u);
  }
  st = block_reduce(st, sh.wst);
  const float vmax = block_max(vr, sh.fred);

  // ---- pass b (L2): window histogram of the filtered rows
  uint32_t nb = 0, ylt = 0;
  if (any_filter) {
    const uint32_t kmax = bf16_key(__float_as_uint(vmax) >> 16);
    // Elements below these levels (relative to the chunk max, hence also to
    // the row max) never enter the support: min-p keeps 2^(u - m) >= min_p;
    // top-p alone keeps a prefix whose complement holds at most (1 - p) of
    // the mass, while all elements with 2^(u - m) < (1 - p) / (2 V) hold less
    // than half of that (the row total is at least 1).  One more octave of
    // margin each.
    float dlo = -kInf;
    if (use_minp) dlo = log2f(mp) - 1.f;
    if (use_p && !use_k && pp > 0.f) dlo = fmaxf(dlo, log2f((1.f - pp) / static_cast<float>(V)) - 2.f);
    uint32_t nbw = kSelWin;
    if (dlo > -kInf && isfinite(st.m)) {
      // smallest key at or above the level: bins b < kmax - kskip + 1
      uint32_t lo = kmax >= static_cast<uint32_t>(kSelWin - 1) ? kmax - (kSelWin - 1) : 0u, hi = kmax;
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (key_u(mid, c) - st.m >= dlo)
          hi = mid;
        else
          lo = mid + 1;
      }
      nbw = kmax - lo + 1;
    }
    // the chunk holding the target also counts the target's earlier ties
    const int y = P.targets[row];
    const bool cnty = y > j0 && y < j1;
    const uint32_t ky = cnty ? bf16_key(grow[y]) : 0xFFFFFFFFu;
    const uint32_t rmax = __float_as_uint(vmax) >> 16;
    const int mode = kmax - (nbw - 1) > 0x7FFFu ? 1 : (kmax < 0x7FFFu ? 2 : 0);
    if (cnty) {
      if (mode == 1) ylt = hist_pass<1, true>(v4, nv, j0, kmax, rmax, nbw, ky, y, hist);
      else if (mode == 2) ylt = hist_pass<2, true>(v4, nv, j0, kmax, rmax, nbw, ky, y, hist);
      else ylt = hist_pass<0, true>(v4, nv, j0, kmax, rmax, nbw, ky, y, hist);
    } else {
      if (mode == 1) hist_pass<1, false>(v4, nv, j0, kmax, rmax, nbw, ky, y, hist);
      else if (mode == 2) hist_pass<2, false>(v4, nv, j0, kmax, rmax, nbw, ky, y, hist);
      else hist_pass<0, false>(v4, nv, j0, kmax, rmax, nbw, ky, y, hist);
    }
    for (int j = j0 + nv * 8 + tid; j < j1; j += kCT) {
      const uint32_t key = bf16_key(grow[j]);
      if (kmax - key < nbw) atomicAdd(&hist[kmax - key], 1u);
      if (cnty) ylt += static_cast<uint32_t>(key == ky) & static_cast<uint32_t>(j < y);
    }
    if (cnty) ylt = block_sum(ylt, sh.ured);
    __syncthreads();
    uint32_t hi = 0;
    for (int b = tid; b < kSelWin; b += kCT)
      if (hist[b]) hi = b + 1;
    nb = block_max_u(hi, sh.ured);
    const int64_t slot = static_cast<int64_t>(row) * Q.S + cs;
    uint4* hout = reinterpret_cast<uint4*>(Q.hists + slot * kHistWords);
    for (int vv = tid; vv < static_cast<int>((nb + 7) / 8); vv += kCT) {
      const uint32_t* h = hist + vv * 8;
      hout[vv] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                            h[6] | (h[7] << 16));
    }
  }
  if (tid == 0) {
    ChunkRec r;
    r.vmax = vmax;
    r.c0 = st.c0;
    r.zr = st.zr;
    r.a = st.a;
    r.nb = nb;
    r.ylt = ylt;
    r.pad0 = r.pad1 = 0;
    Q.recs[static_cast<int64_t>(row) * Q.S + cs] = r;
  }
}

__global__ void __launch_bounds__(kMT, 1) score_merge_kernel(ScoreParams P, SplitArgs Q) {
  __shared__ __align__(16) uint32_t hist[kSelWin];
  __shared__ MergeShared sh;
  RadixArrays& ra = *reinterpret_cast<RadixArrays*>(hist);

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int V = P.vocab;
  const uint16_t* grow = static_cast<const uint16_t*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const float c = kLog2e / T;
  const int kk = P.top_k ? P.top_k[row] : P.top_k_scalar;
  const float pp = P.top_p ? P.top_p[row] : P.top_p_scalar;
  const float mp = P.min_p ? P.min_p[row] : P.min_p_scalar;
  const bool use_k = kk > 0 && kk < V;
  const bool use_p = pp < 1.f;
  const bool use_minp = mp > 0.f;
  const bool any_filter = use_k || use_p || use_minp;
  const int y = P.targets[row];
  const bool target_ok = y >= 0 && y < V;
  const int S = Q.S;
  const uint32_t ry = target_ok ? static_cast<uint32_t>(grow[y]) : 0u;
  pdl_wait();  // the chunk kernel's records and histograms

  const ChunkRec* rr = Q.recs + static_cast<int64_t>(row) * S;
  Stats st = stats_empty();
  float vr = -kInf;
  for (int k = tid; k < S; k += kMT) {
    const float4 h0 = __ldcg(reinterpret_cast<const float4*>(rr + k));
    const uint4 h1 = __ldcg(reinterpret_cast<const uint4*>(rr + k) + 1);
    Stats t{__fmul_rn(h0.x, c), h0.y, h0.z, h0.w};
    stats_merge(st, t);
    vr = fmaxf(vr, h0.x);
    sh.cnb[k] = h1.x;
    sh.coff[k] = static_cast<int32_t>(bf16_key(__float_as_uint(h0.x) >> 16));  // chunk kmax for now
  }
  st = block_reduce(st, sh.wst);
  vr = block_max(vr, sh.fred);

  const bool nonfinite = !stats_finite(st) || !isfinite(vr);
  const float mr = st.m;  // = fl(vr c)
  const float log2z = stats_log2z(st);
  const float h_full = kLn2 * (log2z - st.a / stats_z(st));
  const bool filtered = !nonfinite && any_filter;
  const bool want_cut = P.ctx != nullptr || P.support_mask != nullptr;

  uint32_t tkey = 0;
  int32_t tie_cut = INT_MAX;
  bool cut_known = true;  // tie_cut resolved (or not needed: every tie kept)
  u64 ckeep = 0;
  float log2zs = log2z, h_support = h_full, c0s = st.c0, zrs = st.zr;
  int32_t n_support = nonfinite ? 0 : V;
  bool from_bins = false;  // the threshold lies inside the merged window

  if (filtered) {
    const float fxs = fx_scale(P.fx_shift);
    const uint32_t kmr = bf16_key(__float_as_uint(vr) >> 16);
    Window w{};
    w.kmax = kmr;
    w.klo = kmr >= static_cast<uint32_t>(kSelWin - 1) ? kmr - (kSelWin - 1) : 0u;
    w.nbins = static_cast<int>(kmr - w.klo) + 1;
    w.hist = hist;
    w.c = c;
    w.m = mr;
    w.fxs = fxs;
    // merged window: hist[key - klo]; chunk bin b holds key kmax_k - b
    for (int k = tid; k < S; k += kMT) {
      const int off = static_cast<int>(kmr) - sh.coff[k];  // >= 0
      sh.coff[k] = w.nbins - 1 - off;  // row bin of chunk bin 0 (negative: none)
    }
    for (int b = tid; b < kSelWin; b += kMT) hist[b] = 0u;
    __syncthreads();
    {
      // thread t adds vector t (bins 8t .. 8t+7) of every chunk histogram
      static_assert(kSelWin / 8 == kMT, "one histogram vector per merge thread");
      const uint4* hrow = reinterpret_cast<const uint4*>(Q.hists + static_cast<int64_t>(row) * S * kHistWords);
      for (int k0 = 0; k0 < S; k0 += 8) {
        uint4 q[8];
        int base[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = k0 + u;
          base[u] = -1;
          q[u] = make_uint4(0, 0, 0, 0);
          if (k < S && static_cast<uint32_t>(tid * 8) < sh.cnb[k] && sh.coff[k] - tid * 8 >= 0) {
            base[u] = sh.coff[k] - tid * 8;  // row bin of this vector's first count
            q[u] = __ldcg(hrow + static_cast<int64_t>(k) * (kHistWords / 4) + tid);
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (base[u] < 0) continue;
          const uint32_t wd[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t cnt = (wd[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu;
            const int rb = base[u] - i;
            if (cnt && rb >= 0) atomicAdd(&hist[rb], cnt);
          }
        }
      }
    }
    __syncthreads();

    bool all_ties = true;
    u64 cnum = 0;
    bool have_t = false;
    bool win_ok = true;
    if (use_k || use_p) {
      Desc dk{}, dp{};
      u64 ck = 0;
      if (use_k) {
        win_ok = win_search<kMT>(w, false, static_cast<u64>(kk), dk, sh.sel);
        if (win_ok) {
          ck = static_cast<u64>(kk) - dk.above_cnt;
          tkey = dk.key;
          cnum = ck;
          all_ties = ck >= dk.at_cnt;
          have_t = true;
        }
      }
      if (win_ok && use_p) {
        double mass1;
        if (use_k) {
          const u64 fx_t = dk.at_cnt ? dk.at_mass / dk.at_cnt : 0;
          mass1 = static_cast<double>(dk.above_mass + ck * fx_t);
        } else {
          mass1 = (static_cast<double>(st.c0) + static_cast<double>(st.zr)) * static_cast<double>(fxs);
        }
        const u64 tp = topp_target(pp, mass1);
        win_ok = win_search<kMT>(w, true, tp, dp, sh.sel);
        if (win_ok) {
          u64 cp = topp_ties(dp, tp);
          if (use_k && dp.key == tkey && cp > ck) cp = ck;
          tkey = dp.key;
          cnum = cp;
          all_ties = cp >= dp.at_cnt;
          have_t = true;
        }
      }
      if (!win_ok) {
        // the k-th element or the crossing lies below the window
        have_t = false;
        all_ties = true;
        if (use_k) {
          const Desc d = descend_row<kMT>(grow, V, c, mr, fxs, false, use_p, static_cast<u64>(kk), 1.f, sh, ra);
          const u64 ck2 = static_cast<u64>(kk) - d.above_cnt;
          tkey = d.key;
          cnum = ck2;
          all_ties = ck2 >= d.at_cnt;
          have_t = true;
          if (use_p) {
            const u64 fx_t = d.at_cnt ? d.at_mass / d.at_cnt : 0;
            const u64 tp = topp_target(pp, static_cast<double>(d.above_mass + ck2 * fx_t));
            const Desc e = descend_row<kMT>(grow, V, c, mr, fxs, true, true, tp, pp, sh, ra);
            u64 cp = topp_ties(e, tp);
            if (e.key == tkey && cp > ck2) cp = ck2;
            tkey = e.key;
            cnum = cp;
            all_ties = cp >= e.at_cnt;
          }
        } else {
          const Desc e = descend_row<kMT>(grow, V, c, mr, fxs, true, true, 0ull, pp, sh, ra);
          const u64 cp = topp_ties(e, sh.ulred[1]);
          tkey = e.key;
          cnum = cp;
          all_ties = cp >= e.at_cnt;
          have_t = true;
        }
      }
    }
    if (use_minp) {
      const uint32_t lo = minp_key<uint16_t>(mp, c, mr);
      if (!have_t || lo > tkey) {
        tkey = lo;
        all_ties = true;
        have_t = true;
      }
    }

    // ---- support sums: keys above tkey (max-valued elements apart) and the
    // tie group at tkey
    from_bins = win_ok && tkey >= w.klo;
    SupSums sums{0u, 0u, 0u, 0.f, 0.f};
    if (from_bins) {
      const int per = (w.nbins + kMT - 1) / kMT;
      const int i0 = tid * per, i1 = min(w.nbins, i0 + per);
      for (int i = i0; i < i1; ++i) {
        const uint32_t cnt = hist[i];
        const uint32_t key = w.klo + i;
        if (cnt && key > tkey) {
          const float d = key_u(key, c) - mr;
          const float e = ex2(d);
          const float fc = static_cast<float>(cnt);
          sums.ngt += cnt;
          if (d == 0.f)
            sums.ntp += cnt;
          else
            sums.smass = fmaf(fc, e, sums.smass);
          sums.sa = fmaf(fc * d, e, sums.sa);
        }
      }
      if (tid == 0) sums.neq = hist[tkey - w.klo];
    } else {
      const uint32_t t = tkey;
      for_each_elem<kMT>(grow, 0, V, [&](uint32_t raw, int) {
        const uint32_t key = bf16_key(raw);
        if (key > t) {
          const float d = __fmul_rn(value_of(static_cast<uint16_t>(raw)), c) - mr;
          const float e = ex2(d);
          ++sums.ngt;
          if (d == 0.f)
            ++sums.ntp;
          else
            sums.smass += e;
          sums.sa = fmaf(d, e, sums.sa);
        } else if (key == t) {
          ++sums.neq;
        }
      });
    }
    sums = block_sum_sup(sums, sh);
    const uint32_t ngt = sums.ngt, neq = sums.neq, ntp = sums.ntp;
    const float smass = sums.smass, sa = sums.sa;
    const u64 tot_eq = neq;
    ckeep = all_ties ? tot_eq : (cnum < tot_eq ? cnum : tot_eq);
    const float dt = key_u(tkey, c) - mr;
    const float et = ex2(dt);
    Stats ss;
    ss.m = mr;
    ss.c0 = static_cast<float>(ntp) + (dt == 0.f ? static_cast<float>(ckeep) : 0.f);
    ss.zr = smass + (dt == 0.f ? 0.f : static_cast<float>(ckeep) * et);
    ss.a = sa + static_cast<float>(ckeep) * dt * et;
    log2zs = stats_log2z(ss);
    h_support = kLn2 * (log2zs - ss.a / stats_z(ss));
    c0s = ss.c0;
    zrs = ss.zr;
    n_support = static_cast<int32_t>(ngt + ckeep);

    // ---- tie cut id: only for the saved state or the bitmask
    if (ckeep < tot_eq) {
      cut_known = false;
      if (want_cut) {
        const int need = static_cast<int>(ckeep);
        if (from_bins) {
          // the chunk holding the need-th tie, from the chunk histograms
          // (every chunk window reaches down to the row window)
          if (tid == 0) {
            sh.found_chunk = -1;
            int before = 0;
            for (int k = 0; k < S && sh.found_chunk < 0; ++k) {
              const float vk = __ldcg(&rr[k].vmax);
              const uint32_t kk2 = bf16_key(__float_as_uint(vk) >> 16);
              const uint32_t nbk = __ldcg(&rr[k].nb);
              uint32_t cnt = 0;
              if (kk2 >= tkey && kk2 - tkey < nbk) {
                const uint32_t b = kk2 - tkey;
                const uint32_t wd = __ldcg(Q.hists + (static_cast<int64_t>(row) * S + k) * kHistWords + (b >> 1));
                cnt = (wd >> ((b & 1) * 16)) & 0xFFFFu;
              }
              if (before + static_cast<int>(cnt) >= need) {
                sh.found_chunk = k;
                sh.found_need = need - before;
              }
              before += static_cast<int>(cnt);
            }
          }
          __syncthreads();
          const int k = sh.found_chunk, nd = sh.found_need;
          __syncthreads();
          tie_cut = k >= 0 ? tie_scan<kMT>(grow, k * Q.chunk, min(V, (k + 1) * Q.chunk), tkey, nd, sh)
                           : INT_MAX;
        } else {
          tie_cut = tie_scan<kMT>(grow, 0, V, tkey, need, sh);
        }
        cut_known = true;
      }
    }
  }

  // ---- the target's earlier ties, when its membership hinges on them
  uint32_t ylt_row = 0;
  if (filtered && !cut_known && target_ok && bf16_key(ry) == tkey) {
    uint32_t part = 0;
    if (from_bins) {
      // chunks before the target's: their histogram count at tkey; the
      // target's chunk counted its own earlier ties
      const int cy = y / Q.chunk;
      for (int k = tid; k <= cy; k += kMT) {
        if (k == cy) {
          part += __ldcg(&rr[k].ylt);
        } else {
          const uint32_t kk2 = bf16_key(__float_as_uint(__ldcg(&rr[k].vmax)) >> 16);
          const uint32_t nbk = __ldcg(&rr[k].nb);
          if (kk2 >= tkey && kk2 - tkey < nbk) {
            const uint32_t b = kk2 - tkey;
            const uint32_t wd = __ldcg(Q.hists + (static_cast<int64_t>(row) * S + k) * kHistWords + (b >> 1));
            part += (wd >> ((b & 1) * 16)) & 0xFFFFu;
          }
        }
      }
    } else {
      const uint32_t t = tkey;
      for_each_elem<kMT>(grow, 0, y, [&](uint32_t raw, int) { part += bf16_key(raw) == t; });
    }
    ylt_row = block_sum(part, sh.ured);
  }

  // ---- per-row outputs
  if (tid == 0) {
    uint32_t status = 0;
    float lp_v = __int_as_float(0x7fc00000), lp_s = __int_as_float(0x7fc00000);
    bool in_s = false;
    if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
    if (nonfinite) {
      status |= VS_ROW_NONFINITE_INPUT;
    } else if (target_ok) {
      const float uy = __fmul_rn(value_of(static_cast<uint16_t>(ry)), c);
      lp_v = kLn2 * (uy - mr - log2z);
      if (!filtered) {
        in_s = true;
      } else {
        const uint32_t kyy = bf16_key(ry);
        in_s = kyy > tkey || (kyy == tkey && (cut_known ? y <= tie_cut : ylt_row < ckeep));
      }
      if (in_s) {
        lp_s = filtered ? kLn2 * (uy - mr - log2zs) : lp_v;
      } else {
        lp_s = -kInf;
        status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
      }
    }
    const float nan = __int_as_float(0x7fc00000);
    if (P.lp_full) P.lp_full[row] = lp_v;
    if (P.lp_support) P.lp_support[row] = lp_s;
    if (P.want_entropy) {
      if (P.h_full) P.h_full[row] = nonfinite ? nan : h_full;
      if (P.h_support) P.h_support[row] = nonfinite ? nan : h_support;
    }
    if (P.valid) P.valid[row] = nonfinite ? 0 : 1;
    if (P.status) P.status[row] = status;
    if (P.support_size) P.support_size[row] = n_support;
    if (P.support_mask) {
      RowDecision d;
      d.tkey = tkey;
      d.tie_cut = tie_cut;
      d.mode = nonfinite ? 0u : (filtered ? 2u : 1u);
      d.pad = 0;
      Q.dec[row] = d;
    }
    if (P.ctx) {
      RowCtx cx{};
      cx.m2 = vr;
      cx.log2z = log2z;
      cx.msup = vr;
      cx.log2zs = log2zs;
      cx.h_full = h_full;
      cx.h_support = h_support;
      cx.c = c;
      cx.tkey = tkey;
      cx.tie_cut = tie_cut;
      uint32_t f = kCtxFullStats;
      if (nonfinite) f |= kCtxNonFinite | kCtxEmpty;
      else if (!filtered) f |= kCtxAllVocab;
      else f |= kCtxThreshold;
      if (target_ok) f |= kCtxTargetOk;
      if (in_s) f |= kCtxTargetInS;
      cx.flags = f;
      cx.n_support = n_support;
      cx.status = status;
      cx.c0_full = st.c0;
      cx.zr_full = st.zr;
      cx.c0_sup = c0s;
      cx.zr_sup = zrs;
      P.ctx[row] = cx;
    }
  }
}

// Support bitmask of each chunk from the row's decision: one 32-id word per
// thread and step (chunks start on word boundaries).
__global__ void __launch_bounds__(kCT) score_split_mask_kernel(ScoreParams P, SplitArgs Q) {
  const int row = blockIdx.x / Q.S;
  const int cs = blockIdx.x - row * Q.S;
  const int V = P.vocab;
  const uint16_t* grow = static_cast<const uint16_t*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  const int j0 = cs * Q.chunk, j1 = min(V, j0 + Q.chunk);
  const RowDecision d = Q.dec[row];
  const int64_t wstride = (V + 31) / 32;
  uint32_t* mrow = P.support_mask + static_cast<int64_t>(row) * wstride;
  const int nw = (j1 - j0 + 31) / 32;
  for (int wd = threadIdx.x; wd < nw; wd += kCT) {
    const int jb = j0 + wd * 32;
    uint32_t bits = 0;
    if (d.mode == 1u) {
      bits = jb + 32 <= V ? 0xFFFFFFFFu : ((1u << (V - jb)) - 1u);
    } else if (d.mode == 2u) {
      if (jb + 32 <= j1) {
        const uint4* q4 = reinterpret_cast<const uint4*>(grow + jb);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 q = __ldcg(q4 + k);
          const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t key = bf16_key((w[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu);
            const int id = jb + k * 8 + i;
            if (key > d.tkey || (key == d.tkey && id <= d.tie_cut)) bits |= 1u << (k * 8 + i);
          }
        }
      } else {
        for (int i = 0; i < 32 && jb + i < j1; ++i) {
          const uint32_t key = bf16_key(grow[jb + i]);
          if (key > d.tkey || (key == d.tkey && jb + i <= d.tie_cut)) bits |= 1u << i;
        }
      }
    }
    mrow[j0 / 32 + wd] = bits;
  }
}

struct SplitPlan {
  int S, chunk, rows_per_launch;
  size_t off_hists, off_dec, bytes;
};

// Chunk CTAs resident on the whole device (one wave).
int resident_ctas() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148 * 8;
  if (cached[dev] == 0) {
    int sms = 0, per = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, score_chunk_kernel, kCT, 0) != cudaSuccess ||
        sms <= 0 || per <= 0)
      return 148 * 8;
    cached[dev] = sms * per;
  }
  return cached[dev];
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

SplitPlan split_plan(int rows, int vocab) {
  SplitPlan p{};
  const int cap = resident_ctas();
  // chunks of about 48 KB keep a wave's working set inside L2; small
  // batches split further so that one wave fills the GPU; at most
  // kMaxChunks chunks (vocab <= kMaxChunks * kMaxChunk is checked upstream)
  int S = (vocab + 24575) / 24576;
  const int fill = rows > 0 ? cap / rows : 1;
  if (fill > S) S = fill;
  if (S > kMaxChunks) S = kMaxChunks;
  int chunk = (vocab + S - 1) / S;
  chunk = (chunk + kChunkAlign - 1) / kChunkAlign * kChunkAlign;
  if (chunk < kChunkAlign * 8) chunk = kChunkAlign * 8;
  if (chunk > kMaxChunk) chunk = kMaxChunk;
  S = (vocab + chunk - 1) / chunk;
  p.S = S;
  p.chunk = chunk;
  const size_t per_row = static_cast<size_t>(S) * (sizeof(ChunkRec) + kHistWords * 4) + sizeof(RowDecision);
  size_t rpl = kSplitWsCap / per_row;
  if (rpl < 1) rpl = 1;
  if (rpl > static_cast<size_t>(rows)) rpl = rows;
  p.rows_per_launch = static_cast<int>(rpl);
  p.off_hists = align256(rpl * S * sizeof(ChunkRec));
  p.off_dec = p.off_hists + align256(rpl * S * static_cast<size_t>(kHistWords) * 4);
  p.bytes = p.off_dec + align256(rpl * sizeof(RowDecision));
  return p;
}

// ScoreParams for rows [r0, r0 + n) of P.
ScoreParams offset_rows(const ScoreParams& P, int r0, int n) {
  ScoreParams q = P;
  q.rows = n;
  q.logits = static_cast<const uint16_t*>(P.logits) + static_cast<int64_t>(r0) * P.ld;
  if (P.temperature) q.temperature = P.temperature + r0;
  q.targets = P.targets + r0;
  if (P.top_k) q.top_k = P.top_k + r0;
  if (P.top_p) q.top_p = P.top_p + r0;
  if (P.min_p) q.min_p = P.min_p + r0;
  if (P.lp_full) q.lp_full = P.lp_full + r0;
  if (P.lp_support) q.lp_support = P.lp_support + r0;
  if (P.h_full) q.h_full = P.h_full + r0;
  if (P.h_support) q.h_support = P.h_support + r0;
  if (P.valid) q.valid = P.valid + r0;
  if (P.status) q.status = P.status + r0;
  if (P.support_size) q.support_size = P.support_size + r0;
  if (P.support_mask) q.support_mask = P.support_mask + static_cast<int64_t>(r0) * ((P.vocab + 31) / 32);
  if (P.ctx) q.ctx = P.ctx + r0;
  return q;
}

}  // namespace

int32_t score_split_max_vocab() { return kMaxChunks * kMaxChunk; }

size_t score_split_workspace_bytes(int rows, int vocab) {
  if (rows <= 0) return 0;
  return split_plan(rows, vocab).bytes;
}

cudaError_t launch_score_split(const ScoreParams& p, void* ws, cudaStream_t s) {
  const SplitPlan plan = split_plan(p.rows, p.vocab);
  char* base = static_cast<char*>(ws);
  SplitArgs q{};
  q.S = plan.S;
  q.chunk = plan.chunk;
  q.recs = reinterpret_cast<ChunkRec*>(base);
  q.hists = reinterpret_cast<uint32_t*>(base + plan.off_hists);
  q.dec = reinterpret_cast<RowDecision*>(base + plan.off_dec);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  for (int r0 = 0; r0 < p.rows; r0 += plan.rows_per_launch) {
    const int n = min(plan.rows_per_launch, p.rows - r0);
    const ScoreParams pr = offset_rows(p, r0, n);
    score_chunk_kernel<<<n * plan.S, kCT, 0, s>>>(pr, q);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(n);
    cfg.blockDim = dim3(kMT);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, score_merge_kernel, pr, q);
    if (e != cudaSuccess) return e;
    if (pr.support_mask) score_split_mask_kernel<<<n * plan.S, kCT, 0, s>>>(pr, q);
  }
  return cudaGetLastError();
}

}  // namespace vs
