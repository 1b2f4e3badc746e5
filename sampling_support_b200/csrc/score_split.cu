// Computed-support forward scoring of bf16 rows (temperature -> stable
// token-id top-k -> inclusive top-p -> min-p against the original row max;
// xorl issue #71, section 3).
//
// Kernel 1 (score_chunk_kernel), one 128-thread CTA per (row, chunk): each
// row is cut into S chunks so that one wave covers the GPU.  The chunk is
// streamed once from HBM with online statistics (max, count of max-valued
// elements, sum 2^(u - m), sum (u - m) 2^(u - m); u = z log2 e) and a 16-byte
// record is written.
// Kernel 2 (score_merge_kernel), one 512-thread CTA per row, launched with
// programmatic dependent launch so that its launch overlaps kernel 1: the
// statistics are rebased onto the row max; for a filtered row the row is
// streamed again from L2 (kernel 1 read it moments before) into a histogram
// of the EXACT 16-bit keys in the window of up to 4,096 keys below the row
// max, skipping elements that provably cannot enter the support.  Each bin
// holds one value, so its mass is count x 2^(u - m); block scans over the
// bins find the k-th element and the top-p crossing, and the support sums.
// A crossing below the window falls back to an 8-bit radix descent over the
// row.  The tie cut (which elements equal to the threshold value are kept:
// the lowest ids) is resolved to an id only for the saved state, the
// bitmask or a sample; the target's membership otherwise uses the count of
// its earlier ties.
// Kernel 3 (score_split_mask_kernel, only when the bitmask is requested)
// writes the support bitmask from the row's decision.
// Kernels 4 and 5 (score_split_sample_kernel and its finalize kernel, only
// when a sample is requested): a seeded Gumbel-max token over the support
// (the noise recipe is in gumbel.cuh).

#include <climits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "gumbel.cuh"
#include "internal.h"
#include "select.cuh"

namespace vs {

namespace {

constexpr int kCT = 128;          // threads per chunk CTA
constexpr int kMT = 512;          // threads per merge CTA
constexpr int kMW = kMT / 32;     // warps per merge CTA
constexpr int kRound = 4;         // vectors per thread and round of the chunk pass
constexpr int kHistUnroll = 8;    // 16-byte loads in flight per merge thread
constexpr int kMaxChunks = 256;   // chunks per row
constexpr int kChunkAlign = 256;  // chunk length granularity (elements)
constexpr size_t kRowsL2Bytes = size_t(48) << 20;  // logits per launch kept for the L2 re-read

// Per (row, chunk) statistics relative to fl(vmax c).
struct alignas(16) ChunkRec {
  float vmax;  // chunk maximum (value)
  float c0, zr, a;
};
static_assert(sizeof(ChunkRec) == 16, "record layout");

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
  int32_t tie_cut;
};

struct SplitArgs {
  int S;              // chunks per row
  int chunk;          // elements per chunk (multiple of kChunkAlign)
  ChunkRec* recs;     // [rows * S]
  RowDecision* dec;   // [rows]
  unsigned long long* best;  // [rows] best Gumbel-max key of the row (sampling)
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

// block_reduce of the statistics that also takes the block max of v (one
// exchange for both maxima, one for the rebased sums).
__device__ __forceinline__ Stats block_reduce_vmax(Stats s, float& v, Stats* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  float m = s.m, vv = v;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    vv = fmaxf(vv, __shfl_xor_sync(0xffffffffu, vv, o));
  }
  if (lane == 0) {
    scratch[warp].m = m;
    scratch[warp].c0 = vv;
  }
  __syncthreads();
  m = -kInf;
  vv = -kInf;
  for (int w = 0; w < nw; ++w) {
    m = fmaxf(m, scratch[w].m);
    vv = fmaxf(vv, scratch[w].c0);
  }
  __syncthreads();
  if (s.c0 != 0.f || s.zr != 0.f) stats_rebase(s, m);
  float c0 = s.c0, zr = s.zr, a = s.a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c0 += __shfl_xor_sync(0xffffffffu, c0, o);
    zr += __shfl_xor_sync(0xffffffffu, zr, o);
    a += __shfl_xor_sync(0xffffffffu, a, o);
  }
  if (lane == 0) scratch[warp] = Stats{m, c0, zr, a};
  __syncthreads();
  Stats t{m, 0.f, 0.f, 0.f};
  for (int w = 0; w < nw; ++w) {
    t.c0 += scratch[w].c0;
    t.zr += scratch[w].zr;
    t.a += scratch[w].a;
  }
  __syncthreads();
  v = vv;
  return t;
}

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

// Number of elements in [j0, j1) whose raw bits are r0 or r1 (the two
// encodings of one key): the block's NT threads read 16-byte vectors
// through L2 with kHistUnroll loads in flight each; j0 need not be a
// multiple of 8.
template <int NT>
__device__ __forceinline__ uint32_t count_raw(const uint16_t* g, int j0, int j1, uint32_t r0,
                                              uint32_t r1) {
  uint32_t n = 0;
  auto one = [&](uint32_t r) { n += (r == r0) | (r == r1) ? 1u : 0u; };
  auto vec = [&](const uint4& q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      one(w[i] & 0xFFFFu);
      one(w[i] >> 16);
    }
  };
  const int ja = min(j1, (j0 + 7) & ~7);
  for (int j = j0 + static_cast<int>(threadIdx.x); j < ja; j += NT) one(g[j]);
  const int nv = (j1 - ja) >> 3;
  const uint4* v4 = reinterpret_cast<const uint4*>(g + ja);
  int v = threadIdx.x;
  for (; v + (kHistUnroll - 1) * NT < nv; v += kHistUnroll * NT) {
    uint4 q[kHistUnroll];
#pragma unroll
    for (int k = 0; k < kHistUnroll; ++k) q[k] = __ldcg(v4 + v + k * NT);
#pragma unroll
    for (int k = 0; k < kHistUnroll; ++k) vec(q[k]);
  }
  for (; v < nv; v += NT) vec(__ldcg(v4 + v));
  for (int j = ja + nv * 8 + static_cast<int>(threadIdx.x); j < j1; j += NT) one(g[j]);
  return n;
}

// 8-bit radix descent over the keys of the whole row: the key where the
// cumulative count (by_mass false) or mass reaches target.  target 0 with
// by_mass asks for the top-p target of the full mass (p).
template <int NT>
__device__ __noinline__ Desc descend_row(const uint16_t* g, int V, float c, float m, float fxs, bool by_mass,
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
__device__ __noinline__ int32_t tie_scan(const uint16_t* g, int j0, int j1, uint32_t t, int need,
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

// One shared-memory count increment at the 32-bit shared address a.
__device__ __forceinline__ void red_inc(uint32_t a) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(a) : "memory");
}

// Per-thread state of the chunk pass: running max (value vr, u units mr),
// the count of max-valued elements, and packed sums of 2^(u - mr) and
// (u - mr) 2^(u - mr) over the others.
struct ChunkAcc {
  float vr, mr;
  uint32_t c0;
  f32x2 z2, a2;
};

// The chunk pass over 16-byte vectors: online statistics.  A vector below
// the running max takes a packed path with no per-element compares; a
// vector that reaches or raises it (rare once the first round has fixed a
// high running max) rebases the sums and counts its max-valued elements.
// The thread's first-round vectors q1 are already loaded.
__device__ __forceinline__ void chunk_pass(const uint4 (&q1)[kRound], const uint4* v4, int nv,
                                           float c, ChunkAcc& acc) {
  const f32x2 c2 = pack2(c, c);
  auto vec = [&](const uint4& q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    const uint32_t mv = bmax2(bmax2(q.x, q.y), bmax2(q.z, q.w));
    const float vm = fmaxf(__uint_as_float(mv << 16), __uint_as_float(mv & 0xFFFF0000u));
    if (vm >= acc.vr) {
      if (vm > acc.vr) {
        const float mn = __fmul_rn(vm, c);
        if (acc.vr != -kInf) {
          // rebase onto the new max: the old max-valued elements join the rest
          float z0, z1, a0, a1;
          unpack2(acc.z2, z0, z1);
          unpack2(acc.a2, a0, a1);
          const float f = ex2(acc.mr - mn);
          const float z = static_cast<float>(acc.c0) + z0 + z1;
          acc.z2 = pack2(f * z, 0.f);
          acc.a2 = pack2(f * fmaf(acc.mr - mn, z, a0 + a1), 0.f);
        }
        acc.c0 = 0;
        acc.vr = vm;
        acc.mr = mn;
      }
      // max-valued elements are counted apart (by value)
      float zs = 0.f, as = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = __uint_as_float(i & 1 ? w[i >> 1] & 0xFFFF0000u : w[i >> 1] << 16);
        if (x == acc.vr) {
          ++acc.c0;
        } else {
          const float d = fmaf(x, c, -acc.mr);
          const float e = ex2(d);
          zs += e;
          as = fmaf(d, e, as);
        }
      }
      acc.z2 = add2(acc.z2, pack2(zs, 0.f));
      acc.a2 = add2(acc.a2, pack2(as, 0.f));
    } else {
      // every element lies below the running max
      const f32x2 nm2 = pack2(-acc.mr, -acc.mr);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const f32x2 d2 = fma2(pack2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u)), c2, nm2);
        float d0, d1;
        unpack2(d2, d0, d1);
        const f32x2 e2 = pack2(ex2(d0), ex2(d1));
        acc.z2 = add2(acc.z2, e2);
        acc.a2 = fma2(d2, e2, acc.a2);
      }
    }
  };
  // rounds of kRound vectors per thread, one copy of the loop body
  uint4 q[kRound];
#pragma unroll
  for (int k = 0; k < kRound; ++k) q[k] = q1[k];
  for (int v0 = threadIdx.x;;) {
#pragma unroll
    for (int k = 0; k < kRound; ++k)
      if (v0 + k * kCT < nv) vec(q[k]);
    v0 += kRound * kCT;
    if (v0 >= nv) break;
#pragma unroll
    for (int k = 0; k < kRound; ++k) q[k] = v0 + k * kCT < nv ? __ldg(v4 + v0 + k * kCT) : make_uint4(0, 0, 0, 0);
  }
}

// Smallest key in [lo, hi] whose u-offset from m reaches dlo (hi if none).
__device__ __forceinline__ uint32_t key_at_level(uint32_t lo, uint32_t hi, float c, float m,
                                                 float dlo) {
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (key_u(mid, c) - m >= dlo)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kCT, 8) score_chunk_kernel(ScoreParams P, SplitArgs Q) {
  __shared__ ChunkShared sh;
  // launched programmatically after whatever kernel precedes it on the
  // stream: wait for that grid (and its memory) before touching anything,
  // then let this call's merge kernel launch
  pdl_wait();
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

  // first round: each thread's first kRound vectors; their block max m1
  // starts every thread's running max, so later rebases are rare
  uint4 q1[kRound];
  uint32_t mx = 0xFF80FF80u;  // (-inf, -inf)
#pragma unroll
  for (int k = 0; k < kRound; ++k) {
    const int v = tid + k * kCT;
    q1[k] = v < nv ? __ldg(v4 + v) : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
    mx = bmax2(mx, bmax2(bmax2(q1[k].x, q1[k].y), bmax2(q1[k].z, q1[k].w)));
  }
  const float m1 = block_max(fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xFFFF0000u)), sh.fred);

  ChunkAcc acc{m1, __fmul_rn(m1, c), 0u, pack2(0.f, 0.f), pack2(0.f, 0.f)};
  chunk_pass(q1, v4, nv, c, acc);
  Stats st;
  {
    float z0, z1, a0, a1;
    unpack2(acc.z2, z0, z1);
    unpack2(acc.a2, a0, a1);
    st = Stats{acc.mr, static_cast<float>(acc.c0), z0 + z1, a0 + a1};
  }
  // ragged tail (the last chunk of a row whose length is not a multiple of 8)
  float vr = acc.vr;
  for (int j = j0 + nv * 8 + tid; j < j1; j += kCT) {
    const float x = value_of(grow[j]);
    float u[1] = {__fmul_rn(x, c)};
    vr = fmaxf(vr, x);
    stats_add(st, u);
  }
  st = block_reduce_vmax(st, vr, sh.wst);
  if (tid == 0) Q.recs[static_cast<int64_t>(row) * Q.S + cs] = ChunkRec{vr, st.c0, st.zr, st.a};
}

// Histogram pass of the merge kernel: counts the row's elements whose key
// lies in [klo, klo + nbins), hist[key - klo], streaming the row from L2
// (hist holds kSelWin + 32 words).
// MODE 1 (every kept key is a positive non-zero value): i = r - rlo; MODE 2
// (every kept key is negative): i = rlo - r; MODE 0: the key map.  Raw
// values outside the window wrap to huge indices in modes 1 and 2.
template <int MODE>
__device__ __forceinline__ void row_hist(const uint16_t* g, int V, uint32_t klo, uint32_t rlo,
                                         uint32_t nbins, uint32_t hist_s) {
  auto idx = [&](uint32_t r) -> uint32_t {
    if constexpr (MODE == 1)
      return r - rlo;
    else if constexpr (MODE == 2)
      return rlo - r;
    else
      return bf16_key(r) - klo;
  };
  const int nv = V / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(g);
  // out-of-window elements count into this lane's spill bin (never read):
  // no predicate or branch, and the spill bins of a warp sit in 32 banks
  const uint32_t spill = kSelWin + (threadIdx.x & 31);
  auto vec = [&](const uint4& q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t i0 = idx(w[i] & 0xFFFFu), i1 = idx(w[i] >> 16);
      red_inc(hist_s + ((i0 < nbins ? i0 : spill) << 2));
      red_inc(hist_s + ((i1 < nbins ? i1 : spill) << 2));
    }
  };
  int v = threadIdx.x;
  for (; v + (kHistUnroll - 1) * kMT < nv; v += kHistUnroll * kMT) {
    uint4 q[kHistUnroll];
#pragma unroll
    for (int k = 0; k < kHistUnroll; ++k) q[k] = __ldcg(v4 + v + k * kMT);
#pragma unroll
    for (int k = 0; k < kHistUnroll; ++k) vec(q[k]);
  }
  for (; v < nv; v += kMT) vec(__ldcg(v4 + v));
  for (int j = nv * 8 + threadIdx.x; j < V; j += kMT) {
    const uint32_t i0 = idx(g[j]);
    red_inc(hist_s + ((i0 < nbins ? i0 : spill) << 2));
  }
}

__global__ void __launch_bounds__(kMT, 1) score_merge_kernel(ScoreParams P, SplitArgs Q) {
  // kSelWin window bins, then one spill bin per lane for out-of-window elements
  __shared__ __align__(16) uint32_t hist[kSelWin + 32];
  __shared__ MergeShared sh;
  RadixArrays& ra = *reinterpret_cast<RadixArrays*>(hist);

  // the next call's chunk kernel may launch now; it waits for this grid
  pdl_launch_dependents();
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
  pdl_wait();  // the chunk kernel's records

  const ChunkRec* rr = Q.recs + static_cast<int64_t>(row) * S;
  Stats st = stats_empty();
  float vr = -kInf;
  for (int k = tid; k < S; k += kMT) {
    const float4 h = __ldcg(reinterpret_cast<const float4*>(rr + k));
    Stats t{__fmul_rn(h.x, c), h.y, h.z, h.w};
    stats_merge(st, t);
    vr = fmaxf(vr, h.x);
  }
  st = block_reduce_vmax(st, vr, sh.wst);

  const bool nonfinite = !stats_finite(st) || !isfinite(vr);
  const float mr = st.m;  // = fl(vr c)
  const float log2z = stats_log2z(st);
  const float h_full = kLn2 * (log2z - st.a / stats_z(st));
  const bool filtered = !nonfinite && any_filter;
  const bool want_cut = P.ctx != nullptr || P.support_mask != nullptr || P.sampled != nullptr;

  uint32_t tkey = 0;
  int32_t tie_cut = INT_MAX;
  bool cut_known = true;  // tie_cut resolved (or not needed: every tie kept)
  u64 ckeep = 0;
  u64 tie_group = 0;  // elements holding the threshold key
  float log2zs = log2z, h_support = h_full, c0s = st.c0, zrs = st.zr;
  int32_t n_support = nonfinite ? 0 : V;
  bool from_bins = false;  // the threshold lies inside the window

  if (filtered) {
    const float fxs = fx_scale(P.fx_shift);
    const uint32_t kmr = bf16_key(__float_as_uint(vr) >> 16);
    // Elements below these levels never enter the support: min-p keeps
    // 2^(u - m) >= min_p; top-p alone keeps a prefix whose complement holds
    // at most (1 - p) of the mass Z, while all elements with 2^(u - m) <
    // (1 - p) Z / (2 V) together hold less than half of that.  One more
    // octave of margin each.
    // (No skipping with top-k: its count and the top-k mass need every key.)
    float dlo = -kInf;
    if (!use_k) {
      if (use_minp) dlo = log2f(mp) - 1.f;
      if (use_p && pp > 0.f)
        dlo = fmaxf(dlo, log2f((1.f - pp) * stats_z(st) / static_cast<float>(V)) - 2.f);
    }
    uint32_t klo = kmr >= static_cast<uint32_t>(kSelWin - 1) ? kmr - (kSelWin - 1) : 0u;
    if (dlo > -kInf) klo = key_at_level(klo, kmr, c, mr, dlo);
    Window w{};
    w.kmax = kmr;
    w.klo = klo;
    w.nbins = static_cast<int>(kmr - klo) + 1;
    w.hist = hist;
    w.c = c;
    w.m = mr;
    w.fxs = fxs;
    for (int b = tid; b < kSelWin; b += kMT) hist[b] = 0u;
    __syncthreads();
    {
      const uint32_t hist_s = smem_addr(hist), nb = static_cast<uint32_t>(w.nbins);
      if (klo > 0x7FFFu)
        row_hist<1>(grow, V, klo, klo - 0x7FFFu, nb, hist_s);
      else if (kmr < 0x7FFFu)
        row_hist<2>(grow, V, klo, 0xFFFFu - klo, nb, hist_s);
      else
        row_hist<0>(grow, V, klo, 0u, nb, hist_s);
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
          mass1 = static_cast<double>(dk.above_mass + ck * bin_fx(w, dk.key));
        } else {
          mass1 = (static_cast<double>(st.c0) + static_cast<double>(st.zr)) * static_cast<double>(fxs);
        }
        const u64 tp = topp_target(pp, mass1);
        win_ok = win_search<kMT>(w, true, tp, dp, sh.sel);
        if (win_ok) {
          u64 cp = topp_ties(dp, tp, bin_fx(w, dp.key));
          if (use_k && dp.key == tkey && cp > ck) cp = ck;
          tkey = dp.key;
          cnum = cp;
          all_ties = cp >= dp.at_cnt;
          have_t = true;
        }
      }
      if (!win_ok && use_p && !use_k && use_minp && minp_key<uint16_t>(mp, c, mr) >= w.klo) {
        // the top-p crossing lies below the window, hence below the min-p
        // level: min-p decides the support (applied below)
        win_ok = true;
        have_t = false;
        all_ties = true;
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
            const u64 fx_t = key_fx<uint16_t>(d.key, c, mr, fxs);
            const u64 tp = topp_target(pp, static_cast<double>(d.above_mass + ck2 * fx_t));
            const Desc e = descend_row<kMT>(grow, V, c, mr, fxs, true, true, tp, pp, sh, ra);
            u64 cp = topp_ties(e, tp, key_fx<uint16_t>(e.key, c, mr, fxs));
            if (e.key == tkey && cp > ck2) cp = ck2;
            tkey = e.key;
            cnum = cp;
            all_ties = cp >= e.at_cnt;
          }
        } else {
          const Desc e = descend_row<kMT>(grow, V, c, mr, fxs, true, true, 0ull, pp, sh, ra);
          const u64 cp = topp_ties(e, sh.ulred[1], key_fx<uint16_t>(e.key, c, mr, fxs));
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
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = 8 * tid + k;
        const uint32_t cnt = i < w.nbins ? hist[i] : 0u;
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
    tie_group = tot_eq;
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
        tie_cut = tie_scan<kMT>(grow, 0, V, tkey, need, sh);
        cut_known = true;
      }
    }
  }

  // ---- the target's earlier ties, when its membership hinges on them
  uint32_t ylt_row = 0;
  if (filtered && !cut_known && target_ok && bf16_key(ry) == tkey) {
    // counted on the shorter side of y: after y, the group less the target
    // and the ties that follow it
    const uint32_t r0 = tkey >= 0x7FFFu ? tkey - 0x7FFFu : 0xFFFFu - tkey;
    const uint32_t r1 = tkey == 0x7FFFu ? 0x8000u : r0;  // -0 shares the key of +0
    const bool before = y <= V - 1 - y;
    const uint32_t part = before ? count_raw<kMT>(grow, 0, y, r0, r1)
                                 : count_raw<kMT>(grow, y + 1, V, r0, r1);
    const uint32_t n = block_sum(part, sh.ured);
    ylt_row = before ? n : static_cast<uint32_t>(tie_group) - 1u - n;
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
    if (P.support_mask || P.sampled) {
      RowDecision d;
      d.tkey = tkey;
      d.tie_cut = tie_cut;
      d.mode = nonfinite ? 0u : (filtered ? 2u : 1u);
      d.pad = 0;
      Q.dec[row] = d;
    }
    if (P.sampled) Q.best[row] = 0ull;
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

// Seeded Gumbel-max candidates of each chunk from the row's decision.  The
// chunk is read from L2 in groups of four tokens (chunks start on multiples
// of 256); each warp queues its groups that hold a member (group index,
// member bits and the four raw values) in shared memory and drains the
// queue 32 groups at a time, so the Philox block and the logarithms run
// on full warps and only for members.  The chunk's best key goes into the
// row's slot by an unsigned max (order-independent).
__global__ void __launch_bounds__(kCT) score_split_sample_kernel(ScoreParams P, SplitArgs Q) {
  __shared__ unsigned long long kred[kCT / 32];
  __shared__ uint4 queue[kCT / 32][64];
  const int row = blockIdx.x / Q.S;
  const int cs = blockIdx.x - row * Q.S;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int V = P.vocab;
  const uint16_t* grow = static_cast<const uint16_t*>(P.logits) + static_cast<int64_t>(row) * P.ld;
  const int j0 = cs * Q.chunk, j1 = min(V, j0 + Q.chunk);
  const RowDecision d = Q.dec[row];
  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const uint32_t nrow = static_cast<uint32_t>(P.row_base + row);
  uint4* wq = queue[warp];
  unsigned long long best = 0ull;
  // one queued group: .x = group index, .y = member bits, .z / .w = raw pairs
  auto take = [&](const uint4& e) {
    uint64_t w[4];
    philox4x64_10(e.x, 0, 0, 0, P.sample_seed, nrow, w);
    const uint32_t r[4] = {e.z & 0xFFFFu, e.z >> 16, e.w & 0xFFFFu, e.w >> 16};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (!((e.y >> i) & 1u)) continue;
      const int j = static_cast<int>(4 * e.x) + i;
      const unsigned long long k =
          gumbel_key(gumbel_score(value_of(static_cast<uint16_t>(r[i])), T, gumbel_of(w[i])), j);
      best = k > best ? k : best;
    }
  };
  if (d.mode != 0u) {
    int count = 0;  // queued groups of this warp (warp-uniform)
    const int q_end = (j1 + 3) / 4;
    for (int qb = j0 / 4 + warp * 32; qb < q_end; qb += kCT) {
      const int q = qb + lane;
      const int jb = 4 * q;
      uint32_t lo = 0u, hi = 0u, mbits = 0u;
      if (q < q_end) {
        if (jb + 4 <= j1) {
          const uint2 v = __ldcg(reinterpret_cast<const uint2*>(grow + jb));
          lo = v.x;
          hi = v.y;
        } else {
          for (int i = 0; i < 4 && jb + i < j1; ++i) {
            const uint32_t r = grow[jb + i];
            if (i < 2) lo |= r << (16 * i);
            else hi |= r << (16 * (i - 2));
          }
        }
        const uint32_t r[4] = {lo & 0xFFFFu, lo >> 16, hi & 0xFFFFu, hi >> 16};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          bool in = jb + i < j1;
          if (in && d.mode == 2u) {
            const uint32_t key = bf16_key(r[i]);
            in = key > d.tkey || (key == d.tkey && jb + i <= d.tie_cut);
          }
          mbits |= in ? (1u << i) : 0u;
        }
      }
      const uint32_t ball = __ballot_sync(0xffffffffu, mbits != 0u);
      if (mbits) wq[count + __popc(ball & ((1u << lane) - 1u))] = make_uint4(q, mbits, lo, hi);
      count += __popc(ball);
      __syncwarp();
      if (count >= 32) {
        count -= 32;
        take(wq[count + lane]);
        __syncwarp();
      }
    }
    if (lane < count) take(wq[lane]);
  }
  best = block_max_key(best, kred);
  if (threadIdx.x == 0 && best != 0ull) atomicMax(Q.best + row, best);
}

// The sampled token of each row from its best key (-1: no member).
__global__ void score_split_sample_final_kernel(ScoreParams P, SplitArgs Q) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row < P.rows) P.sampled[row] = gumbel_key_id(Q.best[row]);
}

struct SplitPlan {
  int S, chunk, rows_per_launch;
  size_t off_dec, off_best, bytes;
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
  // rows per launch: their logits stay in L2 between the two kernels
  size_t rpl = kRowsL2Bytes / (2 * static_cast<size_t>(vocab));
  if (rpl < 1) rpl = 1;
  if (rpl > static_cast<size_t>(rows)) rpl = rows;
  const int cap = resident_ctas();
  // chunks of about 48 KB; small batches split further so that one wave
  // fills the GPU
  int S = (vocab + 24575) / 24576;
  const int fill = cap / static_cast<int>(rpl);
  if (fill > S) S = fill;
  if (S > kMaxChunks) S = kMaxChunks;
  int chunk = (vocab + S - 1) / S;
  chunk = (chunk + kChunkAlign - 1) / kChunkAlign * kChunkAlign;
  if (chunk < kChunkAlign * 8) chunk = kChunkAlign * 8;
  S = (vocab + chunk - 1) / chunk;
  p.S = S;
  p.chunk = chunk;
  p.rows_per_launch = static_cast<int>(rpl);
  p.off_dec = align256(rpl * S * sizeof(ChunkRec));
  p.off_best = p.off_dec + align256(rpl * sizeof(RowDecision));
  p.bytes = p.off_best + align256(rpl * sizeof(unsigned long long));
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
  if (P.sampled) q.sampled = P.sampled + r0;
  q.row_base = P.row_base + r0;
  if (P.ctx) q.ctx = P.ctx + r0;
  return q;
}

}  // namespace

int32_t score_split_max_vocab() { return 1 << 26; }

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
  q.dec = reinterpret_cast<RowDecision*>(base + plan.off_dec);
  q.best = reinterpret_cast<unsigned long long*>(base + plan.off_best);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  for (int r0 = 0; r0 < p.rows; r0 += plan.rows_per_launch) {
    const int n = min(plan.rows_per_launch, p.rows - r0);
    const ScoreParams pr = offset_rows(p, r0, n);
    cudaLaunchConfig_t ccfg{};
    ccfg.gridDim = dim3(n * plan.S);
    ccfg.blockDim = dim3(kCT);
    ccfg.dynamicSmemBytes = 0;
    ccfg.stream = s;
    ccfg.attrs = attr;
    ccfg.numAttrs = 1;
    cudaError_t ec = cudaLaunchKernelEx(&ccfg, score_chunk_kernel, pr, q);
    if (ec != cudaSuccess) return ec;
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
    if (pr.sampled) {
      score_split_sample_kernel<<<n * plan.S, kCT, 0, s>>>(pr, q);
      score_split_sample_final_kernel<<<(n + 127) / 128, 128, 0, s>>>(pr, q);
    }
  }
  return cudaGetLastError();
}

}  // namespace vs
