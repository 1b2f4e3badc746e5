// Computed-support forward scoring (temperature -> stable token-id top-k ->
// inclusive top-p -> min-p against the original row max; xorl issue #71,
// section 3), one CTA per row.
//
// The row is streamed once from HBM through a ring of shared-memory stages
// filled by bulk asynchronous copies (thread 0 requests the first ones; the
// last warp to finish with a stage requests the one that refills its slot).
// In that one pass each element updates
//   * the online statistics: max, count of max-valued elements,
//     sum 2^(u - max), sum (u - max) 2^(u - max)   (u = z log2 e), and
//   * for a filtered bf16 row, a shared-memory histogram of the EXACT 16-bit
//     keys in a window of at most 4,096 keys.  The window is fixed once the
//     row's first piece has arrived: its top lies kWinHi keys above that
//     piece's maximum (a lower bound of the row maximum), and, without top-k, its
//     floor is the first key that can still matter (min-p: 2^(u - m) >=
//     min_p / 2; top-p: 2^(u - m) >= (1 - p) / (4 V), below which all
//     elements together hold under a quarter of the 1 - p tail).  Each bin
//     holds one value, so its mass is count x 2^(u - m).
// After the pass warp 0 finds the k-th element and the top-p crossing by
// warp scans of the bins and takes the support sums from the bins; nothing
// is read again (the target's rank in a partly kept tie group, when it
// decides its membership, is counted from L2).  A row whose maximum lies
// above the window, or whose decision lies below it, falls back to passes that re-read the row (an 8-bit radix
// descent; fp32 rows always take it, exact-key windows do not apply to
// 32-bit keys).  Further passes re-read the row only on request:
//   * the id of the last kept element of the threshold's tie group (ties go
//     to the lower token id), for the saved state, the bitmask or a sample
//     (the block then takes warp 0's decision and only finds that position);
//     without those only the target's membership is needed, and when the
//     target sits in a partly kept tie group the ties before it are counted
//     on the shorter side of it;
//   * the support bitmask;
//   * a seeded Gumbel-max token over the support (noise recipe in gumbel.cuh).
// Everything is block-local (no cluster barriers) and deterministic.

#include <climits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "gumbel.cuh"
#include "select.cuh"
#include "window.cuh"

namespace vs {

namespace {

constexpr int kRT = 512;        // threads per row
constexpr int kRW = kRT / 32;   // warps
constexpr int kNStages = 3;     // ring depth
constexpr int kStageBytes = 65536;
constexpr int kWin = kSelWin;
constexpr int kBins = kSelBins;
constexpr uint32_t kWinHi = 256;  // window keys above the first piece's maximum
constexpr int kCountUnroll = 8;   // 16-byte loads in flight per thread (tie count)
constexpr int kHeadElems = 8192;  // elements of the first piece of stage 0 (bf16)
constexpr int kChains = 4;        // statistics chains (16-byte vectors in flight) per thread

// Everything the per-row outputs are made from.
struct RowOut {
  Stats s;
  float vmax, m, log2z, h_full;
  bool nonfinite, filtered, cut_known;
  uint32_t tkey;
  int32_t tie_cut;
  u64 ckeep;
  uint32_t ylt;
  float log2zs, h_support, c0s, zrs;
  int32_t n_support;
};

struct RowSh {
  uint64_t full[kNStages];
  uint32_t done[kNStages];  // warps done with each ring slot in its current use
  uint64_t first;  // the first piece of stage 0 (bf16 rows), loaded apart
  Stats rs;        // the row's merged statistics (warp 0)
  float rvmax;     // the row maximum (warp 0)
  uint32_t general;  // 1: the block takes the general path
  uint32_t d_tkey, d_flags;  // warp 0's decision (bit 0 non-finite, bit 1 filtered)
  float w_m0;      // the first piece's maximum (warp 0)
  uint32_t w_top, w_lo, w_base;  // the window (warp 0)
  int32_t w_mode;
  uint32_t ylt_group;  // fast path: the target's tie group size when its rank there decides
  RowOut rout;     // fast path: the row's outputs while that rank is counted; or
                   // warp 0's decision handed to the block (reuse)
  uint32_t reuse;  // 1: warp 0 decided, only the tie cut's position is missing
  u64 reuse_tot;   // its tie group size
  Stats wst[kRW];
  float fred[kRW];
  uint32_t ured[kRW];
  u64 ulred[kRW];
  SelShared<kRW> sel;
  SupSums sums[kRW];
  int32_t tie_cut;
  uint32_t timeout;
  unsigned long long kred[kRW];
  uint32_t squeue[kRW][64];  // sampling: per-warp queue of member groups (index | bits << 28)
};

// Programmatic dependent launch (PTX griddepcontrol): the next kernel on the
// stream may be scheduled once every CTA of this grid has signalled; a grid
// waits for the preceding one (and its memory) before touching memory.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// streaming ring

template <typename Raw>
struct Ring {
  static constexpr int SE = kStageBytes / sizeof(Raw);  // elements per stage
  const Raw* g;  // row start in global memory
  int V;
  Raw* buf;      // [kNStages][SE]
  RowSh* sh;
  uint32_t cs;   // stages consumed (every thread, in step)
  uint32_t head;  // bytes at the start of stage 0 already requested apart (thread 0)
  __device__ int nst() const { return (V + SE - 1) / SE; }
  __device__ int count(int si) const { return min(SE, V - si * SE); }

  // one thread: load stage si into ring slot `slot`, which no warp reads
  __device__ void issue(int si, int slot) {
    const uint32_t bytes = static_cast<uint32_t>((count(si) * sizeof(Raw) + 15) & ~size_t(15));
    const uint32_t skip = si == 0 ? min(head, bytes) : 0u;
    if (si == 0) head = 0;
    mbar_arrive_expect_tx(&sh->full[slot], bytes - skip);
    if (bytes > skip)
      bulk_load_all(reinterpret_cast<char*>(buf + static_cast<size_t>(slot) * SE) + skip,
                    reinterpret_cast<const char*>(g + static_cast<size_t>(si) * SE) + skip,
                    bytes - skip, &sh->full[slot]);
  }

  // thread 0 requests the first stages of [s0, s1) into the slots that
  // follow the consumed ones (all free between passes)
  __device__ void start(int s0, int s1) {
    if (threadIdx.x == 0)
      for (int i = 0; i < min(s1 - s0, kNStages); ++i)
        issue(s0 + i, static_cast<int>((cs + static_cast<uint32_t>(i)) % kNStages));
  }

  // Run f(stage_ptr, n, base) over stages [s0, s1) in order, after
  // start(s0, s1); f returns true (uniformly) to stop early.  Each warp
  // counts itself out of a slot once done with it, and the warp that
  // completes the count refills the slot with the stage kNStages further
  // on, so no thread waits for the others to release a slot.  Loads already
  // issued are drained either way.
  template <typename F>
  __device__ void consume(int s0, int s1, F&& f) {
    bool stop = false;
    int si = s0;
    for (; si < s1 && !stop; ++si) {
      const int slot = static_cast<int>(cs % kNStages);
      if (!mbar_wait(&sh->full[slot], (cs / kNStages) & 1u)) atomicOr(&sh->timeout, 1u);
      stop = f(buf + static_cast<size_t>(slot) * SE, count(si), si * SE);
      ++cs;
      __syncwarp();
      if ((threadIdx.x & 31) == 0 && release_slot(&sh->done[slot])) {
        sh->done[slot] = 0u;
        const int next = si + kNStages;
        if (!stop && next < s1) {
          fence_proxy_async();
          issue(next, slot);
        }
      }
    }
    if (stop) {
      // stages [si, min(s1, si - 1 + kNStages)) were requested and not read
      const int end = min(s1, si - 1 + kNStages);
      for (; si < end; ++si) {
        const int slot = static_cast<int>(cs % kNStages);
        if (!mbar_wait(&sh->full[slot], (cs / kNStages) & 1u)) atomicOr(&sh->timeout, 1u);
        ++cs;
      }
    }
    cta_sync();
  }

  template <typename F>
  __device__ void pass(int s0, int s1, F&& f) {
    start(s0, s1);
    consume(s0, s1, static_cast<F&&>(f));
  }

  // One warp done with a slot (acquire-release, CTA scope): true for the
  // warp that completes the slot's count.
  __device__ static bool release_slot(uint32_t* done) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                 : "=r"(old)
                 : "r"(smem_addr(done))
                 : "memory");
    return old == static_cast<uint32_t>(kRW - 1);
  }
};

// ---------------------------------------------------------------------------
// general radix descent (fp32 keys, or a window miss)

template <typename Raw>
__device__ Desc descend(Ring<Raw>& ring, float c, float m, int fx_shift, bool by_mass,
                        bool need_mass, u64 target, float p, RowSh& sh, RadixArrays& ra) {
  constexpr int KB = KeyTraits<Raw>::kBits;
  constexpr int VEC = 16 / sizeof(Raw);
  const float fxs = fx_scale(fx_shift);
  uint32_t prefix = 0;
  u64 above_cnt = 0, above_mass = 0;
  Desc out{};
  for (int shift = KB - 8; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < kBins; b += kRT) {
      ra.cnt[b] = 0;
      ra.mass[b] = 0;
    }
    cta_sync();
    const int pshift = shift + 8;
    const uint32_t pre = prefix;
    auto one = [&](Raw raw) {
      const uint32_t key = key_of(raw);
      if (pshift >= KB || (key >> pshift) == pre) {
        const uint32_t digit = (key >> shift) & 255u;
        atomicAdd(&ra.cnt[digit], 1u);
        if (need_mass) {
          const u64 fx = __float2ull_rn(ex2(__fmul_rn(value_of(raw), c) - m) * fxs);
          if (fx) atomicAdd(&ra.mass[digit], fx);
        }
      }
    };
    ring.pass(0, ring.nst(), [&](const Raw* st, int n, int) {
      const int nv = n / VEC;
      const uint4* v4 = reinterpret_cast<const uint4*>(st);
      for (int v = threadIdx.x; v < nv; v += kRT) {
        Raw r[VEC];
        unpack(v4[v], r);
#pragma unroll
        for (int i = 0; i < VEC; ++i) one(r[i]);
      }
      for (int j = nv * VEC + threadIdx.x; j < n; j += kRT) one(st[j]);
      return false;
    });
    if (threadIdx.x < 32) {
      u64 tgt = target;
      if (tgt == 0) {
        u64 tot = 0;
        for (int i = threadIdx.x; i < kBins; i += 32) tot += ra.mass[i];
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
    cta_sync();
    target = sh.ulred[0];
    above_cnt += sh.sel.b_above_cnt;
    above_mass += sh.sel.b_above_mass;
    prefix = (prefix << 8) | sh.sel.b_key;
    out.at_cnt = sh.sel.b_at_cnt;
    out.at_mass = sh.sel.b_at_mass;
    cta_sync();
  }
  out.key = prefix;
  out.above_cnt = above_cnt;
  out.above_mass = above_mass;
  sh.ulred[1] = target;  // the resolved target (for the implicit top-p case)
  cta_sync();
  return out;
}

// ---------------------------------------------------------------------------
// the streamed pass

// bf16 stage: every thread takes every kRT-th 16-byte vector, kChains in
// flight, each into its own statistics chain and, with a window, into the
// exact-key histogram (elements outside the window into this lane's spill
// bin, nb + lane).
template <int MODE>
__device__ __forceinline__ void stage_bf16(const uint16_t* st, int n, float c, f32x2 c2,
                                           Chain (&ch)[kChains], uint32_t& vmax2, uint32_t wbase,
                                           uint32_t nb, uint32_t hist_s) {
  const int nv = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  const uint32_t spill = nb + (threadIdx.x & 31);
  int v = threadIdx.x;
  for (; v + (kChains - 1) * kRT < nv; v += kChains * kRT) {
    uint4 q[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) q[k] = v4[v + k * kRT];
#pragma unroll
    for (int k = 0; k < kChains; ++k) chain_vec(q[k], c, c2, ch[k], vmax2);
    if constexpr (MODE != kWinNone) {
#pragma unroll
      for (int k = 0; k < kChains; ++k) hist_vec<MODE>(q[k], wbase, spill, hist_s);
    }
  }
  for (; v < nv; v += kRT) {
    const uint4 q = v4[v];
    chain_vec(q, c, c2, ch[0], vmax2);
    if constexpr (MODE != kWinNone) hist_vec<MODE>(q, wbase, spill, hist_s);
  }
  for (int j = nv * 8 + threadIdx.x; j < n; j += kRT) {
    const uint32_t r = st[j];
    vmax2 = bmax2(vmax2, r | (r << 16));
    float u[1] = {__fmul_rn(value_of(static_cast<uint16_t>(r)), c)};
    stats_add(ch[0].s, u);
    if constexpr (MODE != kWinNone) red_inc(hist_s + (min(win_index<MODE>(r, wbase), spill) << 2));
  }
}

__device__ __forceinline__ void stats_stage_f32(const uint32_t* st, int n, float c, Stats (&s2)[2],
                                                float& vmax) {
  Stats& s = s2[0];
  const int nv = n / 4;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  for (int v = threadIdx.x; v < nv; v += kRT) {
    const uint4 q = v4[v];
    const float x[4] = {__uint_as_float(q.x), __uint_as_float(q.y), __uint_as_float(q.z),
                        __uint_as_float(q.w)};
    float u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      vmax = fmaxf(vmax, x[i]);
      u[i] = __fmul_rn(x[i], c);
    }
    stats_add(s, u);
  }
  for (int j = nv * 4 + threadIdx.x; j < n; j += kRT) {
    const float x = __uint_as_float(st[j]);
    vmax = fmaxf(vmax, x);
    float u[1] = {__fmul_rn(x, c)};
    stats_add(s, u);
  }
}

// Block sum of the support sums, valid in every thread (warp 0 reduces the
// warps' partials in a fixed order and broadcasts).
__device__ __forceinline__ SupSums block_sum_sup(SupSums v, RowSh& sh) {
  __shared__ SupSums s_res;
  auto warp_sum = [](SupSums& x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x.ngt += __shfl_xor_sync(0xffffffffu, x.ngt, o);
      x.neq += __shfl_xor_sync(0xffffffffu, x.neq, o);
      x.ntp += __shfl_xor_sync(0xffffffffu, x.ntp, o);
      x.smass += __shfl_xor_sync(0xffffffffu, x.smass, o);
      x.sa += __shfl_xor_sync(0xffffffffu, x.sa, o);
    }
  };
  warp_sum(v);
  if ((threadIdx.x & 31) == 0) sh.sums[threadIdx.x >> 5] = v;
  cta_sync();
  if (threadIdx.x < 32) {
    SupSums t = threadIdx.x < kRW ? sh.sums[threadIdx.x] : SupSums{0u, 0u, 0u, 0.f, 0.f};
    warp_sum(t);
    if (threadIdx.x == 0) s_res = t;
  }
  cta_sync();
  return s_res;
}

// Number of elements of g[j0, j1) whose raw bits are r0 or r1 (the two
// encodings of one key), read from global memory by the block with
// kCountUnroll 16-byte loads in flight per thread; j0 need not be a multiple
// of 8.  Result in thread 0 only after the caller's block sum.
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
  for (int j = j0 + static_cast<int>(threadIdx.x); j < ja; j += kRT) one(g[j]);
  const int nv = (j1 - ja) >> 3;
  const uint4* v4 = reinterpret_cast<const uint4*>(g + ja);
  int v = threadIdx.x;
  for (; v + (kCountUnroll - 1) * kRT < nv; v += kCountUnroll * kRT) {
    uint4 q[kCountUnroll];
#pragma unroll
    for (int k = 0; k < kCountUnroll; ++k) q[k] = __ldcg(v4 + v + k * kRT);
#pragma unroll
    for (int k = 0; k < kCountUnroll; ++k) vec(q[k]);
  }
  for (; v < nv; v += kRT) vec(__ldcg(v4 + v));
  for (int j = ja + nv * 8 + static_cast<int>(threadIdx.x); j < j1; j += kRT) one(g[j]);
  return n;
}

// Elements before position y holding the target's key tkey, for a target in
// a tie group of `group` elements: counted by the block on the shorter side
// of y (after y: the group less the target and the ties that follow it).
// Every thread gets the count.
__device__ __forceinline__ uint32_t ties_before_target(const uint16_t* g16, int V, int y,
                                                       uint32_t tkey, uint32_t group,
                                                       uint32_t* red) {
  const uint32_t r0 = tkey >= 0x7FFFu ? tkey - 0x7FFFu : 0xFFFFu - tkey;
  const uint32_t r1 = tkey == 0x7FFFu ? 0x8000u : r0;  // -0 shares the key of +0
  const bool before = y <= V - 1 - y;
  const uint32_t part = before ? count_raw(g16, 0, y, r0, r1) : count_raw(g16, y + 1, V, r0, r1);
  const uint32_t n = block_sum(part, red);
  return before ? n : group - 1u - n;
}

// ---------------------------------------------------------------------------
// warp-level pieces of the decision (warp 0, no block barriers)

// Warp maximum by one redux.sync over order-preserving keys of the values
// (a NaN takes the lowest key, so it is ignored as fmaxf ignores it, and an
// all-NaN warp gets NaN back).
__device__ __forceinline__ float warp_max(float v) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t k = v != v ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
  const uint32_t m = __reduce_max_sync(0xffffffffu, k);
  return __uint_as_float((m & 0x80000000u) ? (m & 0x7FFFFFFFu) : ~m);
}

// Statistics merged over the warp (every lane gets them): the warp maximum
// first, each lane rebased onto it once, then plain sums in a fixed order.
__device__ __forceinline__ Stats warp_stats(Stats s) {
  const float m = warp_max(s.m);
  if (s.c0 != 0.f || s.zr != 0.f) stats_rebase(s, m);
  float c0 = s.c0, zr = s.zr, a = s.a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c0 += __shfl_xor_sync(0xffffffffu, c0, o);
    zr += __shfl_xor_sync(0xffffffffu, zr, o);
    a += __shfl_xor_sync(0xffffffffu, a, o);
  }
  return Stats{m, c0, zr, a};
}

// From bin `top` of the window down, the bin at which the cumulative count
// (by_mass false) or fixed-point mass first reaches need (>= 1); chunks of
// 256 bins, lane l holding bins hi - 8l - k (k = 0..7) of a chunk.  False
// when the bins [0, top] hold less than need.
__device__ bool warp_search(const Window& w, int top, bool by_mass, u64 need, Desc& out,
                            SupSums* above = nullptr) {
  const int lane = threadIdx.x & 31;
  u64 ac = 0, am = 0;  // above the current chunk
  SupSums acc{0u, 0u, 0u, 0.f, 0.f};  // this lane's bins above the current chunk
  for (int hi = top; hi >= 0; hi -= 256) {
    uint32_t cnt[8];
    u64 fx[8];
    float em8[8], ea8[8];
    uint32_t topm = 0;  // bins holding the row maximum (d == 0)
    u64 lc = 0, lm = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int b = hi - 8 * lane - k;
      cnt[k] = b >= 0 ? w.hist[b] : 0u;
      const float d = key_u(w.klo + static_cast<uint32_t>(b), w.c) - w.m;
      const float e = ex2(d);
      const float fc = static_cast<float>(cnt[k]);
      fx[k] = cnt[k] ? static_cast<u64>(cnt[k]) * __float2ull_rn(e * w.fxs) : 0ull;
      if (d == 0.f) topm |= 1u << k;
      em8[k] = cnt[k] && d != 0.f ? fc * e : 0.f;  // the sums' terms, as in warp_sums
      ea8[k] = cnt[k] ? fc * d * e : 0.f;
      lc += cnt[k];
      lm += fx[k];
    }
    u64 pc = lc, pm = lm;  // inclusive prefix from lane 0 (the largest keys)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const u64 tc = __shfl_up_sync(0xffffffffu, pc, o), tm = __shfl_up_sync(0xffffffffu, pm, o);
      if (lane >= o) {
        pc += tc;
        pm += tm;
      }
    }
    const u64 ec = ac + pc - lc, em = am + pm - lm;
    const u64 base = by_mass ? em : ec, mine = by_mass ? lm : lc;
    const uint32_t ball = __ballot_sync(0xffffffffu, base < need && need <= base + mine);
    const int src = ball ? __ffs(ball) - 1 : 32;
    // kx = this lane's bins above the crossing: all 8 before the crossing
    // lane, none after it, and in it those before its first bin whose
    // running sum reaches need (a hit mask and predicated selects: no
    // divergent branch per bin)
    uint32_t hit = 0;
    {
      u64 run = base;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        run += by_mass ? fx[k] : static_cast<u64>(cnt[k]);
        hit |= (cnt[k] != 0u && run >= need) ? (1u << k) : 0u;
      }
    }
    const int kx = lane < src ? 8 : (lane > src ? 0 : __ffs(hit) - 1);
    uint32_t key = 0, at_c = 0;
    u64 rc = ec, rm = em, at_m = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool take = k < kx;
      rc += take ? cnt[k] : 0u;
      rm += take ? fx[k] : 0ull;
      acc.ngt += take ? cnt[k] : 0u;
      acc.ntp += take && ((topm >> k) & 1u) ? cnt[k] : 0u;
      acc.smass += take ? em8[k] : 0.f;
      acc.sa += take ? ea8[k] : 0.f;
      if (k == kx) {
        key = w.klo + static_cast<uint32_t>(hi - 8 * lane - k);
        at_c = cnt[k];
        at_m = fx[k];
      }
    }
    if (ball) {
      out.key = __shfl_sync(0xffffffffu, key, src);
      out.above_cnt = __shfl_sync(0xffffffffu, rc, src);
      out.above_mass = __shfl_sync(0xffffffffu, rm, src);
      out.at_cnt = __shfl_sync(0xffffffffu, static_cast<u64>(at_c), src);
      out.at_mass = __shfl_sync(0xffffffffu, at_m, src);
      if (above) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          acc.smass += __shfl_xor_sync(0xffffffffu, acc.smass, o);
          acc.sa += __shfl_xor_sync(0xffffffffu, acc.sa, o);
        }
        acc.ngt = __reduce_add_sync(0xffffffffu, acc.ngt);
        acc.ntp = __reduce_add_sync(0xffffffffu, acc.ntp);
        acc.neq = static_cast<uint32_t>(out.at_cnt);
        *above = acc;
      }
      return true;
    }
    ac += __shfl_sync(0xffffffffu, pc, 31);
    am += __shfl_sync(0xffffffffu, pm, 31);
  }
  return false;
}

// Support sums over the bins of keys (tkey, kmr] and the count at tkey,
// reduced over the warp in a fixed order (every lane gets them).
__device__ SupSums warp_sums(const Window& w, uint32_t tkey, uint32_t kmr) {
  const int lane = threadIdx.x & 31;
  SupSums v{0u, 0u, 0u, 0.f, 0.f};
  float sm[4] = {0.f, 0.f, 0.f, 0.f}, sa[4] = {0.f, 0.f, 0.f, 0.f};
  const int hi = static_cast<int>(kmr - w.klo);
  int b = static_cast<int>(tkey - w.klo) + 1 + lane;
  // four bins per lane in flight, each into its own accumulators
  for (; b + 96 <= hi; b += 128) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int bk = b + 32 * k;
      const uint32_t cnt = w.hist[bk];
      const float d = key_u(w.klo + static_cast<uint32_t>(bk), w.c) - w.m;
      const float e = cnt ? ex2(d) : 0.f;
      const float fc = static_cast<float>(cnt);
      v.ngt += cnt;
      if (d == 0.f)
        v.ntp += cnt;
      else
        sm[k] = fmaf(fc, e, sm[k]);
      sa[k] = fmaf(fc * d, e, sa[k]);
    }
  }
  for (; b <= hi; b += 32) {
    const uint32_t cnt = w.hist[b];
    const float d = key_u(w.klo + static_cast<uint32_t>(b), w.c) - w.m;
    const float e = cnt ? ex2(d) : 0.f;
    const float fc = static_cast<float>(cnt);
    v.ngt += cnt;
    if (d == 0.f)
      v.ntp += cnt;
    else
      sm[0] = fmaf(fc, e, sm[0]);
    sa[0] = fmaf(fc * d, e, sa[0]);
  }
  v.smass = (sm[0] + sm[1]) + (sm[2] + sm[3]);
  v.sa = (sa[0] + sa[1]) + (sa[2] + sa[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.ngt += __shfl_xor_sync(0xffffffffu, v.ngt, o);
    v.ntp += __shfl_xor_sync(0xffffffffu, v.ntp, o);
    v.smass += __shfl_xor_sync(0xffffffffu, v.smass, o);
    v.sa += __shfl_xor_sync(0xffffffffu, v.sa, o);
  }
  v.neq = w.hist[tkey - w.klo];
  return v;
}


__device__ __forceinline__ RowOut row_out_init(const Stats& s, float vmax, bool any_filter, int V) {
  RowOut o;
  o.s = s;
  o.vmax = vmax;
  o.nonfinite = !stats_finite(s) || !isfinite(vmax);
  o.m = s.m;  // = fl(vmax c)
  o.log2z = stats_log2z(s);
  o.h_full = kLn2 * (o.log2z - s.a / stats_z(s));
  o.filtered = !o.nonfinite && any_filter;
  o.cut_known = true;
  o.tkey = 0;
  o.tie_cut = INT_MAX;
  o.ckeep = 0;
  o.ylt = 0;
  o.log2zs = o.log2z;
  o.h_support = o.h_full;
  o.c0s = s.c0;
  o.zrs = s.zr;
  o.n_support = o.nonfinite ? 0 : V;
  return o;
}

// Support statistics from the sums above the threshold and the ckeep kept
// elements of its tie group.
__device__ __forceinline__ void support_stats(RowOut& o, const SupSums& sums, float c) {
  const float dt = __fmul_rn(KeyTraits<uint16_t>::decode(o.tkey), c) - o.m;
  const float et = ex2(dt);
  Stats ss;
  ss.m = o.m;
  ss.c0 = static_cast<float>(sums.ntp) + (dt == 0.f ? static_cast<float>(o.ckeep) : 0.f);
  ss.zr = sums.smass + (dt == 0.f ? 0.f : static_cast<float>(o.ckeep) * et);
  ss.a = sums.sa + static_cast<float>(o.ckeep) * dt * et;
  o.log2zs = stats_log2z(ss);
  o.h_support = kLn2 * (o.log2zs - ss.a / stats_z(ss));
  o.c0s = ss.c0;
  o.zrs = ss.zr;
  o.n_support = static_cast<int32_t>(sums.ngt + o.ckeep);
}

// The per-row outputs (one thread).
template <typename Raw>
__device__ void emit_row(const ScoreParams& P, int row, const RowOut& o, bool target_ok, int y,
                         Raw ry, float c, uint32_t timeout) {
  uint32_t status = 0;
  float lp_v = __int_as_float(0x7fc00000), lp_s = __int_as_float(0x7fc00000);
  bool in_s = false;
  if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
  if (o.nonfinite) {
    status |= VS_ROW_NONFINITE_INPUT;
  } else if (target_ok) {
    const float uy = __fmul_rn(value_of(ry), c);
    lp_v = kLn2 * (uy - o.m - o.log2z);
    if (!o.filtered) {
      in_s = true;
    } else {
      const uint32_t ky = key_of(ry);
      in_s = ky > o.tkey || (ky == o.tkey && (o.cut_known ? y <= o.tie_cut : o.ylt < o.ckeep));
    }
    if (in_s) {
      lp_s = o.filtered ? kLn2 * (uy - o.m - o.log2zs) : lp_v;
    } else {
      lp_s = -kInf;
      status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
    }
  }
  if (timeout) status |= kRowDeviceTimeout;
  const float nan = __int_as_float(0x7fc00000);
  if (P.lp_full) P.lp_full[row] = lp_v;
  if (P.lp_support) P.lp_support[row] = lp_s;
  if (P.want_entropy) {
    if (P.h_full) P.h_full[row] = o.nonfinite ? nan : o.h_full;
    if (P.h_support) P.h_support[row] = o.nonfinite ? nan : o.h_support;
  }
  if (P.valid) P.valid[row] = o.nonfinite ? 0 : 1;
  if (P.status) P.status[row] = status;
  if (P.support_size) P.support_size[row] = o.n_support;
  if (P.ctx) {
    RowCtx cx{};
    cx.m2 = o.vmax;
    cx.log2z = o.log2z;
    cx.msup = o.vmax;
    cx.log2zs = o.log2zs;
    cx.h_full = o.h_full;
    cx.h_support = o.h_support;
    cx.c = c;
    cx.tkey = o.tkey;
    cx.tie_cut = o.tie_cut;
    uint32_t f = kCtxFullStats;
    if (o.nonfinite) f |= kCtxNonFinite | kCtxEmpty;
    else if (!o.filtered) f |= kCtxAllVocab;
    else f |= kCtxThreshold;
    if (target_ok) f |= kCtxTargetOk;
    if (in_s) f |= kCtxTargetInS;
    cx.flags = f;
    cx.n_support = o.n_support;
    cx.status = status;
    cx.c0_full = o.s.c0;
    cx.zr_full = o.s.zr;
    cx.c0_sup = o.c0s;
    cx.zr_sup = o.zrs;
    P.ctx[row] = cx;
  }
}

// ---------------------------------------------------------------------------

template <typename Raw>
__global__ void __launch_bounds__(kRT, 1) score_row_kernel(ScoreParams P) {
  constexpr bool kBf16 = sizeof(Raw) == 2;
  constexpr int VEC = 16 / sizeof(Raw);
  using KT = KeyTraits<Raw>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Raw* ringbuf = reinterpret_cast<Raw*>(smem_raw);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw + kNStages * kStageBytes);
  RadixArrays& ra = *reinterpret_cast<RadixArrays*>(hist);
  RowSh& sh = *reinterpret_cast<RowSh*>(smem_raw + kNStages * kStageBytes + (kWin + 32) * 4);

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int V = P.vocab;
  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld;

  if (tid == 0) {
    for (int s = 0; s < kNStages; ++s) {
      mbar_init(&sh.full[s], 1);
      sh.done[s] = 0u;
    }
    mbar_init(&sh.first, 1);
    sh.timeout = 0;
    sh.tie_cut = INT_MAX;
    fence_barrier_init();
  }
  // launched programmatically after whatever kernel precedes it on the
  // stream: wait for that grid (and its memory) before reading anything;
  // the next kernel may be scheduled from here on
  pdl_wait();
  pdl_launch_dependents();
  cta_sync();
  Ring<Raw> ring{grow, V, ringbuf, &sh, 0u, 0u};

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
  const Raw ry = target_ok ? grow[y] : Raw(0);

  // ---- the streamed pass: online statistics and the row maximum; for a
  // filtered bf16 row also the exact-key window histogram
  Chain ch2[kChains];                             // bf16 rows
  uint32_t vmax2 = 0xFF80FF80u;                    // bf16 rows: packed running max
  Stats s2[2] = {stats_empty(), stats_empty()};    // fp32 rows
  float vmax = -kInf;
  const bool hist_on = kBf16 && any_filter;
  uint32_t wtop = 0, wlo = 0;  // window keys [wlo, wtop]
  int wmode = kWinNone;
  uint32_t wbase = 0;
  const uint32_t hist_s = smem_addr(hist);
  const int nst = ring.nst();
  if constexpr (kBf16) {
    // the first piece of stage 0 is requested apart, ahead of the ring: its
    // maximum m0, a lower bound of the row maximum m, fixes the window and
    // seeds every chain's running maximum (so that later vectors rarely
    // raise it and take the packed path) while the ring fills
    const int nh = min(V, kHeadElems);
    const uint32_t hbytes = static_cast<uint32_t>((nh * 2 + 15) & ~15);
    if (tid == 0) {
      mbar_arrive_expect_tx(&sh.first, hbytes);
      bulk_load(ringbuf, grow, hbytes, &sh.first);
      ring.head = hbytes;
    }
    ring.start(0, nst);
    // warp 0 finds m0 and the window while the other warps clear every bin
    if (hist_on && warp != 0)
      for (int b = tid - 32; b < kWin + 32; b += kRT - 32) hist[b] = 0u;
    if (warp == 0) {
      if (!mbar_wait(&sh.first, 0)) atomicOr(&sh.timeout, 1u);
      const uint16_t* h16 = reinterpret_cast<const uint16_t*>(ringbuf);
      const uint4* h4 = reinterpret_cast<const uint4*>(ringbuf);
      uint32_t mx = 0xFF80FF80u;
      for (int v = lane; v < nh / 8; v += 32) {
        const uint4 q = h4[v];
        mx = bmax2(mx, bmax2(bmax2(q.x, q.y), bmax2(q.z, q.w)));
      }
      float mh = vmax_of(mx);
      for (int j = (nh / 8) * 8 + lane; j < nh; j += 32) mh = fmaxf(mh, value_of(h16[j]));
      const float m0 = warp_max(mh);
      if (hist_on) {
        // elements below the level found with m0 are below the level of m too
        const uint32_t kref = key_of(static_cast<uint16_t>(__float_as_uint(m0) >> 16));
        wtop = min(kref + kWinHi, KT::kInfKey);
        wlo = wtop >= static_cast<uint32_t>(kWin - 1) ? wtop - (kWin - 1) : 0u;
        if (!use_k && isfinite(m0)) {
          float dlo = -kInf;
          if (use_minp) dlo = log2f(mp) - 1.f;
          if (use_p && pp > 0.f) dlo = fmaxf(dlo, log2f((1.f - pp) / static_cast<float>(V)) - 2.f);
          if (dlo > -kInf) wlo = key_at_level(wlo, wtop, c, __fmul_rn(m0, c), dlo);
        }
        win_mode(wlo, wtop, wmode, wbase);
      }
      if (lane == 0) {
        sh.w_m0 = m0;
        sh.w_top = wtop;
        sh.w_lo = wlo;
        sh.w_base = wbase;
        sh.w_mode = wmode;
      }
    }
    cta_sync();
    const float m0 = sh.w_m0;
    wtop = sh.w_top;
    wlo = sh.w_lo;
    wbase = sh.w_base;
    wmode = sh.w_mode;
#pragma unroll
    for (int k = 0; k < kChains; ++k) chain_seed(ch2[k], m0, c);
    const uint32_t nb = (wtop - wlo) + 1u;
    const f32x2 c2 = pack2(c, c);
    ring.consume(0, nst, [&](const Raw* st, int n, int) {
      const uint16_t* st16 = reinterpret_cast<const uint16_t*>(st);
      if (wmode == kWinNone)
        stage_bf16<kWinNone>(st16, n, c, c2, ch2, vmax2, wbase, nb, hist_s);
      else if (wmode == kWinPos)
        stage_bf16<kWinPos>(st16, n, c, c2, ch2, vmax2, wbase, nb, hist_s);
      else if (wmode == kWinNeg)
        stage_bf16<kWinNeg>(st16, n, c, c2, ch2, vmax2, wbase, nb, hist_s);
      else
        stage_bf16<kWinKey>(st16, n, c, c2, ch2, vmax2, wbase, nb, hist_s);
      return false;
    });
  } else {
    ring.pass(0, nst, [&](const Raw* st, int n, int) {
      stats_stage_f32(st, n, c, s2, vmax);
      return false;
    });
  }
  // ---- per-warp partial statistics; warp 0 merges them and, in the
  // common case, takes the whole decision from the bins with warp shuffles
  // (no block barriers); otherwise the block takes the general path below
  Stats s;
  if constexpr (kBf16) {
    s = ch2[0].s;
#pragma unroll
    for (int k = 1; k < kChains; ++k) stats_merge(s, ch2[k].s);
    vmax = vmax_of(vmax2);
  } else {
    s = s2[0];
    stats_merge(s, s2[1]);
  }
  s = warp_stats(s);
  vmax = warp_max(vmax);
  if (lane == 0) {
    sh.wst[warp] = s;
    sh.fred[warp] = vmax;
  }
  cta_sync();
  const bool want_cut = P.ctx != nullptr || P.support_mask != nullptr || P.sampled != nullptr;
  if (warp == 0) {
    s = warp_stats(lane < kRW ? sh.wst[lane] : stats_empty());
    vmax = warp_max(lane < kRW ? sh.fred[lane] : -kInf);
    RowOut o = row_out_init(s, vmax, any_filter, V);
    bool fast = kBf16;
    uint32_t ylt_group = 0;  // size of the target's tie group when its rank there decides
    bool reuse = false;      // the decision is made; only the cut's position is missing
    u64 reuse_tot = 0;
    if constexpr (kBf16) {
    if (o.filtered) {
      const float fxs = fx_scale(P.fx_shift);
      const uint32_t kmr = key_of(static_cast<uint16_t>(__float_as_uint(vmax) >> 16));
      const Window w{wlo, wtop, static_cast<int>(wtop - wlo) + 1, wmode, 0u, hist, c, o.m, fxs};
      bool win_ok = kmr <= wtop;
      bool all_ties = true, have_t = false;
      u64 cnum = 0;
      SupSums psums{0u, 0u, 0u, 0.f, 0.f};  // the sums above the top-p crossing
      bool have_psums = false;
      uint32_t dp_key = 0;
      if (win_ok && (use_k || use_p)) {
        const int top = static_cast<int>(kmr - wlo);
        Desc dk{}, dp{};
        u64 ck = 0;
        if (use_k) {
          win_ok = warp_search(w, top, false, static_cast<u64>(kk), dk);
          if (win_ok) {
            ck = static_cast<u64>(kk) - dk.above_cnt;
            o.tkey = dk.key;
            cnum = ck;
            all_ties = ck >= dk.at_cnt;
            have_t = true;
          }
        }
        if (win_ok && use_p) {
          const double mass1 = use_k ? static_cast<double>(dk.above_mass + ck * bin_fx(w, dk.key))
                                     : (static_cast<double>(s.c0) + static_cast<double>(s.zr)) *
                                           static_cast<double>(fxs);
          const u64 tp = topp_target(pp, mass1);
          win_ok = warp_search(w, top, true, tp, dp, &psums);
          have_psums = win_ok;
          dp_key = dp.key;
          if (win_ok) {
            u64 cp = topp_ties(dp, tp, bin_fx(w, dp.key));
            if (use_k && dp.key == o.tkey && cp > ck) cp = ck;
            o.tkey = dp.key;
            cnum = cp;
            all_ties = cp >= dp.at_cnt;
            have_t = true;
          }
        }
        if (!win_ok && use_p && !use_k && use_minp && minp_key<Raw>(mp, c, o.m) >= w.klo) {
          win_ok = true;
          have_t = false;
          all_ties = true;
        }
      }
      if (!win_ok && (use_k || use_p)) {
        fast = false;  // the decision lies outside the window
      } else {
        if (use_minp) {
          const uint32_t lo = minp_key<Raw>(mp, c, o.m);
          if (!have_t || lo > o.tkey) {
            o.tkey = lo;
            all_ties = true;
          }
        }
        if (!win_ok || o.tkey < wlo) {
          fast = false;  // the support sums need a pass over the row
        } else {
          // the top-p search summed the bins above its key on the way down
          const SupSums sums = have_psums && o.tkey == dp_key ? psums : warp_sums(w, o.tkey, kmr);
          const u64 tot_eq = sums.neq;
          o.ckeep = all_ties ? tot_eq : (cnum < tot_eq ? cnum : tot_eq);
          support_stats(o, sums, c);
          if (o.ckeep < tot_eq) {
            o.cut_known = false;
            // the cut's position needs a pass over the row (the block takes
            // warp 0's decision and finds it below); so does the target's
            // rank in a partly kept tie group (counted by the block below,
            // from L2)
            if (want_cut) {
              fast = false;
              reuse = true;
              reuse_tot = tot_eq;
            } else if (target_ok && key_of(ry) == o.tkey) {
              ylt_group = tot_eq;
            }
          }
        }
      }
    }
    }
    if (lane == 0) {
      sh.rs = s;
      sh.rvmax = vmax;
      sh.general = fast ? 0u : 1u;
      sh.ylt_group = fast ? ylt_group : 0u;
      sh.reuse = reuse ? 1u : 0u;
      if (reuse) {
        sh.rout = o;
        sh.reuse_tot = reuse_tot;
      }
      if (fast) {
        sh.d_tkey = o.tkey;
        sh.d_flags = (o.nonfinite ? 1u : 0u) | (o.filtered ? 2u : 0u);
        if (ylt_group)
          sh.rout = o;
        else
          emit_row(P, row, o, target_ok, y, ry, c, sh.timeout);
      }
    }
  }
  cta_sync();
  if constexpr (kBf16) {
    if (sh.ylt_group) {
      // the target sits in the partly kept tie group of the threshold key:
      // its rank there decides its membership
      const uint32_t ylt = ties_before_target(reinterpret_cast<const uint16_t*>(grow), V, y,
                                              sh.d_tkey, sh.ylt_group, sh.ured);
      if (tid == 0) {
        RowOut o = sh.rout;
        o.ylt = ylt;
        emit_row(P, row, o, target_ok, y, ry, c, sh.timeout);
      }
    }
  }
  bool nonfinite, filtered;
  uint32_t tkey = 0;
  int32_t tie_cut = INT_MAX;
  if (!sh.general) {
    nonfinite = (sh.d_flags & 1u) != 0;
    filtered = (sh.d_flags & 2u) != 0;
    tkey = sh.d_tkey;
  } else {
  s = sh.rs;
  vmax = sh.rvmax;
  nonfinite = !stats_finite(s) || !isfinite(vmax);
  const float m = s.m;  // = fl(vmax c)
  const float log2z = stats_log2z(s);
  const float h_full = kLn2 * (log2z - s.a / stats_z(s));
  filtered = !nonfinite && any_filter;

  bool cut_known = true;  // tie_cut resolved (or not needed: every tie kept)
  u64 ckeep = 0;
  u64 tie_group = 0;  // elements holding the threshold key
  float log2zs = log2z, h_support = h_full, c0s = s.c0, zrs = s.zr;
  int32_t n_support = nonfinite ? 0 : V;

  const bool reuse = kBf16 && sh.reuse != 0u;
  u64 tot_eq = 0;
  if (filtered && reuse) {
    // warp 0's decision and support statistics, as the fast path has them
    const RowOut& o = sh.rout;
    tkey = o.tkey;
    ckeep = o.ckeep;
    tot_eq = sh.reuse_tot;
    tie_group = tot_eq;
    log2zs = o.log2zs;
    h_support = o.h_support;
    c0s = o.c0s;
    zrs = o.zrs;
    n_support = o.n_support;
  } else if (filtered) {
    const float fxs = fx_scale(P.fx_shift);
    bool all_ties = true;
    u64 cnum = 0;
    bool have_t = false;
    Window w{};
    // the window holds every key at or above its floor only when the row
    // maximum lies inside it
    bool win_ok = false;
    if constexpr (kBf16) {
      const uint32_t kmr = key_of(static_cast<uint16_t>(__float_as_uint(vmax) >> 16));
      w.kmax = wtop;
      w.klo = wlo;
      w.nbins = static_cast<int>(wtop - wlo) + 1;
      w.hist = hist;
      w.c = c;
      w.m = m;
      w.fxs = fxs;
      win_ok = kmr <= wtop;
      if (win_ok && (use_k || use_p)) {
        Desc dk{}, dp{};
        u64 ck = 0;
        if (use_k) {
          win_ok = win_search<kRT>(w, false, static_cast<u64>(kk), dk, sh.sel);
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
            mass1 = (static_cast<double>(s.c0) + static_cast<double>(s.zr)) * static_cast<double>(fxs);
          }
          const u64 tp = topp_target(pp, mass1);
          win_ok = win_search<kRT>(w, true, tp, dp, sh.sel);
          if (win_ok) {
            u64 cp = topp_ties(dp, tp, bin_fx(w, dp.key));
            if (use_k && dp.key == tkey && cp > ck) cp = ck;
            tkey = dp.key;
            cnum = cp;
            all_ties = cp >= dp.at_cnt;
            have_t = true;
          }
        }
        if (!win_ok && use_p && !use_k && use_minp && kmr <= wtop &&
            minp_key<Raw>(mp, c, m) >= w.klo) {
          // the top-p crossing lies below the window, whose floor is at or
          // below the min-p level: min-p decides the support (applied below)
          win_ok = true;
          have_t = false;
          all_ties = true;
        }
      }
    }
    if (!win_ok && (use_k || use_p)) {
      // ---- general radix descent (fp32 keys, or the decision lies outside
      // the window)
      have_t = false;
      all_ties = true;
      if (use_k) {
        Desc d = descend(ring, c, m, P.fx_shift, false, use_p, static_cast<u64>(kk), 1.f, sh, ra);
        const u64 ck = static_cast<u64>(kk) - d.above_cnt;
        tkey = d.key;
        cnum = ck;
        all_ties = ck >= d.at_cnt;
        have_t = true;
        if (use_p) {
          const u64 fx_t = key_fx<Raw>(d.key, c, m, fx_scale(P.fx_shift));
          const u64 tp = topp_target(pp, static_cast<double>(d.above_mass + ck * fx_t));
          Desc e = descend(ring, c, m, P.fx_shift, true, true, tp, pp, sh, ra);
          u64 cp = topp_ties(e, tp, key_fx<Raw>(e.key, c, m, fx_scale(P.fx_shift)));
          if (e.key == tkey && cp > ck) cp = ck;
          tkey = e.key;
          cnum = cp;
          all_ties = cp >= e.at_cnt;
        }
      } else {
        Desc e = descend(ring, c, m, P.fx_shift, true, true, 0ull, pp, sh, ra);
        const u64 tp = sh.ulred[1];
        const u64 cp = topp_ties(e, tp, key_fx<Raw>(e.key, c, m, fx_scale(P.fx_shift)));
        tkey = e.key;
        cnum = cp;
        all_ties = cp >= e.at_cnt;
        have_t = true;
      }
    }
    if (use_minp) {
      const uint32_t lo = minp_key<Raw>(mp, c, m);
      if (!have_t || lo > tkey) {
        tkey = lo;
        all_ties = true;
        have_t = true;
      }
    }

    // ---- support sums: keys above tkey (max-valued elements counted apart)
    // and the tie group at tkey; from the bins when the window holds them
    SupSums sums{0u, 0u, 0u, 0.f, 0.f};
    bool from_bins = false;
    if constexpr (kBf16) from_bins = win_ok && tkey >= w.klo;
    if (from_bins) {
      const int per = (w.nbins + kRT - 1) / kRT;
      const int i0 = tid * per, i1 = min(w.nbins, i0 + per);
      for (int i = i0; i < i1; ++i) {
        const uint32_t cnt = w.hist[i];
        const uint32_t key = w.klo + i;
        if (cnt && key > tkey) {
          const float d = key_u(key, c) - m;
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
      if (tid == 0) sums.neq = w.hist[tkey - w.klo];
    } else {
      const uint32_t t = tkey;
      auto one = [&](Raw raw) {
        const uint32_t key = key_of(raw);
        if (key > t) {
          const float d = __fmul_rn(value_of(raw), c) - m;
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
      };
      ring.pass(0, ring.nst(), [&](const Raw* st, int n, int) {
        const int nv = n / VEC;
        const uint4* v4 = reinterpret_cast<const uint4*>(st);
        for (int v = threadIdx.x; v < nv; v += kRT) {
          Raw r[VEC];
          unpack(v4[v], r);
#pragma unroll
          for (int i = 0; i < VEC; ++i) one(r[i]);
        }
        for (int j = nv * VEC + threadIdx.x; j < n; j += kRT) one(st[j]);
        return false;
      });
    }
    sums = block_sum_sup(sums, sh);
    tot_eq = sums.neq;
    tie_group = tot_eq;
    ckeep = all_ties ? tot_eq : (cnum < tot_eq ? cnum : tot_eq);
    const float dt = __fmul_rn(KT::decode(tkey), c) - m;
    const float et = ex2(dt);
    Stats ss;
    ss.m = m;
    ss.c0 = static_cast<float>(sums.ntp) + (dt == 0.f ? static_cast<float>(ckeep) : 0.f);
    ss.zr = sums.smass + (dt == 0.f ? 0.f : static_cast<float>(ckeep) * et);
    ss.a = sums.sa + static_cast<float>(ckeep) * dt * et;
    log2zs = stats_log2z(ss);
    h_support = kLn2 * (log2zs - ss.a / stats_z(ss));
    c0s = ss.c0;
    zrs = ss.zr;
    n_support = static_cast<int32_t>(sums.ngt + ckeep);
  }
  if (filtered) {
    // ---- id of the last tie kept (ascending id order), when the saved
    // state, the bitmask or a sample needs it (fp32 rows: always)
    if (ckeep < tot_eq) {
      cut_known = false;
      if (want_cut || !kBf16) {
        const int need = static_cast<int>(ckeep);
        const uint32_t t = tkey;
        int seen = 0;  // ties in earlier stages (uniform)
        ring.pass(0, ring.nst(), [&](const Raw* st, int n, int base) {
          // thread tid owns the contiguous elements [j0, j1) of this stage
          const int per = ((n + kRT - 1) / kRT + VEC - 1) / VEC * VEC;
          const int j0 = min(n, tid * per), j1 = min(n, j0 + per);
          int mine = 0;
          int j = j0;
          const uint4* v4 = reinterpret_cast<const uint4*>(st);
          for (; j + 4 * VEC <= j1; j += 4 * VEC) {
            uint4 q[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) q[k] = v4[j / VEC + k];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              Raw r[VEC];
              unpack(q[k], r);
#pragma unroll
              for (int i = 0; i < VEC; ++i) mine += key_of(r[i]) == t;
            }
          }
          for (; j + VEC <= j1; j += VEC) {
            Raw r[VEC];
            unpack(v4[j / VEC], r);
#pragma unroll
            for (int i = 0; i < VEC; ++i) mine += key_of(r[i]) == t;
          }
          for (; j < j1; ++j) mine += key_of(st[j]) == t;
          int total;
          const int excl = seen + block_excl_int<kRT>(mine, total, sh.sel);
          if (excl < need && need <= excl + mine) {
            int cn = excl;
            for (int jj = j0; jj < j1; ++jj)
              if (key_of(st[jj]) == t && ++cn == need) {
                sh.tie_cut = base + jj;
                break;
              }
          }
          seen += total;
          return seen >= need;
        });
        tie_cut = sh.tie_cut;
        cut_known = true;
      }
    }
  }

  // ---- the target's earlier ties, when its membership hinges on them (bf16
  // rows; fp32 rows always resolve the cut above when it is needed)
  uint32_t ylt = 0;
  if (filtered && !cut_known && target_ok && key_of(ry) == tkey) {
    if constexpr (kBf16)
      ylt = ties_before_target(reinterpret_cast<const uint16_t*>(grow), V, y, tkey,
                               static_cast<uint32_t>(tie_group), sh.ured);
  }

  {
    RowOut o;
    o.s = s;
    o.vmax = vmax;
    o.m = m;
    o.log2z = log2z;
    o.h_full = h_full;
    o.nonfinite = nonfinite;
    o.filtered = filtered;
    o.tkey = tkey;
    o.tie_cut = tie_cut;
    o.cut_known = cut_known;
    o.ckeep = ckeep;
    o.ylt = ylt;
    o.log2zs = log2zs;
    o.h_support = h_support;
    o.c0s = c0s;
    o.zrs = zrs;
    o.n_support = n_support;
    if (tid == 0) emit_row(P, row, o, target_ok, y, ry, c, sh.timeout);
  }
  }  // general path

  // ---- support bitmask, one 32-id word per thread and stage
  if (P.support_mask) {
    const int64_t wstride = (V + 31) / 32;
    uint32_t* mrow = P.support_mask + static_cast<int64_t>(row) * wstride;
    ring.pass(0, ring.nst(), [&](const Raw* st, int n, int base) {
      for (int wd = tid; wd < (n + 31) / 32; wd += kRT) {
        uint32_t bits = 0;
        for (int i = 0; i < 32; ++i) {
          const int j = wd * 32 + i;
          if (j >= n || nonfinite) break;
          bool in = true;
          if (filtered) {
            const uint32_t key = key_of(st[j]);
            in = key > tkey || (key == tkey && base + j <= tie_cut);
          }
          if (in) bits |= 1u << i;
        }
        mrow[(base >> 5) + wd] = bits;
      }
      return false;
    });
  }

  // ---- seeded Gumbel-max token over the support.  Tokens go in groups of
  // four (stages start on multiples of four); each warp queues its groups
  // that hold a member and drains the queue 32 groups at a time (and at the
  // end of each stage), so the Philox block and the logarithms run on full
  // warps and only for members.
  if (P.sampled) {
    unsigned long long best = 0ull;
    if (!nonfinite) {
      const uint32_t nrow = static_cast<uint32_t>(P.row_base + row);
      const int lane = tid & 31, warp = tid >> 5;
      uint32_t* wq = sh.squeue[warp];
      ring.pass(0, ring.nst(), [&](const Raw* st, int n, int base) {
        auto take = [&](uint32_t e) {
          const int q = static_cast<int>(e & 0x0FFFFFFFu);
          uint64_t w[4];
          philox4x64_10(static_cast<uint64_t>(base >> 2) + q, 0, 0, 0, P.sample_seed, nrow, w);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (!((e >> (28 + i)) & 1u)) continue;
            const int j = 4 * q + i;
            const unsigned long long k =
                gumbel_key(gumbel_score(value_of(st[j]), T, gumbel_of(w[i])), base + j);
            best = k > best ? k : best;
          }
        };
        const int ng = (n + 3) / 4;
        int count = 0;  // queued groups of this warp (warp-uniform)
        for (int qb = warp * 32; qb < ng; qb += kRT) {
          const int q = qb + lane;
          uint32_t mbits = 0u;
          if (q < ng) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int j = 4 * q + i;
              bool in = j < n;
              if (in && filtered) {
                const uint32_t key = key_of(st[j]);
                in = key > tkey || (key == tkey && base + j <= tie_cut);
              }
              mbits |= in ? (1u << i) : 0u;
            }
          }
          const uint32_t ball = __ballot_sync(0xffffffffu, mbits != 0u);
          if (mbits) wq[count + __popc(ball & ((1u << lane) - 1u))] = static_cast<uint32_t>(q) | (mbits << 28);
          count += __popc(ball);
          __syncwarp();
          if (count >= 32) {
            count -= 32;
            take(wq[count + lane]);
            __syncwarp();
          }
        }
        if (lane < count) take(wq[lane]);
        __syncwarp();
        return false;
      });
    }
    best = block_max_key(best, sh.kred);
    if (tid == 0) P.sampled[row] = gumbel_key_id(best);
  }
}

size_t score_row_smem_bytes() {
  return static_cast<size_t>(kNStages) * kStageBytes + (kWin + 32) * 4 +
         ((sizeof(RowSh) + 127) & ~size_t(127));
}

// The dynamic shared-memory opt-in of a kernel, set once per device.
template <typename K>
cudaError_t ensure_smem(K kernel, int which) {
  static bool done[2][64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[which][dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(score_row_smem_bytes()));
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[which][dev] = true;
  return e;
}

template <typename Raw>
cudaError_t launch_row(const ScoreParams& p, cudaStream_t s, int which) {
  cudaError_t e = ensure_smem(score_row_kernel<Raw>, which);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.rows);
  cfg.blockDim = dim3(kRT);
  cfg.dynamicSmemBytes = score_row_smem_bytes();
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, score_row_kernel<Raw>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_computed(const ScoreParams& p, vs_dtype dtype, cudaStream_t s) {
  return dtype == VS_BF16 ? launch_row<uint16_t>(p, s, 0) : launch_row<uint32_t>(p, s, 1);
}

}  // namespace vs
