// Computed-support forward scoring (temperature -> stable token-id top-k ->
// inclusive top-p -> min-p against the original row max; xorl issue #71,
// section 3), one CTA per row.
//
// The row is streamed through a ring of shared-memory stages filled by bulk
// asynchronous copies (one elected thread issues them; every warp releases a
// stage after use):
//   pass 1 (HBM)  online max / count of max / sum 2^(u - max) /
//                 sum (u - max) 2^(u - max)   (u = z log2 e), and the row max;
//   pass 2 (L2)   bf16 rows with a filter: histogram of the EXACT 16-bit keys
//                 in a window of at most 4,096 keys at and below the row max
//                 (each bin holds one value, so its mass is count x 2^(u-m));
//                 the k-th element and the top-p crossing are found by block
//                 scans of the bins, the support sums by a block reduction;
//   pass 3 (L2)   only when the support ends inside a tie group: an ordered
//                 count of that group's elements finds the id of the last one
//                 kept (ties go to the lower token id);
//   pass 4 (L2)   only when the support bitmask is requested;
//   pass 5 (L2)   only when a sample is requested: a seeded Gumbel-max token
//                 over the support (noise recipe in gumbel.cuh).
// fp32 rows, and bf16 rows whose crossing lies below the window, fall back to
// an 8-bit radix descent over all keys (one streamed pass per digit).
// Everything is block-local (no cluster barriers), deterministic, and each
// row's logits are read from HBM once.

#include <climits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "gumbel.cuh"
#include "select.cuh"

namespace vs {

namespace {

constexpr int kRT = 512;        // threads per row
constexpr int kRW = kRT / 32;   // warps
constexpr int kNStages = 4;     // ring depth
constexpr int kStageBytes = 32768;
constexpr int kWin = kSelWin;
constexpr int kBins = kSelBins;

struct RowSh {
  uint64_t full[kNStages];
  uint64_t empty[kNStages];
  Stats wst[kRW];
  float fred[kRW];
  uint32_t ured[kRW];
  u64 ulred[kRW];
  SelShared<kRW> sel;
  uint32_t outstanding;  // loads issued and not yet consumed (broadcast by thread 0)
  int32_t tie_cut;
  uint32_t timeout;
  unsigned long long kred[kRW];
  uint32_t squeue[kRW][64];  // sampling: per-warp queue of member groups (index | bits << 28)
};

// ---------------------------------------------------------------------------
// streaming ring

template <typename Raw>
struct Ring {
  static constexpr int SE = kStageBytes / sizeof(Raw);  // elements per stage
  const Raw* g;  // row start in global memory
  int V;
  Raw* buf;      // [kNStages][SE]
  RowSh* sh;
  uint32_t ld;   // loads issued (thread 0)
  uint32_t cs;   // stages consumed (all threads)
  __device__ int nst() const { return (V + SE - 1) / SE; }
  __device__ int count(int si) const { return min(SE, V - si * SE); }

  // thread 0: load stage si into the next ring slot
  __device__ void issue(int si) {
    const uint32_t L = ld++;
    const int slot = L % kNStages;
    if (L >= kNStages && !mbar_wait(&sh->empty[slot], ((L / kNStages) - 1u) & 1u)) {
      sh->timeout = 1u;
    }
    const uint32_t bytes = static_cast<uint32_t>((count(si) * sizeof(Raw) + 15) & ~size_t(15));
    mbar_arrive_expect_tx(&sh->full[slot], bytes);
    bulk_load_all(buf + static_cast<size_t>(slot) * SE, g + static_cast<size_t>(si) * SE, bytes,
                  &sh->full[slot]);
  }

  // Run f(stage_ptr, n, base) over stages [s0, s1) in order; f returns true
  // (uniformly) to stop early.  Loads already issued are drained either way.
  template <typename F>
  __device__ void pass(int s0, int s1, F&& f) {
    if (threadIdx.x == 0)
      for (int si = s0; si < min(s1, s0 + kNStages); ++si) issue(si);
    int next = s0 + kNStages;
    bool stop = false;
    for (int si = s0; si < s1 && !stop; ++si) {
      const int slot = cs % kNStages;
      if (!mbar_wait(&sh->full[slot], (cs / kNStages) & 1u)) atomicOr(&sh->timeout, 1u);
      stop = f(buf + static_cast<size_t>(slot) * SE, count(si), si * SE);
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive_cnt(&sh->empty[slot]);
      ++cs;
      if (threadIdx.x == 0 && !stop && next < s1) issue(next);
      ++next;
    }
    // drain loads that were issued but not consumed (early stop)
    if (threadIdx.x == 0) sh->outstanding = ld - 0u;  // ld is thread 0's count
    __syncthreads();
    const uint32_t issued = sh->outstanding;
    while (cs < issued) {
      const int slot = cs % kNStages;
      if (!mbar_wait(&sh->full[slot], (cs / kNStages) & 1u)) atomicOr(&sh->timeout, 1u);
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive_cnt(&sh->empty[slot]);
      ++cs;
    }
    __syncthreads();
  }

  __device__ static void mbar_arrive_cnt(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
  }
};

// ---------------------------------------------------------------------------
// the exact-key window (bf16)

enum WinMode : int { kWinNone = 0, kWinPos = 1, kWinNeg = 2, kWinKey = 3 };

// bin of a raw bf16 (as fp32 bits F) or nbins when outside the window
__device__ __forceinline__ uint32_t win_bin(const Window& w, uint32_t F) {
  uint32_t b;
  if (w.mode == kWinPos) {
    b = (F - w.fconst) >> 16;
    if ((F - w.fconst) >= (static_cast<uint32_t>(w.nbins) << 16)) b = w.nbins;
  } else if (w.mode == kWinNeg) {
    b = (w.fconst - F) >> 16;
    if ((w.fconst - F) >= (static_cast<uint32_t>(w.nbins) << 16)) b = w.nbins;
  } else {
    b = key_of(static_cast<uint16_t>(F >> 16)) - w.klo;
    if (b >= static_cast<uint32_t>(w.nbins)) b = w.nbins;
  }
  return b;
}

// Count the in-window elements of one vector: collected as a bit mask and
// counted with as few shared atomics as the busiest lane of the warp needs.
// Uniform call (every lane of the warp).
__device__ __forceinline__ void win_vec(const Window& w, const uint4& q, bool valid) {
  uint32_t bins[8];
  uint32_t pend = 0;
  const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bins[2 * i] = win_bin(w, wd[i] << 16);
    bins[2 * i + 1] = win_bin(w, wd[i] & 0xFFFF0000u);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (valid && bins[i] < static_cast<uint32_t>(w.nbins)) pend |= 1u << i;
  while (__any_sync(0xffffffffu, pend != 0)) {
    if (pend) {
      const int i = __ffs(pend) - 1;
      uint32_t b = bins[0];
#pragma unroll
      for (int k = 1; k < 8; ++k)
        if (i == k) b = bins[k];
      atomicAdd(&w.hist[b], 1u);
      pend &= pend - 1;
    }
  }
}

// Histogram of one stage (four vectors per thread in flight).
__device__ void win_stage(const Window& w, const uint16_t* st, int n) {
  const int nv = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  const int rounds = (nv + 4 * kRT - 1) / (4 * kRT);
  for (int r = 0; r < rounds; ++r) {
    const int v0 = r * 4 * kRT + threadIdx.x;
    uint4 q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) q[k] = v0 + k * kRT < nv ? v4[v0 + k * kRT] : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int k = 0; k < 4; ++k) win_vec(w, q[k], v0 + k * kRT < nv);
  }
  for (int j = nv * 8 + threadIdx.x; j < n; j += kRT) {
    const uint32_t b = win_bin(w, static_cast<uint32_t>(st[j]) << 16);
    if (b < static_cast<uint32_t>(w.nbins)) atomicAdd(&w.hist[b], 1u);
  }
}

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
    __syncthreads();
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
  sh.ulred[1] = target;  // the resolved target (for the implicit top-p case)
  __syncthreads();
  return out;
}

// ---------------------------------------------------------------------------
// pass 1 helpers

// One 8-element bf16 vector into online statistics s (and the max raw value).
__device__ __forceinline__ void stats_vec_bf16(const uint4& q, float c, f32x2 c2, Stats& s,
                                               float& vmax) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  const __nv_bfloat162 m01 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[0]),
                                     *reinterpret_cast<const __nv_bfloat162*>(&w[1]));
  const __nv_bfloat162 m23 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[2]),
                                     *reinterpret_cast<const __nv_bfloat162*>(&w[3]));
  const __nv_bfloat162 mm = __hmax2(m01, m23);
  const float bmv = fmaxf(__low2float(mm), __high2float(mm));
  vmax = fmaxf(vmax, bmv);
  const float bm = __fmul_rn(bmv, c);
  if (bm > s.m) {
    if (s.c0 != 0.f || s.zr != 0.f) stats_rebase(s, bm);
    s.m = bm;
  }
  if (bm == s.m || !(bm == bm)) {
    // the vector holds this chain's running maximum (or NaN): scalar, with
    // the max-valued elements counted apart
    float u[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), c);
      u[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), c);
    }
    stats_add(s, u);
  } else {
    const f32x2 m2 = pack2(s.m, s.m);
    f32x2 zr2 = pack2(0.f, 0.f), a2 = pack2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const f32x2 x2 = pack2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
      const f32x2 d2 = sub2(mul2(x2, c2), m2);
      float d0, d1;
      unpack2(d2, d0, d1);
      const f32x2 e2 = pack2(ex2(d0), ex2(d1));
      zr2 = add2(zr2, e2);
      a2 = fma2(d2, e2, a2);
    }
    float z0, z1, a0, a1;
    unpack2(zr2, z0, z1);
    unpack2(a2, a0, a1);
    s.zr += z0 + z1;
    s.a += a0 + a1;
  }
}

// bf16 stage: four vectors per thread in flight, each with its own chain.
__device__ __forceinline__ void stats_stage_bf16(const uint16_t* st, int n, float c, Stats (&s)[4],
                                                 float& vmax) {
  const int nv = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  const f32x2 c2 = pack2(c, c);
  int v = threadIdx.x;
  for (; v + 3 * kRT < nv; v += 4 * kRT) {
    uint4 q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) q[k] = v4[v + k * kRT];
#pragma unroll
    for (int k = 0; k < 4; ++k) stats_vec_bf16(q[k], c, c2, s[k], vmax);
  }
  for (; v < nv; v += kRT) stats_vec_bf16(v4[v], c, c2, s[0], vmax);
  for (int j = nv * 8 + threadIdx.x; j < n; j += kRT) {
    const float x = value_of(st[j]);
    vmax = fmaxf(vmax, x);
    float u[1] = {__fmul_rn(x, c)};
    stats_add(s[0], u);
  }
}

__device__ __forceinline__ void stats_stage_f32(const uint32_t* st, int n, float c, Stats (&s4)[4],
                                                float& vmax) {
  Stats& s = s4[0];
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
  RowSh& sh = *reinterpret_cast<RowSh*>(smem_raw + kNStages * kStageBytes + kWin * 4);

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int V = P.vocab;
  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld;

  if (tid == 0) {
    for (int s = 0; s < kNStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kRW);
    }
    sh.timeout = 0;
    sh.tie_cut = INT_MAX;
    fence_barrier_init();
  }
  __syncthreads();
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

  // ---- pass 1 (HBM): online statistics and the row maximum
  Stats s4[4] = {stats_empty(), stats_empty(), stats_empty(), stats_empty()};
  float vmax = -kInf;
  ring.pass(0, ring.nst(), [&](const Raw* st, int n, int) {
    if constexpr (kBf16)
      stats_stage_bf16(st, n, c, s4, vmax);
    else
      stats_stage_f32(st, n, c, s4, vmax);
    return false;
  });
  Stats s = s4[0];
  stats_merge(s, s4[1]);
  stats_merge(s, s4[2]);
  stats_merge(s, s4[3]);
  s = block_reduce(s, sh.wst);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  if ((tid & 31) == 0) sh.fred[tid >> 5] = vmax;
  __syncthreads();
  vmax = -kInf;
  for (int w = 0; w < kRW; ++w) vmax = fmaxf(vmax, sh.fred[w]);
  __syncthreads();

  const bool nonfinite = !stats_finite(s) || !isfinite(vmax);
  const float m = s.m;  // = fl(vmax c)
  const float log2z = stats_log2z(s);
  const float h_full = kLn2 * (log2z - s.a / stats_z(s));
  const bool filtered = !nonfinite && any_filter;

  uint32_t tkey = 0;
  int32_t tie_cut = INT_MAX;
  float log2zs = log2z, h_support = h_full, c0s = s.c0, zrs = s.zr;
  int32_t n_support = nonfinite ? 0 : V;

  if (filtered) {
    const float fxs = fx_scale(P.fx_shift);
    bool all_ties = true;
    u64 cnum = 0;
    bool have_t = false;
    // ---- pass 2 (L2): exact-key window (bf16)
    Window w{};
    bool win_ok = false;
    if constexpr (kBf16) {
      const uint32_t hmax = __float_as_uint(vmax) >> 16;
      w.kmax = key_of(static_cast<uint16_t>(hmax));
      uint32_t klo = w.kmax >= static_cast<uint32_t>(kWin - 1) ? w.kmax - (kWin - 1) : 0u;
      if (use_p && !use_k && !use_minp && pp > 0.f) {
        // top-p alone: elements with 2^(u - m) < (1 - p) / (2 V) cannot be in
        // the support (together they hold less than (1 - p) of the mass, the
        // row total being at least 1); start the window at the first key
        // above that level
        const float dcut = log2f((1.f - pp) / static_cast<float>(V)) - 1.f;
        uint32_t lo = klo, hi = w.kmax;
        while (lo < hi) {
          const uint32_t mid = lo + ((hi - lo) >> 1);
          if (key_u(mid, c) - m >= dcut)
            hi = mid;
          else
            lo = mid + 1;
        }
        klo = lo;
      }
      w.klo = klo;
      w.nbins = static_cast<int>(w.kmax - klo) + 1;
      w.hist = hist;
      w.c = c;
      w.m = m;
      w.fxs = fxs;
      if (klo > 0x7FFFu && (w.kmax - 0x7FFFu) < 0x7000u) {
        w.mode = kWinPos;  // positive nonzero keys below 2^97
        w.fconst = (klo - 0x7FFFu) << 16;
      } else if (w.kmax < 0x7FFFu) {
        w.mode = kWinNeg;  // negative nonzero keys (every value is negative)
        w.fconst = (0xFFFFu - klo) << 16;
      } else {
        w.mode = kWinKey;
        w.fconst = 0;
      }
      for (int b = tid; b < w.nbins; b += kRT) hist[b] = 0u;
      __syncthreads();
      ring.pass(0, ring.nst(), [&](const Raw* st, int n, int) {
        win_stage(w, reinterpret_cast<const uint16_t*>(st), n);
        return false;
      });
      win_ok = true;
      if (use_k || use_p) {
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
      }
    }
    if (!win_ok && (use_k || use_p)) {
      // ---- general radix descent (fp32 keys, or the crossing lies below the window)
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
    // and the tie group at tkey
    uint32_t ngt = 0, neq = 0, ntop = 0;
    float smass = 0.f, sa = 0.f;
    bool sums_done = false;
    if constexpr (kBf16) {
      if (win_ok && tkey >= w.klo) {
        const int per = (w.nbins + kRT - 1) / kRT;
        const int i0 = tid * per, i1 = min(w.nbins, i0 + per);
        for (int i = i0; i < i1; ++i) {
          const uint32_t cnt = hist[i];
          const uint32_t key = w.klo + i;
          if (cnt && key > tkey) {
            const float d = key_u(key, c) - m;
            const float e = ex2(d);
            const float fc = static_cast<float>(cnt);
            ngt += cnt;
            if (d == 0.f)
              ntop += cnt;
            else
              smass = fmaf(fc, e, smass);
            sa = fmaf(fc * d, e, sa);
          }
        }
        if (tid == 0) neq = hist[tkey - w.klo];
        sums_done = true;
      }
    }
    if (!sums_done) {
      const uint32_t t = tkey;
      auto one = [&](Raw raw) {
        const uint32_t key = key_of(raw);
        if (key > t) {
          const float d = __fmul_rn(value_of(raw), c) - m;
          const float e = ex2(d);
          ++ngt;
          if (d == 0.f)
            ++ntop;
          else
            smass += e;
          sa = fmaf(d, e, sa);
        } else if (key == t) {
          ++neq;
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
    ngt = block_sum(ngt, sh.ured);
    neq = block_sum(neq, sh.ured);
    ntop = block_sum(ntop, sh.ured);
    smass = block_sum(smass, sh.fred);
    sa = block_sum(sa, sh.fred);
    const u64 tot_eq = neq;
    const u64 ckeep = all_ties ? tot_eq : (cnum < tot_eq ? cnum : tot_eq);
    const float dt = __fmul_rn(KT::decode(tkey), c) - m;
    const float et = ex2(dt);
    Stats ss;
    ss.m = m;
    ss.c0 = static_cast<float>(ntop) + (dt == 0.f ? static_cast<float>(ckeep) : 0.f);
    ss.zr = smass + (dt == 0.f ? 0.f : static_cast<float>(ckeep) * et);
    ss.a = sa + static_cast<float>(ckeep) * dt * et;
    log2zs = stats_log2z(ss);
    h_support = kLn2 * (log2zs - ss.a / stats_z(ss));
    c0s = ss.c0;
    zrs = ss.zr;
    n_support = static_cast<int32_t>(ngt + ckeep);

    // ---- pass 3 (L2): id of the last tie kept (ascending id order)
    if (ckeep < tot_eq) {
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
    }
  }

  // ---- per-row outputs
  if (tid == 0) {
    const int y = P.targets[row];
    const bool target_ok = y >= 0 && y < V;
    uint32_t status = 0;
    float lp_v = __int_as_float(0x7fc00000), lp_s = __int_as_float(0x7fc00000);
    bool in_s = false;
    if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
    if (nonfinite) {
      status |= VS_ROW_NONFINITE_INPUT;
    } else if (target_ok) {
      const Raw ry = grow[y];
      const float uy = __fmul_rn(value_of(ry), c);
      lp_v = kLn2 * (uy - m - log2z);
      if (!filtered) {
        in_s = true;
      } else {
        const uint32_t ky = key_of(ry);
        in_s = ky > tkey || (ky == tkey && y <= tie_cut);
      }
      if (in_s) {
        lp_s = filtered ? kLn2 * (uy - m - log2zs) : lp_v;
      } else {
        lp_s = -kInf;
        status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
      }
    }
    if (sh.timeout) status |= kRowDeviceTimeout;
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
    if (P.ctx) {
      RowCtx cx{};
      cx.m2 = vmax;
      cx.log2z = log2z;
      cx.msup = vmax;
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
      cx.c0_full = s.c0;
      cx.zr_full = s.zr;
      cx.c0_sup = c0s;
      cx.zr_sup = zrs;
      P.ctx[row] = cx;
    }
  }

  // ---- pass 4 (L2): support bitmask, one 32-id word per thread and stage
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

  // ---- pass 5 (L2): seeded Gumbel-max token over the support.  Tokens go
  // in groups of four (stages start on multiples of four); each warp queues
  // its groups that hold a member and drains the queue 32 groups at a time
  // (and at the end of each stage), so the Philox block and the logarithms
  // run on full warps and only for members.
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

}  // namespace

size_t score_row_smem_bytes() {
  return static_cast<size_t>(kNStages) * kStageBytes + kWin * 4 + ((sizeof(RowSh) + 127) & ~size_t(127));
}

cudaError_t launch_score_computed(const ScoreParams& p, vs_dtype dtype, cudaStream_t s) {
  const size_t smem = score_row_smem_bytes();
  if (dtype == VS_BF16) {
    cudaError_t e = cudaFuncSetAttribute(score_row_kernel<uint16_t>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_row_kernel<uint16_t><<<p.rows, kRT, smem, s>>>(p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(score_row_kernel<uint32_t>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    score_row_kernel<uint32_t><<<p.rows, kRT, smem, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace vs
