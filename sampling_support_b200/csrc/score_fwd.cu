// Forward scoring kernels.
//
//  * score_computed_kernel: computed support (temperature -> stable token-id
//    top-k -> inclusive top-p -> min-p against the original row max; xorl
//    issue #71, section 3).  One thread-block cluster per row; each CTA pulls
//    its slice of the row from HBM once, with bulk asynchronous copies, into
//    shared memory, and every later pass (radix select, support sums, tie
//    resolution, mask) reads that copy.  Row statistics and histograms are
//    combined across the cluster through distributed shared memory in a
//    fixed rank order, so results are deterministic.
//  * score_recorded_kernel: recorded support (SkyRL PR #2004,
//    "Implementation": dense -1-padded id list).  One CTA per row gathers the
//    support logits; rows with an empty support (full-vocabulary fallback),
//    or every row when full statistics are requested, also stream the whole
//    row once with 16-byte loads.

#include <climits>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace vs {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;
// Exact-key window of the bf16 select: the kWin keys at and below the row's
// maximum key (32 binades of bf16 below the maximum value, same sign).
constexpr int kWin = 4096;

typedef unsigned long long u64;

// Arrays of the general radix descent (fp32 keys, or a bf16 row whose
// crossing lies below the window).  They alias the window area.
struct RadixArrays {
  u64 mass[2][kBins];  // fixed-point mass histogram (double-buffered)
  u64 gmass[kBins];    // cluster-reduced
  uint32_t cnt[2][kBins];
  uint32_t gcnt[kBins];
};

// Bytes of the window / radix area of a CTA in a cluster of `cl`.
__host__ __device__ constexpr size_t big_area_bytes(int cl) {
  return (static_cast<size_t>(kWin) + (kWin + cl - 1) / cl) * 4 > sizeof(RadixArrays)
             ? (static_cast<size_t>(kWin) + (kWin + cl - 1) / cl) * 4
             : sizeof(RadixArrays);
}

// Small shared state of one CTA.
struct SelShared {
  uint64_t bar;
  Stats part;  // this CTA's row statistics
  float vmax_part;
  Stats gathered[8];
  float vmax_g[8];
  Stats red[kWarps];
  float fred[kWarps];
  uint32_t ured[kWarps];
  u64 ulred[kWarps];
  u64 scan_a[kWarps], scan_b[kWarps];
  // window slice totals (this CTA) and their cluster gather
  u64 slice_cnt, slice_mass;
  u64 g_slice_cnt[8], g_slice_mass[8];
  // window search results (written by the owning CTA; one slot per search so
  // that a second search never overwrites a result a peer may still read)
  uint32_t res_key[2];
  u64 res_above_cnt[2], res_above_mass[2], res_at_cnt[2], res_at_mass[2];
  // support-sum partials (this CTA)
  float agg_mass, agg_a;
  uint32_t agg_ngt, agg_eq, agg_top;
  // radix broadcast slots
  u64 b_target, b_above_cnt, b_above_mass, b_at_cnt, b_at_mass;
  uint32_t b_digit;
  int32_t tie_cut;
  uint32_t timeout;
  uint32_t scan_tot[kWarps];
};

struct Desc {
  uint32_t key;
  u64 above_cnt, above_mass, at_cnt, at_mass;
};

__device__ __forceinline__ float fx_scale(int shift) {
  return __int_as_float((127 + shift) << 23);
}

// Visit every element of the CTA's slice: f(local_index, raw).
template <typename Raw, typename F>
__device__ __forceinline__ void for_each(const Raw* buf, int n, F&& f) {
  constexpr int VEC = 16 / sizeof(Raw);
  const int nfull = n / VEC;
  const uint4* v4 = reinterpret_cast<const uint4*>(buf);
  for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
    Raw r[VEC];
    unpack(v4[v], r);
#pragma unroll
    for (int i = 0; i < VEC; ++i) f(v * VEC + i, r[i]);
  }
  for (int j = nfull * VEC + threadIdx.x; j < n; j += blockDim.x) f(j, buf[j]);
}

// Exclusive suffix sums over the threads of the block (thread t gets the sum
// of a and b over threads t' > t).  Uniform call.
__device__ __forceinline__ void block_suffix_excl(u64 a, u64 b, u64& ea, u64& eb, SelShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  u64 ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const u64 ta = __shfl_down_sync(0xffffffffu, ia, o);
    const u64 tb = __shfl_down_sync(0xffffffffu, ib, o);
    if (lane + o < 32) {
      ia += ta;
      ib += tb;
    }
  }
  if (lane == 0) {
    sh.scan_a[warp] = ia;
    sh.scan_b[warp] = ib;
  }
  __syncthreads();
  u64 wa = 0, wb = 0;
  const int nw = blockDim.x >> 5;
  for (int w = warp + 1; w < nw; ++w) {
    wa += sh.scan_a[w];
    wb += sh.scan_b[w];
  }
  ea = wa + ia - a;
  eb = wb + ib - b;
  __syncthreads();
}

// Warp 0: find, scanning bins from the top (largest key first), the bin where
// the cumulative `by` quantity first reaches `need` (>= 1).  Returns the
// digit and the sums (count and mass) of the bins strictly above it, in lane 0.
__device__ void scan_bins(const uint32_t* gcnt, const u64* gmass, bool by_mass, u64 need,
                          uint32_t& digit, u64& above_cnt, u64& above_mass) {
  const int lane = threadIdx.x & 31;
  u64 v[8];
  u64 lsum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = 255 - 8 * lane - i;
    v[i] = by_mass ? gmass[b] : static_cast<u64>(gcnt[b]);
    lsum += v[i];
  }
  u64 incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const u64 t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const u64 excl = incl - lsum;
  const bool hit = excl < need && need <= incl;
  const uint32_t ballot = __ballot_sync(0xffffffffu, hit);
  int d;
  if (ballot != 0) {
    const int hl = __ffs(ballot) - 1;
    int local = -1;
    if (lane == hl) {
      u64 s = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (local < 0 && s + v[i] >= need) local = 255 - 8 * lane - i;
        if (local < 0) s += v[i];
      }
    }
    d = __shfl_sync(0xffffffffu, local, hl);
  } else {
    // target beyond the total (cannot happen for consistent targets): take
    // the lowest non-empty bin so that the result stays well defined.
    int lowest = 256;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = 255 - 8 * lane - i;
      if (gcnt[b] != 0) lowest = b;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lowest = min(lowest, __shfl_xor_sync(0xffffffffu, lowest, o));
    d = lowest == 256 ? 0 : lowest;
  }
  u64 ac = 0, am = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int b = 255 - 8 * lane - i;
    if (b > d) {
      ac += gcnt[b];
      am += gmass[b];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ac += __shfl_xor_sync(0xffffffffu, ac, o);
    am += __shfl_xor_sync(0xffffffffu, am, o);
  }
  digit = static_cast<uint32_t>(d);
  above_cnt = ac;
  above_mass = am;
}

// Radix descent over 8-bit digits of the key (most significant first) for
// the position where the cumulative count (by_mass = false) or fixed-point
// mass (by_mass = true) of the total order first reaches `target`.
// target == 0 with by_mass means "ceil(p * total mass)", with the total taken
// from the first level's histogram.  `hb` selects the histogram buffer and
// alternates per level, so one cluster barrier per level suffices.
template <typename Raw>
__device__ Desc descend(const Raw* buf, int n, float c, float vmax, int fx_shift, bool by_mass,
                        bool need_mass, u64 target, float p, SelShared& sh, RadixArrays& ra,
                        cg::cluster_group& cluster, int& hb) {
  constexpr int KB = KeyTraits<Raw>::kBits;
  const uint32_t CL = cluster.num_blocks();
  const float fxs = fx_scale(fx_shift);
  uint32_t prefix = 0;
  u64 above_cnt = 0, above_mass = 0;
  Desc out{};
  for (int shift = KB - 8; shift >= 0; shift -= 8) {
    uint32_t* cnt = ra.cnt[hb];
    u64* mass = ra.mass[hb];
    for (int b = threadIdx.x; b < kBins; b += blockDim.x) {
      cnt[b] = 0;
      mass[b] = 0;
    }
    __syncthreads();
    const int pshift = shift + 8;
    const uint32_t pre = prefix;
    for_each(buf, n, [&](int, Raw raw) {
      const uint32_t key = key_of(raw);
      const bool match = pshift >= KB ? true : ((key >> pshift) == pre);
      if (match) {
        const uint32_t digit = (key >> shift) & 255u;
        atomicAdd(&cnt[digit], 1u);
        if (need_mass) {
          const float e = ex2((value_of(raw) - vmax) * c);
          const u64 fx = __float2ull_rn(e * fxs);
          if (fx) atomicAdd(&mass[digit], fx);
        }
      }
    });
    __syncthreads();
    cluster.sync();
    for (int b = threadIdx.x; b < kBins; b += blockDim.x) {
      uint32_t scnt = 0;
      u64 smass = 0;
      for (uint32_t r = 0; r < CL; ++r) {
        scnt += *cluster.map_shared_rank(&cnt[b], r);
        smass += *cluster.map_shared_rank(&mass[b], r);
      }
      ra.gcnt[b] = scnt;
      ra.gmass[b] = smass;
    }
    __syncthreads();
    hb ^= 1;
    if (threadIdx.x < 32) {
      u64 tgt = target;
      if (tgt == 0) {
        // implicit target: ceil(p * total mass), clamped to [1, total]
        u64 tot = 0;
        for (int i = threadIdx.x; i < kBins; i += 32) tot += ra.gmass[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        const double want = ceil(static_cast<double>(p) * static_cast<double>(tot));
        const u64 t = want <= 1.0 ? 1ull
                      : want >= static_cast<double>(tot) ? tot
                                                         : static_cast<u64>(want);
        tgt = t < 1 ? 1 : t;
      }
      const u64 have = by_mass ? above_mass : above_cnt;
      const u64 need = tgt > have ? tgt - have : 1;
      uint32_t digit;
      u64 ac, am;
      scan_bins(ra.gcnt, ra.gmass, by_mass, need, digit, ac, am);
      if (threadIdx.x == 0) {
        sh.b_target = tgt;
        sh.b_digit = digit;
        sh.b_above_cnt = ac;
        sh.b_above_mass = am;
        sh.b_at_cnt = ra.gcnt[digit];
        sh.b_at_mass = ra.gmass[digit];
      }
    }
    __syncthreads();
    target = sh.b_target;
    above_cnt += sh.b_above_cnt;
    above_mass += sh.b_above_mass;
    prefix = (prefix << 8) | sh.b_digit;
    out.at_cnt = sh.b_at_cnt;
    out.at_mass = sh.b_at_mass;
    __syncthreads();
  }
  out.key = prefix;
  out.above_cnt = above_cnt;
  out.above_mass = above_mass;
  return out;
}

// ---------------------------------------------------------------------------
// exact-key window (bf16): the histogram of keys klo .. klo + kWin - 1,
// cluster-reduced so that CTA r holds bins [r S, r S + S).

struct Window {
  uint32_t klo, kmax;
  int nbins;      // kmax - klo + 1 (<= kWin)
  int S;          // bins per CTA slice
  uint32_t* hist;  // this CTA's unreduced histogram [kWin]
  uint32_t* red;   // this CTA's reduced slice [S]
  float c, vmax, fxs;
};

// Fixed-point mass 2^((v - vmax) c) * 2^fx_shift of one element of a bin.
__device__ __forceinline__ u64 bin_fx(const Window& w, uint32_t key) {
  const float e = ex2((KeyTraits<uint16_t>::decode(key) - w.vmax) * w.c);
  return __float2ull_rn(e * w.fxs);
}

// Reduce the (already filled) window histograms across the cluster, CTA r
// keeping bins [r S, r S + S), and gather the per-slice totals (count and
// fixed-point mass) into every CTA.  The caller has passed a cluster barrier
// since the histograms were filled.
__device__ void window_reduce(Window& w, SelShared& sh, cg::cluster_group& cluster) {
  const uint32_t CL = cluster.num_blocks();
  const uint32_t rank = cluster.block_rank();
  const uint32_t klo = w.klo;
  uint32_t* hist = w.hist;
  const int b0 = static_cast<int>(rank) * w.S;
  const int b1 = min(w.nbins, b0 + w.S);
  u64 tc = 0, tm = 0;
  for (int b = b0 + threadIdx.x; b < b1; b += blockDim.x) {
    uint32_t sum = 0;
    for (uint32_t r = 0; r < CL; ++r) sum += *cluster.map_shared_rank(&hist[b], r);
    w.red[b - b0] = sum;
    if (sum) {
      tc += sum;
      tm += static_cast<u64>(sum) * bin_fx(w, klo + b);
    }
  }
  tc = block_sum(tc, sh.ulred);
  tm = block_sum(tm, sh.ulred);
  if (threadIdx.x == 0) {
    sh.slice_cnt = tc;
    sh.slice_mass = tm;
  }
  cluster.sync();
  if (threadIdx.x < static_cast<int>(CL)) {
    const SelShared* rsh = cluster.map_shared_rank(&sh, threadIdx.x);
    sh.g_slice_cnt[threadIdx.x] = rsh->slice_cnt;
    sh.g_slice_mass[threadIdx.x] = rsh->slice_mass;
  }
  __syncthreads();
}

// Find, from the largest key down, the window bin where the cumulative count
// (by_mass false) or fixed-point mass first reaches `need` (>= 1).  Returns
// false (uniformly across the cluster) when the window holds less.
__device__ bool window_search(const Window& w, bool by_mass, u64 need, int slot, Desc& out,
                              SelShared& sh, cg::cluster_group& cluster) {
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  u64 cum = 0, cum_c = 0, cum_m = 0;
  int rs = -1;
  for (int r = CL - 1; r >= 0; --r) {
    const u64 t = by_mass ? sh.g_slice_mass[r] : sh.g_slice_cnt[r];
    if (cum + t >= need) {
      rs = r;
      break;
    }
    cum += t;
    cum_c += sh.g_slice_cnt[r];
    cum_m += sh.g_slice_mass[r];
  }
  if (rs < 0) return false;
  if (rank == rs) {
    const int b0 = rs * w.S;
    const int nb = max(0, min(w.nbins, b0 + w.S) - b0);
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    const int i0 = threadIdx.x * per, i1 = min(nb, i0 + per);
    u64 lc = 0, lm = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t cnt = w.red[i];
      if (cnt) {
        lc += cnt;
        lm += static_cast<u64>(cnt) * bin_fx(w, w.klo + b0 + i);
      }
    }
    u64 ec, em;
    block_suffix_excl(lc, lm, ec, em, sh);
    const u64 base = cum + (by_mass ? em : ec);
    const u64 mine = by_mass ? lm : lc;
    if (base < need && need <= base + mine) {
      u64 ac = cum_c + ec, am = cum_m + em;
      for (int i = i1 - 1; i >= i0; --i) {
        const uint32_t cnt = w.red[i];
        const u64 fx = cnt ? static_cast<u64>(cnt) * bin_fx(w, w.klo + b0 + i) : 0ull;
        const u64 v = by_mass ? fx : cnt;
        if (cnt && (by_mass ? am : ac) + v >= need) {
          sh.res_key[slot] = w.klo + b0 + i;
          sh.res_above_cnt[slot] = ac;
          sh.res_above_mass[slot] = am;
          sh.res_at_cnt[slot] = cnt;
          sh.res_at_mass[slot] = fx;
          break;
        }
        ac += cnt;
        am += fx;
      }
    }
  }
  cluster.sync();
  const SelShared* rsh = cluster.map_shared_rank(&sh, rs);
  out.key = rsh->res_key[slot];
  out.above_cnt = rsh->res_above_cnt[slot];
  out.above_mass = rsh->res_above_mass[slot];
  out.at_cnt = rsh->res_at_cnt[slot];
  out.at_mass = rsh->res_at_mass[slot];
  return true;
}

// Target mass of inclusive top-p: ceil(p * mass), clamped to [1, mass].
__device__ __forceinline__ u64 topp_target(float p, double mass) {
  const double want = ceil(static_cast<double>(p) * mass);
  if (want <= 1.0) return 1ull;
  if (want >= mass) return static_cast<u64>(mass);
  return static_cast<u64>(want);
}

// Window mode of the fused pass (bf16): how an element's bin is derived.
enum WinMode : int {
  kWinNone = 0,  // no histogram
  kWinPos = 1,   // window within positive values: bin = (F - Fconst) >> 16 on raw float bits
  kWinNeg = 2,   // window within negative values: bin = (Fconst - F) >> 16
  kWinKey = 3,   // general: bin = key - klo
};

// Sums of a slice relative to the known row maximum vmax (base 2, d =
// (v - vmax) c <= 0): count of elements equal to vmax, the sum of 2^d over the
// others, and the sum of d 2^d.
struct FSums {
  float c0, zr, a;
};

// One element of the fused pass.  kTop: the element's vector holds the row
// maximum, so elements with d == 0 are counted apart (exactly 1 each).
template <bool kTop>
__device__ __forceinline__ void fused_elem(float x, float vmax, float c, FSums& s) {
  const float d = (x - vmax) * c;
  const float e = ex2(d);
  if (kTop && d == 0.f)
    s.c0 += 1.f;
  else
    s.zr += e;
  s.a = fmaf(d, e, s.a);
}

// Count one element (raw float bits F) in the window of `nbins` exact keys.
template <int kMode>
__device__ __forceinline__ void win_count(uint32_t F, uint32_t nbins, uint32_t fconst,
                                          uint32_t klo, uint32_t* hist) {
  if constexpr (kMode == kWinPos) {
    const uint32_t b = F - fconst;
    if (b < (nbins << 16)) atomicAdd(&hist[b >> 16], 1u);
  } else if constexpr (kMode == kWinNeg) {
    const uint32_t b = fconst - F;
    if (b < (nbins << 16)) atomicAdd(&hist[b >> 16], 1u);
  } else if constexpr (kMode == kWinKey) {
    const uint32_t b = key_of(static_cast<uint16_t>(F >> 16)) - klo;
    if (b < nbins) atomicAdd(&hist[b], 1u);
  }
}

// Fused pass over a bf16 slice: statistics relative to vmax and, when
// kMode != kWinNone, the exact-key window histogram.
template <int kMode>
__device__ void fused_pass_bf16(const uint16_t* buf, int n, float vmax, float c, uint32_t nbins,
                                uint32_t fconst, uint32_t klo, uint32_t* hist, FSums& s) {
  const int nfull = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(buf);
  const f32x2 vm2 = pack2(vmax, vmax), c2 = pack2(c, c);
  f32x2 zr2 = pack2(0.f, 0.f), a2 = pack2(0.f, 0.f);
  for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
    const uint4 q = v4[v];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    // does this vector hold the row maximum?  (packed max, rare)
    __nv_bfloat162 m01 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[0]),
                                 *reinterpret_cast<const __nv_bfloat162*>(&w[1]));
    __nv_bfloat162 m23 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[2]),
                                 *reinterpret_cast<const __nv_bfloat162*>(&w[3]));
    const __nv_bfloat162 mm = __hmax2(m01, m23);
    const bool top = fmaxf(__low2float(mm), __high2float(mm)) == vmax;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t F0 = w[i] << 16, F1 = w[i] & 0xFFFF0000u;
      // both elements at once: d = (x - vmax) c
      const f32x2 d2 = mul2(sub2(pack2(__uint_as_float(F0), __uint_as_float(F1)), vm2), c2);
      float d0, d1;
      unpack2(d2, d0, d1);
      if (top) {
        fused_elem<true>(__uint_as_float(F0), vmax, c, s);
        fused_elem<true>(__uint_as_float(F1), vmax, c, s);
      } else {
        // e = 2^d, zr += e, a += d e
        const f32x2 e2 = pack2(ex2(d0), ex2(d1));
        zr2 = add2(zr2, e2);
        a2 = fma2(d2, e2, a2);
      }
      win_count<kMode>(F0, nbins, fconst, klo, hist);
      win_count<kMode>(F1, nbins, fconst, klo, hist);
    }
  }
  {
    float z0, z1, a0, a1;
    unpack2(zr2, z0, z1);
    unpack2(a2, a0, a1);
    s.zr += z0 + z1;
    s.a += a0 + a1;
  }
  for (int j = nfull * 8 + threadIdx.x; j < n; j += blockDim.x) {
    const uint32_t F = static_cast<uint32_t>(buf[j]) << 16;
    fused_elem<true>(__uint_as_float(F), vmax, c, s);
    win_count<kMode>(F, nbins, fconst, klo, hist);
  }
}

// Statistics pass over an fp32 slice relative to vmax.
__device__ void fused_pass_f32(const uint32_t* buf, int n, float vmax, float c, FSums& s) {
  const int nfull = n / 4;
  const uint4* v4 = reinterpret_cast<const uint4*>(buf);
  for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
    const uint4 q = v4[v];
    const float x[4] = {__uint_as_float(q.x), __uint_as_float(q.y), __uint_as_float(q.z),
                        __uint_as_float(q.w)};
    const float bm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    if (bm == vmax) {
#pragma unroll
      for (int i = 0; i < 4; ++i) fused_elem<true>(x[i], vmax, c, s);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) fused_elem<false>(x[i], vmax, c, s);
    }
  }
  for (int j = nfull * 4 + threadIdx.x; j < n; j += blockDim.x)
    fused_elem<true>(__uint_as_float(buf[j]), vmax, c, s);
}

// Largest value of a slice (NaN ignored).
template <typename Raw>
__device__ float slice_max(const Raw* buf, int n) {
  float m = -kInf;
  if constexpr (sizeof(Raw) == 2) {
    const int nfull = n / 8;
    const uint4* v4 = reinterpret_cast<const uint4*>(buf);
    __nv_bfloat162 acc = __float2bfloat162_rn(-kInf);
    for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
      const uint4 q = v4[v];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
      acc = __hmax2(acc, __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3])));
    }
    m = fmaxf(__low2float(acc), __high2float(acc));
    for (int j = nfull * 8 + threadIdx.x; j < n; j += blockDim.x) m = fmaxf(m, value_of(buf[j]));
  } else {
    const int nfull = n / 4;
    const uint4* v4 = reinterpret_cast<const uint4*>(buf);
    for (int v = threadIdx.x; v < nfull; v += blockDim.x) {
      const uint4 q = v4[v];
      m = fmaxf(m, fmaxf(fmaxf(__uint_as_float(q.x), __uint_as_float(q.y)),
                         fmaxf(__uint_as_float(q.z), __uint_as_float(q.w))));
    }
    for (int j = nfull * 4 + threadIdx.x; j < n; j += blockDim.x) m = fmaxf(m, value_of(buf[j]));
  }
  return m;
}

template <typename Raw>
__global__ void __launch_bounds__(kThreads, 2) score_computed_kernel(ScoreParams P) {
  constexpr bool kBf16 = sizeof(Raw) == 2;
  using KT = KeyTraits<Raw>;
  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t rank = cluster.block_rank();
  const uint32_t CL = cluster.num_blocks();
  const int row = blockIdx.x / CL;
  const int tid = threadIdx.x;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  Raw* buf = reinterpret_cast<Raw*>(smem_raw);
  const size_t chunk_bytes = static_cast<size_t>(P.chunk) * sizeof(Raw);
  SelShared& sh = *reinterpret_cast<SelShared*>(smem_raw + chunk_bytes);
  uint8_t* big = smem_raw + chunk_bytes + ((sizeof(SelShared) + 127) & ~size_t(127));
  RadixArrays& ra = *reinterpret_cast<RadixArrays*>(big);

  const int V = P.vocab;
  const int c0 = static_cast<int>(rank) * P.chunk;
  const int c1 = min(V, c0 + P.chunk);
  const int n = max(0, c1 - c0);
  const Raw* grow = static_cast<const Raw*>(P.logits) + static_cast<int64_t>(row) * P.ld;

  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_barrier_init();
    sh.timeout = 0;
    sh.tie_cut = INT_MAX;
  }
  __syncthreads();
  const uint32_t bytes = static_cast<uint32_t>((static_cast<size_t>(n) * sizeof(Raw) + 15) & ~size_t(15));
  if (tid == 0 && bytes > 0) {
    mbar_arrive_expect_tx(&sh.bar, bytes);
    bulk_load_all(buf, grow + c0, bytes, &sh.bar);
  }
  if (bytes > 0 && !mbar_wait(&sh.bar, 0)) {
    atomicOr(&sh.timeout, 1u);
    mbar_wait(&sh.bar, 0);  // give the copy a second bounded chance to land
  }
  __syncthreads();

  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const float c = kLog2e / T;
  const int kk = P.top_k ? P.top_k[row] : P.top_k_scalar;
  const float pp = P.top_p ? P.top_p[row] : P.top_p_scalar;
  const float mp = P.min_p ? P.min_p[row] : P.min_p_scalar;
  const bool use_k = kk > 0 && kk < V;
  const bool use_p = pp < 1.f;
  const bool use_minp = mp > 0.f;
  const bool any_filter = use_k || use_p || use_minp;

  // ---- pass 0: row maximum (cluster-wide, rank order)
  {
    float vm = slice_max(buf, n);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
    if ((tid & 31) == 0) sh.fred[tid >> 5] = vm;
    __syncthreads();
    if (tid == 0) {
      float m = -kInf;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sh.fred[w]);
      sh.vmax_part = m;
    }
  }
  cluster.sync();
  if (tid < static_cast<int>(CL)) sh.vmax_g[tid] = cluster.map_shared_rank(&sh, tid)->vmax_part;
  __syncthreads();
  float vmax = -kInf;
  for (uint32_t r = 0; r < CL; ++r) vmax = fmaxf(vmax, sh.vmax_g[r]);

  // ---- window geometry (bf16 with a filter): exact keys klo .. kmax, at most
  // kWin of them.  With top-p alone the window starts at the first key whose
  // d = (v - vmax) c reaches dcut = log2((1 - p) / V) - 1: every element
  // below it lies outside the support (together they hold less than (1 - p)
  // of the mass, the row total being at least 1).
  Window w{};
  int wmode = kWinNone;
  if constexpr (kBf16) {
    if (any_filter && isfinite(vmax)) {
      const uint32_t hmax = __float_as_uint(vmax) >> 16;
      w.kmax = key_of(static_cast<uint16_t>(hmax));
      uint32_t klo = w.kmax >= static_cast<uint32_t>(kWin - 1) ? w.kmax - (kWin - 1) : 0u;
      if (use_p && !use_k && !use_minp && pp > 0.f) {
        const float dcut = log2f((1.f - pp) / static_cast<float>(V)) - 1.f;
        uint32_t lo = klo, hi = w.kmax;  // smallest key with d >= dcut (kmax has d = 0)
        while (lo < hi) {
          const uint32_t mid = lo + ((hi - lo) >> 1);
          if ((KT::decode(mid) - vmax) * c >= dcut)
            hi = mid;
          else
            lo = mid + 1;
        }
        klo = lo;
      }
      w.klo = klo;
      w.nbins = static_cast<int>(w.kmax - klo) + 1;
      w.S = (w.nbins + CL - 1) / CL;
      w.hist = reinterpret_cast<uint32_t*>(big);
      w.red = w.hist + kWin;
      w.c = c;
      w.vmax = vmax;
      w.fxs = fx_scale(P.fx_shift);
      if (klo > 0x7FFFu && (w.kmax - 0x7FFFu) < 0x7000u)
        wmode = kWinPos;  // every window key is a positive nonzero value (below 2^97, so
                          // no negative raw pattern lands within kWin bins of raw(klo))
      else if (w.kmax < 0x7FFFu)
        wmode = kWinNeg;  // every window key is a negative nonzero value
      else
        wmode = kWinKey;
      for (int b = tid; b < w.nbins; b += blockDim.x) w.hist[b] = 0u;
      __syncthreads();
    }
  }

  // ---- pass 1 (fused): sums relative to vmax (+ window histogram)
  FSums fs{0.f, 0.f, 0.f};
  if constexpr (kBf16) {
    const uint32_t nb = static_cast<uint32_t>(w.nbins);
    switch (wmode) {
      case kWinPos:  // bin = raw - raw(klo), on the fp32 bit pattern
        fused_pass_bf16<kWinPos>(buf, n, vmax, c, nb, (w.klo - 0x7FFFu) << 16, 0u, w.hist, fs);
        break;
      case kWinNeg:  // bin = raw(klo) - raw
        fused_pass_bf16<kWinNeg>(buf, n, vmax, c, nb, (0xFFFFu - w.klo) << 16, 0u, w.hist, fs);
        break;
      case kWinKey:
        fused_pass_bf16<kWinKey>(buf, n, vmax, c, nb, 0u, w.klo, w.hist, fs);
        break;
      default:
        fused_pass_bf16<kWinNone>(buf, n, vmax, c, 0u, 0u, 0u, nullptr, fs);
        break;
    }
  } else {
    fused_pass_f32(reinterpret_cast<const uint32_t*>(buf), n, vmax, c, fs);
  }
  fs.c0 = block_sum(fs.c0, sh.fred);
  fs.zr = block_sum(fs.zr, sh.fred);
  fs.a = block_sum(fs.a, sh.fred);
  if (tid == 0) sh.part = Stats{vmax, fs.c0, fs.zr, fs.a};
  cluster.sync();  // sums and window histograms complete everywhere
  if (tid < static_cast<int>(CL)) sh.gathered[tid] = cluster.map_shared_rank(&sh, tid)->part;
  __syncthreads();
  Stats rs{vmax, 0.f, 0.f, 0.f};
  for (uint32_t r = 0; r < CL; ++r) {
    rs.c0 += sh.gathered[r].c0;
    rs.zr += sh.gathered[r].zr;
    rs.a += sh.gathered[r].a;
  }

  const bool nonfinite = !(isfinite(vmax) && isfinite(rs.zr) && isfinite(rs.a) && rs.c0 >= 1.f);
  const float log2z = stats_log2z(rs);
  const float h_full = kLn2 * (log2z - rs.a / stats_z(rs));
  const bool filtered = !nonfinite && any_filter;

  uint32_t tkey = 0;
  int32_t tie_cut = INT_MAX;
  float log2zs = log2z;
  float h_support = h_full;
  float c0s = rs.c0, zrs = rs.zr;
  int32_t n_support = nonfinite ? 0 : V;

  if (filtered) {
    bool all_ties = true;  // every element with key == tkey is kept
    u64 cnum = 0;          // ties kept at tkey when !all_ties
    bool have_t = false;
    bool sums_done = false;
    uint32_t tot_gt = 0, tot_eq = 0, tot_top = 0;
    float tot_mass = 0.f, tot_a = 0.f;
    uint32_t eq_rank[8];
    const float fxs = fx_scale(P.fx_shift);

    // ---- exact-key window select (bf16)
    bool win_ok = false;
    if constexpr (kBf16) {
      window_reduce(w, sh, cluster);
      win_ok = true;
      if (use_k || use_p) {
        Desc dk{}, dp{};
        u64 ck = 0;
        if (use_k) {
          win_ok = window_search(w, false, static_cast<u64>(kk), 0, dk, sh, cluster);
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
            mass1 = (static_cast<double>(rs.c0) + static_cast<double>(rs.zr)) * static_cast<double>(fxs);
          }
          const u64 tp = topp_target(pp, mass1);
          win_ok = window_search(w, true, tp, 1, dp, sh, cluster);
          if (win_ok) {
            const u64 fxe = dp.at_cnt ? dp.at_mass / dp.at_cnt : 0;
            const u64 need = tp > dp.above_mass ? tp - dp.above_mass : 0;
            u64 cp = fxe ? (need + fxe - 1) / fxe : dp.at_cnt;
            if (cp < 1) cp = 1;
            if (cp > dp.at_cnt) cp = dp.at_cnt;
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
      int hb = 0;
      have_t = false;
      all_ties = true;
      if (use_k) {
        Desc d = descend(buf, n, c, vmax, P.fx_shift, false, use_p, static_cast<u64>(kk), 1.f,
                         sh, ra, cluster, hb);
        const u64 ck = static_cast<u64>(kk) - d.above_cnt;
        tkey = d.key;
        cnum = ck;
        all_ties = ck >= d.at_cnt;
        have_t = true;
        if (use_p) {
          const u64 fx_t = d.at_cnt ? d.at_mass / d.at_cnt : 0;
          const u64 tp = topp_target(pp, static_cast<double>(d.above_mass + ck * fx_t));
          Desc e = descend(buf, n, c, vmax, P.fx_shift, true, true, tp, pp, sh, ra, cluster, hb);
          const u64 fxe = e.at_cnt ? e.at_mass / e.at_cnt : 0;
          const u64 need = tp > e.above_mass ? tp - e.above_mass : 0;
          u64 cp = fxe ? (need + fxe - 1) / fxe : e.at_cnt;
          if (cp < 1) cp = 1;
          if (cp > e.at_cnt) cp = e.at_cnt;
          if (e.key == tkey && cp > ck) cp = ck;
          tkey = e.key;
          cnum = cp;
          all_ties = cp >= e.at_cnt;
        }
      } else {
        Desc e = descend(buf, n, c, vmax, P.fx_shift, true, true, 0ull, pp, sh, ra, cluster, hb);
        const u64 tp = sh.b_target;
        const u64 fxe = e.at_cnt ? e.at_mass / e.at_cnt : 0;
        const u64 need = tp > e.above_mass ? tp - e.above_mass : 0;
        u64 cp = fxe ? (need + fxe - 1) / fxe : e.at_cnt;
        if (cp < 1) cp = 1;
        if (cp > e.at_cnt) cp = e.at_cnt;
        tkey = e.key;
        cnum = cp;
        all_ties = cp >= e.at_cnt;
        have_t = true;
      }
    }

    if (use_minp) {
      // smallest key whose probability ratio to the row max reaches min_p
      uint32_t lo = 0, hi = KT::kInfKey;
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        const float r = ex2((KT::decode(mid) - vmax) * c);
        if (r >= mp)
          hi = mid;
        else
          lo = mid + 1;
      }
      if (!have_t || lo > tkey) {
        tkey = lo;
        all_ties = true;
        have_t = true;
      }
    }

    // ---- support sums: keys above tkey, and the tie group at tkey
    // (elements equal to the row max are counted apart, as in Stats)
    uint32_t ngt = 0, neq = 0, ntop = 0;
    float smass = 0.f, sa = 0.f;
    if constexpr (kBf16) {
      if (win_ok && tkey >= w.klo) {
        // from the reduced window bins of this CTA's slice
        const int b0 = static_cast<int>(rank) * w.S;
        const int b1 = min(w.nbins, b0 + w.S);
        for (int b = b0 + tid; b < b1; b += blockDim.x) {
          const uint32_t cnt = w.red[b - b0];
          const uint32_t key = w.klo + b;
          if (cnt && key > tkey) {
            const float d = (KT::decode(key) - vmax) * c;
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
        if (tid == 0) neq = w.hist[tkey - w.klo];  // this CTA's own elements at tkey
        sums_done = true;
      }
    }
    if (!sums_done) {
      const uint32_t t = tkey;
      for_each(buf, n, [&](int, Raw raw) {
        const uint32_t key = key_of(raw);
        if (key > t) {
          const float d = (value_of(raw) - vmax) * c;
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
      });
    }
    ngt = block_sum(ngt, sh.ured);
    neq = block_sum(neq, sh.ured);
    ntop = block_sum(ntop, sh.ured);
    smass = block_sum(smass, sh.fred);
    sa = block_sum(sa, sh.fred);
    if (tid == 0) {
      sh.agg_ngt = ngt;
      sh.agg_eq = neq;
      sh.agg_top = ntop;
      sh.agg_mass = smass;
      sh.agg_a = sa;
    }
    cluster.sync();
    for (uint32_t r = 0; r < CL; ++r) {
      const SelShared* rsh = cluster.map_shared_rank(&sh, r);
      tot_gt += rsh->agg_ngt;
      eq_rank[r] = rsh->agg_eq;
      tot_eq += eq_rank[r];
      tot_top += rsh->agg_top;
      tot_mass += rsh->agg_mass;
      tot_a += rsh->agg_a;
    }
    const u64 ckeep = all_ties ? tot_eq : (cnum < tot_eq ? cnum : tot_eq);
    const float dt = (KT::decode(tkey) - vmax) * c;
    const float et = ex2(dt);
    Stats ss;
    ss.m = vmax;
    ss.c0 = static_cast<float>(tot_top) + (dt == 0.f ? static_cast<float>(ckeep) : 0.f);
    ss.zr = tot_mass + (dt == 0.f ? 0.f : static_cast<float>(ckeep) * et);
    ss.a = tot_a + static_cast<float>(ckeep) * dt * et;
    log2zs = stats_log2z(ss);
    h_support = kLn2 * (log2zs - ss.a / stats_z(ss));
    c0s = ss.c0;
    zrs = ss.zr;
    n_support = static_cast<int32_t>(tot_gt + ckeep);

    // ---- tie resolution: id of the last tie kept (ascending id order)
    if (ckeep < tot_eq) {
      u64 off = 0;
      uint32_t owner = 0;
      for (uint32_t r = 0; r < CL; ++r) {
        if (off + eq_rank[r] >= ckeep) {
          owner = r;
          break;
        }
        off += eq_rank[r];
      }
      if (rank == owner) {
        // each thread owns a contiguous id range of the slice: count its ties,
        // one exclusive scan over threads, then the thread holding the
        // need-th tie walks its range again to find it
        const int need = static_cast<int>(ckeep - off);
        const uint32_t t = tkey;
        constexpr int kV = 16 / sizeof(Raw);
        const int per = ((n + kThreads - 1) / kThreads + kV - 1) / kV * kV;
        const int j0 = tid * per, j1 = min(n, j0 + per);
        int mine = 0;
        {
          int j = j0;
          const uint4* v4 = reinterpret_cast<const uint4*>(buf);
          for (; j + kV <= j1; j += kV) {
            Raw r[kV];
            unpack(v4[j / kV], r);
#pragma unroll
            for (int i = 0; i < kV; ++i) mine += key_of(r[i]) == t;
          }
          for (; j < j1; ++j) mine += key_of(buf[j]) == t;
        }
        const int lane = tid & 31, warp = tid >> 5;
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int x = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += x;
        }
        if (lane == 31) sh.scan_tot[warp] = incl;
        __syncthreads();
        int wpre = 0;
        for (int ww = 0; ww < warp; ++ww) wpre += sh.scan_tot[ww];
        const int excl = wpre + incl - mine;
        if (excl < need && need <= excl + mine) {
          int cn = excl;
          for (int j = j0; j < j1; ++j) {
            if (key_of(buf[j]) == t && ++cn == need) {
              sh.tie_cut = c0 + j;
              break;
            }
          }
        }
      }
      cluster.sync();
      tie_cut = *cluster.map_shared_rank(&sh.tie_cut, owner);
    } else {
      tie_cut = INT_MAX;
    }
  }

  // ---- per-row outputs (rank 0, thread 0)
  if (rank == 0 && tid == 0) {
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
      const float dy = (value_of(ry) - vmax) * c;
      lp_v = kLn2 * (dy - log2z);
      if (!filtered) {
        in_s = true;
      } else {
        const uint32_t ky = key_of(ry);
        in_s = ky > tkey || (ky == tkey && y <= tie_cut);
      }
      if (in_s) {
        lp_s = filtered ? kLn2 * (dy - log2zs) : lp_v;
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
      cx.c0_full = rs.c0;
      cx.zr_full = rs.zr;
      cx.c0_sup = c0s;
      cx.zr_sup = zrs;
      P.ctx[row] = cx;
    }
  }

  // ---- support bitmask for this CTA's slice (words never straddle CTAs)
  if (P.support_mask) {
    const int words = (n + 31) / 32;
    const int64_t wstride = (V + 31) / 32;
    uint32_t* mrow = P.support_mask + static_cast<int64_t>(row) * wstride + c0 / 32;
    const int lane = tid & 31, warp = tid >> 5;
    for (int wd = warp; wd < words; wd += kWarps) {
      const int j = wd * 32 + lane;
      bool in = false;
      if (j < n && !nonfinite) {
        if (!filtered) {
          in = true;
        } else {
          const uint32_t key = key_of(buf[j]);
          in = key > tkey || (key == tkey && (c0 + j) <= tie_cut);
        }
      }
      const uint32_t bits = __ballot_sync(0xffffffffu, in);
      if (lane == 0) mrow[wd] = bits;
    }
  }
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------------------
// recorded support

constexpr int kRecThreads = 256;

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

constexpr int kMaxChunkBytes = 96 * 1024;

}  // namespace

int score_max_vocab(vs_dtype dtype) {
  const int esize = dtype == VS_BF16 ? 2 : 4;
  return 8 * (kMaxChunkBytes / esize);
}

// Cluster size and per-CTA slice (elements, multiple of 32) for a row of
// `vocab` elements: the smallest cluster whose slices fit an 80 KB budget
// (two CTAs per SM; small clusters pack the GPCs densely); larger rows grow
// the slice up to 96 KB.
int score_cluster_size(int vocab, vs_dtype dtype, int* chunk) {
  const int esize = dtype == VS_BF16 ? 2 : 4;
  const int target = 80 * 1024 / esize;
  int cl = 1;
  while (cl < 8 && (vocab + cl - 1) / cl > target) ++cl;
  int e = (vocab + cl - 1) / cl;
  e = (e + 31) & ~31;
  *chunk = e;
  return cl;
}

cudaError_t launch_score_computed(const ScoreParams& p, vs_dtype dtype, int cluster,
                                  cudaStream_t s) {
  const size_t esize = dtype == VS_BF16 ? 2 : 4;
  const size_t smem = static_cast<size_t>(p.chunk) * esize +
                      ((sizeof(SelShared) + 127) & ~size_t(127)) + big_area_bytes(cluster);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.rows) * cluster, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (dtype == VS_BF16) {
    e = cudaFuncSetAttribute(score_computed_kernel<uint16_t>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, score_computed_kernel<uint16_t>, p);
  }
  e = cudaFuncSetAttribute(score_computed_kernel<uint32_t>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, score_computed_kernel<uint32_t>, p);
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
