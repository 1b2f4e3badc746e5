// Exact support selection helpers shared by the computed-support kernels:
// fixed-point masses, block scans, the exact-key bf16 window search and the
// 8-bit radix digit scan (xorl issue #71, section 3: stable token-id top-k,
// inclusive top-p on the top-k mass, min-p against the original row max).
//
// Masses are 64-bit fixed point, 2^(u - m) * 2^fx_shift with
// vocab * 2^fx_shift <= 2^63, so every sum is exact and order-independent.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace vs {

typedef unsigned long long u64;

constexpr int kSelWin = 4096;  // exact-key window (bins)
constexpr int kSelBins = 256;  // radix digit bins

__device__ __forceinline__ float fx_scale(int shift) {
  return __int_as_float((127 + shift) << 23);
}

// Target mass of inclusive top-p: ceil(p * mass), clamped to [1, mass].
__device__ __forceinline__ u64 topp_target(float p, double mass) {
  const double want = ceil(static_cast<double>(p) * mass);
  if (want <= 1.0) return 1ull;
  if (want >= mass) return static_cast<u64>(mass);
  return static_cast<u64>(want);
}

// One threshold candidate: its key, the count and mass strictly above it,
// and the count and mass of its tie group.
struct Desc {
  uint32_t key;
  u64 above_cnt, above_mass, at_cnt, at_mass;
};

// Radix digit histogram (aliases the window storage in the kernels).
struct RadixArrays {
  u64 mass[kSelBins];
  uint32_t cnt[kSelBins];
};
static_assert(sizeof(RadixArrays) <= kSelWin * 4, "radix arrays alias the window");

// Shared scratch for the scans of a block of NW warps.
template <int NW>
struct SelShared {
  u64 scan_a[NW], scan_b[NW];
  int32_t iscan[NW];
  uint32_t b_key;
  u64 b_above_cnt, b_above_mass, b_at_cnt, b_at_mass;
  int32_t b_found;
  int32_t i_total;  // block_excl_int: the block total
};

// Exclusive suffix sums of (a, b) over the threads of the block, thread
// order = ascending.  Every thread calls.  Warp 0 turns the warps' totals
// into per-warp exclusive suffixes.
template <int NT>
__device__ __forceinline__ void block_suffix_excl(u64 a, u64 b, u64& ea, u64& eb,
                                                  SelShared<NT / 32>& sh) {
  constexpr int NW = NT / 32;
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
  cta_sync();
  if (warp == 0) {
    // inclusive suffix over the warps' totals, then exclusive
    const u64 ta0 = lane < NW ? sh.scan_a[lane] : 0ull, tb0 = lane < NW ? sh.scan_b[lane] : 0ull;
    u64 xa = ta0, xb = tb0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const u64 ya = __shfl_down_sync(0xffffffffu, xa, o);
      const u64 yb = __shfl_down_sync(0xffffffffu, xb, o);
      if (lane + o < 32) {
        xa += ya;
        xb += yb;
      }
    }
    if (lane < NW) {
      sh.scan_a[lane] = xa - ta0;
      sh.scan_b[lane] = xb - tb0;
    }
  }
  cta_sync();
  ea = sh.scan_a[warp] + ia - a;
  eb = sh.scan_b[warp] + ib - b;
  cta_sync();
}

// Exclusive prefix sum of v over the block; total in `total`.
template <int NT>
__device__ __forceinline__ int block_excl_int(int v, int& total, SelShared<NT / 32>& sh) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh.iscan[warp] = incl;
  cta_sync();
  if (warp == 0) {
    const int t0 = lane < NW ? sh.iscan[lane] : 0;
    int x = t0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < NW) sh.iscan[lane] = x - t0;  // exclusive prefix of the warp totals
    if (lane == 31) sh.i_total = x;
  }
  cta_sync();
  const int pre = sh.iscan[warp];
  total = sh.i_total;
  cta_sync();
  return pre + incl - v;
}

// ---------------------------------------------------------------------------
// exact-key window over bf16 keys [klo, klo + nbins): hist[key - klo] counts
// the elements holding that exact value, so a bin's mass is count x 2^(u - m).

struct Window {
  uint32_t klo, kmax;
  int nbins;
  int mode;         // row kernel: how raw bits map to bins
  uint32_t fconst;  // row kernel: raw-bit offset of the sign-specific modes
  uint32_t* hist;   // [nbins]
  float c, m, fxs;  // u = v c; mass 2^(u - m) in fixed point 2^fx_shift
};

__device__ __forceinline__ float key_u(uint32_t key, float c) {
  return __fmul_rn(KeyTraits<uint16_t>::decode(key), c);
}

__device__ __forceinline__ u64 bin_fx(const Window& w, uint32_t key) {
  return __float2ull_rn(ex2(key_u(key, w.c) - w.m) * w.fxs);
}

// Search the window from the largest key for the bin where the cumulative
// count (by_mass false) or fixed-point mass first reaches need (>= 1).
// False when the whole window holds less than need.  Each thread owns a run
// of NB = ceil(4096 / NT) consecutive bins, loads them and their fixed-point
// masses into registers at once (independent loads and exponentials, no
// chain through the loop), and the one thread whose run holds the crossing
// walks its registers back down.
template <int NT>
__device__ __forceinline__ bool win_search(const Window& w, bool by_mass, u64 need, Desc& out,
                                        SelShared<NT / 32>& sh) {
  constexpr int NB = (kSelWin + NT - 1) / NT;
  const int i0 = threadIdx.x * NB;
  const int nb = w.nbins;
  const uint32_t* hist = w.hist;
  const uint32_t klo = w.klo;
  uint32_t cnt[NB];
  u64 fx[NB];
#pragma unroll
  for (int k = 0; k < NB; ++k) cnt[k] = i0 + k < nb ? hist[i0 + k] : 0u;
  u64 lc = 0, lm = 0;
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    fx[k] = cnt[k] ? static_cast<u64>(cnt[k]) * bin_fx(w, klo + i0 + k) : 0ull;
    lc += cnt[k];
    lm += fx[k];
  }
  u64 ec, em;
  block_suffix_excl<NT>(lc, lm, ec, em, sh);
  if (threadIdx.x == 0) sh.b_found = 0;
  cta_sync();
  const u64 base = by_mass ? em : ec;
  const u64 mine = by_mass ? lm : lc;
  if (base < need && need <= base + mine) {
    u64 ac = ec, am = em;
    bool done = false;
#pragma unroll
    for (int k = NB - 1; k >= 0; --k) {
      if (!done && cnt[k] && (by_mass ? am + fx[k] : ac + cnt[k]) >= need) {
        sh.b_key = klo + i0 + k;
        sh.b_above_cnt = ac;
        sh.b_above_mass = am;
        sh.b_at_cnt = cnt[k];
        sh.b_at_mass = fx[k];
        sh.b_found = 1;
        done = true;
      }
      if (!done) {
        ac += cnt[k];
        am += fx[k];
      }
    }
  }
  cta_sync();
  const bool ok = sh.b_found != 0;
  out.key = sh.b_key;
  out.above_cnt = sh.b_above_cnt;
  out.above_mass = sh.b_above_mass;
  out.at_cnt = sh.b_at_cnt;
  out.at_mass = sh.b_at_mass;
  cta_sync();
  return ok;
}

// Warp 0: from the top digit down, the bin where the cumulative `by`
// quantity reaches need; sums of the bins strictly above it.  When no bin
// reaches need, the lowest non-empty bin.
__device__ inline void scan_bins(const uint32_t* gcnt, const u64* gmass, bool by_mass, u64 need,
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
  const uint32_t ballot = __ballot_sync(0xffffffffu, excl < need && need <= incl);
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
    int lowest = 256;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (gcnt[255 - 8 * lane - i] != 0) lowest = 255 - 8 * lane - i;
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

// Fixed-point mass of one element with this key: 2^(u - m) 2^fx_shift.
template <typename Raw>
__device__ __forceinline__ u64 key_fx(uint32_t key, float c, float m, float fxs) {
  return __float2ull_rn(ex2(__fmul_rn(KeyTraits<Raw>::decode(key), c) - m) * fxs);
}

// Number of the top-p tie group's elements to keep (each of fixed-point
// mass fxe): enough that the mass reaches the target, at least one, at most
// the group.  The quotient comes from one double division, made exact by
// an integer correction (products stay below 2^64).
__device__ __forceinline__ u64 topp_ties(const Desc& d, u64 target, u64 fxe) {
  const u64 need = target > d.above_mass ? target - d.above_mass : 0;
  u64 cp = d.at_cnt;
  if (fxe != 0) {
    const double q = ceil(static_cast<double>(need) / static_cast<double>(fxe));
    cp = q >= static_cast<double>(d.at_cnt) + 1.0 ? d.at_cnt + 1 : static_cast<u64>(q);
    if (cp > 0 && (cp - 1) * fxe >= need)
      --cp;
    else if (cp * fxe < need)
      ++cp;
  }
  if (cp < 1) cp = 1;
  if (cp > d.at_cnt) cp = d.at_cnt;
  return cp;
}

// Smallest key whose probability ratio to the row max reaches min_p.
template <typename Raw>
__device__ __forceinline__ uint32_t minp_key(float mp, float c, float m) {
  uint32_t lo = 0, hi = KeyTraits<Raw>::kInfKey;
  while (lo < hi) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (ex2(__fmul_rn(KeyTraits<Raw>::decode(mid), c) - m) >= mp)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

}  // namespace vs
