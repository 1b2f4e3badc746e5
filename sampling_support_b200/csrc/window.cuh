// The exact-key bf16 window of the computed-support kernels: which raw
// bits map to which histogram bin, the counting of one 16-byte vector into
// the bins, and the level below which no key can matter (xorl issue #71,
// section 3: the support's threshold lies at or above it).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "select.cuh"

namespace vs {

// Support sums: counts above the threshold, of its tie group and of the
// max-valued elements; mass and (u - m)-weighted mass of the others.
struct SupSums {
  uint32_t ngt, neq, ntp;
  float smass, sa;
};

enum WinMode : int { kWinNone = 0, kWinPos = 1, kWinNeg = 2, kWinKey = 3 };

// Window index of the raw bf16 bits r (>= the bin count outside the window).
// kWinPos (every window key is a positive value): base = raw bits of the
// lowest window key, and negative values wrap to huge indices; kWinNeg
// (every window key is a negative value): base = raw bits of the lowest
// window key (the most negative value); kWinKey: base = lowest window key.
template <int MODE>
__device__ __forceinline__ uint32_t win_index(uint32_t r, uint32_t base) {
  if constexpr (MODE == kWinPos)
    return r - base;
  else if constexpr (MODE == kWinNeg)
    return base - r;
  else
    return key_of(static_cast<uint16_t>(r)) - base;
}

// One shared-memory count increment at the 32-bit shared address a.
__device__ __forceinline__ void red_inc(uint32_t a) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(a) : "memory");
}

// Count the eight elements of one vector: in-window elements into their bin,
// the others into this lane's spill bin (bins >= the window's bin count are
// never read), so there is no predicate or branch.  For the sign-specific
// windows both elements of a 32-bit word are indexed at once with 16-bit
// lane arithmetic (add.u16x2, min.u16x2): kWinPos adds -base to the raw
// bits, kWinNeg adds -(lowest key) to their complement (0xFFFF - r is the
// key of a negative value); out-of-window values land at 16-bit indices of
// at least the bin count and clamp to the spill bin.
template <int MODE>
__device__ __forceinline__ void hist_vec(const uint4& q, uint32_t base, uint32_t spill,
                                         uint32_t hist_s) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  if constexpr (MODE == kWinPos || MODE == kWinNeg) {
    // 16-bit offsets, replicated in both halves
    const uint32_t off = MODE == kWinPos ? ((0u - base) & 0xFFFFu) : ((0u - (0xFFFFu - base)) & 0xFFFFu);
    const uint32_t off2 = off | (off << 16), sp2 = spill | (spill << 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t x = MODE == kWinNeg ? ~w[i] : w[i];
      asm("add.u16x2 %0, %1, %2;" : "=r"(x) : "r"(x), "r"(off2));
      asm("min.u16x2 %0, %1, %2;" : "=r"(x) : "r"(x), "r"(sp2));
      red_inc(hist_s + ((x & 0xFFFFu) << 2));
      red_inc(hist_s + ((x >> 16) << 2));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red_inc(hist_s + (min(win_index<MODE>(w[i] & 0xFFFFu, base), spill) << 2));
      red_inc(hist_s + (min(win_index<MODE>(w[i] >> 16, base), spill) << 2));
    }
  }
}

// The bin mapping of the window of keys [lo, hi] (at most kSelWin keys).
// The sign-specific modes index with 16-bit lane arithmetic; they are
// chosen only when every raw pattern of the other sign lands at an index of
// at least the bin count (their wrapped offsets start at 0x8000 - base for
// kWinPos and at base - 0x7FFF for kWinNeg), which fails only for windows
// of values beyond about 2^97 in magnitude; kWinKey maps through key_of.
__device__ __forceinline__ void win_mode(uint32_t lo, uint32_t hi, int& mode, uint32_t& base) {
  const uint32_t nb = hi - lo + 1u;
  if (lo > 0x7FFFu && 0x8000u - (lo - 0x7FFFu) >= nb) {
    mode = kWinPos;
    base = lo - 0x7FFFu;
  } else if (hi < 0x7FFFu && (0xFFFFu - lo) - 0x7FFFu >= nb) {
    mode = kWinNeg;
    base = 0xFFFFu - lo;
  } else {
    mode = kWinKey;
    base = lo;
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

}  // namespace vs
