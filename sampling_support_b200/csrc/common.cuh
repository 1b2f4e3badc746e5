// Device helpers shared by the scoring kernels (sm_100a).
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cg = cooperative_groups;

namespace vs {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kInf = __builtin_huge_valf();

// Iteration cap for every mbarrier wait: try_wait suspends the thread for a
// hardware-defined interval per attempt, so this bounds a wait to seconds.
constexpr uint32_t kWaitLimit = 1u << 24;

// Block barrier entered by whole warps.  A warp whose lanes took different
// paths since their last common instruction (one lane issuing a copy or an
// atomic, lanes leaving a wait loop at different times) meets at __syncwarp
// first: the block barrier instruction is an aligned one, which every lane
// of a warp must execute together, and a warp that reaches it in pieces can
// be counted more than once, letting the other warps through early.
__device__ __forceinline__ void cta_sync() {
  __syncwarp();
  __syncthreads();
}

// Per-row status bit set when a bounded device wait gave up (never expected).
constexpr uint32_t kRowDeviceTimeout = 1u << 5;  // VS_ROW_DEVICE_TIMEOUT

// 2^x on the MUFU unit (ex2.approx.ftz.f32: PTX ISA instruction, relative
// error about 2^-22; -inf -> +0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// monotone integer keys:  key(a) < key(b)  <=>  a < b  for finite values, and
// key(-0) == key(+0).  For raw IEEE bits x of width W with sign bit S:
//   negative x:      key = (2^W - 1) - x      (0 .. S - 1;  -0 -> S - 1)
//   non-negative x:  key = x + (S - 1)        (S - 1 .. 2^W - 2; +0 -> S - 1)

__device__ __forceinline__ uint32_t key_of(uint16_t raw) {
  const uint32_t x = raw;
  return (x & 0x8000u) ? (0xFFFFu - x) : (x + 0x7FFFu);
}
__device__ __forceinline__ uint32_t key_of(uint32_t raw) {
  return (raw & 0x80000000u) ? (0xFFFFFFFFu - raw) : (raw + 0x7FFFFFFFu);
}
__device__ __forceinline__ float value_of(uint16_t raw) {
  return __uint_as_float(static_cast<uint32_t>(raw) << 16);
}
__device__ __forceinline__ float value_of(uint32_t raw) { return __uint_as_float(raw); }

template <typename Raw>
struct KeyTraits;
template <>
struct KeyTraits<uint16_t> {
  static constexpr int kBits = 16;
  static constexpr uint32_t kInfKey = 0x7F80u + 0x7FFFu;  // key of +inf
  __device__ static float decode(uint32_t k) {
    const uint32_t bits = k >= 0x7FFFu ? k - 0x7FFFu : 0xFFFFu - k;
    return __uint_as_float(bits << 16);
  }
};
template <>
struct KeyTraits<uint32_t> {
  static constexpr int kBits = 32;
  static constexpr uint32_t kInfKey = 0x7F800000u + 0x7FFFFFFFu;
  __device__ static float decode(uint32_t k) {
    const uint32_t bits = k >= 0x7FFFFFFFu ? k - 0x7FFFFFFFu : 0xFFFFFFFFu - k;
    return __uint_as_float(bits);
  }
};

// Unpack one 16-byte vector of raw elements.
__device__ __forceinline__ void unpack(const uint4& q, uint16_t (&r)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r[2 * i] = static_cast<uint16_t>(w[i] & 0xFFFFu);
    r[2 * i + 1] = static_cast<uint16_t>(w[i] >> 16);
  }
}
__device__ __forceinline__ void unpack(const uint4& q, uint32_t (&r)[4]) {
  r[0] = q.x;
  r[1] = q.y;
  r[2] = q.z;
  r[3] = q.w;
}

// ---------------------------------------------------------------------------
// online log-sum-exp and entropy statistics in base-2 units (u = z log2 e):
//   m  = max u
//   c0 = number of elements with u == m      (each contributes 2^0 = 1)
//   zr = sum over the other elements of 2^(u - m)
//   a  = sum over all elements of (u - m) 2^(u - m)      (<= 0)
// Keeping the max elements' count apart from the rest lets
//   log2 Z = log2 c0 + log1p(zr / c0) / ln 2,   Z = c0 + zr
// keep full relative precision when one token dominates (Z close to 1),
// and then  LSE = ln2 (m + log2 Z),  H = ln2 (log2 Z - a / Z).

struct Stats {
  float m, c0, zr, a;
};

__device__ __forceinline__ Stats stats_empty() { return {-kInf, 0.f, 0.f, 0.f}; }

__device__ __forceinline__ float stats_z(const Stats& s) { return s.c0 + s.zr; }

// log2 Z = log2 c0 + log2(1 + t), t = zr / c0: for t < 2^-6 the series
// t - t^2/2 + t^3/3 - t^4/4 + t^5/5 (remainder below t^6/6 < 2^-38) keeps
// full precision of a small t; above, log2 of the rounded sum c0 + zr is
// within 2^-24 / ln 2 absolute, under 4e-6 relative to log2 Z.
__device__ __forceinline__ float stats_log2z(const Stats& s) {
  const float t = s.zr / s.c0;
  const bool small = t < 0.015625f;
  const float l = log2f(small ? s.c0 : s.c0 + s.zr);
  const float p = fmaf(fmaf(fmaf(fmaf(t, 0.2f, -0.25f), t, 1.f / 3.f), t, -0.5f), t, 1.f);
  return small ? fmaf(t * p, kLog2e, l) : l;
}

// True when the statistics describe only finite values.
__device__ __forceinline__ bool stats_finite(const Stats& s) {
  return isfinite(s.m) && isfinite(s.zr) && isfinite(s.a) && s.c0 >= 1.f;
}

// Re-express `s` relative to a new maximum mn >= s.m (s non-empty).
__device__ __forceinline__ void stats_rebase(Stats& s, float mn) {
  if (s.m == mn) return;
  const float f = ex2(s.m - mn);
  const float z = s.c0 + s.zr;
  s.a = f * fmaf(s.m - mn, z, s.a);
  s.zr = f * z;
  s.c0 = 0.f;
  s.m = mn;
}

// Merge b into s.  An empty side (c0 == 0 and zr == 0) is skipped; NaN/inf
// propagate through zr / a.
__device__ __forceinline__ void stats_merge(Stats& s, Stats b) {
  if (b.c0 == 0.f && b.zr == 0.f) return;
  if (s.c0 == 0.f && s.zr == 0.f) {
    s = b;
    return;
  }
  const float mn = fmaxf(s.m, b.m);
  stats_rebase(s, mn);
  stats_rebase(b, mn);
  s.c0 += b.c0;
  s.zr += b.zr;
  s.a += b.a;
}

// Add a batch of N values u[] (already scaled to base-2 units).
template <int N>
__device__ __forceinline__ void stats_add(Stats& s, const float (&u)[N]) {
  float bm = u[0];
#pragma unroll
  for (int i = 1; i < N; ++i) bm = fmaxf(bm, u[i]);
  if (bm > s.m) {
    if (s.c0 != 0.f || s.zr != 0.f) stats_rebase(s, bm);
    s.m = bm;
  }
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float d = u[i] - s.m;
    const float e = ex2(d);
    const bool top = d == 0.f;
    s.c0 += top ? 1.f : 0.f;
    s.zr += top ? 0.f : e;
    s.a = fmaf(d, e, s.a);
  }
}

__device__ __forceinline__ Stats shfl_xor(const Stats& s, int lane_mask) {
  return {__shfl_xor_sync(0xffffffffu, s.m, lane_mask), __shfl_xor_sync(0xffffffffu, s.c0, lane_mask),
          __shfl_xor_sync(0xffffffffu, s.zr, lane_mask), __shfl_xor_sync(0xffffffffu, s.a, lane_mask)};
}

// Deterministic block reduction; result valid in every thread.  `scratch`
// holds at least blockDim.x / 32 entries.  The block max comes first, then
// every thread rebases its own statistics onto it once and plain sums
// follow (no chain of rebases).  Per phase: warp shuffles, one partial per
// warp, warp 0 reduces the partials (a fixed order) and broadcasts.
__device__ __forceinline__ Stats block_reduce(Stats s, Stats* scratch) {
  __shared__ float s_m;
  __shared__ Stats s_res;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  float m = s.m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) scratch[warp].m = m;
  cta_sync();
  if (warp == 0) {
    float x = lane < nw ? scratch[lane].m : -kInf;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    if (lane == 0) s_m = x;
  }
  cta_sync();
  m = s_m;
  if (s.c0 != 0.f || s.zr != 0.f) stats_rebase(s, m);
  float c0 = s.c0, zr = s.zr, a = s.a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c0 += __shfl_xor_sync(0xffffffffu, c0, o);
    zr += __shfl_xor_sync(0xffffffffu, zr, o);
    a += __shfl_xor_sync(0xffffffffu, a, o);
  }
  if (lane == 0) scratch[warp] = Stats{m, c0, zr, a};
  cta_sync();
  if (warp == 0) {
    float x0 = 0.f, x1 = 0.f, x2 = 0.f;
    if (lane < nw) {
      x0 = scratch[lane].c0;
      x1 = scratch[lane].zr;
      x2 = scratch[lane].a;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x0 += __shfl_xor_sync(0xffffffffu, x0, o);
      x1 += __shfl_xor_sync(0xffffffffu, x1, o);
      x2 += __shfl_xor_sync(0xffffffffu, x2, o);
    }
    if (lane == 0) s_res = Stats{m, x0, x1, x2};
  }
  cta_sync();
  return s_res;
}

// Sum of v over the block, valid in every thread (warp shuffles, one
// partial per warp in `scratch`, warp 0 reduces them in a fixed order).
template <typename T>
__device__ __forceinline__ T block_sum(T v, T* scratch) {
  __shared__ T s_res;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) scratch[warp] = v;
  cta_sync();
  if (warp == 0) {
    T x = lane < static_cast<int>(blockDim.x >> 5) ? scratch[lane] : T(0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) s_res = x;
  }
  cta_sync();
  return s_res;
}

// ---------------------------------------------------------------------------
// packed fp32x2 arithmetic (sm_100a: add/sub/mul/fma.rn.f32x2), two lanes per
// 64-bit register; each lane rounds exactly as the scalar instruction.

typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// ---------------------------------------------------------------------------
// mbarrier + bulk async copy (global -> shared), PTX ISA.

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false after the
// iteration cap.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Bulk copy `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global memory into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Largest bulk piece issued at once (keeps each instruction modest).
constexpr uint32_t kBulkPiece = 32768;

// Load `bytes` from src into dst via bulk copies on `bar` (thread 0 only).
// The caller arms the barrier with the full byte count first.
__device__ __forceinline__ void bulk_load_all(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  for (uint32_t off = 0; off < bytes; off += kBulkPiece) {
    const uint32_t n = min(kBulkPiece, bytes - off);
    bulk_load(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off, n, bar);
  }
}

// ---------------------------------------------------------------------------
// bf16 streaming statistics

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  const __nv_bfloat162 r = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                   *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// The eight elements of a bf16 vector into s one by one, the max-valued
// ones counted apart (the vector reaches or raises s's maximum, or holds a
// NaN: rare once the maximum is seeded).
static __device__ __forceinline__ Stats stats_vec_bf16_scalar(uint32_t w0, uint32_t w1, uint32_t w2,
                                                   uint32_t w3, float c, Stats s) {
  const uint32_t w[4] = {w0, w1, w2, w3};
  float u[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    u[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), c);
    u[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), c);
  }
  stats_add(s, u);
  return s;
}

// A statistics chain over bf16 vectors with its running maximum also kept as
// raw bf16 bits in both halves of a word, so that the per-vector test "does
// any element reach the maximum" is one packed bf16x2 comparison.
struct Chain {
  Stats s;
  uint32_t thr2;  // raw bf16 of the value whose fl(value c) is s.m, both halves
};

__device__ __forceinline__ Chain chain_empty() { return Chain{stats_empty(), 0xFF80FF80u}; }

// Start a chain at the value v (a lower bound of the maximum of the data it
// will see): no element counted yet.
__device__ __forceinline__ void chain_seed(Chain& ch, float v, float c) {
  const uint32_t r = __float_as_uint(v) >> 16;
  ch.s = Stats{__fmul_rn(v, c), 0.f, 0.f, 0.f};
  ch.thr2 = r | (r << 16);
}

// True when an element of the packed pair mm is >= the threshold pair (NaN
// compares false: it reaches the sums through the packed path).
__device__ __forceinline__ bool any_ge_bf16x2(uint32_t mm, uint32_t thr2) {
  uint32_t r;
  asm("{\n .reg .pred p, q;\n setp.ge.bf16x2 p|q, %1, %2;\n selp.u32 %0, 1, 0, p;\n"
      " @q mov.u32 %0, 1;\n}\n"
      : "=r"(r)
      : "r"(mm), "r"(thr2));
  return r != 0u;
}

// One 8-element bf16 vector into the chain; vmax2 keeps the running maximum
// of the raw values (packed bf16x2).
__device__ __forceinline__ void chain_vec(const uint4& q, float c, f32x2 c2, Chain& ch,
                                          uint32_t& vmax2) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  const uint32_t mm = bmax2(bmax2(w[0], w[1]), bmax2(w[2], w[3]));
  vmax2 = bmax2(vmax2, mm);
  if (any_ge_bf16x2(mm, ch.thr2)) {
    const float bmv = fmaxf(__uint_as_float(mm << 16), __uint_as_float(mm & 0xFFFF0000u));
    const float bm = __fmul_rn(bmv, c);
    if (bm > ch.s.m) {
      if (ch.s.c0 != 0.f || ch.s.zr != 0.f) stats_rebase(ch.s, bm);
      ch.s.m = bm;
      const uint32_t r = __float_as_uint(bmv) >> 16;
      ch.thr2 = r | (r << 16);
    }
    ch.s = stats_vec_bf16_scalar(w[0], w[1], w[2], w[3], c, ch.s);
  } else {
    const f32x2 nm2 = pack2(-ch.s.m, -ch.s.m);
    f32x2 zr2 = pack2(0.f, 0.f), a2 = pack2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const f32x2 x2 = pack2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
      const f32x2 d2 = fma2(x2, c2, nm2);
      float d0, d1;
      unpack2(d2, d0, d1);
      const f32x2 e2 = pack2(ex2(d0), ex2(d1));
      zr2 = add2(zr2, e2);
      a2 = fma2(d2, e2, a2);
    }
    float z0, z1, a0, a1;
    unpack2(zr2, z0, z1);
    unpack2(a2, a0, a1);
    ch.s.zr += z0 + z1;
    ch.s.a += a0 + a1;
  }
}

// Largest value of a packed bf16x2 running maximum.
__device__ __forceinline__ float vmax_of(uint32_t vmax2) {
  return fmaxf(__uint_as_float(vmax2 << 16), __uint_as_float(vmax2 & 0xFFFF0000u));
}

}  // namespace vs
