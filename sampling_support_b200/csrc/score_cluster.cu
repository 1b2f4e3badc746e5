// Computed-support forward scoring of bf16 rows (temperature -> stable
// token-id top-k -> inclusive top-p -> min-p against the original row max;
// xorl issue #71, section 3) with each row split over a thread-block
// cluster.
//
// A row of V logits is cut into CL contiguous slices (CL = 8, 4, 2 or 1,
// the largest that keeps every cluster of the launch resident at once);
// CTA r of the row's cluster streams slice r once from HBM through a small
// ring of shared-memory stages filled by bulk copies.  In that one pass each
// element updates
//   * the online statistics: max, count of max-valued elements,
//     sum 2^(u - max), sum (u - max) 2^(u - max)   (u = z log2 e), and
//   * for a filtered row, this CTA's histogram of the EXACT 16-bit keys in a
//     window of at most 4,096 keys.  The window is fixed once every CTA's
//     first stage has arrived: its top lies kWinHi keys above the cluster's
//     largest first-stage value (a lower bound of the row maximum), and,
//     without top-k, its floor is the first key that can still matter
//     (min-p: 2^(u - m) >= min_p / 2; top-p: 2^(u - m) >= (1 - p) / (4 V)).
// Then, through distributed shared memory, the CTAs' statistics merge in
// rank order, and the histograms are reduce-scattered (CTA r sums its share
// of the bins over the cluster) and gathered back: every CTA holds the row's
// histogram and takes the same decisions from it.  Each bin holds one
// value, so its mass is count x 2^(u - m): the k-th element, the top-p
// crossing and the support sums all come from the bins, and nothing is read
// again.  A row whose maximum lies above the window, or whose decision lies
// below it, re-streams its slices into 4,096-key windows from the top down.
// Further passes re-read the slices (from L2 as a rule) only on request:
//   * the position of the last kept element of a partly kept tie group (ties
//     go to the lower token id), for the saved state, the bitmask or a
//     sample; without those only the ties before the target are counted,
//     when its membership hinges on them;
//   * the support bitmask;
//   * a seeded Gumbel-max token over the support (noise recipe in gumbel.cuh).
// Every decision is computed identically by all CTAs of a cluster from the
// same merged data, so the cluster barriers are reached uniformly; results
// are deterministic.

#include <climits>
#include <mutex>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"
#include "gumbel.cuh"
#include "select.cuh"
#include "window.cuh"

namespace vs {

namespace {

constexpr int kCT = 128;               // threads per CTA
constexpr int kCW = kCT / 32;          // warps per CTA
constexpr int kCStages = 3;            // ring depth
constexpr int kCStageBytes = 4096;
constexpr int kCSE = kCStageBytes / 2;  // elements per stage
constexpr int kCMinBlocks = 7;         // resident CTAs per SM the kernel is built for
constexpr uint32_t kCWinHi = 256;      // window keys above the first stages' maximum
constexpr int kCHistWords = kSelWin + 32;  // bins + one spill bin per lane

// What a CTA hands to its cluster after the streamed pass.
struct alignas(16) PassPart {
  Stats s;
  float vmax;
  uint32_t timeout;
};

struct ClSh {
  uint64_t full[kCStages];
  uint64_t empty[kCStages];
  Stats wst[kCW];
  float fred[kCW];
  uint32_t ured[kCW];
  SelShared<kCW> sel;
  SupSums sums[kCW];
  unsigned long long kred[kCW];
  u64 tot_c, tot_m;     // window search: totals of the current chunk
  uint32_t outstanding;  // loads issued and not yet consumed (broadcast by thread 0)
  uint32_t timeout;
  // cluster exchange slots: written by their CTA before a cluster barrier,
  // read by the peers after it
  float m0part;
  PassPart part;
  SupSums sumpart;
  uint32_t cntpart;
  uint32_t ylpart;
  unsigned long long keypart;
  int32_t tie_cut;  // written into every CTA by the one whose slice holds the cut
  uint32_t squeue[kCW][64];  // sampling: per-warp queue of member groups (index | bits << 28)
};

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Cluster barrier in two halves.  sync() is a full barrier; release() only
// arrives, after this CTA's last read of the peers' shared memory in a
// phase, and the matching wait comes with the next sync(), finish() or
// before this CTA overwrites a slot the peers may still be reading.  Every
// thread of every CTA of the cluster calls the same sequence.
struct ClBar {
  bool pending;
  __device__ void arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
  __device__ void wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
  __device__ void finish() {
    if (pending) wait();
    pending = false;
  }
  __device__ void sync() {
    finish();
    arrive();
    wait();
  }
  __device__ void release() {
    finish();
    arrive();
    pending = true;
  }
};

template <typename T>
__device__ __forceinline__ T* peer(T* p, uint32_t r) {
  return cg::this_cluster().map_shared_rank(p, r);
}

// ---------------------------------------------------------------------------
// streaming ring over this CTA's slice

struct CRing {
  const uint16_t* g;  // slice start in global memory
  int n;              // slice length (elements)
  uint16_t* buf;      // [kCStages][kCSE]
  ClSh* sh;
  uint32_t ld;  // loads issued (thread 0)
  uint32_t cs;  // stages consumed (all threads)
  __device__ int nst() const { return (n + kCSE - 1) / kCSE; }
  __device__ int count(int si) const { return min(kCSE, n - si * kCSE); }

  // thread 0: load stage si into the next ring slot
  __device__ void issue(int si) {
    const uint32_t L = ld++;
    const int slot = L % kCStages;
    if (L >= kCStages && !mbar_wait(&sh->empty[slot], ((L / kCStages) - 1u) & 1u)) sh->timeout = 1u;
    const uint32_t bytes = static_cast<uint32_t>((count(si) * 2 + 15) & ~15);
    mbar_arrive_expect_tx(&sh->full[slot], bytes);
    bulk_load(buf + static_cast<size_t>(slot) * kCSE, g + static_cast<size_t>(si) * kCSE, bytes,
              &sh->full[slot]);
  }
  __device__ void start(int s0, int s1) {
    if (threadIdx.x == 0) {
      // the ring buffer may have held a histogram share written and read
      // through the generic proxy: order those accesses before the copies
      fence_proxy_async();
      for (int si = s0; si < min(s1, s0 + kCStages); ++si) issue(si);
    }
  }
  __device__ const uint16_t* wait() {
    const int slot = cs % kCStages;
    if (!mbar_wait(&sh->full[slot], (cs / kCStages) & 1u)) atomicOr(&sh->timeout, 1u);
    return buf + static_cast<size_t>(slot) * kCSE;
  }
  // every warp releases the stage it consumed; thread 0 then issues `next`
  // (when below s1)
  __device__ void release(int next, int s1) {
    const int slot = cs % kCStages;
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&sh->empty[slot]))
                   : "memory");
    ++cs;
    if (threadIdx.x == 0 && next < s1) issue(next);
  }
  // loads issued and not consumed (after an early stop) are drained
  __device__ void drain() {
    if (threadIdx.x == 0) sh->outstanding = ld;
    __syncthreads();
    const uint32_t issued = sh->outstanding;
    while (cs < issued) {
      wait();
      release(0, 0);
    }
    __syncthreads();
  }
  // Run f(stage_ptr, n, base) over stages [s0, s1) in order; f returns true
  // (uniformly over the CTA) to stop early.
  template <typename F>
  __device__ void pass(int s0, int s1, F&& f) {
    start(s0, s1);
    bool stop = false;
    for (int si = s0; si < s1 && !stop; ++si) {
      const uint16_t* st = wait();
      stop = f(st, count(si), si * kCSE);
      release(stop ? s1 : si + kCStages, s1);
    }
    drain();
  }
};

// ---------------------------------------------------------------------------
// block helpers (kCT threads)

__device__ __forceinline__ float cblock_max(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = -kInf;
#pragma unroll
  for (int w = 0; w < kCW; ++w) t = fmaxf(t, scratch[w]);
  __syncthreads();
  return t;
}

__device__ __forceinline__ SupSums cblock_sum_sup(SupSums v, ClSh& sh) {
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
#pragma unroll
  for (int w = 0; w < kCW; ++w) {
    t.ngt += sh.sums[w].ngt;
    t.neq += sh.sums[w].neq;
    t.ntp += sh.sums[w].ntp;
    t.smass += sh.sums[w].smass;
    t.sa += sh.sums[w].sa;
  }
  __syncthreads();
  return t;
}

// Maximum value of one bf16 stage over the CTA.
__device__ __forceinline__ float cstage_max(const uint16_t* st, int n, float* scratch) {
  const int nv = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  uint32_t mx = 0xFF80FF80u;
  for (int v = threadIdx.x; v < nv; v += kCT) {
    const uint4 q = v4[v];
    mx = bmax2(mx, bmax2(bmax2(q.x, q.y), bmax2(q.z, q.w)));
  }
  float m = vmax_of(mx);
  for (int j = nv * 8 + threadIdx.x; j < n; j += kCT) m = fmaxf(m, value_of(st[j]));
  return cblock_max(m, scratch);
}

// One stage: statistics chains and, with a window, the histogram; each
// thread takes every kCT-th 16-byte vector, two in flight.
template <int MODE>
__device__ __forceinline__ void stage_main(const uint16_t* st, int n, float c, f32x2 c2,
                                           Chain (&ch)[2], uint32_t& vmax2, uint32_t wbase,
                                           uint32_t spill, uint32_t hist_s) {
  const int nv = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  int v = threadIdx.x;
  for (; v + kCT < nv; v += 2 * kCT) {
    const uint4 q0 = v4[v], q1 = v4[v + kCT];
    chain_vec(q0, c, c2, ch[0], vmax2);
    chain_vec(q1, c, c2, ch[1], vmax2);
    if constexpr (MODE != kWinNone) {
      hist_vec<MODE>(q0, wbase, spill, hist_s);
      hist_vec<MODE>(q1, wbase, spill, hist_s);
    }
  }
  if (v < nv) {
    const uint4 q = v4[v];
    chain_vec(q, c, c2, ch[0], vmax2);
    if constexpr (MODE != kWinNone) hist_vec<MODE>(q, wbase, spill, hist_s);
  }
  for (int j = nv * 8 + threadIdx.x; j < n; j += kCT) {
    const uint32_t r = st[j];
    vmax2 = bmax2(vmax2, r | (r << 16));
    float u[1] = {__fmul_rn(value_of(static_cast<uint16_t>(r)), c)};
    stats_add(ch[0].s, u);
    if constexpr (MODE != kWinNone) red_inc(hist_s + (min(win_index<MODE>(r, wbase), spill) << 2));
  }
}

// One stage of histogram only (re-streamed windows).
template <int MODE>
__device__ __forceinline__ void stage_hist(const uint16_t* st, int n, uint32_t wbase,
                                           uint32_t spill, uint32_t hist_s) {
  const int nv = n / 8;
  const uint4* v4 = reinterpret_cast<const uint4*>(st);
  int v = threadIdx.x;
  for (; v + kCT < nv; v += 2 * kCT) {
    const uint4 q0 = v4[v], q1 = v4[v + kCT];
    hist_vec<MODE>(q0, wbase, spill, hist_s);
    hist_vec<MODE>(q1, wbase, spill, hist_s);
  }
  if (v < nv) hist_vec<MODE>(v4[v], wbase, spill, hist_s);
  for (int j = nv * 8 + threadIdx.x; j < n; j += kCT)
    red_inc(hist_s + (min(win_index<MODE>(st[j], wbase), spill) << 2));
}

// The row's histogram in every CTA: bins [0, nb) of each CTA's `hist` are
// summed over the cluster, CTA r summing the share [r s, (r + 1) s) into
// `rs` (its idle ring buffer), and every CTA gathers the shares back into
// its own `hist`.  The caller has completed `hist` (__syncthreads).
__device__ void hist_exchange(uint32_t* hist, uint32_t* rs, int nb, uint32_t rank, uint32_t CL,
                              ClBar& bar) {
  if (CL == 1) return;
  const int share = ((nb + static_cast<int>(CL) - 1) / static_cast<int>(CL) + 3) & ~3;
  bar.sync();  // every CTA's histogram is complete
  const int b0 = static_cast<int>(rank) * share, b1 = min(nb, b0 + share);
  for (int b = b0 + 4 * static_cast<int>(threadIdx.x); b < b1; b += 4 * kCT) {
    uint4 acc = make_uint4(0u, 0u, 0u, 0u);
    for (uint32_t r = 0; r < CL; ++r) {
      const uint4 x = *reinterpret_cast<const uint4*>(peer(hist, r) + b);
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    *reinterpret_cast<uint4*>(rs + (b - b0)) = acc;
  }
  fence_proxy_async();  // the share lives where bulk copies land later
  bar.sync();  // every share is reduced; no CTA reads a histogram any more
  for (int b = 4 * static_cast<int>(threadIdx.x); b < nb; b += 4 * kCT) {
    const uint32_t r = static_cast<uint32_t>(b / share);
    *reinterpret_cast<uint4*>(hist + b) =
        *reinterpret_cast<const uint4*>(peer(rs, r) + (b - static_cast<int>(r) * share));
  }
  bar.release();  // a share may be overwritten once every CTA has gathered
  __syncthreads();
}

// From bin `top` down, the bin at which the cumulative count (by_mass
// false) or fixed-point mass first reaches need (>= 1), in chunks of 4 kCT
// bins (thread t holds bins 4t .. 4t + 3 of a chunk, ascending).  False
// when the bins [0, top] hold less than need; their totals are then in
// tc / tm.
__device__ bool csearch(const Window& w, int top, bool by_mass, u64 need, Desc& out, u64& tc,
                        u64& tm, ClSh& sh) {
  u64 ac = 0, am = 0;  // above the current chunk
  for (int hi = top; hi >= 0; hi -= 4 * kCT) {
    const int b0 = hi - 4 * kCT + 1 + 4 * static_cast<int>(threadIdx.x);
    uint32_t cnt[4];
    u64 fx[4];
    u64 lc = 0, lm = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int b = b0 + k;
      cnt[k] = b >= 0 ? w.hist[b] : 0u;
      fx[k] = cnt[k] ? static_cast<u64>(cnt[k]) * bin_fx(w, w.klo + static_cast<uint32_t>(b)) : 0ull;
      lc += cnt[k];
      lm += fx[k];
    }
    u64 ec, em;
    block_suffix_excl<kCT>(lc, lm, ec, em, sh.sel);
    if (threadIdx.x == 0) {
      sh.tot_c = ec + lc;
      sh.tot_m = em + lm;
      sh.sel.b_found = 0;
    }
    __syncthreads();
    const u64 base = by_mass ? am + em : ac + ec;
    const u64 mine = by_mass ? lm : lc;
    if (base < need && need <= base + mine) {
      u64 rc = ac + ec, rm = am + em;
      bool done = false;
#pragma unroll
      for (int k = 3; k >= 0; --k) {
        if (!done && cnt[k] && (by_mass ? rm + fx[k] : rc + cnt[k]) >= need) {
          sh.sel.b_key = w.klo + static_cast<uint32_t>(b0 + k);
          sh.sel.b_above_cnt = rc;
          sh.sel.b_above_mass = rm;
          sh.sel.b_at_cnt = cnt[k];
          sh.sel.b_at_mass = fx[k];
          sh.sel.b_found = 1;
          done = true;
        }
        if (!done) {
          rc += cnt[k];
          rm += fx[k];
        }
      }
    }
    __syncthreads();
    const bool found = sh.sel.b_found != 0;
    if (found) {
      out.key = sh.sel.b_key;
      out.above_cnt = sh.sel.b_above_cnt;
      out.above_mass = sh.sel.b_above_mass;
      out.at_cnt = sh.sel.b_at_cnt;
      out.at_mass = sh.sel.b_at_mass;
    }
    ac += sh.tot_c;
    am += sh.tot_m;
    __syncthreads();
    if (found) return true;
  }
  tc = ac;
  tm = am;
  return false;
}

// Support sums over the bins of keys (tkey, kmr], and the count at tkey.
__device__ SupSums sums_from_bins(const Window& w, uint32_t tkey, uint32_t kmr, ClSh& sh) {
  SupSums s{0u, 0u, 0u, 0.f, 0.f};
  const int hi = static_cast<int>(kmr - w.klo);
  for (int b = static_cast<int>(tkey - w.klo) + 1 + static_cast<int>(threadIdx.x); b <= hi; b += kCT) {
    const uint32_t cnt = w.hist[b];
    if (cnt) {
      const float d = key_u(w.klo + static_cast<uint32_t>(b), w.c) - w.m;
      const float e = ex2(d);
      const float fc = static_cast<float>(cnt);
      s.ngt += cnt;
      if (d == 0.f)
        s.ntp += cnt;
      else
        s.smass = fmaf(fc, e, s.smass);
      s.sa = fmaf(fc * d, e, s.sa);
    }
  }
  if (threadIdx.x == 0) s.neq = w.hist[tkey - w.klo];
  return cblock_sum_sup(s, sh);
}

struct Row {
  CRing ring;
  uint32_t* hist;
  uint32_t* rs;
  uint32_t rank, CL;
  int c0;  // slice start (row element index)
  ClBar bar;
};

// Re-stream this CTA's slice into the window of keys [lo, hi] and make the
// row's histogram of it in every CTA.
__device__ void rehist(Row& R, uint32_t lo, uint32_t hi, ClSh& sh) {
  R.bar.finish();  // the peers have gathered from this CTA's ring buffer
  int mode;
  uint32_t base;
  win_mode(lo, hi, mode, base);
  const int nb = static_cast<int>(hi - lo) + 1;
  for (int b = threadIdx.x; b < nb + 32; b += kCT) R.hist[b] = 0u;
  __syncthreads();
  const uint32_t spill = static_cast<uint32_t>(nb) + (threadIdx.x & 31);
  const uint32_t hs = smem_addr(R.hist);
  R.ring.pass(0, R.ring.nst(), [&](const uint16_t* st, int n, int) {
    if (mode == kWinPos)
      stage_hist<kWinPos>(st, n, base, spill, hs);
    else if (mode == kWinNeg)
      stage_hist<kWinNeg>(st, n, base, spill, hs);
    else
      stage_hist<kWinKey>(st, n, base, spill, hs);
    return false;
  });
  hist_exchange(R.hist, R.rs, nb, R.rank, R.CL, R.bar);
}

// Threshold search over re-streamed 4,096-key windows from key `ktop` down:
// the key at which the cumulative count (by_mass false) or mass reaches
// need.  When the row holds less than need (a top-p target from the
// floating-point statistics can exceed the fixed-point total by rounding),
// the lowest key of the row with all its ties.
__device__ Desc cascade(Row& R, bool by_mass, u64 need, uint32_t ktop, float c, float m, float fxs,
                        ClSh& sh) {
  u64 ac = 0, am = 0;
  uint32_t hi = ktop;
  uint32_t last_lo = 0, last_hi = 0;  // the lowest window holding an element
  u64 last_ac = 0, last_am = 0, last_tc = 0;
  bool any = false;
  Desc d{};
  for (;;) {
    const uint32_t lo = hi >= static_cast<uint32_t>(kSelWin - 1) ? hi - (kSelWin - 1) : 0u;
    rehist(R, lo, hi, sh);
    const Window w{lo, hi, static_cast<int>(hi - lo) + 1, kWinNone, 0u, R.hist, c, m, fxs};
    u64 tc = 0, tm = 0;
    const u64 have = by_mass ? am : ac;
    if (csearch(w, static_cast<int>(hi - lo), by_mass, need - have, d, tc, tm, sh)) {
      d.above_cnt += ac;
      d.above_mass += am;
      return d;
    }
    if (tc) {
      any = true;
      last_lo = lo;
      last_hi = hi;
      last_ac = ac;
      last_am = am;
      last_tc = tc;
    }
    ac += tc;
    am += tm;
    if (lo == 0) break;
    hi = lo - 1;
  }
  if (!any) return d;  // an empty row: unreachable for V >= 1
  rehist(R, last_lo, last_hi, sh);
  const Window w{last_lo, last_hi, static_cast<int>(last_hi - last_lo) + 1, kWinNone, 0u, R.hist,
                 c, m, fxs};
  u64 tc, tm;
  csearch(w, static_cast<int>(last_hi - last_lo), false, last_tc, d, tc, tm, sh);
  d.above_cnt += last_ac;
  d.above_mass += last_am;
  return d;
}

// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kCT, kCMinBlocks) score_cluster_kernel(ScoreParams P, int S) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint16_t* ringbuf = reinterpret_cast<uint16_t*>(smem_raw);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw + kCStages * kCStageBytes);
  ClSh& sh = *reinterpret_cast<ClSh*>(smem_raw + kCStages * kCStageBytes + kCHistWords * 4);

  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t rank = cluster.block_rank();
  const uint32_t CL = cluster.num_blocks();
  const int row = static_cast<int>(blockIdx.x / CL);
  const int tid = threadIdx.x;
  const int V = P.vocab;
  const int c0 = min(V, static_cast<int>(rank) * S);
  const int c1 = min(V, c0 + S);
  const uint16_t* grow = static_cast<const uint16_t*>(P.logits) + static_cast<int64_t>(row) * P.ld;

  if (tid == 0) {
    for (int s = 0; s < kCStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], kCW);
    }
    sh.timeout = 0;
    sh.tie_cut = INT_MAX;
    fence_barrier_init();
  }
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();

  Row R{CRing{grow + c0, c1 - c0, ringbuf, &sh, 0u, 0u}, hist,
        reinterpret_cast<uint32_t*>(ringbuf), rank, CL, c0, ClBar{false}};
  CRing& ring = R.ring;
  ClBar& bar = R.bar;

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
  const uint16_t ry = target_ok ? grow[y] : uint16_t(0);
  const int nst = ring.nst();

  // ---- the first stage of every slice: the cluster's largest first-stage
  // value m0, a lower bound of the row maximum, fixes the window and seeds
  // the statistics chains
  ring.start(0, nst);
  const uint16_t* st0 = nullptr;
  float m0l = -kInf;
  if (nst > 0) {
    st0 = ring.wait();
    m0l = cstage_max(st0, ring.count(0), sh.fred);
  }
  if (tid == 0) sh.m0part = m0l;
  bar.sync();
  float m0 = -kInf;
  for (uint32_t r = 0; r < CL; ++r) m0 = fmaxf(m0, *peer(&sh.m0part, r));
  bar.release();

  uint32_t wtop = 0, wlo = 0;  // window keys [wlo, wtop]
  int wmode = kWinNone;
  uint32_t wbase = 0;
  if (any_filter) {
    const uint32_t kref = key_of(static_cast<uint16_t>(__float_as_uint(m0) >> 16));
    wtop = min(kref + kCWinHi, KeyTraits<uint16_t>::kInfKey);
    wlo = wtop >= static_cast<uint32_t>(kSelWin - 1) ? wtop - (kSelWin - 1) : 0u;
    if (!use_k && isfinite(m0)) {
      float dlo = -kInf;
      if (use_minp) dlo = log2f(mp) - 1.f;
      if (use_p && pp > 0.f) dlo = fmaxf(dlo, log2f((1.f - pp) / static_cast<float>(V)) - 2.f);
      if (dlo > -kInf) wlo = key_at_level(wlo, wtop, c, __fmul_rn(m0, c), dlo);
    }
    win_mode(wlo, wtop, wmode, wbase);
    const int nb = static_cast<int>(wtop - wlo) + 1;
    for (int b = tid; b < nb + 32; b += kCT) hist[b] = 0u;
    __syncthreads();
  }

  // ---- the streamed pass
  Chain ch2[2];
  chain_seed(ch2[0], m0, c);
  chain_seed(ch2[1], m0, c);
  uint32_t vmax2 = 0xFF80FF80u;
  {
    const f32x2 c2 = pack2(c, c);
    const uint32_t spill = (wtop - wlo) + 1u + (tid & 31);
    const uint32_t hs = smem_addr(hist);
    for (int si = 0; si < nst; ++si) {
      const uint16_t* st = si == 0 ? st0 : ring.wait();
      const int n = ring.count(si);
      if (wmode == kWinNone)
        stage_main<kWinNone>(st, n, c, c2, ch2, vmax2, wbase, spill, hs);
      else if (wmode == kWinPos)
        stage_main<kWinPos>(st, n, c, c2, ch2, vmax2, wbase, spill, hs);
      else if (wmode == kWinNeg)
        stage_main<kWinNeg>(st, n, c, c2, ch2, vmax2, wbase, spill, hs);
      else
        stage_main<kWinKey>(st, n, c, c2, ch2, vmax2, wbase, spill, hs);
      ring.release(si + kCStages, nst);
    }
  }
  Stats sl = ch2[0].s;
  stats_merge(sl, ch2[1].s);
  sl = block_reduce(sl, sh.wst);
  const float vml = cblock_max(vmax_of(vmax2), sh.fred);
  if (tid == 0) sh.part = PassPart{sl, vml, sh.timeout};
  bar.sync();
  Stats s = stats_empty();
  float vmax = -kInf;
  uint32_t tmo = 0;
  for (uint32_t r = 0; r < CL; ++r) {
    const PassPart pr = *peer(&sh.part, r);
    stats_merge(s, pr.s);
    vmax = fmaxf(vmax, pr.vmax);
    tmo |= pr.timeout;
  }
  bar.release();

  const bool nonfinite = !stats_finite(s) || !isfinite(vmax);
  const float m = s.m;  // = fl(vmax c)
  const float log2z = stats_log2z(s);
  const float h_full = kLn2 * (log2z - s.a / stats_z(s));
  const bool filtered = !nonfinite && any_filter;
  const bool want_cut = P.ctx != nullptr || P.support_mask != nullptr || P.sampled != nullptr;

  if (any_filter) {
    __syncthreads();
    hist_exchange(hist, R.rs, static_cast<int>(wtop - wlo) + 1, rank, CL, bar);
  }

  uint32_t tkey = 0;
  int32_t tie_cut = INT_MAX;
  bool cut_known = true;
  u64 ckeep = 0;
  float log2zs = log2z, h_support = h_full, c0s = s.c0, zrs = s.zr;
  int32_t n_support = nonfinite ? 0 : V;

  if (filtered) {
    const float fxs = fx_scale(P.fx_shift);
    bool all_ties = true;
    u64 cnum = 0;
    bool have_t = false;
    const uint32_t kmr = key_of(static_cast<uint16_t>(__float_as_uint(vmax) >> 16));
    const Window w{wlo, wtop, static_cast<int>(wtop - wlo) + 1, wmode, 0u, hist, c, m, fxs};
    // the window holds every key at or above its floor only when the row
    // maximum lies inside it
    bool win_ok = kmr <= wtop;
    if (win_ok && (use_k || use_p)) {
      const int top = static_cast<int>(kmr - wlo);
      Desc dk{}, dp{};
      u64 ck = 0, tc, tm;
      if (use_k) {
        win_ok = csearch(w, top, false, static_cast<u64>(kk), dk, tc, tm, sh);
        if (win_ok) {
          ck = static_cast<u64>(kk) - dk.above_cnt;
          tkey = dk.key;
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
        win_ok = csearch(w, top, true, tp, dp, tc, tm, sh);
        if (win_ok) {
          u64 cp = topp_ties(dp, tp, bin_fx(w, dp.key));
          if (use_k && dp.key == tkey && cp > ck) cp = ck;
          tkey = dp.key;
          cnum = cp;
          all_ties = cp >= dp.at_cnt;
          have_t = true;
        }
      }
      if (!win_ok && use_p && !use_k && use_minp && minp_key<uint16_t>(mp, c, m) >= w.klo) {
        // the top-p crossing lies below the window, whose floor is at or
        // below the min-p level: min-p decides the support (applied below)
        win_ok = true;
        have_t = false;
        all_ties = true;
      }
    }
    if (!win_ok && (use_k || use_p)) {
      // ---- the decision lies outside the window: re-streamed windows from
      // the row maximum down
      have_t = false;
      all_ties = true;
      if (use_k) {
        const Desc d = cascade(R, false, static_cast<u64>(kk), kmr, c, m, fxs, sh);
        const u64 ck = static_cast<u64>(kk) - d.above_cnt;
        tkey = d.key;
        cnum = ck;
        all_ties = ck >= d.at_cnt;
        have_t = true;
        if (use_p) {
          const u64 fx_t = key_fx<uint16_t>(d.key, c, m, fxs);
          const u64 tp = topp_target(pp, static_cast<double>(d.above_mass + ck * fx_t));
          const Desc e = cascade(R, true, tp, kmr, c, m, fxs, sh);
          u64 cp = topp_ties(e, tp, key_fx<uint16_t>(e.key, c, m, fxs));
          if (e.key == tkey && cp > ck) cp = ck;
          tkey = e.key;
          cnum = cp;
          all_ties = cp >= e.at_cnt;
        }
      } else {
        const u64 tp = topp_target(pp, (static_cast<double>(s.c0) + static_cast<double>(s.zr)) *
                                           static_cast<double>(fxs));
        const Desc e = cascade(R, true, tp, kmr, c, m, fxs, sh);
        const u64 cp = topp_ties(e, tp, key_fx<uint16_t>(e.key, c, m, fxs));
        tkey = e.key;
        cnum = cp;
        all_ties = cp >= e.at_cnt;
        have_t = true;
      }
    }
    if (use_minp) {
      const uint32_t lo = minp_key<uint16_t>(mp, c, m);
      if (!have_t || lo > tkey) {
        tkey = lo;
        all_ties = true;
        have_t = true;
      }
    }

    // ---- support sums: from the bins when the window holds every key from
    // tkey up, else by a pass over the slices merged in rank order
    SupSums sums;
    if (win_ok && tkey >= wlo) {
      sums = sums_from_bins(w, tkey, kmr, sh);
    } else {
      SupSums part{0u, 0u, 0u, 0.f, 0.f};
      const uint32_t t = tkey;
      bar.finish();
      ring.pass(0, nst, [&](const uint16_t* st, int n, int) {
        const int nv = n / 8;
        const uint4* v4 = reinterpret_cast<const uint4*>(st);
        auto one = [&](uint16_t raw) {
          const uint32_t key = key_of(raw);
          if (key > t) {
            const float d = __fmul_rn(value_of(raw), c) - m;
            const float e = ex2(d);
            ++part.ngt;
            if (d == 0.f)
              ++part.ntp;
            else
              part.smass += e;
            part.sa = fmaf(d, e, part.sa);
          } else if (key == t) {
            ++part.neq;
          }
        };
        for (int v = tid; v < nv; v += kCT) {
          uint16_t r[8];
          unpack(v4[v], r);
#pragma unroll
          for (int i = 0; i < 8; ++i) one(r[i]);
        }
        for (int j = nv * 8 + tid; j < n; j += kCT) one(st[j]);
        return false;
      });
      part = cblock_sum_sup(part, sh);
      if (tid == 0) sh.sumpart = part;
      bar.sync();
      sums = SupSums{0u, 0u, 0u, 0.f, 0.f};
      for (uint32_t r = 0; r < CL; ++r) {
        const SupSums q = *peer(&sh.sumpart, r);
        sums.ngt += q.ngt;
        sums.neq += q.neq;
        sums.ntp += q.ntp;
        sums.smass += q.smass;
        sums.sa += q.sa;
      }
      bar.release();
    }
    const u64 tot_eq = sums.neq;
    ckeep = all_ties ? tot_eq : (cnum < tot_eq ? cnum : tot_eq);
    const float dt = __fmul_rn(KeyTraits<uint16_t>::decode(tkey), c) - m;
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

    // ---- id of the last tie kept (ascending id order), when the saved
    // state, the bitmask or a sample needs it: each CTA counts the ties in
    // its slice; the one holding the cut finds it and writes it into every
    // CTA
    if (ckeep < tot_eq) {
      cut_known = false;
      if (want_cut) {
        const uint32_t t = tkey;
        bar.finish();
        uint32_t mine = 0;
        ring.pass(0, nst, [&](const uint16_t* st, int n, int) {
          for (int j = tid; j < n; j += kCT) mine += key_of(st[j]) == t;
          return false;
        });
        mine = block_sum(mine, sh.ured);
        if (tid == 0) sh.cntpart = mine;
        bar.sync();
        u64 before = 0;
        for (uint32_t r = 0; r < rank; ++r) before += *peer(&sh.cntpart, r);
        bar.release();
        if (before < ckeep && ckeep <= before + mine) {
          const int need = static_cast<int>(ckeep - before);  // the cut's rank within this slice
          int seen = 0;  // ties in earlier stages (uniform)
          ring.pass(0, nst, [&](const uint16_t* st, int n, int base) {
            const int per = ((n + kCT - 1) / kCT + 7) / 8 * 8;
            const int j0 = min(n, tid * per), j1 = min(n, j0 + per);
            int cnt = 0;
            for (int j = j0; j < j1; ++j) cnt += key_of(st[j]) == t;
            int total;
            const int excl = seen + block_excl_int<kCT>(cnt, total, sh.sel);
            if (excl < need && need <= excl + cnt) {
              int cn = excl;
              for (int jj = j0; jj < j1; ++jj)
                if (key_of(st[jj]) == t && ++cn == need) {
                  sh.tie_cut = c0 + base + jj;
                  break;
                }
            }
            seen += total;
            return seen >= need;
          });
          __syncthreads();
          if (tid < static_cast<int>(CL)) *peer(&sh.tie_cut, static_cast<uint32_t>(tid)) = sh.tie_cut;
        }
        bar.sync();
        tie_cut = sh.tie_cut;
        cut_known = true;
      }
    }
  }

  // ---- the target's earlier ties, when its membership hinges on them
  uint32_t ylt = 0;
  if (filtered && !cut_known && target_ok && key_of(ry) == tkey) {
    const uint32_t t = tkey;
    const int yl = y - c0;  // ties at slice positions < yl precede the target
    uint32_t mine = 0;
    if (yl > 0) {
      bar.finish();
      const int s1 = min(nst, (yl + kCSE - 1) / kCSE);
      ring.pass(0, s1, [&](const uint16_t* st, int n, int base) {
        const int lim = min(n, yl - base);
        for (int j = tid; j < lim; j += kCT) mine += key_of(st[j]) == t;
        return false;
      });
    }
    mine = block_sum(mine, sh.ured);
    bar.finish();
    if (tid == 0) sh.ylpart = mine;
    bar.sync();
    for (uint32_t r = 0; r < CL; ++r) ylt += *peer(&sh.ylpart, r);
    bar.release();
  }

  // ---- per-row outputs (rank 0)
  if (rank == 0 && tid == 0) {
    uint32_t status = 0;
    float lp_v = __int_as_float(0x7fc00000), lp_s = __int_as_float(0x7fc00000);
    bool in_s = false;
    if (!target_ok) status |= VS_ROW_TARGET_OUT_OF_RANGE;
    if (nonfinite) {
      status |= VS_ROW_NONFINITE_INPUT;
    } else if (target_ok) {
      const float uy = __fmul_rn(value_of(ry), c);
      lp_v = kLn2 * (uy - m - log2z);
      if (!filtered) {
        in_s = true;
      } else {
        const uint32_t ky = key_of(ry);
        in_s = ky > tkey || (ky == tkey && (cut_known ? y <= tie_cut : ylt < ckeep));
      }
      if (in_s) {
        lp_s = filtered ? kLn2 * (uy - m - log2zs) : lp_v;
      } else {
        lp_s = -kInf;
        status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
      }
    }
    if (tmo || sh.timeout) status |= kRowDeviceTimeout;
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

  // ---- support bitmask of this slice, one 32-id word per thread and stage
  // (slices and stages start on multiples of 32 ids)
  if (P.support_mask) {
    const int64_t wstride = (V + 31) / 32;
    uint32_t* mrow = P.support_mask + static_cast<int64_t>(row) * wstride + c0 / 32;
    bar.finish();
    ring.pass(0, nst, [&](const uint16_t* st, int n, int base) {
      for (int wd = tid; wd < (n + 31) / 32; wd += kCT) {
        uint32_t bits = 0;
        for (int i = 0; i < 32; ++i) {
          const int j = wd * 32 + i;
          if (j >= n || nonfinite) break;
          bool in = true;
          if (filtered) {
            const uint32_t key = key_of(st[j]);
            in = key > tkey || (key == tkey && c0 + base + j <= tie_cut);
          }
          if (in) bits |= 1u << i;
        }
        mrow[(base >> 5) + wd] = bits;
      }
      return false;
    });
  }

  // ---- seeded Gumbel-max token over the support.  Tokens go in groups of
  // four (slices and stages start on multiples of four); each warp queues
  // its groups that hold a member and drains the queue 32 groups at a time,
  // so the Philox block and the logarithms run on full warps and only for
  // members.  The CTAs' best candidates meet at rank 0.
  if (P.sampled) {
    unsigned long long best = 0ull;
    bar.finish();
    if (!nonfinite) {
      const uint32_t nrow = static_cast<uint32_t>(P.row_base + row);
      const int lane = tid & 31, warp = tid >> 5;
      uint32_t* wq = sh.squeue[warp];
      ring.pass(0, nst, [&](const uint16_t* st, int n, int sbase) {
        const int base = c0 + sbase;
        auto take = [&](uint32_t e) {
          const int q = static_cast<int>(e & 0x0FFFFFFFu);
          uint64_t wv[4];
          philox4x64_10(static_cast<uint64_t>(base >> 2) + q, 0, 0, 0, P.sample_seed, nrow, wv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (!((e >> (28 + i)) & 1u)) continue;
            const int j = 4 * q + i;
            const unsigned long long k =
                gumbel_key(gumbel_score(value_of(st[j]), T, gumbel_of(wv[i])), base + j);
            best = k > best ? k : best;
          }
        };
        const int ng = (n + 3) / 4;
        int count = 0;  // queued groups of this warp (warp-uniform)
        for (int qb = warp * 32; qb < ng; qb += kCT) {
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
    if (tid == 0) sh.keypart = best;
    bar.sync();
    if (rank == 0 && tid == 0) {
      unsigned long long b = 0ull;
      for (uint32_t r = 0; r < CL; ++r) {
        const unsigned long long k = *peer(&sh.keypart, r);
        b = k > b ? k : b;
      }
      P.sampled[row] = gumbel_key_id(b);
    }
    bar.release();
  }
  // no CTA leaves while a peer may still read its shared memory
  bar.finish();
}

size_t cluster_smem_bytes() {
  return static_cast<size_t>(kCStages) * kCStageBytes + kCHistWords * 4 +
         ((sizeof(ClSh) + 127) & ~size_t(127));
}

// Largest cluster size whose clusters for `rows` rows are all resident at
// once (per device, from the occupancy calculator); at least one stage per
// CTA's slice.
cudaError_t pick_cluster(int rows, int vocab, int* cl) {
  static std::mutex mu;
  static int maxc[64][4] = {};  // [device][log2 cluster size] max active clusters, +1 (0 = unknown)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int pick = 1;
  for (int lg = 3; lg >= 1; --lg) {
    const int size = 1 << lg;
    if ((vocab + size - 1) / size < 2 * kCSE) continue;
    int n = 0;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (dev >= 0 && dev < 64 && maxc[dev][lg] > 0) n = maxc[dev][lg] - 1;
      else {
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(static_cast<unsigned>(size) * 64u);
        cfg.blockDim = dim3(kCT);
        cfg.dynamicSmemBytes = cluster_smem_bytes();
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(size);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&n, score_cluster_kernel, &cfg);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) maxc[dev][lg] = n + 1;
      }
    }
    if (rows <= n) {
      pick = size;
      break;
    }
  }
  *cl = pick;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_score_cluster(const ScoreParams& p, cudaStream_t s) {
  int cl = 1;
  cudaError_t e = pick_cluster(p.rows, p.vocab, &cl);
  if (e != cudaSuccess) return e;
  const int S = ((p.vocab + cl - 1) / cl + 31) & ~31;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p.rows) * static_cast<unsigned>(cl));
  cfg.blockDim = dim3(kCT);
  cfg.dynamicSmemBytes = cluster_smem_bytes();
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, score_cluster_kernel, p, S);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace vs
