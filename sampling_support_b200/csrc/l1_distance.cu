// Draft/target probability distance (DeepSpec PR #87, DSpark, section
// "Purpose"): one softmax of the draft row and one of the target row, one
// |p - q| reduction, reused for accept_rate = clamp(1 - 0.5 L1, 0, 1) and for
// the weighted L1 loss; gradient with respect to the draft logits only.
//
// One thread-block cluster per row.  Each CTA bulk-copies its slice of BOTH
// rows into shared memory once; the passes (maxima, sums for p and q, the
// |p - q| and sum p s reduction, the gradient) read that copy, so the whole
// job reads each logit from HBM exactly once and writes the gradient once.
// The CTAs exchange their partial records by pushing them into each other's
// shared memory (distributed shared memory) and combine them in a fixed
// order; cross-row sums (the loss) are reduced by a single block in row order.

#include <mutex>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace vs {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCluster = 8;  // CTAs per row pair at most (portable cluster size)

struct L1Shared {
  uint64_t bar;
  uint64_t xbar[2];  // the two exchanges: every CTA's records received
  alignas(16) Stats gathered[kMaxCluster][2];  // exchange 1: [rank] = that CTA's (draft, target) statistics
  alignas(16) float2 agg[kMaxCluster];         // exchange 2: [rank] = that CTA's (sum |p - q|, sum p s)
  Stats merged[2];                   // exchange 1's records merged (draft, target)
  Stats red[kWarps];
  float fred[kWarps];
  float2 red2[2][kWarps];  // block reductions: one partial per warp (two buffers in turn)
  uint32_t timeout;
};

// Two values reduced over the block at once with one barrier: warp
// shuffles, one partial per warp in buffer `buf`, and every thread combines
// the partials in warp order (the same order everywhere, so every thread
// gets the same result).  MAX selects the maximum, else the sum.
// Consecutive calls take the two buffers in turn, so a buffer is rewritten
// only after a barrier that follows its last read.
template <bool MAX>
__device__ __forceinline__ float2 block_reduce2(float a, float b, L1Shared& sh, int buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float oa = __shfl_xor_sync(0xffffffffu, a, o), ob = __shfl_xor_sync(0xffffffffu, b, o);
    a = MAX ? fmaxf(a, oa) : a + oa;
    b = MAX ? fmaxf(b, ob) : b + ob;
  }
  if (lane == 0) sh.red2[buf][warp] = make_float2(a, b);
  cta_sync();
  float2 x = sh.red2[buf][0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) {
    const float2 y = sh.red2[buf][w];
    x.x = MAX ? fmaxf(x.x, y.x) : x.x + y.x;
    x.y = MAX ? fmaxf(x.y, y.y) : x.y + y.y;
  }
  return x;
}

struct L1Params {
  int32_t rows, vocab;
  int64_t ld;
  const void* draft;
  const void* target;
  const float* row_weight;
  float* l1;
  float* accept;
  void* grad;
  int64_t grad_ld;
  double* ws_wsum;  // [1] sum of this call's weights (written by l1_wsum_kernel)
  double* ws_wl1;   // [rows] w_i * L1_i
  const double* wsum_norm;  // [1] the loss denominator: ws_wsum, or the caller's sum over all shards
  int32_t chunk;
};

// Programmatic dependent launch within one call: the weight-sum kernel lets
// the distance kernel start at once, and the distance kernel lets the loss
// kernel start; each waits on its predecessor only before it reads that
// predecessor's output (the weight sum before the gradient pass; the
// per-row terms in the loss kernel).
__device__ __forceinline__ void l1_pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void l1_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// The exit barrier of a cluster: no CTA leaves while a record pushed by the
// exchanges below may still be on its way to a peer.  Each CTA arrives once
// every record sent to it is in (after its second exchange) and waits only
// at its exit, so the barrier's latency overlaps the gradient pass instead
// of following the gradient's stores.
__device__ __forceinline__ void exit_arrive() {
  asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
}
__device__ __forceinline__ void exit_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Exchanges between the CTAs of a cluster: each CTA pushes its record into
// slot [its rank] of every CTA's array (st.async into the peer's shared
// memory, counted in bytes on the peer's mbarrier for that exchange) and
// waits on its own mbarrier until the CL records are in.  No CTA reads
// another's shared memory and no cluster barrier is taken per exchange.
__device__ __forceinline__ uint32_t cl_map(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void push_stats(uint32_t raddr, uint32_t rbar, const Stats& v) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%2, %3, %4, %5}, [%1];" ::"r"(raddr),
      "r"(rbar), "r"(__float_as_uint(v.m)), "r"(__float_as_uint(v.c0)), "r"(__float_as_uint(v.zr)),
      "r"(__float_as_uint(v.a))
      : "memory");
}
__device__ __forceinline__ void push_f2(uint32_t raddr, uint32_t rbar, float a, float b) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%2, %3}, [%1];" ::"r"(raddr),
               "r"(rbar), "r"(__float_as_uint(a)), "r"(__float_as_uint(b))
               : "memory");
}
// exchange 1: thread r < CL sends this CTA's (draft, target) statistics to CTA r
__device__ __forceinline__ void exchange_stats(L1Shared& sh, uint32_t rank, uint32_t CL, const Stats& d,
                                               const Stats& t) {
  const uint32_t r = threadIdx.x;
  if (r < CL) {
    const uint32_t rbar = cl_map(&sh.xbar[0], r);
    push_stats(cl_map(&sh.gathered[rank][0], r), rbar, d);
    push_stats(cl_map(&sh.gathered[rank][1], r), rbar, t);
  }
  if (!mbar_wait(&sh.xbar[0], 0)) atomicOr(&sh.timeout, 1u);
}
// Exchange 1's CL records merged by warp 0 along a fixed shuffle tree over
// lanes 0-7 (((0,1),(2,3)),((4,5),(6,7))): the same tree in every CTA and
// for draft and target alike, so every CTA and every thread get the same
// statistics, and identical rows stay identical.
__device__ __forceinline__ Stats stats_shfl_down(const Stats& s, int o) {
  return Stats{__shfl_down_sync(0xffffffffu, s.m, o), __shfl_down_sync(0xffffffffu, s.c0, o),
               __shfl_down_sync(0xffffffffu, s.zr, o), __shfl_down_sync(0xffffffffu, s.a, o)};
}
static_assert((kMaxCluster & (kMaxCluster - 1)) == 0 && kMaxCluster <= 32,
              "merge_records' shuffle tree spans a power-of-two lane range within a warp");
__device__ __forceinline__ void merge_records(L1Shared& sh, uint32_t CL, Stats& d, Stats& t) {
  if (threadIdx.x < 32) {
    const uint32_t lane = threadIdx.x;
    Stats a = lane < CL ? sh.gathered[lane][0] : stats_empty();
    Stats b = lane < CL ? sh.gathered[lane][1] : stats_empty();
#pragma unroll
    for (int o = 1; o < kMaxCluster; o <<= 1) {
      const Stats a2 = stats_shfl_down(a, o), b2 = stats_shfl_down(b, o);
      stats_merge(a, a2);
      stats_merge(b, b2);
    }
    if (lane == 0) {
      sh.merged[0] = a;
      sh.merged[1] = b;
    }
  }
  cta_sync();
  d = sh.merged[0];
  t = sh.merged[1];
}
// exchange 2: thread r < CL sends this CTA's (sum |p - q|, sum p s) to CTA r
__device__ __forceinline__ void exchange_sums(L1Shared& sh, uint32_t rank, uint32_t CL, float l1, float ps) {
  const uint32_t r = threadIdx.x;
  if (r < CL) push_f2(cl_map(&sh.agg[rank], r), cl_map(&sh.xbar[1], r), l1, ps);
  if (!mbar_wait(&sh.xbar[1], 0)) atomicOr(&sh.timeout, 1u);
}

__device__ __forceinline__ float sgn(float d) { return d > 0.f ? 1.f : (d < 0.f ? -1.f : 0.f); }

// p_j (in [0, 1], so bits 30 and 31 of its fp32 pattern are zero) and
// s_j = sign(p_j - q_j) in one 32-bit word: bit 31 set for s = -1, bit 30 set
// for s = 0.  Pass 2 writes it over the element's two shared-memory slots so
// the gradient pass needs no second exponentiation.
__device__ __forceinline__ uint32_t enc_ps(float p, float d) {
  uint32_t w = __float_as_uint(p);
  if (d < 0.f)
    w |= 0x80000000u;
  else if (!(d > 0.f))
    w |= 0x40000000u;
  return w;
}
__device__ __forceinline__ float dec_grad(uint32_t w, float coef, float ps) {
  const float p = __uint_as_float(w & 0x3FFFFFFFu);
  const float s = (w & 0x40000000u) ? 0.f : ((w & 0x80000000u) ? -1.f : 1.f);
  return coef * p * (s - ps);
}

__device__ __forceinline__ float l1_block_max(float v, float* scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  cta_sync();
  float t = -kInf;
  for (int w = 0; w < kWarps; ++w) t = fmaxf(t, scratch[w]);
  cta_sync();
  return t;
}

// Largest of the eight bf16 values of a vector.
__device__ __forceinline__ float vec_max(const uint4& a) {
  const uint32_t m = bmax2(bmax2(a.x, a.y), bmax2(a.z, a.w));
  return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
}

// Element i of the eight bf16 values in w[4].
__device__ __forceinline__ float bf16_at(const uint32_t (&w)[4], int i) {
  return __uint_as_float(i & 1 ? w[i >> 1] & 0xFFFF0000u : w[i >> 1] << 16);
}

// One element of pass 2: accumulates |p - q| and p sign(p - q) and returns
// the in-place (p, sign) word: p (in [0, 1], so bits 31 and 30 of its fp32
// pattern are clear) with bit 31 = the sign bit of p - q and bit 30 set when
// p == q (sign 0).
__device__ __forceinline__ uint32_t l1_step(float p, float q, float& l1, float& ps) {
  const float d = p - q;
  l1 += fabsf(d);
  const uint32_t sbit = __float_as_uint(d) & 0x80000000u;
  const bool zero = d == 0.f;
  const float s = zero ? 0.f : __uint_as_float(sbit | 0x3F800000u);  // sign(d)
  ps = fmaf(p, s, ps);
  return __float_as_uint(p) | sbit | (zero ? 0x40000000u : 0u);
}

// Gradient of one element from its (p, sign) word: k_pos, k_neg, k_zero are
// coef (s - sum p s) for s = +1, -1, 0.
__device__ __forceinline__ float l1_grad(uint32_t w, float k_pos, float k_neg, float k_zero) {
  const float p = __uint_as_float(w & 0x3FFFFFFFu);
  return p * ((w & 0x40000000u) ? k_zero : ((w & 0x80000000u) ? k_neg : k_pos));
}

// bf16 rows: the row pair's slice sits in shared memory; four passes over it
// with packed fp32x2 arithmetic.  Pass 0: slice maxima.  Pass 1: sum of
// 2^(u - m) over the slice for both rows (u = z log2 e; the log-sum-exp
// needs no count of max-valued elements here), merged across the cluster.
// Pass 2: |p - q|, p sign(p - q), (p, sign) written in place: a full
// vector's eight words over its two 16-byte slots in element order, a tail
// element's word split into its two 16-bit slots (high half in the draft's).
// Pass 3: the gradient.
template <typename G>
__device__ __forceinline__ void l1_rows_bf16(uint16_t* bd, uint16_t* bt, int n, int c0, int row,
                                             uint32_t rank, uint32_t CL, cg::cluster_group& cluster,
                                             L1Shared& sh, const L1Params& P) {
  const int tid = threadIdx.x;
  const int nfull = n / 8;
  const uint4* d4 = reinterpret_cast<const uint4*>(bd);
  const uint4* t4 = reinterpret_cast<const uint4*>(bt);
  const f32x2 l2e = pack2(kLog2e, kLog2e);

  // pass 0
  uint32_t mxd = 0xFF80FF80u, mxt = 0xFF80FF80u;
  for (int v = tid; v < nfull; v += kThreads) {
    const uint4 a = d4[v], b = t4[v];
    mxd = bmax2(mxd, bmax2(bmax2(a.x, a.y), bmax2(a.z, a.w)));
    mxt = bmax2(mxt, bmax2(bmax2(b.x, b.y), bmax2(b.z, b.w)));
  }
  float vd = fmaxf(__uint_as_float(mxd << 16), __uint_as_float(mxd & 0xFFFF0000u));
  float vt = fmaxf(__uint_as_float(mxt << 16), __uint_as_float(mxt & 0xFFFF0000u));
  for (int j = nfull * 8 + tid; j < n; j += kThreads) {
    vd = fmaxf(vd, value_of(bd[j]));
    vt = fmaxf(vt, value_of(bt[j]));
  }
  {
    const float2 mm = block_reduce2<true>(vd, vt, sh, 0);
    vd = mm.x;
    vt = mm.y;
  }

  // pass 1: sum of 2^(x log2 e - m) over the slice, with x log2 e rounded
  // before the subtraction (a max-valued element gives exactly 2^0); draft
  // and target go through the same code, so identical rows give identical
  // sums
  const float md = __fmul_rn(vd, kLog2e), mt = __fmul_rn(vt, kLog2e);
  {
    const f32x2 nmd = pack2(-md, -md), nmt = pack2(-mt, -mt);
    f32x2 zd = pack2(0.f, 0.f), zt = pack2(0.f, 0.f);
    for (int v = tid; v < nfull; v += kThreads) {
      const uint4 a = d4[v], b = t4[v];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float e0, e1, f0, f1;
        unpack2(add2(mul2(pack2(__uint_as_float(wa[i] << 16), __uint_as_float(wa[i] & 0xFFFF0000u)), l2e), nmd), e0, e1);
        unpack2(add2(mul2(pack2(__uint_as_float(wb[i] << 16), __uint_as_float(wb[i] & 0xFFFF0000u)), l2e), nmt), f0, f1);
        zd = add2(zd, pack2(ex2(e0), ex2(e1)));
        zt = add2(zt, pack2(ex2(f0), ex2(f1)));
      }
    }
    float z0, z1, y0, y1;
    unpack2(zd, z0, z1);
    unpack2(zt, y0, y1);
    float sz = z0 + z1, sy = y0 + y1;
    for (int j = nfull * 8 + tid; j < n; j += kThreads) {
      sz += ex2(__fmul_rn(value_of(bd[j]), kLog2e) - md);
      sy += ex2(__fmul_rn(value_of(bt[j]), kLog2e) - mt);
    }
    const float2 zz = block_reduce2<false>(sz, sy, sh, 1);
    Stats sd{md, 0.f, zz.x, 0.f}, st{mt, 0.f, zz.y, 0.f};
    if (vd == -kInf && zz.x == 0.f) sd = stats_empty();
    if (vt == -kInf && zz.y == 0.f) st = stats_empty();
    exchange_stats(sh, rank, CL, sd, st);
  }
  Stats Sd, St;
  merge_records(sh, CL, Sd, St);
  const float ld2 = stats_log2z(Sd), lt2 = stats_log2z(St);
  const float cd = Sd.m + ld2, ct = St.m + lt2;

  // pass 2: p = 2^(fl(x log2 e) - (m + log2 Z)) and q alike (the same code
  // for both rows; a one-element row gets p = q = 1 exactly), |p - q| and
  // p sign(p - q), and (p, sign) in place for pass 3
  float l1 = 0.f, ps = 0.f;
  const bool keep = P.grad != nullptr;
  uint4* d4w = reinterpret_cast<uint4*>(bd);
  uint4* t4w = reinterpret_cast<uint4*>(bt);
  {
    const f32x2 ncd = pack2(-cd, -cd), nct = pack2(-ct, -ct);
    for (int v = tid; v < nfull; v += kThreads) {
      const uint4 a = d4[v], b = t4[v];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
      uint32_t enc[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float p0, p1, q0, q1;
        unpack2(add2(mul2(pack2(__uint_as_float(wa[i] << 16), __uint_as_float(wa[i] & 0xFFFF0000u)), l2e), ncd), p0, p1);
        unpack2(add2(mul2(pack2(__uint_as_float(wb[i] << 16), __uint_as_float(wb[i] & 0xFFFF0000u)), l2e), nct), q0, q1);
        enc[2 * i] = l1_step(ex2(p0), ex2(q0), l1, ps);
        enc[2 * i + 1] = l1_step(ex2(p1), ex2(q1), l1, ps);
      }
      if (keep) {
        // the vector's eight words fill its two 16-byte slots in order:
        // elements 0-3 over the draft slot, 4-7 over the target slot
        d4w[v] = make_uint4(enc[0], enc[1], enc[2], enc[3]);
        t4w[v] = make_uint4(enc[4], enc[5], enc[6], enc[7]);
      }
    }
    for (int j = nfull * 8 + tid; j < n; j += kThreads) {
      const uint32_t e = l1_step(ex2(__fmul_rn(value_of(bd[j]), kLog2e) - cd),
                                 ex2(__fmul_rn(value_of(bt[j]), kLog2e) - ct), l1, ps);
      if (keep) {
        bd[j] = static_cast<uint16_t>(e >> 16);
        bt[j] = static_cast<uint16_t>(e & 0xFFFFu);
      }
    }
  }
  {
    const float2 lp = block_reduce2<false>(l1, ps, sh, 0);
    exchange_sums(sh, rank, CL, lp.x, lp.y);
  }
  float L1 = 0.f, PS = 0.f;
  for (uint32_t r = 0; r < CL; ++r) {
    L1 += sh.agg[r].x;
    PS += sh.agg[r].y;
  }
  exit_arrive();  // every record sent to this CTA is in
  const float w = P.row_weight ? P.row_weight[row] : 1.f;
  if (rank == 0 && tid == 0) {
    if (P.l1) P.l1[row] = L1;
    if (P.accept) P.accept[row] = fminf(1.f, fmaxf(0.f, 1.f - 0.5f * L1));
    if (P.ws_wl1) P.ws_wl1[row] = static_cast<double>(w) * static_cast<double>(L1);
  }

  // pass 3: d loss / d draft_j = (w / sum w) p_j (s_j - sum_k p_k s_k)
  if (P.grad) {
    l1_pdl_wait();  // the weight-sum kernel's result
    const double wsum = *P.wsum_norm;
    const float coef = wsum > 0.0 ? static_cast<float>(static_cast<double>(w) / wsum) : 0.f;
    const float k_pos = coef * (1.f - PS), k_neg = coef * (-1.f - PS), k_zero = coef * (-PS);
    G* go = static_cast<G*>(P.grad) + static_cast<int64_t>(row) * P.grad_ld + c0;
    for (int v = tid; v < nfull; v += kThreads) {
      const uint4 hv = d4[v], lv = t4[v];
      const uint32_t wd[8] = {hv.x, hv.y, hv.z, hv.w, lv.x, lv.y, lv.z, lv.w};
      float out[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = l1_grad(wd[i], k_pos, k_neg, k_zero);
      G* dst = go + v * 8;
      if constexpr (sizeof(G) == 2) {
        uint32_t wv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(out[2 * i], out[2 * i + 1]);
          wv[i] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        __stcs(reinterpret_cast<uint4*>(dst), make_uint4(wv[0], wv[1], wv[2], wv[3]));
      } else {
        __stcs(reinterpret_cast<float4*>(dst), make_float4(out[0], out[1], out[2], out[3]));
        __stcs(reinterpret_cast<float4*>(dst + 4), make_float4(out[4], out[5], out[6], out[7]));
      }
    }
    for (int j = nfull * 8 + tid; j < n; j += kThreads) {
      const float g = l1_grad((static_cast<uint32_t>(bd[j]) << 16) | static_cast<uint32_t>(bt[j]),
                              k_pos, k_neg, k_zero);
      if constexpr (sizeof(G) == 2)
        go[j] = static_cast<G>(__bfloat16_as_ushort(__float2bfloat16_rn(g)));
      else
        go[j] = g;
    }
  }
}

template <typename Raw, typename G>
__global__ void __launch_bounds__(kThreads) l1_kernel(L1Params P) {
  l1_pdl_launch();  // the loss kernel may be scheduled (it waits for this grid)
  constexpr int VEC = 16 / sizeof(Raw);
  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t rank = cluster.block_rank();
  const uint32_t CL = cluster.num_blocks();
  const int row = blockIdx.x / CL;
  const int tid = threadIdx.x;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Raw* bd = reinterpret_cast<Raw*>(smem_raw);
  Raw* bt = bd + P.chunk;
  L1Shared& sh = *reinterpret_cast<L1Shared*>(smem_raw + 2 * static_cast<size_t>(P.chunk) * sizeof(Raw));

  const int V = P.vocab;
  const int c0 = static_cast<int>(rank) * P.chunk;
  const int c1 = min(V, c0 + P.chunk);
  const int n = max(0, c1 - c0);
  const Raw* gd = static_cast<const Raw*>(P.draft) + static_cast<int64_t>(row) * P.ld;
  const Raw* gt = static_cast<const Raw*>(P.target) + static_cast<int64_t>(row) * P.ld;

  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    mbar_init(&sh.xbar[0], 1);
    mbar_init(&sh.xbar[1], 1);
    fence_barrier_init();
    sh.timeout = 0;
    // each exchange: the CL records of every CTA (this one included)
    mbar_arrive_expect_tx(&sh.xbar[0], CL * 2u * static_cast<uint32_t>(sizeof(Stats)));
    mbar_arrive_expect_tx(&sh.xbar[1], CL * static_cast<uint32_t>(sizeof(float2)));
  }
  cta_sync();
  // no CTA may push into a peer before the peer's mbarriers exist: the
  // initialisation is released to the cluster here and acquired below,
  // once the slice's copy is in
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const uint32_t bytes = static_cast<uint32_t>((static_cast<size_t>(n) * sizeof(Raw) + 15) & ~size_t(15));
  if (tid == 0 && bytes > 0) {
    mbar_arrive_expect_tx(&sh.bar, 2 * bytes);
    bulk_load_all(bd, gd + c0, bytes, &sh.bar);
    bulk_load_all(bt, gt + c0, bytes, &sh.bar);
  }
  if (bytes > 0 && !mbar_wait(&sh.bar, 0)) {
    atomicOr(&sh.timeout, 1u);
    mbar_wait(&sh.bar, 0);
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  cta_sync();

  if constexpr (sizeof(Raw) == 2) {
    l1_rows_bf16<G>(bd, bt, n, c0, row, rank, CL, cluster, sh, P);
  } else {
  // fp32 rows: pass 1, online statistics of both rows (base-2 units)
  Stats sd = stats_empty(), st = stats_empty();
  const int nfull = n / VEC;
  const uint4* d4 = reinterpret_cast<const uint4*>(bd);
  const uint4* t4 = reinterpret_cast<const uint4*>(bt);
  for (int v = tid; v < nfull; v += blockDim.x) {
    Raw rd[VEC], rt[VEC];
    unpack(d4[v], rd);
    unpack(t4[v], rt);
    float ud[VEC], ut[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      ud[i] = __fmul_rn(value_of(rd[i]), kLog2e);
      ut[i] = __fmul_rn(value_of(rt[i]), kLog2e);
    }
    stats_add(sd, ud);
    stats_add(st, ut);
  }
  for (int j = nfull * VEC + tid; j < n; j += blockDim.x) {
    float ud[1] = {__fmul_rn(value_of(bd[j]), kLog2e)};
    float ut[1] = {__fmul_rn(value_of(bt[j]), kLog2e)};
    stats_add(sd, ud);
    stats_add(st, ut);
  }
  sd = block_reduce(sd, sh.red);
  st = block_reduce(st, sh.red);
  exchange_stats(sh, rank, CL, sd, st);
  Stats Sd, St;
  merge_records(sh, CL, Sd, St);
  const float md = Sd.m, ld2 = stats_log2z(Sd);
  const float mt = St.m, lt2 = stats_log2z(St);

  // pass 2: L1 = sum |p - q| and sum_k p_k sign(p_k - q_k); (p, s) kept in
  // place for the gradient pass
  float l1 = 0.f, ps = 0.f;
  const bool keep = P.grad != nullptr;
  uint4* d4w = reinterpret_cast<uint4*>(bd);
  uint4* t4w = reinterpret_cast<uint4*>(bt);
  for (int v = tid; v < nfull; v += blockDim.x) {
    Raw rd[VEC], rt[VEC];
    unpack(d4[v], rd);
    unpack(t4[v], rt);
    uint32_t enc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      const float p = ex2((__fmul_rn(value_of(rd[i]), kLog2e) - md) - ld2);
      const float q = ex2((__fmul_rn(value_of(rt[i]), kLog2e) - mt) - lt2);
      const float d = p - q;
      l1 += fabsf(d);
      ps = fmaf(p, sgn(d), ps);
      enc[i] = enc_ps(p, d);
    }
    if (keep) {
      if constexpr (sizeof(Raw) == 2) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          hi[i] = (enc[2 * i] >> 16) | (enc[2 * i + 1] & 0xFFFF0000u);
          lo[i] = (enc[2 * i] & 0xFFFFu) | (enc[2 * i + 1] << 16);
        }
        d4w[v] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        t4w[v] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      } else {
        d4w[v] = make_uint4(enc[0], enc[1], enc[2], enc[3]);
      }
    }
  }
  for (int j = nfull * VEC + tid; j < n; j += blockDim.x) {
    const float p = ex2((__fmul_rn(value_of(bd[j]), kLog2e) - md) - ld2);
    const float q = ex2((__fmul_rn(value_of(bt[j]), kLog2e) - mt) - lt2);
    const float d = p - q;
    l1 += fabsf(d);
    ps = fmaf(p, sgn(d), ps);
    if (keep) {
      const uint32_t e = enc_ps(p, d);
      if constexpr (sizeof(Raw) == 2) {
        bd[j] = static_cast<Raw>(e >> 16);
        bt[j] = static_cast<Raw>(e & 0xFFFFu);
      } else {
        bd[j] = e;
      }
    }
  }
  l1 = block_sum(l1, sh.fred);
  ps = block_sum(ps, sh.fred);
  exchange_sums(sh, rank, CL, l1, ps);
  float L1 = 0.f, PS = 0.f;
  for (uint32_t r = 0; r < CL; ++r) {
    L1 += sh.agg[r].x;
    PS += sh.agg[r].y;
  }
  exit_arrive();  // every record sent to this CTA is in
  const float w = P.row_weight ? P.row_weight[row] : 1.f;
  if (rank == 0 && tid == 0) {
    if (P.l1) P.l1[row] = L1;
    if (P.accept) P.accept[row] = fminf(1.f, fmaxf(0.f, 1.f - 0.5f * L1));
    if (P.ws_wl1) P.ws_wl1[row] = static_cast<double>(w) * static_cast<double>(L1);
  }

  // pass 3: d loss / d draft_j = (w / sum w) p_j (s_j - sum_k p_k s_k)
  if (P.grad) {
    l1_pdl_wait();  // the weight-sum kernel's result
    const double wsum = *P.wsum_norm;
    const float coef = wsum > 0.0 ? static_cast<float>(static_cast<double>(w) / wsum) : 0.f;
    G* go = static_cast<G*>(P.grad) + static_cast<int64_t>(row) * P.grad_ld + c0;
    for (int v = tid; v < nfull; v += blockDim.x) {
      float out[VEC];
      if constexpr (sizeof(Raw) == 2) {
        const uint4 hv = d4[v], lv = t4[v];
        const uint32_t hi[4] = {hv.x, hv.y, hv.z, hv.w}, lo[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          out[2 * i] = dec_grad((hi[i] << 16) | (lo[i] & 0xFFFFu), coef, PS);
          out[2 * i + 1] = dec_grad((hi[i] & 0xFFFF0000u) | (lo[i] >> 16), coef, PS);
        }
      } else {
        const uint4 e = d4[v];
        const uint32_t ee[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
        for (int i = 0; i < VEC; ++i) out[i] = dec_grad(ee[i], coef, PS);
      }
      G* dst = go + v * VEC;
      if constexpr (sizeof(G) == 2) {
        uint32_t wv[VEC / 2];
#pragma unroll
        for (int i = 0; i < VEC / 2; ++i)
          wv[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(out[2 * i]))) |
                  (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(out[2 * i + 1]))) << 16);
        if constexpr (VEC == 8)
          __stcs(reinterpret_cast<uint4*>(dst), make_uint4(wv[0], wv[1], wv[2], wv[3]));
        else
          __stcs(reinterpret_cast<uint2*>(dst), make_uint2(wv[0], wv[1]));
      } else {
#pragma unroll
        for (int i = 0; i < VEC; i += 4)
          __stcs(reinterpret_cast<float4*>(dst + i), make_float4(out[i], out[i + 1], out[i + 2], out[i + 3]));
      }
    }
    for (int j = nfull * VEC + tid; j < n; j += blockDim.x) {
      uint32_t e;
      if constexpr (sizeof(Raw) == 2)
        e = (static_cast<uint32_t>(bd[j]) << 16) | static_cast<uint32_t>(bt[j]);
      else
        e = bd[j];
      const float g = dec_grad(e, coef, PS);
      if constexpr (sizeof(G) == 2)
        go[j] = static_cast<G>(__bfloat16_as_ushort(__float2bfloat16_rn(g)));
      else
        go[j] = g;
    }
  }
  }
  if (sh.timeout && tid == 0 && P.l1) P.l1[row] = __int_as_float(0x7fc00000);
  // this grid completes only after the weight-sum grid, so that the loss
  // kernel, which waits for this grid alone, also sees the weight sum
  l1_pdl_wait();
  exit_wait();
}

// sum of row weights, in row order (one block)
__global__ void l1_wsum_kernel(const float* w, int rows, double* out) {
  l1_pdl_launch();
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < rows; i += blockDim.x) s += w ? static_cast<double>(w[i]) : 1.0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[warp] = s;
  cta_sync();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += red[i];
    *out = t;
  }
}

// loss numerator / denominator / value (one block): numerator and
// denominator over this call's rows; the value divides the numerator by
// `norm` (this call's denominator, or the sum over all shards, so that the
// values of the shards add up to the loss of the whole batch)
__global__ void l1_loss_kernel(const double* wl1, const double* wsum, const double* norm, int rows,
                               float* out3) {
  l1_pdl_wait();  // the distance kernel's per-row terms
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < rows; i += blockDim.x) s += wl1[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[warp] = s;
  cta_sync();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += red[i];
    const double den = *wsum, nrm = *norm;
    out3[0] = static_cast<float>(t);
    out3[1] = static_cast<float>(den);
    out3[2] = nrm > 0.0 ? static_cast<float>(t / nrm) : 0.f;
  }
}

}  // namespace

cudaError_t launch_l1_weight_sum(int rows, const float* row_weight, double* out, cudaStream_t s) {
  l1_wsum_kernel<<<1, 1024, 0, s>>>(row_weight, rows, out);
  return cudaGetLastError();
}

size_t l1_workspace_bytes(int rows) { return 16 + 8 * static_cast<size_t>(rows > 0 ? rows : 0); }

// Cluster size and per-CTA slice for a pair of rows of `vocab` elements.
int l1_cluster_size(int vocab, vs_dtype dtype, int* chunk) {
  const int esize = dtype == VS_BF16 ? 2 : 4;
  const int target = 40 * 1024 / (2 * esize);
  int cl = 1;
  while (cl < kMaxCluster && (vocab + cl - 1) / cl > target) ++cl;
  int e = (vocab + cl - 1) / cl;
  e = (e + 31) & ~31;
  *chunk = e;
  return cl;
}

int l1_max_vocab(vs_dtype dtype) {
  const int esize = dtype == VS_BF16 ? 2 : 4;
  return kMaxCluster * (96 * 1024 / (2 * esize));
}

cudaError_t launch_l1(int rows, int vocab, int64_t ld, vs_dtype dtype, const void* draft,
                      const void* target, const float* row_weight, float* l1, float* accept,
                      float* loss3, void* grad, vs_dtype gdtype, int64_t grad_ld, void* ws,
                      const double* global_wsum, cudaStream_t s) {
  int chunk = 0;
  const int cl = l1_cluster_size(vocab, dtype, &chunk);
  L1Params P{};
  P.rows = rows;
  P.vocab = vocab;
  P.ld = ld;
  P.draft = draft;
  P.target = target;
  P.row_weight = row_weight;
  P.l1 = l1;
  P.accept = accept;
  P.grad = grad;
  P.grad_ld = grad_ld;
  P.chunk = chunk;
  const bool need_ws = loss3 != nullptr || grad != nullptr;
  P.ws_wsum = need_ws ? static_cast<double*>(ws) : nullptr;
  P.ws_wl1 = need_ws ? static_cast<double*>(ws) + 2 : nullptr;
  P.wsum_norm = global_wsum ? global_wsum : P.ws_wsum;
  if (need_ws) {
    l1_wsum_kernel<<<1, 1024, 0, s>>>(row_weight, rows, P.ws_wsum);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t esize = dtype == VS_BF16 ? 2 : 4;
  const size_t smem = 2 * static_cast<size_t>(chunk) * esize + sizeof(L1Shared);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(rows) * cl, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // early start only behind this call's own weight-sum kernel, whose
  // output the kernel waits for before using it
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = need_ws ? 2 : 1;
  cudaError_t e = cudaSuccess;
#define VS_L1_LAUNCH(RAW, G)                                                                  \
  do {                                                                                        \
    e = cudaFuncSetAttribute(l1_kernel<RAW, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(smem));                                         \
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, l1_kernel<RAW, G>, P);                 \
  } while (0)
  if (rows > 0) {
    if (dtype == VS_BF16) {
      if (gdtype == VS_BF16) VS_L1_LAUNCH(uint16_t, uint16_t);
      else VS_L1_LAUNCH(uint16_t, float);
    } else {
      if (gdtype == VS_BF16) VS_L1_LAUNCH(uint32_t, uint16_t);
      else VS_L1_LAUNCH(uint32_t, float);
    }
  }
#undef VS_L1_LAUNCH
  if (e != cudaSuccess) return e;
  if (loss3) {
    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3(1);
    lc.blockDim = dim3(1024);
    lc.stream = s;
    cudaLaunchAttribute la[1];
    la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = la;
    lc.numAttrs = rows > 0 ? 1 : 0;  // behind this call's distance kernel only
    e = cudaLaunchKernelEx(&lc, l1_loss_kernel, static_cast<const double*>(P.ws_wl1),
                           static_cast<const double*>(P.ws_wsum), P.wsum_norm, rows, loss3);
  }
  return e;
}

}  // namespace vs

// ---------------------------------------------------------------------------
// Allocation-free variant of vs_l1_distance: the scratch (weight sum and the
// per-row weighted distances) lives in a file-scope device array instead of a
// caller workspace.

namespace vs {
vs_status set_last_error(vs_status code, const char* msg);
}  // namespace vs

namespace {

static_assert(VS_L1_STATIC_SCRATCH_BYTES >= 16 + 8 * VS_L1_STATIC_MAX_ROWS, "scratch size");

// One copy per GPU that loads the library, alive until the process exits.
static __device__ __align__(256) unsigned char g_l1_scratch[VS_L1_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_l1_scratch on the current device, looked up once per
// device (host code sees only a stand-in for the symbol, never its address).
vs_status scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return vs::set_last_error(VS_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return vs::set_last_error(VS_ERR_UNSUPPORTED, "device ordinal beyond the scratch table");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_l1_scratch);
    if (e != cudaSuccess || !p)
      return vs::set_last_error(VS_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                              : "scratch address is NULL");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return VS_OK;
}

}  // namespace

extern "C" vs_status vs_l1_distance_static(int32_t rows, int32_t vocab, int64_t ld,
                                           vs_dtype dtype, const void* draft, const void* target,
                                           const float* row_weight, float* l1,
                                           float* accept_rate, float* loss_num_den_loss,
                                           void* grad_draft, vs_dtype grad_dtype, int64_t grad_ld,
                                           void* stream) {
  if (rows > VS_L1_STATIC_MAX_ROWS)
    return vs::set_last_error(VS_ERR_UNSUPPORTED,
                              "rows exceed VS_L1_STATIC_MAX_ROWS: use vs_l1_distance with a workspace");
  void* scratch = nullptr;
  const vs_status st = scratch_for_current_device(&scratch);
  if (st != VS_OK) return st;
  return vs_l1_distance(rows, vocab, ld, dtype, draft, target, row_weight, l1, accept_rate,
                        loss_num_den_loss, grad_draft, grad_dtype, grad_ld, scratch,
                        VS_L1_STATIC_SCRATCH_BYTES, stream);
}
