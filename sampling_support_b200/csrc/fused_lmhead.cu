// Fused LM-head scoring (xorl issue #71, section 1: chunked projection ->
// fixed-order LSE -> support -> selected logprob; SkyRL PR #2004,
// "Performance": the full-vocabulary logits are never materialised).
//
//   z[i, v] = (sum_k H[i, k] W[v, k]) / T_i
//
// Kernel 1 (lmhead_gemm_kernel), persistent and warp-specialised, one CTA per
// SM.  Work units are (row unit, vocabulary split) pairs; a unit walks its
// split in 256-column tiles.  In pair mode two CTAs of a cluster share each
// tile as one 256 x 256 tcgen05 MMA (cta_group::2): each loads its 128 rows
// of H and its 128 of the tile's 256 W rows, the first CTA issues the MMAs
// for both, and each receives its 128 rows of the accumulator, so a CTA
// moves two thirds of the operand bytes of a single-CTA 128 x 256 tile:
//   warp 0   TMA producer: 128x64 tiles of H and 256x64 tiles of W into a
//            ring of shared-memory stages (128-byte swizzle, mbarriers);
//   warp 1   MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//            M = 128, N = 256, K = 16 per instruction, accumulating each tile
//            in one of two TMEM buffers (256 columns each);
//   warps 2-5 epilogue: one thread per row reads its 256 accumulators with
//            tcgen05.ld, releases the buffer, and folds the values into the
//            row's online (max, count of max, sum 2^(u - max), sum (u - max)
//            2^(u - max)) and into an unsorted top-k list in shared memory
//            (per 32-column chunk each lane marks its candidates against the
//            list's threshold and inserts them itself, so the lanes of a warp
//            insert side by side).  At the end of a unit the row's partials
//            go to the workspace, the list sorted by rank.
// Kernel 2 (lmhead_merge_kernel), one thread per row: merges the split
// partials in a fixed order, takes the top-k, applies inclusive top-p on the
// top-k mass and min-p against the row max, and writes the outputs.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cublasLt.h>

#include <climits>
#include <cmath>
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace vs {

namespace {

constexpr int kBM = 128;  // rows per tile (TMEM lanes)
constexpr int kBN = 256;  // vocabulary columns per tile
constexpr int kBK = 64;   // hidden elements per stage (128 bytes of bf16)
constexpr int kUK = 16;   // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;
constexpr int kStageABytes = kBM * kBK * 2;  // 16 KB
constexpr int kStageBBytes = kBN * kBK * 2;  // 32 KB
constexpr int kStageBytes = kStageABytes + kStageBBytes;
constexpr uint32_t kTmemCols = 2 * kBN;  // two accumulators
constexpr int kMaxStages = 6;

// Pair mode (tcgen05 cta_group::2): a cluster of two CTAs computes a
// 256 x 256 tile; each CTA holds its 128 rows of the H tile and 128 of the
// 256 W rows, and receives its 128 rows x 256 columns of the accumulator.
constexpr int kBNh = kBN / 2;                     // W rows per CTA of a pair
constexpr int kStageBytes2 = kStageABytes + kBNh * kBK * 2;  // 32 KB
// kind::f16 descriptor for M = 256 (the pair), N = 256
constexpr uint32_t kIDesc2 = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                             (uint32_t(256 >> 4) << 24);

// UMMA instruction descriptor, kind::f16: D fp32, A and B bf16, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIDesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                            (uint32_t(kBM >> 4) << 24);

struct LmParams {
  int32_t rows, vocab, hidden;
  int32_t m_units;      // row units: 128-row blocks, or 256-row block pairs in pair mode
  int32_t top_k;
  int32_t splits;       // vocabulary splits
  int32_t tiles_per_split;
  int32_t n_tiles;      // ceil(vocab / kBN)
  int32_t m_blocks;     // ceil(rows / kBM)
  int32_t stages;
  const float* temperature;
  float temperature_scalar;
  const int32_t* targets;
  float4* ws_stats;  // [rows, splits] (m, c0, zr, a) in base-2 units of z log2(e)
  float* ws_val;     // [rows, splits, top_k] accumulator values (desc)
  int32_t* ws_id;    // [rows, splits, top_k]
  float* ws_zy;      // [rows] accumulator at the target id
  uint32_t* ws_err;  // [1] bounded-wait timeouts
  int32_t col_offset;  // vocabulary id of weight row 0 (a shard of a vocabulary-parallel head)
  // backward (kModeDz): per-row (c, log-sum-exp in base-2 units, alpha, beta)
  // of the dense logit gradient p (alpha + beta x), c == 0 for a row with no
  // gradient; the bf16 gradient tile goes to dz [rows, dz_ld]
  const float4* rowc;
  uint16_t* dz;
  int64_t dz_ld;
};

// Epilogues of the GEMM kernel.
enum : int {
  kModeScore = 0,  // forward: online statistics and top-k candidates
  kModeDz = 1,     // backward: the dense part of d loss / d (H W^T), bf16
};

// ---------------------------------------------------------------------------
// PTX wrappers (tcgen05, TMA tensor loads)

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
  // start address >> 4 | LBO 1 (16 B) | SBO 64 (1024 B = 8 rows of 128 B) |
  // version 1 | layout SWIZZLE_128B
  const uint64_t a = (smem_addr(p) >> 4) & 0x3FFFu;
  return a | (uint64_t(1) << 16) | (uint64_t(64) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIDesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Pair-mode tensor load: lands in this CTA's shared memory and completes its
// bytes on the leader CTA's barrier at the same offset (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int c0, int c1,
                                                 uint64_t* bar) {
  asm volatile(
      "{\n .reg .b32 lb;\n mapa.shared::cluster.u32 lb, %4, 0;\n"
      " cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [lb];\n}\n" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIDesc2), "r"(accumulate)
      : "memory");
}

// Completion of the pair's MMAs arrives on the barrier at this offset in
// both CTAs of the pair.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// Arrive on the leader CTA's barrier at this offset.
__device__ __forceinline__ void mbar_arrive_leader(uint64_t* bar) {
  asm volatile(
      "{\n .reg .b32 ra;\n mapa.shared::cluster.u32 ra, %0, 0;\n"
      " mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n}\n" ::"r"(smem_addr(bar))
      : "memory");
}

// Bounded wait for a barrier phase whose arrivals come from the peer CTA
// (acquire at cluster scope); false after the iteration cap.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// shared-memory layout of the GEMM kernel (after 1024-byte alignment):
//   [stages x (A 16 KB | B 32 KB)] [top-k values 128 x k] [top-k ids 128 x k]
//   [barriers] [tmem slot]

struct Barriers {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  uint32_t abort;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Barriers* bs,
                                              uint32_t* err) {
  if (mbar_wait(bar, parity)) return true;
  atomicOr(&bs->abort, 1u);
  atomicOr(err, 1u);
  return false;
}

// A row's running top-k is an unsorted list of up to k (value, id) entries.
// Within a work unit ids arrive in ascending order, so a new element ranks
// below every listed entry of equal value: once the list is full it is taken
// only when it exceeds `thr`, the smallest listed value, and it replaces the
// lowest-ranked entry (smallest value, then largest id) at `low`.
__device__ __forceinline__ void topk_push(float* vals, int32_t* ids, int k, int& count, int& low,
                                          float& thr, float x, int32_t id) {
  const int slot = count < k ? count++ : low;
  vals[slot] = x;
  ids[slot] = id;
  if (count == k) {
    float mv = vals[0];
    int32_t mi = ids[0];
    int mp = 0;
    for (int j = 1; j < k; ++j) {
      const float vj = vals[j];
      const int32_t ij = ids[j];
      if (vj < mv || (vj == mv && ij > mi)) {
        mv = vj;
        mi = ij;
        mp = j;
      }
    }
    low = mp;
    thr = mv;
  }
}

// v[i] for a per-lane index i, by a five-level select tree on the bits of i
// (static register indices only, so v stays in registers).
__device__ __forceinline__ float pick32(const float (&v)[32], int i) {
  float a[16], b[8], c[4];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = (i & 1) ? v[2 * j + 1] : v[2 * j];
#pragma unroll
  for (int j = 0; j < 8; ++j) b[j] = (i & 2) ? a[2 * j + 1] : a[2 * j];
#pragma unroll
  for (int j = 0; j < 4; ++j) c[j] = (i & 4) ? b[2 * j + 1] : b[2 * j];
  const float d0 = (i & 8) ? c[1] : c[0];
  const float d1 = (i & 8) ? c[3] : c[2];
  return (i & 16) ? d1 : d0;
}

// Work unit u -> (row unit mu, vocabulary split sp).  Units go in groups of
// at most kUnitGroup row units: a group's units of every split come before
// the next group's, so the units running at the same time share a few
// vocabulary splits (their weight tiles are read once from DRAM and then
// from L2) and at most kUnitGroup row blocks of the hidden states (which
// stay in L2 while the group sweeps the vocabulary).
constexpr int kUnitGroup = 16;

__device__ __forceinline__ void unit_coords(int u, const LmParams& P, int& mu, int& sp) {
  const int gsz = P.m_units < kUnitGroup ? P.m_units : kUnitGroup;
  const int per_group = gsz * P.splits;
  const int g = u / per_group;
  const int r = u - g * per_group;
  const int g0 = g * gsz;
  const int gn = P.m_units - g0 < gsz ? P.m_units - g0 : gsz;  // the last group may be smaller
  mu = g0 + r % gn;
  sp = r / gn;
}

template <bool PAIR, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    lmhead_gemm_kernel(const __grid_constant__ CUtensorMap map_h,
                       const __grid_constant__ CUtensorMap map_w, LmParams P) {
  constexpr int SB = PAIR ? kStageBytes2 : kStageBytes;  // bytes per stage in this CTA
  constexpr int SA = kStageABytes;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~uintptr_t(1023));
  const int S = P.stages;
  uint8_t* stage0 = base;
  float* tk_val = reinterpret_cast<float*>(base + S * SB);
  int32_t* tk_id = reinterpret_cast<int32_t*>(tk_val + kBM * P.top_k);
  Barriers* bs = reinterpret_cast<Barriers*>(
      (reinterpret_cast<uintptr_t>(tk_id + kBM * P.top_k) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = P.m_units * P.splits;
  const int nkb = P.hidden / kBK;
  // work-unit walk: CTAs (or CTA pairs) stride over (row unit, split)
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int u_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int u_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bs->full[s], 1);
      mbar_init(&bs->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bs->tfull[b], 1);
      mbar_init(&bs->tempty[b], PAIR ? 2 * kBM : kBM);  // both CTAs' epilogues in pair mode
    }
    bs->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    // allocate the two accumulators (512 TMEM columns) for this CTA (both
    // CTAs of a pair, same warp, same slot)
    if constexpr (PAIR) {
      asm volatile(
          "tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
              smem_addr(&bs->tmem_base)),
          "r"(kTmemCols)
          : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile(
          "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
              smem_addr(&bs->tmem_base)),
          "r"(kTmemCols)
          : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  cta_sync();
  if constexpr (PAIR) cluster_barrier();  // the peer's barriers are initialised
  tc_fence_after();
  const uint32_t tmem = bs->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_h)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int u = u_first; u < units && ok; u += u_step) {
        int mu, sp;
        unit_coords(u, P, mu, sp);
        const int mb = PAIR ? 2 * mu + static_cast<int>(rank) : mu;
        const int t0 = sp * P.tiles_per_split, t1 = min(P.n_tiles, t0 + P.tiles_per_split);
        for (int t = t0; t < t1 && ok; ++t) {
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % S;
            const uint32_t wrap = it / S;
            if (!wait_or_abort(&bs->empty[s], (wrap & 1u) ^ 1u, bs, P.ws_err)) {
              ok = false;
              break;
            }
            uint8_t* sa = stage0 + s * SB;
            if constexpr (PAIR) {
              // the leader's barrier counts both CTAs' bytes
              if (leader) mbar_arrive_expect_tx(&bs->full[s], 2 * SB);
              tma_load_2d_pair(sa, &map_h, kb * kBK, mb * kBM, &bs->full[s]);
              tma_load_2d_pair(sa + SA, &map_w, kb * kBK, t * kBN + static_cast<int>(rank) * kBNh,
                               &bs->full[s]);
            } else {
              mbar_arrive_expect_tx(&bs->full[s], SB);
              tma_load_2d(sa, &map_h, kb * kBK, mb * kBM, &bs->full[s]);
              tma_load_2d(sa + SA, &map_w, kb * kBK, t * kBN, &bs->full[s]);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // (pair mode: the leader CTA issues for both)
    if (lane == 0 && leader) {
      uint32_t it = 0, tile = 0;
      bool ok = true;
      for (int u = u_first; u < units && ok; u += u_step) {
        int mu, sp;
        unit_coords(u, P, mu, sp);
        const int t0 = sp * P.tiles_per_split, t1 = min(P.n_tiles, t0 + P.tiles_per_split);
        for (int t = t0; t < t1 && ok; ++t, ++tile) {
          const int b = tile & 1;
          const uint32_t use = tile >> 1;
          const bool freed = PAIR ? mbar_wait_cluster(&bs->tempty[b], (use & 1u) ^ 1u)
                                  : wait_or_abort(&bs->tempty[b], (use & 1u) ^ 1u, bs, P.ws_err);
          if (!freed) {
            atomicOr(&bs->abort, 1u);
            atomicOr(P.ws_err, 1u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dacc = tmem + b * kBN;
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % S;
            const uint32_t wrap = it / S;
            if (!wait_or_abort(&bs->full[s], wrap & 1u, bs, P.ws_err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* sa = stage0 + s * SB;
            const uint64_t ad = smem_desc_sw128(sa);
            const uint64_t bd = smem_desc_sw128(sa + SA);
#pragma unroll
            for (int kk = 0; kk < kBK / kUK; ++kk) {
              // advance 16 elements (32 bytes) along K inside the swizzle atom
              if constexpr (PAIR)
                umma_f16_pair(dacc, ad + 2 * kk, bd + 2 * kk, (kb | kk) ? 1u : 0u);
              else
                umma_f16(dacc, ad + 2 * kk, bd + 2 * kk, (kb | kk) ? 1u : 0u);
            }
            // frees the stage (in both CTAs of a pair) once these MMAs finish
            if constexpr (PAIR)
              umma_commit_pair(&bs->empty[s]);
            else
              umma_commit(&bs->empty[s]);
          }
          if (ok) {  // accumulator b complete
            if constexpr (PAIR)
              umma_commit_pair(&bs->tfull[b]);
            else
              umma_commit(&bs->tfull[b]);
          }
        }
      }
    }
  } else if constexpr (MODE == kModeDz) {
    // ------------------------------------------------------------ epilogue (backward)
    // d loss / d x for each accumulator x of the row: the dense part
    // p (alpha + beta x), p = 2^(x c - lse); the support and target entries
    // are rewritten afterwards by the fix-up kernel
    const int q = warp & 3;
    const int r = q * 32 + lane;
    uint32_t tile = 0;
    bool ok = true;
    for (int u = u_first; u < units && ok; u += u_step) {
      int mu, sp;
      unit_coords(u, P, mu, sp);
      const int mb = PAIR ? 2 * mu + static_cast<int>(rank) : mu;
      const int t0 = sp * P.tiles_per_split, t1 = min(P.n_tiles, t0 + P.tiles_per_split);
      const int row = mb * kBM + r;
      const bool row_ok = row < P.rows;
      const float4 rc = row_ok ? P.rowc[row] : make_float4(0.f, 0.f, 0.f, 0.f);
      uint16_t* drow = P.dz + static_cast<int64_t>(row_ok ? row : 0) * P.dz_ld;
      for (int t = t0; t < t1 && ok; ++t, ++tile) {
        const int b = tile & 1;
        const uint32_t use = tile >> 1;
        if (!wait_or_abort(&bs->tfull[b], use & 1u, bs, P.ws_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + b * kBN;
        for (int ch = 0; ch < kBN / 32; ++ch) {
          float v[32];
          tmem_ld32(taddr + ch * 32, v);
          if (ch == kBN / 32 - 1) {
            tc_fence_before();
            if constexpr (PAIR)
              mbar_arrive_leader(&bs->tempty[b]);
            else
              mbar_arrive(&bs->tempty[b]);
          }
          const int col0 = t * kBN + ch * 32;
          if (!row_ok || col0 >= P.vocab) continue;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float g0 = 0.f, g1 = 0.f;
            if (rc.x != 0.f) {
              g0 = ex2(fmaf(v[2 * i], rc.x, -rc.y)) * fmaf(rc.w, v[2 * i], rc.z);
              g1 = ex2(fmaf(v[2 * i + 1], rc.x, -rc.y)) * fmaf(rc.w, v[2 * i + 1], rc.z);
            }
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(g0, g1);
            pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          uint16_t* dst = drow + col0;
          if (col0 + 32 <= P.vocab) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (col0 + 2 * i < P.vocab) dst[2 * i] = static_cast<uint16_t>(pk[i] & 0xFFFFu);
              if (col0 + 2 * i + 1 < P.vocab) dst[2 * i + 1] = static_cast<uint16_t>(pk[i] >> 16);
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const int k = P.top_k;
    float* my_val = tk_val + r * k;
    int32_t* my_id = tk_id + r * k;
    uint32_t tile = 0;
    bool ok = true;
    for (int u = u_first; u < units && ok; u += u_step) {
      int mu, sp;
      unit_coords(u, P, mu, sp);
      const int mb = PAIR ? 2 * mu + static_cast<int>(rank) : mu;
      const int t0 = sp * P.tiles_per_split, t1 = min(P.n_tiles, t0 + P.tiles_per_split);
      const int row = mb * kBM + r;
      const bool row_ok = row < P.rows;
      const float T = row_ok ? (P.temperature ? P.temperature[row] : P.temperature_scalar) : 1.f;
      const float c = kLog2e / T;
      // the target as a column of this weight (outside [0, vocab): not here)
      const int y = row_ok ? P.targets[row] - P.col_offset : -1;
      const bool y_here = y >= 0 && y < P.vocab;
      Stats st = stats_empty();
      int count = 0, low = 0;
      float thr = -kInf;  // smallest listed value once the list is full
      for (int t = t0; t < t1 && ok; ++t, ++tile) {
        const int b = tile & 1;
        const uint32_t use = tile >> 1;
        if (!wait_or_abort(&bs->tfull[b], use & 1u, bs, P.ws_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + b * kBN;
        for (int ch = 0; ch < kBN / 32; ++ch) {
          float v[32];
          tmem_ld32(taddr + ch * 32, v);
          if (ch == kBN / 32 - 1) {
            // every column of this buffer has been read: hand it back (to
            // the leader, which issues the pair's MMAs)
            tc_fence_before();
            if constexpr (PAIR)
              mbar_arrive_leader(&bs->tempty[b]);
            else
              mbar_arrive(&bs->tempty[b]);
          }
          const int col0 = t * kBN + ch * 32;
          if (!row_ok) continue;
          // top-k candidates of this chunk against the threshold at its
          // start (a stale threshold only admits extra candidates, which the
          // exact test below drops); each lane walks its own candidates in
          // ascending column order, so the warp's lanes insert side by side
          uint32_t cand = 0;
          if (col0 + 32 <= P.vocab) {
            float uu[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) uu[i] = __fmul_rn(v[i], c);
            stats_add(st, uu);
#pragma unroll
            for (int i = 0; i < 32; ++i) cand |= (v[i] > thr ? 1u : 0u) << i;
          } else {
            for (int i = 0; i < 32 && col0 + i < P.vocab; ++i) {
              float uu[1] = {__fmul_rn(pick32(v, i), c)};
              stats_add(st, uu);
            }
            const int nv = P.vocab - col0;
#pragma unroll
            for (int i = 0; i < 32; ++i) cand |= (i < nv && v[i] > thr ? 1u : 0u) << i;
          }
          if (y_here && y >= col0 && y < col0 + 32) P.ws_zy[row] = pick32(v, y - col0);
          while (cand != 0u) {
            const int i = __ffs(cand) - 1;
            cand &= cand - 1u;
            const float x = pick32(v, i);
            if (x > thr) topk_push(my_val, my_id, k, count, low, thr, x, col0 + i + P.col_offset);
          }
        }
      }
      if (row_ok) {
        const int64_t slot = static_cast<int64_t>(row) * P.splits + sp;
        P.ws_stats[slot] = make_float4(st.m, st.c0, st.zr, st.a);
        float* dv = P.ws_val + slot * k;
        int32_t* di = P.ws_id + slot * k;
        // the split's list in the total order (value desc, id asc): each
        // entry goes to its rank (ids are distinct, so ranks are too)
        for (int j = 0; j < count; ++j) {
          const float vj = my_val[j];
          const int32_t ij = my_id[j];
          int rk = 0;
          for (int l = 0; l < count; ++l) {
            const float vl = my_val[l];
            rk += (vl > vj || (vl == vj && my_id[l] < ij)) ? 1 : 0;
          }
          dv[rk] = vj;
          di[rk] = ij;
        }
        for (int j = count; j < k; ++j) {
          dv[j] = -kInf;
          di[j] = -1;
        }
      }
    }
  }

  // teardown: every role has left its loop (bounded waits); make sure the
  // MMAs of this CTA have completed before the accumulators are freed
  tc_fence_before();
  cta_sync();
  if constexpr (PAIR) cluster_barrier();  // the pair's MMAs and arrivals are done
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
  }
}

// ---------------------------------------------------------------------------
// merge: one thread per row

// Saved per-row state of the fused head for its backward
// (VS_CTX_BYTES_PER_ROW bytes), base-2 units u = x c, x = (H W^T)[i, v]:
struct alignas(16) LmCtx {
  float m;       // max_v u
  float log2z;   // log2 sum_v 2^(u - m)
  float ms;      // support sums reference (u of the top-1)
  float log2zs;  // log2 sum_{v in S} 2^(u - ms)
  float h_full, h_support;  // nat
  float c;       // log2(e) / T
  int32_t n;     // |S| (S = the first n top-k ids)
  uint32_t flags;  // kLmCtx*
  uint32_t pad[7];
};
static_assert(sizeof(LmCtx) == VS_CTX_BYTES_PER_ROW, "fused-head ctx layout");
enum : uint32_t {
  kLmCtxNonFinite = 1u << 0,
  kLmCtxTargetOk = 1u << 1,
  kLmCtxTargetInS = 1u << 2,
};

// Inputs of the merge: `splits` partial records per row, at element strides
// (row, split) for the statistics and the lists, the target logit as the sum
// over `parts` entries (one part holds it, the others hold 0) and the
// timeout flags ORed over `parts` entries.
struct MergeParams {
  int32_t rows, vocab, splits, top_k;
  float top_p, min_p;
  const float* temperature;
  float temperature_scalar;
  const int32_t* targets;
  const float4* ws_stats;
  const float* ws_val;
  const int32_t* ws_id;
  const float* ws_zy;
  const uint32_t* ws_err;
  int64_t st_row, st_split;  // float4 elements
  int64_t ls_row, ls_split;  // list elements
  int32_t parts;
  int64_t zy_part, err_part;  // elements
  // partial output (one shard of a vocabulary-parallel head): the merged
  // statistics, top-k list, target logit and flag of this shard's splits
  // are written here and nothing is finalised
  float4* out_stats;
  float* out_val;
  int32_t* out_id;
  float* out_zy;
  uint32_t* out_err;
  float* lp_full;
  float* lp_support;
  float* h_full;
  float* h_support;
  uint8_t* valid;
  uint32_t* status;
  int32_t* support_size;
  int32_t* topk_ids;
  float* topk_logprob;
  LmCtx* ctx;
  int32_t want_entropy;
};

constexpr int kMaxSplits = 64;
constexpr int kMergeAhead = 4;  // list entries per split loaded before the merge rounds

// One warp per row.  Lane l owns splits l and l + 32: their statistics are
// merged by a fixed shuffle tree, and their sorted lists by k rounds of a
// warp-wide argmax over the lanes' list heads.  Each lane loads the first
// kMergeAhead entries of its two lists up front (all lanes' loads in flight
// at once), so that a round rarely waits for memory: only a list that gives
// more than kMergeAhead entries to the top-k reads its next head from global
// memory.  Entry i of the merged top-k lives in lane i % 32, slot i / 32.
__global__ void __launch_bounds__(128) lmhead_merge_kernel(MergeParams P) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= P.rows) return;  // whole warps leave together
  const int k = P.top_k;
  const int64_t lbase = row * P.ls_row;
  // the first kMergeAhead entries of this lane's two lists
  float av[2][kMergeAhead];
  int32_t ai[2][kMergeAhead];
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    const int sp = lane + 32 * sl;
#pragma unroll
    for (int d = 0; d < kMergeAhead; ++d) {
      const bool ok = sp < P.splits && d < k;
      av[sl][d] = ok ? P.ws_val[lbase + sp * P.ls_split + d] : -kInf;
      ai[sl][d] = ok ? P.ws_id[lbase + sp * P.ls_split + d] : -1;
    }
  }
  const float T = P.temperature ? P.temperature[row] : P.temperature_scalar;
  const float c = kLog2e / T;
  const float nan = __int_as_float(0x7fc00000);
  // statistics over the full vocabulary
  Stats st = stats_empty();
  for (int sp = lane; sp < P.splits; sp += 32) {
    const float4 v = P.ws_stats[row * P.st_row + sp * P.st_split];
    stats_merge(st, Stats{v.x, v.y, v.z, v.w});
  }
  {
    float m = st.m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (st.c0 != 0.f || st.zr != 0.f) stats_rebase(st, m);
    float c0 = st.c0, zr = st.zr, a = st.a;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c0 += __shfl_xor_sync(0xffffffffu, c0, o);
      zr += __shfl_xor_sync(0xffffffffu, zr, o);
      a += __shfl_xor_sync(0xffffffffu, a, o);
    }
    st = Stats{m, c0, zr, a};
  }
  uint32_t errs = 0;
  for (int q = 0; q < P.parts; ++q) errs |= P.ws_err[q * P.err_part];
  const bool timeout = errs != 0;
  const bool nonfinite = !stats_finite(st);
  const float log2z = stats_log2z(st);
  const float h_full = kLn2 * (log2z - st.a / stats_z(st));
  // top-k by (value desc, id asc): k-way merge of the sorted split lists
  int cur0 = 0, cur1 = 0;
  const bool has0 = lane < P.splits, has1 = lane + 32 < P.splits;
  auto head = [&](int sp, int cur, float& v, int32_t& id) {
    v = -kInf;
    id = -1;
    if (cur < k) {
      const int sl = sp >= 32 ? 1 : 0;
      if (cur < kMergeAhead) {
#pragma unroll
        for (int d = 0; d < kMergeAhead; ++d)
          if (d == cur) {
            v = sl ? av[1][d] : av[0][d];
            id = sl ? ai[1][d] : ai[0][d];
          }
      } else {
        v = P.ws_val[lbase + sp * P.ls_split + cur];
        id = P.ws_id[lbase + sp * P.ls_split + cur];
      }
    }
  };
  float h0v = -kInf, h1v = -kInf;
  int32_t h0i = -1, h1i = -1;
  if (has0) head(lane, 0, h0v, h0i);
  if (has1) head(lane + 32, 0, h1v, h1i);
  // each head as one 64-bit key ordered as (value desc, id asc): the value's
  // bits made monotone (-0 as +0, NaN below every number), then the id
  // complemented; an exhausted list is 0
  auto mkkey = [](float v, int32_t id) -> unsigned long long {
    if (id < 0) return 0ull;
    uint32_t b = __float_as_uint(v);
    if ((b & 0x7FFFFFFFu) == 0u) b = 0u;
    uint32_t mono = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    if (v != v) mono = 0u;
    return (static_cast<unsigned long long>(mono) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(id));
  };
  unsigned long long k0 = mkkey(h0v, h0i), k1 = mkkey(h1v, h1i);
  float tv[2] = {-kInf, -kInf};
  int32_t ti[2] = {-1, -1};
  for (int i = 0; i < k; ++i) {
    // the warp's largest 64-bit key: the largest high word (redux.sync),
    // then the largest low word among the lanes holding it
    unsigned long long best = k0 > k1 ? k0 : k1;
    {
      const uint32_t bh = static_cast<uint32_t>(best >> 32), bl = static_cast<uint32_t>(best);
      const uint32_t mh = __reduce_max_sync(0xffffffffu, bh);
      const uint32_t ml = __reduce_max_sync(0xffffffffu, bh == mh ? bl : 0u);
      best = (static_cast<unsigned long long>(mh) << 32) | ml;
    }
    if (lane == (i & 31)) {
      float bv = -kInf;
      int32_t bi = -1;
      if (best != 0ull) {
        const uint32_t mono = static_cast<uint32_t>(best >> 32);
        bv = __uint_as_float((mono & 0x80000000u) ? (mono & 0x7FFFFFFFu) : ~mono);
        bi = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(best));
      }
      if (i < 32) {
        tv[0] = bv;
        ti[0] = bi;
      } else {
        tv[1] = bv;
        ti[1] = bi;
      }
    }
    if (best != 0ull) {
      // the owner of the winning head (ids are unique in a row) advances
      if (k0 == best) {
        ++cur0;
        head(lane, cur0, h0v, h0i);
        k0 = mkkey(h0v, h0i);
      } else if (k1 == best) {
        ++cur1;
        head(lane + 32, cur1, h1v, h1i);
        k1 = mkkey(h1v, h1i);
      }
    }
  }
  float zy = 0.f;
  for (int q = 0; q < P.parts; ++q) zy += P.ws_zy[q * P.zy_part + row];
  if (P.out_stats) {
    // one shard of a vocabulary-parallel head: hand on the merged record
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const int i = sl * 32 + lane;
      if (i < k) {
        P.out_val[static_cast<int64_t>(row) * k + i] = tv[sl];
        P.out_id[static_cast<int64_t>(row) * k + i] = ti[sl];
      }
    }
    if (lane == 0) {
      P.out_stats[row] = make_float4(st.m, st.c0, st.zr, st.a);
      P.out_zy[row] = zy;
      if (timeout) atomicOr(P.out_err, 1u);
    }
    return;
  }
  // support: inclusive top-p on the top-k mass (fp64 prefix sums in rank
  // order), then min-p against the row max
  double e[2], pre[2];
  bool live[2];
#pragma unroll
  for (int sl = 0; sl < 2; ++sl) {
    const int i = sl * 32 + lane;
    live[sl] = i < k && ti[sl] >= 0;
    e[sl] = live[sl] ? static_cast<double>(ex2(__fmul_rn(tv[sl], c) - st.m)) : 0.0;
    double x = e[sl];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    pre[sl] = x;
  }
  const double tot0 = __shfl_sync(0xffffffffu, pre[0], 31);
  pre[1] += tot0;
  const double mass1 = __shfl_sync(0xffffffffu, pre[1], 31);
  const uint32_t lv0 = __ballot_sync(0xffffffffu, live[0]), lv1 = __ballot_sync(0xffffffffu, live[1]);
  const int nlive = __popc(lv0) + __popc(lv1);  // live entries form a prefix
  int n = nlive;
  if (P.top_p < 1.f) {
    const double tgt = static_cast<double>(P.top_p) * mass1;
    const uint32_t r0 = __ballot_sync(0xffffffffu, live[0] && pre[0] >= tgt);
    const uint32_t r1 = __ballot_sync(0xffffffffu, live[1] && pre[1] >= tgt);
    if (r0)
      n = __ffs(r0);
    else if (r1)
      n = 32 + __ffs(r1);
  }
  if (P.min_p > 0.f) {
    const uint32_t q0 = __ballot_sync(0xffffffffu, live[0] && lane < n &&
                                                      static_cast<float>(e[0]) >= P.min_p);
    const uint32_t q1 = __ballot_sync(0xffffffffu, live[1] && 32 + lane < n &&
                                                      static_cast<float>(e[1]) >= P.min_p);
    n = __popc(q0) + __popc(q1);  // the ratio falls along the order: a prefix
  }
  // support statistics relative to its maximum, the top-1 value
  const float ms = __shfl_sync(0xffffffffu, __fmul_rn(tv[0], c), 0);
  Stats ss = stats_empty();
  if (n > 0) {
    float c0 = 0.f, zr = 0.f, a = 0.f;
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      if (sl * 32 + lane < n) {
        const float d = __fmul_rn(tv[sl], c) - ms;
        const float ev = ex2(d);
        if (d == 0.f)
          c0 += 1.f;
        else
          zr += ev;
        a = fmaf(d, ev, a);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c0 += __shfl_xor_sync(0xffffffffu, c0, o);
      zr += __shfl_xor_sync(0xffffffffu, zr, o);
      a += __shfl_xor_sync(0xffffffffu, a, o);
    }
    ss = Stats{ms, c0, zr, a};
  }
  const float log2zs = n > 0 ? stats_log2z(ss) : nan;
  const float h_sup = n > 0 ? kLn2 * (log2zs - ss.a / stats_z(ss)) : 0.f;
  const int y = P.targets[row];
  const bool in_s = __ballot_sync(0xffffffffu, (lane < n && ti[0] == y) ||
                                                   (32 + lane < n && ti[1] == y)) != 0u;
  // the writes: per-row values by lane 0, the top-k entries by their lanes
  if (P.topk_ids || P.topk_logprob) {
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
      const int i = sl * 32 + lane;
      if (i >= k) continue;
      if (P.topk_ids) P.topk_ids[static_cast<int64_t>(row) * k + i] = ti[sl];
      if (P.topk_logprob)
        P.topk_logprob[static_cast<int64_t>(row) * k + i] =
            (ti[sl] >= 0 && !nonfinite) ? kLn2 * (__fmul_rn(tv[sl], c) - st.m - log2z) : nan;
    }
  }
  if (lane != 0) return;
  uint32_t status = 0;
  float lp_v = nan, lp_s = nan;
  if (y < 0 || y >= P.vocab) status |= VS_ROW_TARGET_OUT_OF_RANGE;
  if (nonfinite) {
    status |= VS_ROW_NONFINITE_INPUT;
  } else if (!(status & VS_ROW_TARGET_OUT_OF_RANGE)) {
    const float uy = __fmul_rn(zy, c);
    lp_v = kLn2 * (uy - st.m - log2z);
    if (in_s) {
      lp_s = kLn2 * (uy - ss.m - log2zs);
    } else {
      lp_s = -kInf;
      status |= VS_ROW_TARGET_NOT_IN_SUPPORT;
    }
  }
  if (timeout) status |= kRowDeviceTimeout;
  if (P.lp_full) P.lp_full[row] = lp_v;
  if (P.lp_support) P.lp_support[row] = lp_s;
  if (P.want_entropy) {
    if (P.h_full) P.h_full[row] = nonfinite ? nan : h_full;
    if (P.h_support) P.h_support[row] = nonfinite ? nan : h_sup;
  }
  if (P.valid) P.valid[row] = (!nonfinite && n > 0) ? 1 : 0;
  if (P.status) P.status[row] = status;
  if (P.support_size) P.support_size[row] = nonfinite ? 0 : n;
  if (P.ctx) {
    LmCtx cx{};
    cx.m = st.m;
    cx.log2z = log2z;
    cx.ms = ss.m;
    cx.log2zs = log2zs;
    cx.h_full = h_full;
    cx.h_support = h_sup;
    cx.c = c;
    cx.n = nonfinite ? 0 : n;
    uint32_t f = 0;
    if (nonfinite || timeout) f |= kLmCtxNonFinite;
    if (!(status & VS_ROW_TARGET_OUT_OF_RANGE)) f |= kLmCtxTargetOk;
    if (in_s && !nonfinite) f |= kLmCtxTargetInS;
    cx.flags = f;
    P.ctx[row] = cx;
  }
}

// The merge: a warp per row, four rows per CTA.
cudaError_t launch_merge(const MergeParams& M, int rows, cudaStream_t s) {
  lmhead_merge_kernel<<<(rows + 3) / 4, 128, 0, s>>>(M);
  return cudaGetLastError();
}

// Clears the timeout flag and, when given, the target logits (a shard that
// does not hold a row's target leaves 0 there).
__global__ void lmhead_clear_kernel(uint32_t* err, float* zy, int rows) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *err = 0u;
  if (zy)
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x)
      zy[r] = 0.f;
}

// ---------------------------------------------------------------------------
// backward (xorl issue #71, section 1: selected logprob + VJP), with respect
// to x = H W^T (so dz / T for z = x / T):
//   dx_j = (1/T) ( g_lpV ([j == y] - p_j) + g_lpS 1_S(j) ([j == y] - q_j)
//                 - g_HV p_j (log p_j + H_V) - g_HS 1_S(j) q_j (log q_j + H_S) )
// Dense part for every j: p_j (alpha + beta x_j) with
//   alpha = -(1/T) (g_lpV + g_HV (H_V - LSE)),  beta = -(1/T^2) g_HV;
// the target and support entries (at most top_k + 1 per row) are rewritten
// whole by the fix-up kernel.  An empty support folds g_lpS into g_lpV (lp_S
// is lp_V there); a target outside [0, V) drops the logprob terms; a
// non-finite row has no gradient.

struct BwdRowParams {
  int32_t rows, top_k;
  const LmCtx* ctx;
  const float* g_lpv;
  const float* g_lps;
  const float* g_hv;
  const float* g_hs;
  float4* rowc;
};

__device__ __forceinline__ float gval(const float* g, int row) { return g ? g[row] : 0.f; }

// g_lpV as it enters the row's gradient (see above)
__device__ __forceinline__ float row_gv(const LmCtx& cx, const float* g_lpv, const float* g_lps,
                                        int row) {
  if (!(cx.flags & kLmCtxTargetOk)) return 0.f;
  return gval(g_lpv, row) + (cx.n == 0 ? gval(g_lps, row) : 0.f);
}

__global__ void lmhead_bwd_prep_kernel(BwdRowParams P) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= P.rows) return;
  const LmCtx cx = P.ctx[row];
  float4 rc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!(cx.flags & kLmCtxNonFinite)) {
    const float gv = row_gv(cx, P.g_lpv, P.g_lps, row);
    const float ghv = gval(P.g_hv, row);
    const float lse = cx.m + cx.log2z;  // base-2 units
    const float k = cx.c * kLn2;        // 1 / T
    rc = make_float4(cx.c, lse, -k * (gv + ghv * (cx.h_full - kLn2 * lse)), -k * ghv * kLn2 * cx.c);
  }
  P.rowc[row] = rc;
}

struct FixParams {
  int32_t rows, hidden, top_k, c0, c1;  // the vocabulary chunk [c0, c1)
  const uint16_t* H;
  int64_t ldh;
  const uint16_t* W;
  int64_t ldw;
  const LmCtx* ctx;
  const int32_t* targets;
  const int32_t* topk_ids;
  const float* g_lpv;
  const float* g_lps;
  const float* g_hv;
  const float* g_hs;
  const float4* rowc;
  const uint32_t* err;
  uint16_t* dz;
  int64_t dz_ld;
};

// One CTA per row: the row's support ids and target inside the chunk, each
// by one warp: x_j = H_i . W_j (bf16 products accumulated in fp32), then the
// whole gradient entry, rounded to bf16 over the dense value.
__global__ void __launch_bounds__(128) lmhead_bwd_fix_kernel(FixParams P) {
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint16_t* drow = P.dz + static_cast<int64_t>(row) * P.dz_ld;
  if (*P.err != 0u) {
    // a bounded wait of the dense pass gave up: make the failure loud
    if (threadIdx.x == 0 && P.c1 > P.c0) drow[0] = 0x7FC0u;  // NaN
    return;
  }
  const LmCtx cx = P.ctx[row];
  if (cx.flags & kLmCtxNonFinite) return;
  const int n = cx.n;
  const int y = P.targets[row];
  const bool yok = cx.flags & kLmCtxTargetOk;
  const bool yin = cx.flags & kLmCtxTargetInS;
  const int nid = n + ((yok && !yin) ? 1 : 0);
  const uint4* h4 = reinterpret_cast<const uint4*>(P.H + static_cast<int64_t>(row) * P.ldh);
  const int nv = P.hidden / 8;
  for (int e = warp; e < nid; e += 4) {
    const int j = e < n ? P.topk_ids[static_cast<int64_t>(row) * P.top_k + e] : y;
    if (j < P.c0 || j >= P.c1) continue;
    const uint4* w4 = reinterpret_cast<const uint4*>(P.W + static_cast<int64_t>(j) * P.ldw);
    float acc = 0.f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 a = h4[v], b = w4[v];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc = fmaf(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16), acc);
        acc = fmaf(__uint_as_float(wa[i] & 0xFFFF0000u), __uint_as_float(wb[i] & 0xFFFF0000u), acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float4 rc = P.rowc[row];
      const float k = cx.c * kLn2;  // 1 / T
      float g = ex2(fmaf(acc, rc.x, -rc.y)) * fmaf(rc.w, acc, rc.z);
      if (j == y && yok) g += k * row_gv(cx, P.g_lpv, P.g_lps, row);
      if (e < n && n > 1) {
        // a singleton support has q = 1 and H_S = 0: both support terms vanish
        const float dq = fmaf(acc, cx.c, -(cx.ms + cx.log2zs));  // log2 q_j
        const float qv = ex2(dq);
        float sp = gval(P.g_hs, row) * (-qv * fmaf(kLn2, dq, cx.h_support));
        if (yin) sp += gval(P.g_lps, row) * ((j == y ? 1.f : 0.f) - qv);
        g += k * sp;
      }
      drow[j - P.c0] = __bfloat16_as_ushort(__float2bfloat16_rn(g));
    }
  }
}


// ---------------------------------------------------------------------------
// host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
              uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Vocabulary splits: the fewest (up to kMaxSplits) that keep the units
// (row blocks x splits) at >= 97% of a whole number of waves over the SMs.
int choose_splits(int m_blocks, int n_tiles, int sms) {
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= kMaxSplits && s <= n_tiles; ++s) {
    const long units = static_cast<long>(m_blocks) * s;
    const long waves = (units + sms - 1) / sms;
    const double eff = static_cast<double>(units) / static_cast<double>(waves * sms);
    if (eff >= 0.97) return s;
    if (eff > best_eff) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}

struct LmLayout {
  int m_blocks, m_units, n_tiles, splits, tiles_per_split;
  size_t off_stats, off_val, off_id, off_zy, off_err, total;
};

// Work layout and workspace.  Pair mode: row units of 256 rows over half as
// many workers (CTA pairs).
LmLayout lm_layout(int rows, int vocab, int top_k, bool pair) {
  LmLayout L{};
  L.m_blocks = (rows + kBM - 1) / kBM;
  L.m_units = pair ? (L.m_blocks + 1) / 2 : L.m_blocks;
  L.n_tiles = (vocab + kBN - 1) / kBN;
  L.splits = choose_splits(L.m_units, L.n_tiles, pair ? num_sms() / 2 : num_sms());
  L.tiles_per_split = (L.n_tiles + L.splits - 1) / L.splits;
  L.splits = (L.n_tiles + L.tiles_per_split - 1) / L.tiles_per_split;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rs = static_cast<size_t>(rows) * L.splits;
  L.off_stats = 0;
  L.off_val = up(L.off_stats + rs * sizeof(float4));
  L.off_id = up(L.off_val + rs * top_k * sizeof(float));
  L.off_zy = up(L.off_id + rs * top_k * sizeof(int32_t));
  L.off_err = up(L.off_zy + static_cast<size_t>(rows) * sizeof(float));
  L.total = up(L.off_err + 16);
  return L;
}

// Launch shape of the GEMM kernel.  Pair mode (two SMs per 256 x 256 tile,
// half the operand traffic per SM) when the device schedules clusters of two
// with this shared memory; otherwise one CTA per 128 x 256 tile.
struct GemmConfig {
  bool pair;
  int stages;
  size_t smem;
};

template <int MODE>
GemmConfig gemm_config(int top_k) {
  GemmConfig g{};
  const size_t lists = static_cast<size_t>(kBM) * top_k * 8;
  const size_t fixed = 1024 + lists + 16 + sizeof(Barriers);
  int stages2 = static_cast<int>((227 * 1024 - fixed) / kStageBytes2);
  if (stages2 > kMaxStages) stages2 = kMaxStages;
  const size_t smem2 = fixed + static_cast<size_t>(stages2) * kStageBytes2;
  bool pair = stages2 >= 3;
  if (pair) {
    cudaError_t e = cudaFuncSetAttribute(lmhead_gemm_kernel<true, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem2));
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem2;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nc = 0;
    if (e != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&nc, lmhead_gemm_kernel<true, MODE>, &cfg) != cudaSuccess ||
        nc < 1) {
      cudaGetLastError();
      pair = false;
    }
  }
  g.pair = pair;
  if (pair) {
    g.stages = stages2;
    g.smem = smem2;
  } else {
    g.stages = top_k <= 24 ? 4 : 3;
    g.smem = fixed + static_cast<size_t>(g.stages) * kStageBytes;
  }
  return g;
}

template <int MODE>
cudaError_t gemm_launch(const GemmConfig& g, const CUtensorMap& map_h, const CUtensorMap& map_w,
                        const LmParams& P, int units, cudaStream_t s) {
  if (g.pair) {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    const int workers = num_sms() / 2;
    cfg.gridDim = dim3(2 * (units < workers ? units : workers), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = g.smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, lmhead_gemm_kernel<true, MODE>, map_h, map_w, P);
  }
  cudaError_t e = cudaFuncSetAttribute(lmhead_gemm_kernel<false, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(g.smem));
  if (e != cudaSuccess) return e;
  const int grid = units < num_sms() ? units : num_sms();
  lmhead_gemm_kernel<false, MODE><<<grid, kThreads, g.smem, s>>>(map_h, map_w, P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// plain GEMMs of the backward on cuBLASLt (bf16 operands, fp32 accumulation
// and output), with the caller's workspace

constexpr size_t kLtWorkspace = size_t(32) << 20;
constexpr int kBwdChunk = 32768;  // vocabulary columns per backward chunk (multiple of kBN)

std::mutex g_lt_mu;
cublasLtHandle_t g_lt[64] = {};

cublasLtHandle_t lt_handle() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_lt_mu);
  if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) g_lt[dev] = nullptr;
  return g_lt[dev];
}

// Column-major C[m, n] (ldc) = A[m, k] (lda) op(B) + beta C, op(B) = B[k, n]
// (ldb) or, with transb, the transpose of B[n, k] (ldb).
bool lt_gemm(bool transb, int64_t m, int64_t n, int64_t k, const void* A, int64_t lda,
             const void* B, int64_t ldb, float* C, int64_t ldc, float beta, void* ws,
             size_t ws_bytes, cudaStream_t s) {
  cublasLtHandle_t h = lt_handle();
  if (!h) return false;
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  bool ok = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) == CUBLAS_STATUS_SUCCESS;
  const cublasOperation_t ta = CUBLAS_OP_N, tb = transb ? CUBLAS_OP_T : CUBLAS_OP_N;
  ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)) ==
                 CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb)) ==
                 CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, m, k, lda) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, transb ? n : k, transb ? k : n, ldb) ==
                 CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, m, n, ldc) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES,
                                                  &ws_bytes, sizeof(ws_bytes)) ==
                 CUBLAS_STATUS_SUCCESS;
  cublasLtMatmulHeuristicResult_t res{};
  int nres = 0;
  ok = ok && cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &res, &nres) ==
                 CUBLAS_STATUS_SUCCESS && nres > 0;
  const float alpha = 1.f;
  ok = ok && cublasLtMatmul(h, op, &alpha, A, la, B, lb, &beta, C, lc, C, lc, &res.algo, ws,
                            ws_bytes, s) == CUBLAS_STATUS_SUCCESS;
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return ok;
}

struct BwdLayout {
  int chunk;
  size_t off_rowc, off_err, off_dz, off_lt, total;
};

BwdLayout bwd_layout(int rows, int vocab) {
  BwdLayout L{};
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int vr = (vocab + kBN - 1) / kBN * kBN;
  L.chunk = vr < kBwdChunk ? vr : kBwdChunk;
  L.off_rowc = 0;
  L.off_err = up(static_cast<size_t>(rows) * sizeof(float4));
  L.off_dz = up(L.off_err + 16);
  L.off_lt = up(L.off_dz + static_cast<size_t>(rows) * L.chunk * 2);
  L.total = L.off_lt + kLtWorkspace;
  return L;
}

}  // namespace

size_t lmhead_workspace_bytes(int rows, int vocab, int hidden, int top_k) {
  (void)hidden;
  if (rows <= 0 || vocab <= 0 || top_k <= 0) return 0;
  // enough for either launch mode
  const size_t a = lm_layout(rows, vocab, top_k, true).total;
  const size_t b = lm_layout(rows, vocab, top_k, false).total;
  return a > b ? a : b;
}

namespace {

// The projection with the scoring epilogue over weight rows [0, vocab) whose
// vocabulary ids start at col_offset: per (row, split) records in `ws`
// (lm_layout).  clear_zy zeroes the target logits first (a shard may not
// hold a row's target).
vs_status gemm_phase(int rows, int vocab, int col_offset, int hidden, const void* H, int64_t ldh,
                     const void* W, int64_t ldw, const float* temperature,
                     float temperature_scalar, const int32_t* targets, int top_k, void* ws,
                     bool clear_zy, cudaStream_t s, LmParams* Pout, LmLayout* Lout,
                     std::string* err) {
  const GemmConfig G = gemm_config<kModeScore>(top_k);
  const LmLayout L = lm_layout(rows, vocab, top_k, G.pair);
  CUtensorMap map_h, map_w;
  if (!make_map(&map_h, H, rows, hidden, ldh, kBM) ||
      !make_map(&map_w, W, vocab, hidden, ldw, G.pair ? kBNh : kBN)) {
    *err = "cuTensorMapEncodeTiled failed";
    return VS_ERR_CUDA;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  LmParams P{};
  P.rows = rows;
  P.vocab = vocab;
  P.hidden = hidden;
  P.top_k = top_k;
  P.splits = L.splits;
  P.tiles_per_split = L.tiles_per_split;
  P.n_tiles = L.n_tiles;
  P.m_blocks = L.m_blocks;
  P.m_units = L.m_units;
  P.stages = G.stages;
  P.temperature = temperature;
  P.temperature_scalar = temperature_scalar;
  P.targets = targets;
  P.col_offset = col_offset;
  P.ws_stats = reinterpret_cast<float4*>(w8 + L.off_stats);
  P.ws_val = reinterpret_cast<float*>(w8 + L.off_val);
  P.ws_id = reinterpret_cast<int32_t*>(w8 + L.off_id);
  P.ws_zy = reinterpret_cast<float*>(w8 + L.off_zy);
  P.ws_err = reinterpret_cast<uint32_t*>(w8 + L.off_err);
  if (clear_zy)
    lmhead_clear_kernel<<<(rows + 255) / 256, 256, 0, s>>>(P.ws_err, P.ws_zy, rows);
  else
    lmhead_clear_kernel<<<1, 1, 0, s>>>(P.ws_err, nullptr, 0);
  cudaError_t e = gemm_launch<kModeScore>(G, map_h, map_w, P, L.m_units * L.splits, s);
  if (e != cudaSuccess) {
    *err = cudaGetErrorString(e);
    return VS_ERR_CUDA;
  }
  *Pout = P;
  *Lout = L;
  return VS_OK;
}

// Merge inputs: the GEMM's per-(row, split) records.
void merge_from_workspace(MergeParams& M, const LmParams& P, const LmLayout& L, int top_k) {
  M.splits = L.splits;
  M.ws_stats = P.ws_stats;
  M.ws_val = P.ws_val;
  M.ws_id = P.ws_id;
  M.ws_zy = P.ws_zy;
  M.ws_err = P.ws_err;
  M.st_row = L.splits;
  M.st_split = 1;
  M.ls_row = static_cast<int64_t>(L.splits) * top_k;
  M.ls_split = top_k;
  M.parts = 1;
  M.zy_part = 0;
  M.err_part = 0;
}

// One shard's partial record block (vocabulary-parallel head).
struct PartLayout {
  size_t off_stats, off_val, off_id, off_zy, off_err, total;
};

PartLayout part_layout(int rows, int top_k) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  PartLayout L{};
  L.off_stats = 0;
  L.off_val = up(static_cast<size_t>(rows) * sizeof(float4));
  L.off_id = up(L.off_val + static_cast<size_t>(rows) * top_k * sizeof(float));
  L.off_zy = up(L.off_id + static_cast<size_t>(rows) * top_k * sizeof(int32_t));
  L.off_err = up(L.off_zy + static_cast<size_t>(rows) * sizeof(float));
  L.total = up(L.off_err + 16);
  return L;
}

}  // namespace

vs_status lmhead_run(int rows, int vocab, int hidden, const void* H, int64_t ldh, const void* W,
                     int64_t ldw, const float* temperature, float temperature_scalar,
                     const int32_t* targets, int top_k, float top_p, float min_p,
                     uint32_t flags, const vs_score_out* out, int32_t* topk_ids,
                     float* topk_logprob, void* ws, size_t ws_bytes, cudaStream_t s,
                     std::string* err) {
  auto bad = [&](vs_status code, const char* msg) {
    *err = msg;
    return code;
  };
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (rows < 0) return bad(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (vocab < 1) return bad(VS_ERR_INVALID_ARG, "vocab must be >= 1");
  if (hidden < kBK || hidden % kBK != 0) return bad(VS_ERR_UNSUPPORTED, "hidden_dim must be a positive multiple of 64");
  if (top_k < 1 || top_k > VS_MAX_FUSED_TOPK || top_k > vocab)
    return bad(VS_ERR_UNSUPPORTED, "top_k must lie in [1, min(VS_MAX_FUSED_TOPK, vocab)]");
  if (!(top_p > 0.f && top_p <= 1.f)) return bad(VS_ERR_INVALID_ARG, "top_p must lie in (0, 1]");
  if (!(min_p >= 0.f && min_p < 1.f)) return bad(VS_ERR_INVALID_ARG, "min_p must lie in [0, 1)");
  if (!temperature && !(std::isfinite(temperature_scalar) && temperature_scalar > 0.f))
    return bad(VS_ERR_INVALID_ARG, "temperature_scalar must be finite and > 0");
  if (!out) return bad(VS_ERR_INVALID_ARG, "out is NULL");
  if (out->sampled || out->support_mask || (flags & VS_WANT_SAMPLE))
    return bad(VS_ERR_INVALID_ARG, "sampled and support_mask are not offered by the fused head: pass NULL");
  const bool want_grad = flags & VS_WANT_GRAD;
  if (want_grad != (out->ctx != nullptr))
    return bad(VS_ERR_INVALID_ARG, "VS_WANT_GRAD and ctx go together");
  if (want_grad && (!topk_ids || !a16(out->ctx)))
    return bad(VS_ERR_INVALID_ARG, "VS_WANT_GRAD needs topk_ids (the support) and a 16-byte aligned ctx");
  const bool want_entropy = flags & VS_WANT_ENTROPY;
  if (!want_entropy && (out->entropy_full || out->entropy_support))
    return bad(VS_ERR_INVALID_ARG, "entropy outputs need VS_WANT_ENTROPY");
  if (rows == 0) return VS_OK;
  if (!H || !W || !targets) return bad(VS_ERR_INVALID_ARG, "hidden, weight and targets must be non-NULL");
  if (!a16(H) || !a16(W) || ldh % 8 != 0 || ldw % 8 != 0 || ldh < hidden || ldw < hidden)
    return bad(VS_ERR_INVALID_ARG, "hidden/weight must be 16-byte aligned with ld >= hidden_dim, ld % 8 == 0");
  if (!ws || !a16(ws) || ws_bytes < lmhead_workspace_bytes(rows, vocab, hidden, top_k))
    return bad(VS_ERR_WORKSPACE, "workspace missing, misaligned or smaller than vs_fused_lmhead_workspace_size");

  LmParams P{};
  LmLayout L{};
  const vs_status gs = gemm_phase(rows, vocab, 0, hidden, H, ldh, W, ldw, temperature,
                                  temperature_scalar, targets, top_k, ws, false, s, &P, &L, err);
  if (gs != VS_OK) return gs;
  MergeParams M{};
  merge_from_workspace(M, P, L, top_k);
  M.rows = rows;
  M.vocab = vocab;
  M.top_k = top_k;
  M.top_p = top_p;
  M.min_p = min_p;
  M.temperature = temperature;
  M.temperature_scalar = temperature_scalar;
  M.targets = targets;
  M.lp_full = out->logprob_full;
  M.lp_support = out->logprob_support;
  M.h_full = want_entropy ? out->entropy_full : nullptr;
  M.h_support = want_entropy ? out->entropy_support : nullptr;
  M.valid = out->valid;
  M.status = out->status;
  M.support_size = out->support_size;
  M.topk_ids = topk_ids;
  M.topk_logprob = topk_logprob;
  M.ctx = want_grad ? static_cast<LmCtx*>(out->ctx) : nullptr;
  M.want_entropy = want_entropy ? 1 : 0;
  if (const cudaError_t em = launch_merge(M, rows, s); em != cudaSuccess)
    return bad(VS_ERR_CUDA, cudaGetErrorString(em));  // a warp per row
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));
  return VS_OK;
}

// ---------------------------------------------------------------------------
// vocabulary-parallel head: one shard's partial records, then the merge of
// every shard's records

size_t lmhead_partial_bytes(int rows, int top_k) {
  if (rows <= 0 || top_k <= 0) return 0;
  return part_layout(rows, top_k).total;
}

vs_status lmhead_partial_run(int rows, int vocab_total, int vocab_begin, int vocab_count,
                             int hidden, const void* H, int64_t ldh, const void* W, int64_t ldw,
                             const float* temperature, float temperature_scalar,
                             const int32_t* targets, int top_k, void* partial, void* ws,
                             size_t ws_bytes, cudaStream_t s, std::string* err) {
  auto bad = [&](vs_status code, const char* msg) {
    *err = msg;
    return code;
  };
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (rows < 0) return bad(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (vocab_total < 1 || vocab_begin < 0 || vocab_count < 1 || vocab_begin > vocab_total - vocab_count)
    return bad(VS_ERR_INVALID_ARG, "the shard [vocab_begin, vocab_begin + vocab_count) must lie in [0, vocab_total)");
  if (hidden < kBK || hidden % kBK != 0)
    return bad(VS_ERR_UNSUPPORTED, "hidden_dim must be a positive multiple of 64");
  if (top_k < 1 || top_k > VS_MAX_FUSED_TOPK || top_k > vocab_total)
    return bad(VS_ERR_UNSUPPORTED, "top_k must lie in [1, min(VS_MAX_FUSED_TOPK, vocab_total)]");
  if (!temperature && !(std::isfinite(temperature_scalar) && temperature_scalar > 0.f))
    return bad(VS_ERR_INVALID_ARG, "temperature_scalar must be finite and > 0");
  if (rows == 0) return VS_OK;
  if (!H || !W || !targets || !partial)
    return bad(VS_ERR_INVALID_ARG, "hidden, weight, targets and partial must be non-NULL");
  if (!a16(H) || !a16(W) || !a16(partial) || ldh % 8 != 0 || ldw % 8 != 0 || ldh < hidden ||
      ldw < hidden)
    return bad(VS_ERR_INVALID_ARG, "hidden/weight/partial must be 16-byte aligned with ld >= hidden_dim, ld % 8 == 0");
  if (!ws || !a16(ws) || ws_bytes < lmhead_workspace_bytes(rows, vocab_count, hidden, top_k))
    return bad(VS_ERR_WORKSPACE, "workspace missing, misaligned or smaller than vs_fused_lmhead_partial_workspace_size");
  LmParams P{};
  LmLayout L{};
  const vs_status gs = gemm_phase(rows, vocab_count, vocab_begin, hidden, H, ldh, W, ldw,
                                  temperature, temperature_scalar, targets, top_k, ws, true, s,
                                  &P, &L, err);
  if (gs != VS_OK) return gs;
  const PartLayout B = part_layout(rows, top_k);
  uint8_t* b8 = static_cast<uint8_t*>(partial);
  MergeParams M{};
  merge_from_workspace(M, P, L, top_k);
  M.rows = rows;
  M.vocab = vocab_total;
  M.top_k = top_k;
  M.temperature = temperature;
  M.temperature_scalar = temperature_scalar;
  M.targets = targets;
  M.out_stats = reinterpret_cast<float4*>(b8 + B.off_stats);
  M.out_val = reinterpret_cast<float*>(b8 + B.off_val);
  M.out_id = reinterpret_cast<int32_t*>(b8 + B.off_id);
  M.out_zy = reinterpret_cast<float*>(b8 + B.off_zy);
  M.out_err = reinterpret_cast<uint32_t*>(b8 + B.off_err);
  lmhead_clear_kernel<<<1, 1, 0, s>>>(M.out_err, nullptr, 0);
  if (const cudaError_t em = launch_merge(M, rows, s); em != cudaSuccess)
    return bad(VS_ERR_CUDA, cudaGetErrorString(em));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));
  return VS_OK;
}

vs_status lmhead_merge_run(int rows, int vocab_total, int n_shards, const void* partials,
                           const float* temperature, float temperature_scalar,
                           const int32_t* targets, int top_k, float top_p, float min_p,
                           uint32_t flags, const vs_score_out* out, int32_t* topk_ids,
                           float* topk_logprob, cudaStream_t s, std::string* err) {
  auto bad = [&](vs_status code, const char* msg) {
    *err = msg;
    return code;
  };
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (rows < 0) return bad(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (vocab_total < 1) return bad(VS_ERR_INVALID_ARG, "vocab_total must be >= 1");
  if (n_shards < 1 || n_shards > kMaxSplits)
    return bad(VS_ERR_UNSUPPORTED, "n_shards must lie in [1, 64]");
  if (top_k < 1 || top_k > VS_MAX_FUSED_TOPK || top_k > vocab_total)
    return bad(VS_ERR_UNSUPPORTED, "top_k must lie in [1, min(VS_MAX_FUSED_TOPK, vocab_total)]");
  if (!(top_p > 0.f && top_p <= 1.f)) return bad(VS_ERR_INVALID_ARG, "top_p must lie in (0, 1]");
  if (!(min_p >= 0.f && min_p < 1.f)) return bad(VS_ERR_INVALID_ARG, "min_p must lie in [0, 1)");
  if (!temperature && !(std::isfinite(temperature_scalar) && temperature_scalar > 0.f))
    return bad(VS_ERR_INVALID_ARG, "temperature_scalar must be finite and > 0");
  if (!out) return bad(VS_ERR_INVALID_ARG, "out is NULL");
  if (out->sampled || out->support_mask || out->ctx || (flags & (VS_WANT_SAMPLE | VS_WANT_GRAD)))
    return bad(VS_ERR_INVALID_ARG, "sampled, support_mask and ctx are not offered by the merge: pass NULL");
  const bool want_entropy = flags & VS_WANT_ENTROPY;
  if (!want_entropy && (out->entropy_full || out->entropy_support))
    return bad(VS_ERR_INVALID_ARG, "entropy outputs need VS_WANT_ENTROPY");
  if (rows == 0) return VS_OK;
  if (!partials || !a16(partials) || !targets)
    return bad(VS_ERR_INVALID_ARG, "partials (16-byte aligned) and targets must be non-NULL");
  const PartLayout B = part_layout(rows, top_k);
  const uint8_t* b8 = static_cast<const uint8_t*>(partials);
  MergeParams M{};
  M.rows = rows;
  M.vocab = vocab_total;
  M.splits = n_shards;
  M.top_k = top_k;
  M.top_p = top_p;
  M.min_p = min_p;
  M.temperature = temperature;
  M.temperature_scalar = temperature_scalar;
  M.targets = targets;
  M.ws_stats = reinterpret_cast<const float4*>(b8 + B.off_stats);
  M.ws_val = reinterpret_cast<const float*>(b8 + B.off_val);
  M.ws_id = reinterpret_cast<const int32_t*>(b8 + B.off_id);
  M.ws_zy = reinterpret_cast<const float*>(b8 + B.off_zy);
  M.ws_err = reinterpret_cast<const uint32_t*>(b8 + B.off_err);
  M.st_row = 1;
  M.st_split = static_cast<int64_t>(B.total / sizeof(float4));
  M.ls_row = top_k;
  M.ls_split = static_cast<int64_t>(B.total / sizeof(float));
  M.parts = n_shards;
  M.zy_part = static_cast<int64_t>(B.total / sizeof(float));
  M.err_part = static_cast<int64_t>(B.total / sizeof(uint32_t));
  M.lp_full = out->logprob_full;
  M.lp_support = out->logprob_support;
  M.h_full = want_entropy ? out->entropy_full : nullptr;
  M.h_support = want_entropy ? out->entropy_support : nullptr;
  M.valid = out->valid;
  M.status = out->status;
  M.support_size = out->support_size;
  M.topk_ids = topk_ids;
  M.topk_logprob = topk_logprob;
  M.want_entropy = want_entropy ? 1 : 0;
  if (const cudaError_t em = launch_merge(M, rows, s); em != cudaSuccess)
    return bad(VS_ERR_CUDA, cudaGetErrorString(em));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));
  return VS_OK;
}

size_t lmhead_bwd_workspace_bytes(int rows, int vocab, int hidden) {
  (void)hidden;
  if (rows <= 0 || vocab <= 0) return 0;
  return bwd_layout(rows, vocab).total;
}

vs_status lmhead_bwd_run(int rows, int vocab, int hidden, const void* H, int64_t ldh,
                         const void* W, int64_t ldw, const int32_t* targets, int top_k,
                         const void* ctx, const int32_t* topk_ids, const float* g_lp_full,
                         const float* g_lp_support, const float* g_h_full,
                         const float* g_h_support, float* d_hidden, int64_t ld_dh,
                         float* d_weight, int64_t ld_dw, void* ws, size_t ws_bytes,
                         cudaStream_t s, std::string* err) {
  auto bad = [&](vs_status code, const char* msg) {
    *err = msg;
    return code;
  };
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (rows < 0) return bad(VS_ERR_INVALID_ARG, "rows must be >= 0");
  if (vocab < 1) return bad(VS_ERR_INVALID_ARG, "vocab must be >= 1");
  if (hidden < kBK || hidden % kBK != 0)
    return bad(VS_ERR_UNSUPPORTED, "hidden_dim must be a positive multiple of 64");
  if (top_k < 1 || top_k > VS_MAX_FUSED_TOPK || top_k > vocab)
    return bad(VS_ERR_UNSUPPORTED, "top_k must lie in [1, min(VS_MAX_FUSED_TOPK, vocab)]");
  if (rows == 0 || (!d_hidden && !d_weight)) return VS_OK;
  if (!H || !W || !targets || !ctx || !topk_ids)
    return bad(VS_ERR_INVALID_ARG, "hidden, weight, targets, ctx and topk_ids must be non-NULL");
  if (!a16(H) || !a16(W) || ldh % 8 != 0 || ldw % 8 != 0 || ldh < hidden || ldw < hidden ||
      !a16(ctx))
    return bad(VS_ERR_INVALID_ARG, "hidden/weight must be 16-byte aligned with ld >= hidden_dim, ld % 8 == 0; ctx 16-byte aligned");
  if ((d_hidden && (ld_dh < hidden || !a16(d_hidden) || ld_dh % 4 != 0)) ||
      (d_weight && (ld_dw < hidden || !a16(d_weight) || ld_dw % 4 != 0)))
    return bad(VS_ERR_INVALID_ARG, "d_hidden / d_weight must be 16-byte aligned with ld >= hidden_dim, ld % 4 == 0");
  const BwdLayout L = bwd_layout(rows, vocab);
  if (!ws || !a16(ws) || ws_bytes < L.total)
    return bad(VS_ERR_WORKSPACE, "workspace missing, misaligned or smaller than vs_fused_lmhead_bwd_workspace_size");

  uint8_t* w8 = static_cast<uint8_t*>(ws);
  float4* rowc = reinterpret_cast<float4*>(w8 + L.off_rowc);
  uint32_t* werr = reinterpret_cast<uint32_t*>(w8 + L.off_err);
  uint16_t* dz = reinterpret_cast<uint16_t*>(w8 + L.off_dz);
  void* ltws = w8 + L.off_lt;
  const LmCtx* cx = static_cast<const LmCtx*>(ctx);

  lmhead_clear_kernel<<<1, 1, 0, s>>>(werr, nullptr, 0);
  BwdRowParams R{};
  R.rows = rows;
  R.top_k = top_k;
  R.ctx = cx;
  R.g_lpv = g_lp_full;
  R.g_lps = g_lp_support;
  R.g_hv = g_h_full;
  R.g_hs = g_h_support;
  R.rowc = rowc;
  lmhead_bwd_prep_kernel<<<(rows + 127) / 128, 128, 0, s>>>(R);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));

  const GemmConfig G = gemm_config<kModeDz>(0);
  CUtensorMap map_h;
  if (!make_map(&map_h, H, rows, hidden, ldh, kBM)) return bad(VS_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  for (int c0 = 0; c0 < vocab; c0 += L.chunk) {
    const int len = vocab - c0 < L.chunk ? vocab - c0 : L.chunk;
    const uint16_t* Wc = static_cast<const uint16_t*>(W) + static_cast<int64_t>(c0) * ldw;
    CUtensorMap map_w;
    if (!make_map(&map_w, Wc, len, hidden, ldw, G.pair ? kBNh : kBN))
      return bad(VS_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    const LmLayout LL = lm_layout(rows, len, 0, G.pair);
    LmParams P{};
    P.rows = rows;
    P.vocab = len;
    P.hidden = hidden;
    P.top_k = 0;
    P.splits = LL.splits;
    P.tiles_per_split = LL.tiles_per_split;
    P.n_tiles = LL.n_tiles;
    P.m_blocks = LL.m_blocks;
    P.m_units = LL.m_units;
    P.stages = G.stages;
    P.ws_err = werr;
    P.rowc = rowc;
    P.dz = dz;
    P.dz_ld = L.chunk;
    e = gemm_launch<kModeDz>(G, map_h, map_w, P, LL.m_units * LL.splits, s);
    if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));
    FixParams F{};
    F.rows = rows;
    F.hidden = hidden;
    F.top_k = top_k;
    F.c0 = c0;
    F.c1 = c0 + len;
    F.H = static_cast<const uint16_t*>(H);
    F.ldh = ldh;
    F.W = static_cast<const uint16_t*>(W);
    F.ldw = ldw;
    F.ctx = cx;
    F.targets = targets;
    F.topk_ids = topk_ids;
    F.g_lpv = g_lp_full;
    F.g_lps = g_lp_support;
    F.g_hv = g_h_full;
    F.g_hs = g_h_support;
    F.rowc = rowc;
    F.err = werr;
    F.dz = dz;
    F.dz_ld = L.chunk;
    lmhead_bwd_fix_kernel<<<rows, 128, 0, s>>>(F);
    e = cudaGetLastError();
    if (e != cudaSuccess) return bad(VS_ERR_CUDA, cudaGetErrorString(e));
    // d_hidden (+)= dz_c W_c:  column-major [hidden, rows] = W_c^T [hidden, len] dz_c^T [len, rows]
    if (d_hidden && !lt_gemm(false, hidden, rows, len, Wc, ldw, dz, L.chunk, d_hidden, ld_dh,
                             c0 == 0 ? 0.f : 1.f, ltws, kLtWorkspace, s))
      return bad(VS_ERR_CUDA, "cuBLASLt matmul (d_hidden) failed");
    // d_weight[c0 : c0 + len] = dz_c^T H:  column-major [hidden, len] = H^T [hidden, rows] dz_c [rows, len]
    if (d_weight && !lt_gemm(true, hidden, len, rows, H, ldh, dz, L.chunk,
                             d_weight + static_cast<int64_t>(c0) * ld_dw, ld_dw, 0.f, ltws,
                             kLtWorkspace, s))
      return bad(VS_ERR_CUDA, "cuBLASLt matmul (d_weight) failed");
  }
  return VS_OK;
}

}  // namespace vs
