// Paged prefill on 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Many new query tokens per sequence attend causally to the sequence's paged
// cache: query i at absolute position pos_i sees tokens 0..pos_i.  The
// block-wise form of "PagedAttention" (wiki mirror, "Formulació matemàtica")
// applies to every query; with 128 queries a tile the two products are dense
// contractions, S = Q.K^T and O = P.V.
//
// A work item = (sequence, query head, 256 new queries as two 128-row tiles).
// CTAs walk the items heaviest first (fp16: one persistent CTA per SM; bf16:
// the grid covers every item, so each CTA's walk is one item), with
// specialised warps:
//   * warps 0-3 and 4-7: two softmax warpgroups, one per query tile; thread r
//     of a group owns query row r (TMEM lane r).  Each reads its row of S
//     (128 keys) from TMEM, applies the causal mask and the online softmax in
//     fp32 (log2 domain) and writes its row of P (fp16/bf16 pairs) back over
//     S in TMEM, where the P.V product takes its A operand from.  P is handed
//     over in two 64-key pieces, each on its own mbarrier, so that P.V of the
//     first runs while the second is computed.  At the end of an item the
//     group writes its rows of O out and frees O for the next item;
//   * warp 8: the loader.  It loads each item's Q tiles and streams the paged
//     K and V rows of each 128-key tile with TMA tensor copies (one 16-row box
//     per physical block and 64-wide slice of head_dim, hardware 128-byte
//     swizzle) into rings of K and V stages that run on across items; the
//     valid V rows of a partly filled last block are copied by its lanes and
//     the V rows past the context are zeroed;
//   * warp 9: one thread issues the tensor-core products into TMEM and commits
//     them to mbarriers.
// The two query tiles share every K/V stage and take turns on the tensor core:
// while one group runs its softmax, the MMA unit computes the other group's
// P.V and next S.  Keeping P in TMEM leaves shared memory to the Q, K and V
// operands, whose bandwidth bounds the products (128-key tiles halve the Q
// re-reads per flop against 64-key ones).  The running max is only moved
// (and the row of O in TMEM rescaled) when a score exceeds it by more than
// 2^8, which keeps every weight at most 256 and makes the rescale rare.
// Shared-memory operands are described by SW128 matrix descriptors (K-major
// for Q and K; MN-major for V).  Every wait is bounded; a wait that gives
// up stops the CTA's other roles, lets every copy and product already issued
// land, frees TMEM and reports PA_DEVERR_TIMEOUT.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "device_utils.cuh"
#include "mma_utils.cuh"
#include "pagedattn.h"
#include "tma.cuh"

namespace pa {

struct PrefillArgs {
  const void* q;                // [T][HQ][D]
  const void* v_pool;           // rows of a partly filled last block are copied directly
  const int32_t* block_tables;
  const int32_t* context_lens;  // [S] tokens cached, new ones included
  const int32_t* query_start;   // [S+1] CSR: new tokens of s are rows query_start[s].. of q/out
  void* out;                    // [T][HQ][D]
  uint32_t* err;
  int64_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int32_t heads;     // KV heads
  int32_t q_per_kv;  // query heads per KV head
  int32_t max_context_len;
  int32_t q_pairs;   // 256-query units per sequence (work items per (sequence, head))
  int32_t max_new_tokens;  // bound on every sequence's new tokens (the grid covers it)
  int32_t num_tokens;      // rows of q and out
  float scale_log2;
};

// SPLIT_P: the softmax weights go to the tensor core as a high part plus its
// rounding residual (two P operands, two P.V chains).  bf16 needs it (8-bit
// significand); fp16's 11 bits keep the result inside the parity gate alone.
template <int D, bool SPLIT_P>
struct PrefillConfig {
  static constexpr int BM = 128;        // query rows per tile (TMEM lanes)
  static constexpr int QT = 2;          // query tiles per CTA (softmax warpgroups)
  static constexpr int BN = 128;        // keys per tile
  static constexpr int KB = D / 64;     // 128-byte K-blocks across head_dim
  static constexpr int NS = D == 128 ? 2 : 3;  // stages of the K ring and of the V ring
#ifndef PA_PREFILL_P_CHUNKS
#define PA_PREFILL_P_CHUNKS 2
#endif
  // P goes to the tensor core in PC pieces of BN / PC keys, each handed over
  // as soon as it is in TMEM
  static constexpr int PC = PA_PREFILL_P_CHUNKS;
  static_assert(PC == 1 || PC == 2 || PC == 4, "P pieces");
  // keys [piece_begin(c), piece_end(c)) form P piece c
  static constexpr int piece_begin(int c) { return c * (BN / PC); }
  static constexpr int piece_end(int c) { return (c + 1) * (BN / PC); }
  static constexpr int LOAD_WARP = 8, MMA_WARP = 9;  // warps 10-11 only fill the warpgroup
  static constexpr int THREADS = 384;
  // Launched at 168 registers a thread (384 x 168 fit the register file);
  // the loader/MMA warpgroup then drops to 104 and the softmax groups rise to
  // 200: 256 x 200 + 128 x 104 = 64512 = 384 x 168 launched (per SM
  // sub-partition: two softmax warps and one other, 16128 of 16384).
  static constexpr int REGS_LAUNCH = 168, REGS_SOFTMAX = 200, REGS_OTHER = 104;
  static_assert(256 * REGS_SOFTMAX + 128 * REGS_OTHER <= THREADS * REGS_LAUNCH, "register split");
  static constexpr int Q_BYTES = KB * BM * 128;
  static constexpr int KV_BYTES = KB * BN * 128;   // one stage of K or of V
  static constexpr int OFF_Q = 0;                               // [tile]
  static constexpr int OFF_K = OFF_Q + QT * Q_BYTES;            // [stage]
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;           // [stage]
  static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
  // mbarriers: Q full / free, K full/empty[NS], V full/empty[NS], and per
  // query tile s_full, p_full of each P piece (BAR_P + 2 * piece + tile),
  // o_done, o_free (O read out); fin
  static constexpr int BAR_QF = 0, BAR_QFREE = 1, BAR_KF = 2, BAR_KE = BAR_KF + NS,
                       BAR_VF = BAR_KE + NS, BAR_VE = BAR_VF + NS, BAR_S = BAR_VE + NS,
                       BAR_P = BAR_S + 2, BAR_O = BAR_P + 2 * PC,
                       BAR_OFREE = BAR_O + 2, BAR_FIN = BAR_OFREE + 2, NBARS = BAR_FIN + 1;
  static constexpr int OFF_SLOT = OFF_BAR + NBARS * 8;  // TMEM address, abort flag
  // + 1 KB so the swizzled tiles can start on a 1024-byte boundary
  static constexpr size_t SMEM = OFF_SLOT + 16 + 1024;
  // TMEM columns: S of tile w at w * BN (fp32), overwritten by P as packed
  // pairs (high part in its first 64 columns, residual in the next 64); O of
  // tile w at O_COL0 + w * D.
  static constexpr int S_COL0 = 0;
  static constexpr int P_LO = 64;
  static constexpr int O_COL0 = 2 * BN;
  static constexpr int TMEM_COLS = 512;
  static_assert(O_COL0 + 2 * D <= TMEM_COLS, "TMEM columns");
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(SMEM <= 232448, "shared memory");
};

// ---- tcgen05 / TMA helpers -------------------------------------------------------

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// and stride byte offsets (16-byte units), version 1, layout type 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N, bool bf16, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same with A read from TMEM (rows on lanes, pairs of 16-bit elements
// packed along K in each 32-bit column).
__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive TMEM columns of this warp's 32 lanes into v (no wait).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  tmem_ld32_nowait(taddr, v);
  tmem_wait_ld();
}

// 16 consecutive TMEM columns of this warp's 32 lanes from w (no wait).
__device__ __forceinline__ void tmem_st16_nowait(uint32_t taddr, const uint32_t* w) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 3-D tiled tensor copy global -> shared (no multicast); x innermost.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait that also gives up once another role raised the abort flag.
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t bar, uint32_t parity,
                                                   const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u && (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs)) return false;
  }
}

// The same for every lane of a warp: the warp goes on only if all its lanes saw
// the phase complete, so a give-up never splits a warp.
__device__ __forceinline__ bool warp_wait_or_abort(uint32_t bar, uint32_t parity,
                                                   const volatile int* abort_flag) {
  return __all_sync(kFullMask, mbar_wait_or_abort(bar, parity, abort_flag));
}

// max / min of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


template <typename T>
constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;

// tm_k, tm_v: K and V pools viewed as [num_blocks * heads * 16 rows][head_dim],
// box {64, 16} (one physical block, one 64-wide slice), 128-byte swizzle.
// tm_q: q as [tokens][query heads][head_dim], box {64, 1, 128} (128 query
// rows of one head, one 64-wide slice), 128-byte swizzle.
//
// The CTAs walk the work items (query head, sequence, 256-query pair) in
// heaviest-first order, in boustrophedon rounds: persistent (one CTA per SM)
// for fp16, one item per CTA for bf16 (the launch decides).  The K/V rings,
// the TMEM allocation and the barriers live across items: the loader fetches
// the next item's Q as soon as the current item's last S products are done,
// and a softmax group's epilogue overlaps the next item's first products.
template <typename T, int D>
__global__ void __launch_bounds__(384, 1)
    paged_prefill_kernel(PrefillArgs a, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_q) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using Cfg = PrefillConfig<D, kSplitP<T>>;
  constexpr int BM = Cfg::BM, BN = Cfg::BN, KB = Cfg::KB, NS = Cfg::NS;
  constexpr uint32_t IDESC_S = f16_idesc(BM, BN, kBf16, false);
  constexpr uint32_t IDESC_PV = f16_idesc(BM, D, kBf16, true);

  extern __shared__ __align__(1024) uint8_t prefill_smem[];
  uint8_t* smem = prefill_smem + ((1024u - (smem_addr(prefill_smem) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.q_per_kv, HQ = a.heads * G;
  const int num_items = HQ * a.num_seqs * a.q_pairs;
  // The CTA's k-th item: rounds of gridDim.x items, taken left to right in
  // even rounds and right to left in odd ones, so that every CTA gets a fair
  // share of the heavy (early) and light (late) items.
  const int rounds = (num_items + gridDim.x - 1) / gridDim.x;
  auto nth_item = [&](int k) {
    return k * (int)gridDim.x + ((k & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };
  const int cap = min(a.max_context_len, a.max_blocks_per_seq * kBlock);

  // One work item: (query head, sequence, query pair) with the pair slowest,
  // so that every head's and sequence's latest pairs (most keys) come first.
  struct Item {
    int hq, s, qt, q0, n, L, kvh, nkt0, nkt1, nkt;
    bool has1;
  };
  // Whether item w holds work; a sequence the launch cannot take is reported
  // once (by its item with pair 0 and head 0) and skipped.
  auto item_of = [&](int w, Item& it, bool report) {
    it.hq = w % HQ;
    it.s = (w / HQ) % a.num_seqs;
    it.qt = a.q_pairs - 1 - w / (HQ * a.num_seqs);
    it.q0 = a.query_start[it.s];
    it.n = a.query_start[it.s + 1] - it.q0;
    const bool first = it.qt == 0 && it.hq == 0;
    // rows outside q / out, or beyond the launch's bound
    if (it.n > a.max_new_tokens || (it.n > 0 && (it.q0 < 0 || it.q0 > a.num_tokens - it.n))) {
      if (report && first) atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
      return false;
    }
    if (it.n <= 0 || it.qt * 2 * BM >= it.n) return false;
    it.L = a.context_lens[it.s];
    if (it.L < it.n || it.L > cap) {  // the new tokens must be in the cache
      if (report && first) atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
      return false;
    }
    it.kvh = it.hq / G;
    it.has1 = it.qt * 2 * BM + BM < it.n;  // second query tile holds queries
    // key tiles each query tile visits (up to its last query's position)
    it.nkt0 = (it.L - it.n + min(it.n, it.qt * 2 * BM + BM) - 1 + BN) / BN;
    it.nkt1 = it.has1 ? (it.L - it.n + min(it.n, it.qt * 2 * BM + 2 * BM) - 1 + BN) / BN : 0;
    it.nkt = it.has1 ? it.nkt1 : it.nkt0;
    return true;
  };

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  auto bar = [&](int i) { return smem_addr(&bars[i]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_SLOT + 4);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    mbar_init(bar(Cfg::BAR_QF), 1);
    mbar_init(bar(Cfg::BAR_QFREE), 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar(Cfg::BAR_KF + i), 1);
      mbar_init(bar(Cfg::BAR_KE + i), 1);
      mbar_init(bar(Cfg::BAR_VF + i), 1);
      mbar_init(bar(Cfg::BAR_VE + i), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bar(Cfg::BAR_S + w), 1);
      for (int c = 0; c < Cfg::PC; ++c)
        mbar_init(bar(Cfg::BAR_P + 2 * c + w), BM / 32);  // one arrival per softmax warp
      mbar_init(bar(Cfg::BAR_O + w), 1);
      mbar_init(bar(Cfg::BAR_OFREE + w), BM / 32);
    }
    mbar_init(bar(Cfg::BAR_FIN), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto give_up = [&]() {
    if (!*abort_flag) {
      *abort_flag = 1;
      atomicOr(a.err, PA_DEVERR_TIMEOUT);
    }
  };

  // registers move from the loader/MMA warpgroup to the softmax groups; each
  // group changes its limit at one point, before its warps split into roles
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Cfg::REGS_OTHER));
  if (warp == Cfg::LOAD_WARP) {
    // ---- loader: Q of each item, then K and V of key tile j into the next
    // stage of their rings (positions counted across items) ----------------------
    // K runs one tile ahead of V: a K stage frees once both S products of its
    // tile are issued, a V stage only after both P.V products.
    uint32_t kc = 0, vc = 0;  // K / V fills issued
    int items = 0;            // items whose Q was loaded
    bool ok = true;
    for (int k = 0; ok && k < rounds; ++k) {
      const int w = nth_item(k);
      Item it;
      if (w >= num_items || !item_of(w, it, false)) continue;
      const int32_t* table = a.block_tables + (int64_t)it.s * a.max_blocks_per_seq;
      // lane i < blocks in tile j: that block's id (fetched by all lanes at once)
      auto tile_blocks = [&](int j, int& nblk, int& valid) {
        valid = min(BN, it.L - j * BN);
        nblk = (valid + kBlock - 1) / kBlock;
        int32_t blk = 0;
        if (lane < nblk) {
          blk = table[j * (BN / kBlock) + lane];
          if (blk < 0 || blk >= a.num_blocks) {
            atomicOr(a.err, PA_DEVERR_BLOCK_ID);
            blk = 0;
          }
        }
        return blk;
      };
      auto load_k = [&](int j) {
        int nblk, valid;
        const int32_t blk = tile_blocks(j, nblk, valid);
        const int st = kc % NS;
        if (kc >= NS && !warp_wait_or_abort(bar(Cfg::BAR_KE + st), ((kc / NS) - 1) & 1, abort_flag))
          return false;
        if (lane == 0) mbar_arrive_expect_tx(bar(Cfg::BAR_KF + st), (uint32_t)nblk * KB * kBlock * 128);
        __syncwarp();
        if (lane < nblk) {  // K rows past the context are masked out of S by selection
          const int row0 = (int)(((int64_t)blk * a.heads + it.kvh) * kBlock);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sbase + Cfg::OFF_K + st * Cfg::KV_BYTES + kb * (BN * 128) + lane * (kBlock * 128),
                        &tm_k, kb * 64, row0, bar(Cfg::BAR_KF + st));
        }
        ++kc;
        return true;
      };
      auto load_v = [&](int j) {
        int nblk, valid;
        const int32_t blk = tile_blocks(j, nblk, valid);
        const int st = vc % NS;
        if (vc >= NS && !warp_wait_or_abort(bar(Cfg::BAR_VE + st), ((vc / NS) - 1) & 1, abort_flag))
          return false;
        // V rows at or past the context are zeroed (their weights are zero, but
        // stale bits may be NaN).  A partly filled last block's valid rows are
        // copied by the lanes, so every tensor copy moves a whole block.
        const bool partial = valid < nblk * kBlock;
        const int32_t last_blk = __shfl_sync(kFullMask, blk, nblk - 1);
        uint8_t* gV = smem + Cfg::OFF_V + st * Cfg::KV_BYTES;
        if (valid < BN) {
          const int r_lo = partial ? (nblk - 1) * kBlock : valid;
          const T* src = static_cast<const T*>(a.v_pool) +
                         (((int64_t)last_blk * a.heads + it.kvh) * kBlock) * D;
          for (int idx = lane; idx < (BN - r_lo) * KB * 8; idx += 32) {
            const int r = r_lo + idx / (KB * 8), c = idx % (KB * 8);
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < valid) v = *reinterpret_cast<const uint4*>(src + (int64_t)(r - r_lo) * D + c * 8);
            *reinterpret_cast<uint4*>(gV + (c >> 3) * (BN * 128) + sw128_off(r, c & 7)) = v;
          }
          fence_proxy_async_shared();
        }
        const int nfull = partial ? nblk - 1 : nblk;
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(bar(Cfg::BAR_VF + st), (uint32_t)nfull * KB * kBlock * 128);
        __syncwarp();
        if (lane < nfull) {
          const int row0 = (int)(((int64_t)blk * a.heads + it.kvh) * kBlock);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sbase + Cfg::OFF_V + st * Cfg::KV_BYTES + kb * (BN * 128) + lane * (kBlock * 128),
                        &tm_v, kb * 64, row0, bar(Cfg::BAR_VF + st));
        }
        ++vc;
        return true;
      };
      // Q of the item's query tiles, once the previous item's S products are
      // done with the Q buffers (rows past the tokens come in as zeros)
      if (items > 0 && !warp_wait_or_abort(bar(Cfg::BAR_QFREE), (items - 1) & 1, abort_flag)) {
        give_up();
        break;
      }
      if (lane == 0) {
        const int tiles = it.has1 ? 2 : 1;
        mbar_arrive_expect_tx(bar(Cfg::BAR_QF), (uint32_t)tiles * Cfg::Q_BYTES);
        for (int t = 0; t < tiles; ++t)
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sbase + Cfg::OFF_Q + t * Cfg::Q_BYTES + kb * (BM * 128), &tm_q, kb * 64,
                        it.hq, it.q0 + it.qt * 2 * BM + t * BM, bar(Cfg::BAR_QF));
      }
      __syncwarp();
      ++items;
      for (int t = 0; t <= it.nkt; ++t) {
        if ((t < it.nkt && !load_k(t)) || (t >= 1 && !load_v(t - 1))) {
          give_up();
          ok = false;
          break;
        }
      }
    }
    // let the last copies land before the CTA releases its memory
    if (lane == 0) {
      for (uint32_t j = kc > NS ? kc - NS : 0; j < kc; ++j)
        mbar_wait_bounded(bar(Cfg::BAR_KF + j % NS), (j / NS) & 1);
      for (uint32_t j = vc > NS ? vc - NS : 0; j < vc; ++j)
        mbar_wait_bounded(bar(Cfg::BAR_VF + j % NS), (j / NS) & 1);
      if (items > 0) mbar_wait_bounded(bar(Cfg::BAR_QF), (items - 1) & 1);
    }
  } else if (warp == Cfg::MMA_WARP) {
    // ---- MMA issue ------------------------------------------------------------------
    if (lane == 0) {
      // Descriptors are built once: an operand at a byte offset o from a
      // base differs only in the start-address field (o >> 4 added to the
      // low word; every address here stays inside that 14-bit field), so a
      // product costs one add per operand on the issuing thread, which
      // shares its sub-partition with two busy softmax warps.
      const uint64_t dq = sw128_desc(sbase + Cfg::OFF_Q, 16, 1024);
      const uint64_t dk = sw128_desc(sbase + Cfg::OFF_K, 16, 1024);
      const uint64_t dv = sw128_desc(sbase + Cfg::OFF_V, BN * 128, 1024);
      auto at = [](uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); };
      auto issue_s = [&](int w, int st) {
        const uint64_t qd = at(dq, w * Cfg::Q_BYTES), kd = at(dk, st * Cfg::KV_BYTES);
        const uint32_t sd = tmem + Cfg::S_COL0 + w * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kofs = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint32_t kofs_b = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
          umma_f16(sd, at(qd, kofs), at(kd, kofs_b), IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // P.V over the keys of P piece c of a tile
      auto issue_pv = [&](int w, int st, bool first, int c) {
        const uint32_t pa = tmem + Cfg::S_COL0 + w * BN;  // P over S, 8 columns per 16 keys
        const uint32_t od = tmem + Cfg::O_COL0 + w * D;
        const uint64_t vd = at(dv, st * Cfg::KV_BYTES);
#pragma unroll
        for (int kk = Cfg::piece_begin(c) / 16; kk < Cfg::piece_end(c) / 16; ++kk) {
          // V is MN-major: 64-dim blocks LBO apart, 8-key groups 1024 bytes apart
          const uint64_t bd = at(vd, kk * 2048);
          umma_f16_ts(od, pa + kk * 8, bd, IDESC_PV, (!first || kk > 0) ? 1u : 0u);
          if constexpr (kSplitP<T>) umma_f16_ts(od, pa + Cfg::P_LO + kk * 8, bd, IDESC_PV, 1u);
        }
      };
      // ring positions (counted across items) whose K / V stage was seen full
      int64_t k_ready = -1, v_ready = -1;
      auto wait_full = [&](int base, uint32_t pos, int64_t& ready) {
        if ((int64_t)pos <= ready) return true;
        if (!mbar_wait_or_abort(bar(base + pos % NS), (pos / NS) & 1, abort_flag)) return false;
        ready = pos;
        tc_fence_after();
        return true;
      };
      uint32_t kc = 0, vc = 0;    // K / V tiles consumed
      int items = 0;              // items started
      int pc[2] = {0, 0};         // p_full phases consumed, per query tile
      int ow[2] = {0, 0};         // items in which each query tile had work
      bool ok = true;
      for (int k = 0; ok && k < rounds; ++k) {
        const int w = nth_item(k);
        Item it;
        if (w >= num_items || !item_of(w, it, false)) continue;
        const int nkt = it.nkt;
        ok = mbar_wait_or_abort(bar(Cfg::BAR_QF), items & 1, abort_flag) &&
             wait_full(Cfg::BAR_KF, kc, k_ready);
        if (!ok) break;
        ++items;
        tc_fence_after();
        issue_s(0, kc % NS);
        umma_commit(bar(Cfg::BAR_S + 0));
        if (it.has1) {
          issue_s(1, kc % NS);
          umma_commit(bar(Cfg::BAR_S + 1));
        }
        umma_commit(bar(Cfg::BAR_KE + kc % NS));
        if (nkt == 1) umma_commit(bar(Cfg::BAR_QFREE));  // Q is no longer read
        for (int j = 0; ok && j < nkt; ++j) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int nk = t == 0 ? it.nkt0 : it.nkt1;
            if (j >= nk) continue;
            const uint32_t ph = pc[t] & 1;
            if (!(ok = mbar_wait_or_abort(bar(Cfg::BAR_P + t), ph, abort_flag) &&
                       wait_full(Cfg::BAR_VF, vc + j, v_ready)))
              break;
            ++pc[t];
            // the first P.V of an item overwrites O: its last reader must be done
            if (j == 0 && ow[t] > 0 &&
                !(ok = mbar_wait_or_abort(bar(Cfg::BAR_OFREE + t), (ow[t] - 1) & 1, abort_flag)))
              break;
            tc_fence_after();
            // P.V of each piece runs while the softmax finishes the next ones
            issue_pv(t, (vc + j) % NS, j == 0, 0);
#pragma unroll
            for (int c = 1; c < Cfg::PC; ++c) {
              if (!(ok = mbar_wait_or_abort(bar(Cfg::BAR_P + 2 * c + t), ph, abort_flag))) break;
              tc_fence_after();
              issue_pv(t, (vc + j) % NS, j == 0, c);
            }
            if (!ok) break;
            if (j == nk - 1) {
              umma_commit(bar(Cfg::BAR_O + t));
            } else {
              if (!(ok = wait_full(Cfg::BAR_KF, kc + j + 1, k_ready))) break;
              issue_s(t, (kc + j + 1) % NS);
              umma_commit(bar(Cfg::BAR_S + t));
            }
          }
          if (ok) {
            umma_commit(bar(Cfg::BAR_VE + (vc + j) % NS));
            if (j + 1 < nkt) umma_commit(bar(Cfg::BAR_KE + (kc + j + 1) % NS));
            if (j + 2 == nkt) umma_commit(bar(Cfg::BAR_QFREE));  // the item's last S are issued
          }
        }
        kc += nkt;
        vc += nkt;
        ow[0] += it.nkt0 > 0;
        ow[1] += it.nkt1 > 0;
      }
      if (!ok) give_up();
      // every product issued has completed before TMEM and shared memory go
      umma_commit(bar(Cfg::BAR_FIN));
      mbar_wait_bounded(bar(Cfg::BAR_FIN), 0);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Cfg::REGS_SOFTMAX));
    // ---- softmax warpgroups -----------------------------------------------------------
    const int w = warp >> 2, r = threadIdx.x & (BM - 1);
    const float sl2 = a.scale_log2;
    const float masked_raw = sl2 >= 0.f ? -INFINITY : INFINITY;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + Cfg::S_COL0 + w * BN;
    const uint32_t o_addr = tmem + lane_base + Cfg::O_COL0 + w * D;
    int sc_ph = 0, oc_ph = 0;  // s_full / o_done phases consumed (across items)
    bool ok = true;
    for (int k = 0; ok && k < rounds; ++k) {
      const int wi = nth_item(k);
      Item it;
      if (wi >= num_items || !item_of(wi, it, threadIdx.x == 0)) continue;
      const int qbase = it.qt * 2 * BM + w * BM;
      const int nk = w == 0 ? it.nkt0 : it.nkt1;
      if (nk == 0) continue;  // this query tile of the item holds no queries
      const int qi = qbase + r;
      const bool row_valid = qi < it.n;
      const int pos = it.L - it.n + qi;  // this query's position
      float m_used = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nk; ++j) {
        if (!(ok = warp_wait_or_abort(bar(Cfg::BAR_S + w), sc_ph & 1, abort_flag))) break;
        ++sc_ph;
        tc_fence_after();
        float2 sv[BN / 2];
        float* sc = reinterpret_cast<float*>(sv);
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 32) tmem_ld32_nowait(s_addr + c0, sc + c0);
        tmem_wait_ld();
        const bool need_mask = !row_valid || j * BN + BN - 1 > pos;
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (!row_valid || j * BN + c > pos) sc[c] = masked_raw;
        }
        // bf16: the row's max and its weights against the current reference
        // max are computed in one pass (the max on the ALU pipe while the
        // exp2s run on the multi-function unit); only if the max passed the
        // reference by more than 2^8 -- on a row's first tile, and rarely
        // after -- does the reference move and the warp redo the row from S,
        // still in TMEM.  That measured +19 % for bf16, whose high/residual
        // split keeps the ALU busiest, and -1 % for fp16, which finds the max
        // first.
        const float2 sl2v = make_float2(sl2, sl2);
        // weights of the keys [2 * i0, 2 * i1) against the reference max mb
        auto weights = [&](float mb, int i0, int i1) {
          const float2 nmb = make_float2(-mb, -mb);
#pragma unroll
          for (int i = i0; i < i1; ++i) {
            const float2 x = __ffma2_rn(sv[i], sl2v, nmb);
            sv[i] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          }
        };
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = sc[i];
        const bool ahead = kSplitP<T> && __all_sync(kFullMask, m_used != -INFINITY);
        // 8 chains, two scores folded in per three-input instruction
        if (sl2 >= 0.f) {
#pragma unroll
          for (int c = 8; c < BN; c += 2) mx8[(c >> 1) & 7] = fmax3f(mx8[(c >> 1) & 7], sc[c], sc[c + 1]);
        } else {
#pragma unroll
          for (int c = 8; c < BN; c += 2) mx8[(c >> 1) & 7] = fmin3f(mx8[(c >> 1) & 7], sc[c], sc[c + 1]);
        }
        if (ahead) weights(m_used, 0, BN / 2);  // independent of the max: overlaps it
#pragma unroll
        for (int i = 4; i >= 1; i >>= 1)
#pragma unroll
          for (int k = 0; k < i; ++k)
            mx8[k] = sl2 >= 0.f ? fmaxf(mx8[k], mx8[k + i]) : fminf(mx8[k], mx8[k + i]);
        const float m_tile = sl2 == 0.f ? 0.f : mx8[0] * sl2;
        // move the reference max only when a weight would exceed 2^8
        const bool move = m_tile > m_used + 8.f;
        const bool any_move = __any_sync(kFullMask, move);
        float alpha = 1.f;
        bool have_w = ahead;  // the weights above stand unless the reference moves
        if (any_move || !ahead) {
          if (move) {
            alpha = m_used == -INFINITY ? 0.f : ex2_approx(m_used - m_tile);
            m_used = m_tile;
          }
          if (ahead) {  // the weights above are stale: S again from TMEM
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 32) tmem_ld32_nowait(s_addr + c0, sc + c0);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int c = 0; c < BN; ++c)
                if (!row_valid || j * BN + c > pos) sc[c] = masked_raw;
            }
          }
          have_w = false;
        }
        const float mb = m_used == -INFINITY ? 0.f : m_used;
        // rescale this row of O before any P.V of this tile lands in it (P.V
        // of tile j-1 has completed: the product S of tile j was committed
        // after it)
        __syncwarp();
        if (j > 0 && any_move) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tmem_ld32(o_addr + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(o_addr + c0, o);
          }
        }
        // this row of P over S in TMEM, in PC pieces of BN/PC keys, each
        // handed to the MMA warp as soon as it is stored, so that P.V of one
        // piece runs while the next is computed.  Column c holds keys 2c (low
        // half) and 2c + 1; the S values were all read above.
        // the piece index is a compile-time constant, so every index into sc
        // is one and the row stays in registers
        auto piece = [&](auto pc_const) {
          constexpr int pi = decltype(pc_const)::value;
          constexpr int k0 = Cfg::piece_begin(pi), k1 = Cfg::piece_end(pi);
          if (!have_w) weights(mb, k0 / 2, k1 / 2);
          if (need_mask) {  // a zero scale keeps masked scores finite: select them out
#pragma unroll
            for (int c = k0; c < k1; ++c)
              if (!row_valid || j * BN + c > pos) sc[c] = 0.f;
          }
#pragma unroll
          for (int h = k0 / 32; h < k1 / 32; ++h) {
            if constexpr (kSplitP<T>) {
              uint32_t hi[16], lo[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pack_split<T>(sc[32 * h + 2 * i], sc[32 * h + 2 * i + 1], hi[i], lo[i]);
              tmem_st16_nowait(s_addr + Cfg::P_LO + 16 * h, lo);
              tmem_st16_nowait(s_addr + 16 * h, hi);
            } else {
              uint32_t hi[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                hi[i] = MmaType<T>::pack(sc[32 * h + 2 * i], sc[32 * h + 2 * i + 1]);
              tmem_st16_nowait(s_addr + 16 * h, hi);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(Cfg::BAR_P + 2 * pi + w));
        };
        piece(std::integral_constant<int, 0>{});
        if constexpr (Cfg::PC > 1) piece(std::integral_constant<int, 1>{});
        if constexpr (Cfg::PC > 2) {
          piece(std::integral_constant<int, 2>{});
          piece(std::integral_constant<int, 3>{});
        }
        // the row sum, off the path to P.V
        float2 sum4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sum4[i] = sv[i];
#pragma unroll
        for (int i = 4; i < BN / 2; ++i) sum4[i & 3] = __fadd2_rn(sum4[i & 3], sv[i]);
        sum4[0] = __fadd2_rn(__fadd2_rn(sum4[0], sum4[1]), __fadd2_rn(sum4[2], sum4[3]));
        l_run = fmaf(l_run, alpha, sum4[0].x + sum4[0].y);
      }
      if (ok) ok = warp_wait_or_abort(bar(Cfg::BAR_O + w), oc_ph & 1, abort_flag);
      if (!ok) break;
      ++oc_ph;
      tc_fence_after();
      // ---- O / l for this row, then O is free for the next item -------------------------
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      T* dst = static_cast<T*>(a.out) + ((int64_t)(it.q0 + qi) * HQ + it.hq) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tmem_ld32(o_addr + c0, o);
        if (row_valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v;
            v.x = MmaType<T>::pack(o[i] * inv, o[i + 1] * inv);
            v.y = MmaType<T>::pack(o[i + 2] * inv, o[i + 3] * inv);
            v.z = MmaType<T>::pack(o[i + 4] * inv, o[i + 5] * inv);
            v.w = MmaType<T>::pack(o[i + 6] * inv, o[i + 7] * inv);
            *reinterpret_cast<uint4*>(dst + c0 + i) = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(Cfg::BAR_OFREE + w));
    }
    if (!ok) give_up();
  }
  // every role is done and every copy or product it issued has landed
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace pa
