// Paged decode attention for sm_100a: partition kernel and split-K merge (the
// arguments and the work plan are in plan.cuh).
//
// The method: "PagedAttention" (e-fortepiano.pl wiki mirror), "Formulació
// matemàtica" -- the attention of one query token, computed block by block
// over KV blocks reached through the sequence's block table, equals the
// ordinary softmax(q.K^T * scale).V over the cached tokens.  Block table and
// 16-token pages: "Atención paginada en modelos de lenguaje grandes (LLM)"
// (7minutos.es), section 2.
//
// Design (ours; the pages give no kernel):
//   * The unit of work is (sequence s, partition p of partition_size tokens,
//     group g of WARPS heads).  One warp owns one head of the group, so the
//     warps of a CTA share the block-table slice and read adjacent 4 KB tiles
//     of the same physical block.
//   * Each warp runs its own NSTAGE-deep ring of shared-memory stages.  Lane
//     0 issues two 1-D bulk copies per stage (the K and V tiles of one
//     (block, head), contiguous in the [block][head][slot][dim] layout) that
//     complete on that stage's mbarrier; no multicast, no tensor map.
//   * q.k: lane l reads 16-byte chunks l, l+32, ... of the tile from shared
//     memory (512 contiguous bytes per warp instruction, conflict free); a
//     transpose-reduce over the lanes of a row leaves every lane with one
//     token's score in NCH shuffles instead of NCH*log2(LPR).
//   * fp32 online softmax in the log2 domain (q is pre-scaled by
//     scale*log2(e)); P.V accumulates in fp32 registers.
//   * Work items are handed out by an atomic counter in the workspace, in the
//     order a one-CTA plan kernel wrote: the ragged last partitions of split
//     sequences, the full partitions, then the unsplit sequences by
//     decreasing size, so the merges fall mid-launch and the tail of the
//     grid is made of the smallest items, which merge nothing.
//   * Sequences with more than one partition write (m, l, unnormalised acc)
//     per partition and bump a per-(sequence, head group) arrival counter;
//     the CTA that arrives last merges all partitions by log-sum-exp in
//     partition order and re-arms the counter (no second kernel).  No
//     atomics touch values, so results are bit-stable run to run and
//     independent of where the blocks sit in the pool.
//   * Optional fused append: with k_new/v_new given, the CTA that owns a
//     sequence's last block writes the new token's K/V row into the pool
//     (what reshape_and_cache would do) and patches the same row of its
//     shared-memory copy of the tile, so one launch appends and attends.
#pragma once

#include <math.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "pagedattn.h"
#include "plan.cuh"

namespace pa {

// ---- transpose-reduce of NCH partial dot products over LPR lanes --------------------
// Step with xor-mask M halves the values a lane carries: the lane keeps one
// half and adds its partner's copy of that half.  After log2(NCH) steps one
// value is left, summed over NCH lanes; a last xor-1 step completes the row.

template <int M, int N>
__device__ __forceinline__ void halve(float* v, int lane) {
  if constexpr (M >= 2) {
    const bool upper = (lane & M) != 0;
#pragma unroll
    for (int k = 0; k < N / 2; ++k) {
      const float send = upper ? v[k] : v[k + N / 2];
      const float keep = upper ? v[k + N / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(kFullMask, send, M);
    }
    halve<M / 2, N / 2>(v, lane);
  }
}

// ---- the partition kernel -----------------------------------------------------------

// G = query heads per KV head that share one ring: the G warps of a ring
// read the same staged (block, KV head) tile, each with its own query head.
template <typename T, int D, int WARPS, int NSTAGE, int G>
struct DecodeConfig {
  static constexpr int VEC = Chunk<T>::N;      // elements per 16-byte chunk
  static constexpr int CPR = D / VEC;          // chunks (= lanes) per token row
  static constexpr int RPI = 32 / CPR;         // rows covered by one warp-wide load
  static constexpr int NCH = kBlock / RPI;     // chunks per lane per tile
  static constexpr int TILE = kBlock * D * (int)sizeof(T);  // one (block, head) tile
  static constexpr int STAGE_BYTES = 2 * TILE;              // K tile + V tile
  static constexpr int THREADS = WARPS * 32;
  static constexpr int RINGS = WARPS / G;      // KV heads per work item
  static_assert(CPR >= 2 && CPR <= 32 && 32 % CPR == 0, "head_dim / dtype not supported");
  static_assert(NCH * 2 == CPR, "lane mapping");
  static_assert(WARPS % G == 0 && RINGS >= 1, "a ring's warps must fit the CTA");
  // stage rings + one mbarrier per stage + the item's block-table slice
  static size_t smem_bytes(int partition_size) {
    return (size_t)RINGS * NSTAGE * STAGE_BYTES + (size_t)RINGS * NSTAGE * 8 +
           (size_t)(partition_size / kBlock) * 4;
  }
};

// Barrier over the G warps of ring r (named barrier 1 + r); returns whether
// every participating thread passed ok.  With G == 1 it is a warp vote.
template <int G>
__device__ __forceinline__ bool ring_vote(int r, bool ok) {
  if constexpr (G == 1) {
    return __all_sync(kFullMask, ok);
  } else {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)ok), "r"(1 + r), "r"(G * 32)
        : "memory");
    return res != 0;
  }
}

template <int G>
__device__ __forceinline__ void ring_sync(int r) {
  if constexpr (G == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + r), "r"(G * 32) : "memory");
  }
}

// Merge the partitions of (sequence s, head h) by log-sum-exp, in partition
// order, and write the normalised output.  The max over the partitions is
// read by all 32 lanes at once (every 32nd partition each, then combined:
// max is exact, so the split changes no bit); then lanes < CPR each own one
// 16-byte output chunk.  Partials are read with .cg loads (L2), since other
// CTAs wrote them during this launch.  Called by all 32 lanes of the warp.
template <typename T, int D>
__device__ __forceinline__ void merge_partitions(const DecodeArgs& a, int64_t sh, int np, int lane) {
  using C = Chunk<T>;
  constexpr int VEC = C::N;
  constexpr int CPR = D / VEC;
  const float2* ml = a.part_ml + sh * a.max_parts;
  float M = -INFINITY;
  for (int p = lane; p < np; p += 32) M = fmaxf(M, __ldcg(&ml[p]).x);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, m));
  if (lane >= CPR) return;
  float den = 0.f;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  const float* base = a.part_acc + sh * a.max_parts * D + lane * VEC;
#pragma unroll 4
  for (int p = 0; p < np; ++p) {
    const float2 v = __ldcg(&ml[p]);
    const float w = exp2f(v.x - M);
    den = fmaf(v.y, w, den);
    const float4* src = reinterpret_cast<const float4*>(base + (int64_t)p * D);
#pragma unroll
    for (int e = 0; e < VEC; e += 4) {
      const float4 x = __ldcg(src + e / 4);
      acc[e] = fmaf(w, x.x, acc[e]);
      acc[e + 1] = fmaf(w, x.y, acc[e + 1]);
      acc[e + 2] = fmaf(w, x.z, acc[e + 2]);
      acc[e + 3] = fmaf(w, x.w, acc[e + 3]);
    }
  }
  const float inv = 1.f / den;
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] *= inv;
  reinterpret_cast<uint4*>(static_cast<T*>(a.out) + sh * D)[lane] = C::from_float(acc);
}

// Four or two consecutive output values of one lane, rounded like Chunk<T>.
template <typename T, int N>
__device__ __forceinline__ void store_out(T* dst, const float* v) {
  if constexpr (sizeof(T) == 4) {
    if constexpr (N == 4) *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
  } else {
    float f[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = e < N ? v[e] : 0.f;
    const uint4 u = Chunk<T>::from_float(f);  // pairs rounded as in a full chunk
    if constexpr (N == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(u.x, u.y);
    else *reinterpret_cast<uint32_t*>(dst) = u.x;
  }
}

// The merge of merge_partitions for a warp that owns a bulk-copy ring (one
// query head per ring): the partial rows come into the ring buffer `buf` by
// one bulk copy per round of up to BUF / (4 D) partitions, while the lanes
// read the (m, l) pairs (one partition per lane) and the max; every lane then
// owns D/32 output values.  About one memory round trip per round instead of
// one per few partitions.  Rounds complete on the ring's barriers as ring
// fills, the first being fill number `fill0`.  Per element the arithmetic and
// its order are those of merge_partitions, so the results are the same bits.
// Returns the number of fills used, negated if a copy did not land in time
// (nothing is written then).
template <typename T, int D, int NSTAGE, int BUF>
__device__ __forceinline__ int merge_staged(const DecodeArgs& a, int64_t sh, int np, int lane,
                                            uint8_t* buf, uint64_t* bars, uint32_t fill0) {
  constexpr int ROW = D * 4;                        // one partial row, fp32
  constexpr int PC = BUF / ROW < 32 ? BUF / ROW : 32;  // partitions per round
  constexpr int DPL = D / 32;                        // output values per lane
  static_assert(PC >= 1 && (DPL == 4 || DPL == 2), "merge layout");
  const float2* ml = a.part_ml + sh * a.max_parts;
  const float* acc_src = a.part_acc + sh * a.max_parts * D;
  auto issue = [&](int p0, int n, uint32_t k) {
    __syncwarp();  // every lane is done reading buf
    if (lane == 0) {
      const uint32_t bar = smem_addr(&bars[k % NSTAGE]);
      fence_proxy_async_shared();
      fence_proxy_async_global();  // partials other CTAs wrote, seen through the arrival count
      mbar_arrive_expect_tx(bar, (uint32_t)(n * ROW));
      bulk_copy_g2s(smem_addr(buf), acc_src + (int64_t)p0 * D, (uint32_t)(n * ROW), bar);
    }
  };
  uint32_t k = fill0;
  issue(0, min(PC, np), k);
  float M = -INFINITY;
  for (int p = lane; p < np; p += 32) M = fmaxf(M, __ldcg(&ml[p]).x);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, m));
  float den = 0.f;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  bool ok = true;
  for (int p0 = 0; p0 < np; p0 += PC) {
    const int n = min(PC, np - p0);
    const float2 v = lane < n ? __ldcg(&ml[p0 + lane]) : make_float2(0.f, 0.f);
    if (p0 > 0) issue(p0, n, ++k);
    if (!__all_sync(kFullMask, mbar_wait_bounded(smem_addr(&bars[k % NSTAGE]), (k / NSTAGE) & 1u))) {
      ok = false;
      break;
    }
    for (int p = 0; p < n; ++p) {
      const float vx = __shfl_sync(kFullMask, v.x, p), vy = __shfl_sync(kFullMask, v.y, p);
      const float w = exp2f(vx - M);
      den = fmaf(vy, w, den);
      const float* src = reinterpret_cast<const float*>(buf + p * ROW) + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, src[e], acc[e]);
    }
  }
  const int used = (int)(k - fill0) + 1;
  if (!ok) {
    mbar_wait_bounded(smem_addr(&bars[k % NSTAGE]), (k / NSTAGE) & 1u);  // let the copy land
    return -used;
  }
  const float inv = 1.f / den;
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] *= inv;
  store_out<T, DPL>(static_cast<T*>(a.out) + sh * D + lane * DPL, acc);
  __syncwarp();  // buf is read before the ring's next fill
  return used;
}

// The persistent partition kernel: CTAs pull (sequence, partition, head
// group) items from the plan's queue.  Each ring of G warps streams one KV
// head of the item through NSTAGE stages of bulk copies; each warp of the
// ring attends with its own query head (G == 1: one warp per head).
template <typename T, int D, int WARPS, int NSTAGE, int G>
__global__ void __launch_bounds__(WARPS * 32) paged_decode_kernel(DecodeArgs a) {
  using Cfg = DecodeConfig<T, D, WARPS, NSTAGE, G>;
  using C = Chunk<T>;
  constexpr int VEC = Cfg::VEC, CPR = Cfg::CPR, RPI = Cfg::RPI, NCH = Cfg::NCH;
  constexpr int TILE = Cfg::TILE, RINGS = Cfg::RINGS;

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RINGS * NSTAGE * Cfg::STAGE_BYTES);
  int32_t* tbl = reinterpret_cast<int32_t*>(bars + RINGS * NSTAGE);
  __shared__ int32_t s_item;
  __shared__ int32_t s_abort;
  __shared__ int32_t s_merge;
  __shared__ int32_t s_plan_ok;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ring = warp / G;            // which KV head of the item this warp serves
  const bool leader = (warp % G) == 0;  // lane 0 of the leader warp issues the ring's copies
  const int HK = a.heads;               // KV heads
  const int HQ = a.heads * G;           // query heads
  const int PS = a.partition_size;

  // launched right behind its plan (one call that plans and runs): the CTAs
  // set up while the plan kernel runs, and wait for it here
  if (a.after_plan) grid_dependency_wait();
  int32_t next = -1;  // thread 0: the next item, once reserved
  if (threadIdx.x == 0) {
    for (int i = 0; i < RINGS * NSTAGE; ++i) mbar_init(smem_addr(&bars[i]), 1);
    mbar_init_fence();
    s_abort = 0;
    // a plan that is not this launch's, or that an earlier launch gave up
    // on, is not run: nothing in the workspace is touched
    s_plan_ok = plan_header_ok(a);
    if (s_plan_ok) next = atomicAdd(&a.plan->work_counter, 1);
    else atomicOr(a.err, PA_DEVERR_PLAN);
  }
  __syncthreads();
  if (!s_plan_ok) return;
  const int32_t num_items = a.plan->num_items;

  uint32_t fills = 0;  // stage fills this ring has consumed so far (drives ring slot + parity)
  uint8_t* my_stages = stages + ring * NSTAGE * Cfg::STAGE_BYTES;
  uint64_t* my_bars = bars + ring * NSTAGE;

  for (;;) {
    if (threadIdx.x == 0) {  // reserved near the end of the previous item, else taken now
      s_item = next >= 0 ? next : atomicAdd(&a.plan->work_counter, 1);
      next = -1;
    }
    __syncthreads();
    const int item = s_item;
    if (item >= num_items || s_abort) break;

    PlanItem it;
    if (!plan_item(a, item, &it)) {  // a damaged plan entry: report and skip the item
      if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_PLAN);
      __syncthreads();
      continue;
    }
    const int g = item % a.head_groups;
    const int s = it.s, p = it.p, L = it.L, np = it.np, ni = it.ni;
    const bool split = np > 1;
    const int tok0 = it.base + p * PS;
    const int ntok = max(0, min(L, tok0 + PS) - tok0);
    const int nblk = (ntok + kBlock - 1) / kBlock;
    const int blk0 = tok0 / kBlock;
    // the item holding the sequence's last token appends the new one (fused mode)
    const bool append = a.k_new != nullptr && L > 0 && p == ni - 1 && tok0 + ntok == L;
    const int new_row = (L - 1) % kBlock;  // in-block offset of the appended token

    // block-table slice of this partition, bounds-checked once
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
      int32_t b = a.block_tables[(int64_t)s * a.max_blocks_per_seq + blk0 + i];
      if (b < 0 || b >= a.num_blocks) {
        atomicOr(a.err, PA_DEVERR_BLOCK_ID);
        b = 0;
      }
      tbl[i] = b;
    }
    __syncthreads();

    const int kvh = g * RINGS + ring;          // KV head
    const int hq = kvh * G + (warp % G);       // this warp's query head
    if (kvh < HK) {
      const int c = lane % CPR;  // this lane's chunk within a token row
      const int64_t sh = (int64_t)s * HQ + hq;
      float qf[VEC];
      {
        const uint4 u = reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) + sh * D)[c];
        C::to_float(u, qf);
#pragma unroll
        for (int e = 0; e < VEC; ++e) qf[e] *= a.scale_log2;
      }
      float m_run = -INFINITY, l_run = 0.f;
      float acc[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] = 0.f;

      const char* kbase = static_cast<const char*>(a.k_pool) + (int64_t)kvh * TILE;
      const char* vbase = static_cast<const char*>(a.v_pool) + (int64_t)kvh * TILE;
      const int64_t block_bytes = (int64_t)HK * TILE;
      auto issue = [&](uint32_t k, int bi) {
        const int st = k % NSTAGE;
        const uint32_t bar = smem_addr(&my_bars[st]);
        uint8_t* dst = my_stages + st * Cfg::STAGE_BYTES;
        const int64_t off = (int64_t)tbl[bi] * block_bytes;
        mbar_arrive_expect_tx(bar, 2 * TILE);
        bulk_copy_g2s(smem_addr(dst), kbase + off, TILE, bar);
        bulk_copy_g2s(smem_addr(dst + TILE), vbase + off, TILE, bar);
      };

      const uint32_t k0 = fills;
      if (leader && lane == 0) {
        fence_proxy_async_shared();  // the previous item's reads of these stages are done
        for (int j = 0; j < NSTAGE && j < nblk; ++j) issue(k0 + j, j);
      }
      // rows this lane reads: r_j = lane / CPR + RPI * j; score row after the reduce:
      const int my_row = lane / CPR + RPI * ((lane % CPR) >> 1);
      bool ok = true;
      int i = 0;
      for (; i < nblk; ++i) {
        const uint32_t k = k0 + i;
        const int st = k % NSTAGE;
        const bool landed = mbar_wait_bounded(smem_addr(&my_bars[st]), (k / NSTAGE) & 1u);
        uint4* kt = reinterpret_cast<uint4*>(my_stages + st * Cfg::STAGE_BYTES);
        uint4* vt = kt + TILE / 16;
        const int valid = min(kBlock, ntok - i * kBlock);
        if (append && i == nblk - 1 && leader && __all_sync(kFullMask, landed)) {
          // fused reshape_and_cache: the new token's row goes to the pool and
          // replaces the stale row of the staged tile (before the ring reads it)
          if (lane < CPR) {
            const int64_t skv = (int64_t)s * HK + kvh;
            const uint4 kn = reinterpret_cast<const uint4*>(static_cast<const T*>(a.k_new) + skv * D)[lane];
            const uint4 vn = reinterpret_cast<const uint4*>(static_cast<const T*>(a.v_new) + skv * D)[lane];
            kt[new_row * CPR + lane] = kn;
            vt[new_row * CPR + lane] = vn;
            const int64_t row_off = (int64_t)tbl[i] * block_bytes + (int64_t)new_row * (TILE / kBlock);
            reinterpret_cast<uint4*>(const_cast<char*>(kbase) + row_off)[lane] = kn;
            reinterpret_cast<uint4*>(const_cast<char*>(vbase) + row_off)[lane] = vn;
          }
          __syncwarp();
        }
        if (!ring_vote<G>(ring, landed)) {  // the ring gives up together
          ok = false;
          break;
        }

        float part[NCH];
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          float kf[VEC];
          C::to_float(kt[lane + 32 * j], kf);
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; ++e) d = fmaf(qf[e], kf[e], d);
          part[j] = d;
        }
        halve<CPR / 2, NCH>(part, lane);
        float sc = part[0] + __shfl_xor_sync(kFullMask, part[0], 1);
        if (my_row >= valid) sc = -INFINITY;

        float bmax = sc;
#pragma unroll
        for (int m = 2; m < 32; m <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFullMask, bmax, m));
        const float m_new = fmaxf(m_run, bmax);
        const float alpha = exp2f(m_run - m_new);
        const float pw = exp2f(sc - m_new);
        float bsum = pw;
#pragma unroll
        for (int m = 2; m < 32; m <<= 1) bsum += __shfl_xor_sync(kFullMask, bsum, m);
        l_run = fmaf(l_run, alpha, bsum);
        m_run = m_new;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] *= alpha;

#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          const float pj = __shfl_sync(kFullMask, pw, (lane / CPR) * CPR + 2 * j);
          float vf[VEC];
          C::to_float(vt[lane + 32 * j], vf);
          if (valid < kBlock && lane / CPR + RPI * j >= valid) continue;  // slot past the end
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] = fmaf(pj, vf[e], acc[e]);
        }
        ring_sync<G>(ring);  // every warp of the ring is done with this stage
        if (leader && lane == 0 && i + NSTAGE < nblk) {
          fence_proxy_async_shared();
          issue(k + NSTAGE, i + NSTAGE);
        }
        // The next item is reserved four tiles before this one ends: late enough
        // that the queue's last items go to the CTAs that free up first (an
        // item reserved at the start of the current one waited out all of
        // it, and CTAs that drew the end of the queue sat idle meanwhile),
        // early enough that the atomic's round trip is hidden.
        if (threadIdx.x == 0 && i == max(nblk - 5, 0)) next = atomicAdd(&a.plan->work_counter, 1);
      }
      if (!ok) {
        // give up on this item: report, let the copies already issued land,
        // stop the CTA, and mark the plan so that no merge trusts its
        // counters again until it is rewritten
        if (lane == 0) {
          atomicOr(a.err, PA_DEVERR_TIMEOUT);
          s_abort = 1;
          a.plan->poisoned = 1;
          __threadfence();
        }
        const int issued = min(nblk, i + NSTAGE);
        for (int j = i; j < issued; ++j) {
          const uint32_t k = k0 + j;
          mbar_wait_bounded(smem_addr(&my_bars[k % NSTAGE]), (k / NSTAGE) & 1u);
        }
      } else {
        fills = k0 + nblk;
        // combine the RPI lanes that hold the same chunk (different rows)
#pragma unroll
        for (int m = CPR; m < 32; m <<= 1) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(kFullMask, acc[e], m);
        }
        if (lane < CPR) {
          if (!split) {
            float o[VEC];
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) o[e] = l_run > 0.f ? acc[e] * inv : 0.f;
            reinterpret_cast<uint4*>(static_cast<T*>(a.out) + sh * D)[c] = C::from_float(o);
          } else {
            float4* dst = reinterpret_cast<float4*>(a.part_acc + (sh * a.max_parts + p) * D + c * VEC);
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
              dst[e / 4] = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
            if (lane == 0) a.part_ml[sh * a.max_parts + p] = make_float2(m_run, l_run);
          }
        }
      }
    }
    if (split) {
      // count this partition in; the last of the sequence's partitions merges.
      // The barrier orders every warp's partial stores before thread 0's
      // gpu-scope fence, which publishes them before the arrival count.
      __syncthreads();
      if (threadIdx.x == 0) {
        int32_t* cnt = a.merge_cnt + (int64_t)s * a.head_groups + g;
        __threadfence();
        const int arrived = atomicAdd(cnt, 1) + 1;  // own partitions only
        __threadfence();
        // no merge once any CTA of this launch gave up (its partial may be missing)
        s_merge = arrived == ni && !s_abort && *(volatile int32_t*)&a.plan->poisoned == 0;
        if (arrived == ni) *cnt = 0;  // re-arm for the next launch on this plan
      }
      __syncthreads();
      if (s_merge && kvh < HK) {
        // shared-prefix partials come from the preceding launch, which this
        // one may overlap (programmatic dependent launch): wait for it to
        // complete before reading them (returns at once otherwise)
        if (np > ni) grid_dependency_wait();
        __threadfence();
        if constexpr (G == 1) {
          // one query head per ring: the partials come through the warp's ring
          constexpr int BUF = NSTAGE * Cfg::STAGE_BYTES;
          const int used =
              merge_staged<T, D, NSTAGE, BUF>(a, (int64_t)s * HQ + hq, np, lane, my_stages, my_bars, fills);
          fills += used > 0 ? used : -used;
          if (used < 0 && lane == 0) {  // as for a copy of the item: report, stop, poison the plan
            atomicOr(a.err, PA_DEVERR_TIMEOUT);
            s_abort = 1;
            a.plan->poisoned = 1;
            __threadfence();
          }
        } else {
          merge_partitions<T, D>(a, (int64_t)s * HQ + hq, np, lane);
        }
      }
    }
    __syncthreads();
  }

  // the last CTA out re-arms the queue so the plan can be reused
  if (threadIdx.x == 0) {
    __threadfence();
    const int done = atomicAdd(&a.plan->done_counter, 1);
    if (done == (int)gridDim.x - 1) {
      a.plan->work_counter = 0;
      a.plan->done_counter = 0;
      __threadfence();
    }
  }
}

}  // namespace pa
