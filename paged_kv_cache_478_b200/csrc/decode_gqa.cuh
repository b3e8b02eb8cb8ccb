// Grouped-query decode on tensor cores (fp16 / bf16 pools).
//
// With G query heads per KV head, each staged (block, KV head) tile serves G
// queries: per 16-token block that is a [G x D] . [D x 16] score product and
// a [G x 16] . [16 x D] value product, i.e. two m16n8k16 chains with the G
// query heads as the rows.  Two warps own one KV head of the work item and
// all of its query heads (each half of the partition's blocks, states
// combined at the end), so the CUDA-core cost per byte no longer grows
// with G.  With bf16 the softmax weights enter P.V as a high part plus its
// rounding residual (8 significand bits alone would cost the result
// precision); fp16 weights go in as they are.  The running max only moves,
// and the accumulators are only rescaled, when a score passes it by more than
// 2^8, so the rescale is rare and the weights stay at most 256.  The pipeline
// is the MHA kernel's: a per-warp NSTAGE ring on mbarriers, items from the
// plan's queue, split-K partials merged by the last CTA to finish a
// sequence, optional fused append.
// Staging: each (block, KV head) tile of K and of V arrives whole, as D/64
// tiled tensor copies of one 16-row x 128-byte box each (the pool viewed as
// [blocks * heads * 16 rows][head_dim]), written with 128-byte swizzle so the
// ldmatrix reads of the products are free of bank conflicts.  Four copies per
// block at head_dim 128, issued by one lane.  V rows past the end of a ragged
// block (stale, possibly NaN) are zeroed in shared memory after they land,
// so they never reach the product; K rows there only produce scores that are
// masked out.
#pragma once

#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "decode.cuh"
#include "device_utils.cuh"
#include "mma_utils.cuh"
#include "tma.cuh"

namespace pa {

#ifndef PA_GQA_WARPS
#define PA_GQA_WARPS 4
#endif

template <typename T, int D, int NSTAGE>
struct GqaConfig {
  static constexpr int WARPS = PA_GQA_WARPS;  // warps per CTA, two per KV head of the work item
  static_assert(WARPS == 2 || WARPS == 4, "warps per CTA");
  static constexpr int KVPI = WARPS / 2;      // KV heads per work item
  static constexpr int THREADS = WARPS * 32;
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int BOXES = D / 64;              // 64-wide slices of head_dim
  static constexpr int BOX_BYTES = kBlock * 128;    // 16 rows x 128 bytes, swizzled
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile + V tile
  static_assert(BOX_BYTES % 1024 == 0, "swizzled boxes start 1024-byte aligned");
  // 1 KB of slack to align the stages, the stages, one mbarrier per stage,
  // and the item's block-table slice
  static size_t smem_bytes(int partition_size) {
    return 1024 + (size_t)WARPS * NSTAGE * STAGE_BYTES + (size_t)WARPS * NSTAGE * 8 +
           (size_t)(partition_size / kBlock) * 4;
  }
};

// Merge the partitions of all G query heads of one KV head (query heads
// sh0 .. sh0+G-1) with one warp: 32/G lanes per query head, each lane owning
// D*G/32 output dimensions, so the G merges run side by side.  A lane owns
// every (32/G)-th 16-byte chunk of its head's row, so that one load
// instruction of the warp reads whole 128-byte lines of the staged rows; with
// 8 heads (64 bytes per head and instruction) the odd heads take their
// chunks in the opposite order of each pair, so that the 8 heads fill all 32
// banks and no two lanes meet in one.  The partial
// rows are staged through the warp's ring buffer `buf` by bulk copies, PC
// partitions of every head per round (one copy per head and round, all in
// flight at once), and the (m, l) pairs of a round are loaded while the
// copies fly: a merge costs about one memory round trip per round instead
// of one per partition.  Rounds complete on the ring's barriers as ring
// fills (`fills` counts them).  Per element the arithmetic and its order are
// those of merge_partitions (max over the partitions, then the weighted sums
// in partition order), so the results are the same bits.  Returns false if
// a copy did not land in time (nothing is written then).
template <typename T, int D, int G, int NSTAGE, int BUF>
__device__ __forceinline__ bool merge_group(const DecodeArgs& a, int64_t sh0, int np, int lane,
                                            uint8_t* buf, uint64_t* bars, uint32_t& fills) {
  constexpr int LPH = 32 / G;        // lanes per query head
  constexpr int DPL = D / LPH;       // output dimensions per lane
  constexpr int ROW = D * 4;         // one partial row, fp32
  constexpr int PC = BUF / (G * ROW);  // partitions per round
  constexpr int CPL = DPL / 4;        // 16-byte chunks per lane
  static_assert(DPL % 4 == 0, "a lane owns whole 16-byte chunks");
  static_assert(PC >= 1, "the ring holds one partition of every head");
  static_assert(LPH * 16 >= 64 && (LPH * 16 >= 128 || CPL % 2 == 0), "bank layout of the staged rows");
  const int j = lane / LPH;
  const int64_t sh = sh0 + j;
  // chunk of acc[4e .. 4e+3]: cl + LPH * (e ^ flip)
  const int cl = lane % LPH;
  const int flip = LPH * 16 < 128 ? (j & 1) : 0;
  const float2* ml = a.part_ml + sh * a.max_parts;

  // one round: lane 0 copies partitions [p0, p0 + n) of every head into buf
  auto issue = [&](int p0, int n, uint32_t k) {
    __syncwarp();  // every lane is done reading buf
    if (lane == 0) {
      const uint32_t bar = smem_addr(&bars[k % NSTAGE]);
      fence_proxy_async_shared();
      fence_proxy_async_global();  // partials other CTAs wrote, seen through the arrival count
      mbar_arrive_expect_tx(bar, (uint32_t)(G * n * ROW));
#pragma unroll
      for (int h = 0; h < G; ++h)
        bulk_copy_g2s(smem_addr(buf + h * PC * ROW),
                      a.part_acc + ((sh0 + h) * a.max_parts + p0) * D, (uint32_t)(n * ROW), bar);
    }
  };
  int n0 = min(PC, np);
  uint32_t k = fills++;
  issue(0, n0, k);

  // the max over the partitions while the first round flies: the head's LPH
  // lanes read every LPH-th partition, then combine (max is exact)
  float M = -INFINITY;
#pragma unroll 4
  for (int p = lane % LPH; p < np; p += LPH) M = fmaxf(M, __ldcg(&ml[p]).x);  // loads in flight together
#pragma unroll
  for (int m = 1; m < LPH; m <<= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, m));

  float den = 0.f;
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  bool ok = true;
  for (int p0 = 0; p0 < np; p0 += PC) {
    const int n = min(PC, np - p0);
    float2 v[PC];
#pragma unroll
    for (int p = 0; p < PC; ++p) v[p] = p < n ? __ldcg(&ml[p0 + p]) : make_float2(0.f, 0.f);
    if (p0 > 0) {
      k = fills++;
      issue(p0, n, k);
    }
    if (!__all_sync(kFullMask, mbar_wait_bounded(smem_addr(&bars[k % NSTAGE]), (k / NSTAGE) & 1u))) {
      ok = false;
      break;
    }
#pragma unroll
    for (int p = 0; p < PC; ++p) {
      if (p < n) {
        const float w = exp2f(v[p].x - M);
        den = fmaf(v[p].y, w, den);
        const float4* src = reinterpret_cast<const float4*>(buf + (j * PC + p) * ROW) + cl;
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
          const float4 x = src[LPH * (e ^ flip)];
          acc[4 * e] = fmaf(w, x.x, acc[4 * e]);
          acc[4 * e + 1] = fmaf(w, x.y, acc[4 * e + 1]);
          acc[4 * e + 2] = fmaf(w, x.z, acc[4 * e + 2]);
          acc[4 * e + 3] = fmaf(w, x.w, acc[4 * e + 3]);
        }
      }
    }
  }
  if (!ok) {
    mbar_wait_bounded(smem_addr(&bars[k % NSTAGE]), (k / NSTAGE) & 1u);  // let the copies land
    return false;
  }
  const float inv = 1.f / den;
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] *= inv;
  uint2* dst = reinterpret_cast<uint2*>(static_cast<T*>(a.out) + sh * D) + cl;
#pragma unroll
  for (int e = 0; e < CPL; ++e)
    dst[LPH * (e ^ flip)] = make_uint2(MmaType<T>::pack(acc[4 * e], acc[4 * e + 1]),
                                       MmaType<T>::pack(acc[4 * e + 2], acc[4 * e + 3]));
  __syncwarp();  // buf is read before the ring's next fill
  return true;
}

// tm_k, tm_v: the K and V pools as [num_blocks * heads * 16 rows][head_dim],
// box {64, 16}, 128-byte swizzle.
template <typename T, int D, int NSTAGE>
__global__ void __launch_bounds__(128, 3)  // 3 CTAs per SM: at most 168 registers a thread
    paged_decode_gqa_kernel(DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v) {
  using Cfg = GqaConfig<T, D, NSTAGE>;
  constexpr int KSTEPS = D / 16;
  constexpr int NT = D / 8;
  constexpr int WARPS = Cfg::WARPS;

  extern __shared__ __align__(1024) uint8_t gqa_smem[];
  uint8_t* smem = gqa_smem + ((1024u - (smem_addr(gqa_smem) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WARPS * NSTAGE * Cfg::STAGE_BYTES);
  int32_t* tbl = reinterpret_cast<int32_t*>(bars + WARPS * NSTAGE);
  __shared__ int32_t s_item;
  __shared__ int32_t s_abort;
  __shared__ int32_t s_merge;
  __shared__ int32_t s_plan_ok;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = a.q_per_kv;  // query heads per KV head, <= 8
  const int HK = a.heads, HQ = a.heads * G;
  const int PS = a.partition_size;

  // launched right behind its plan (one call that plans and runs): the CTAs
  // set up while the plan kernel runs, and wait for it here
  if (a.after_plan) grid_dependency_wait();
  int32_t next = -1;  // thread 0: the next item, once reserved
  if (threadIdx.x == 0) {
    for (int i = 0; i < WARPS * NSTAGE; ++i) mbar_init(smem_addr(&bars[i]), 1);
    mbar_init_fence();
    s_abort = 0;
    s_plan_ok = plan_header_ok(a);  // see the MHA kernel
    if (s_plan_ok) next = atomicAdd(&a.plan->work_counter, 1);
    else atomicOr(a.err, PA_DEVERR_PLAN);
  }
  __syncthreads();
  if (!s_plan_ok) return;
  const int32_t num_items = a.plan->num_items;

  uint32_t fills = 0;
  uint8_t* my_stages = stages + warp * NSTAGE * Cfg::STAGE_BYTES;
  uint64_t* my_bars = bars + warp * NSTAGE;
  // the query row (head within the group) of each accumulator half: lane/4 and lane/4 + 8
  const int qrow = lane >> 2;
  const bool row_ok = qrow < G;  // rows 8..15 are never used (G <= 8)

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
    const bool append = a.k_new != nullptr && L > 0 && p == ni - 1 && tok0 + ntok == L;
    const int new_row = (L - 1) % kBlock;

    for (int i = threadIdx.x; i < nblk; i += blockDim.x) {
      int32_t b = a.block_tables[(int64_t)s * a.max_blocks_per_seq + blk0 + i];
      if (b < 0 || b >= a.num_blocks) {
        atomicOr(a.err, PA_DEVERR_BLOCK_ID);
        b = 0;
      }
      tbl[i] = b;
    }
    __syncthreads();

    // Two warps per KV head: warp 2h streams the first half of the
    // partition's blocks, warp 2h + 1 the second half, and their softmax
    // states are combined below.  An item then carries the bytes of two KV
    // heads, not four: at a given partition size the queue's items are half
    // as long, which makes longer partitions (fewer merges) affordable.
    const int kvh = g * Cfg::KVPI + (warp >> 1);
    const int half = warp & 1;
    const int n0 = (nblk + 1) >> 1;
    const int jb = half ? n0 : 0;            // this warp's first block of the partition
    const int my_n = half ? nblk - n0 : n0;  // and its number of blocks
    float m_run = -INFINITY, l_run = 0.f;
    float o[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = 0.f;
    if (kvh < HK) {
      // Q fragments of this KV head's query heads (rows >= G are zero)
      uint32_t qa[KSTEPS][4];
      {
        const T* q0 = static_cast<const T*>(a.q) + ((int64_t)s * HQ + kvh * G + qrow) * D;
        const int kc = (lane & 3) * 2;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          qa[ks][0] = row_ok ? *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + kc) : 0u;
          qa[ks][1] = 0u;
          qa[ks][2] = row_ok ? *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + kc + 8) : 0u;
          qa[ks][3] = 0u;
        }
      }
      char* kbase = static_cast<char*>(const_cast<void*>(a.k_pool)) + (int64_t)kvh * kBlock * Cfg::ROW_BYTES;
      char* vbase = static_cast<char*>(const_cast<void*>(a.v_pool)) + (int64_t)kvh * kBlock * Cfg::ROW_BYTES;
      const int64_t block_bytes = (int64_t)HK * kBlock * Cfg::ROW_BYTES;
      // fill stage k with block bi: lane 0 issues the tile copies of K and V
      // (the host keeps every row coordinate below 2^31)
      auto issue = [&](uint32_t k, int bi) {
        const int st = k % NSTAGE;
        const uint32_t bar = smem_addr(&my_bars[st]);
        const uint32_t dst = smem_addr(my_stages + st * Cfg::STAGE_BYTES);
        const int y = (tbl[bi] * HK + kvh) * kBlock;
        fence_proxy_async_shared();  // this lane ordered the warp's reads of the stage (syncwarp)
        mbar_arrive_expect_tx(bar, Cfg::STAGE_BYTES);
#pragma unroll
        for (int b = 0; b < Cfg::BOXES; ++b) {
          tma_load_2d(dst + b * Cfg::BOX_BYTES, &tm_k, b * 64, y, bar);
          tma_load_2d(dst + Cfg::TILE_BYTES + b * Cfg::BOX_BYTES, &tm_v, b * 64, y, bar);
        }
      };

      const uint32_t k0 = fills;
      __syncwarp();  // every lane is done with the previous item's stages
      if (lane == 0)
        for (int j = 0; j < NSTAGE && j < my_n; ++j) issue(k0 + j, jb + j);
      bool ok = true;
      int i = 0;
      for (; i < my_n; ++i) {
        const uint32_t k = k0 + i;
        const int st = k % NSTAGE;
        const bool landed = mbar_wait_bounded(smem_addr(&my_bars[st]), (k / NSTAGE) & 1u);
        if (!__all_sync(kFullMask, landed)) {
          ok = false;
          break;
        }
        uint8_t* ktile = my_stages + st * Cfg::STAGE_BYTES;
        uint8_t* vtile = ktile + Cfg::TILE_BYTES;
        const int valid = min(kBlock, ntok - (jb + i) * kBlock);
        if (valid < kBlock) {
          // V rows past the context hold stale values (maybe NaN): zero them
          // so that 0-weight x stale never reaches P.V
          constexpr int CH = Cfg::BOXES * 8;  // 16-byte chunks per row
          for (int c = lane; c < (kBlock - valid) * CH; c += 32) {
            const int r = valid + c / CH;
            *reinterpret_cast<uint4*>(vtile + (c % CH / 8) * Cfg::BOX_BYTES + r * 128 +
                                      (c % 8) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        if (append && jb + i == nblk - 1 && lane < Cfg::ROW_BYTES / 16) {
          // fused reshape_and_cache of the KV head's new row: into the pool,
          // and over the stale row of the staged tiles
          const int64_t skv = (int64_t)s * HK + kvh;
          const uint4 kn = reinterpret_cast<const uint4*>(static_cast<const T*>(a.k_new) + skv * D)[lane];
          const uint4 vn = reinterpret_cast<const uint4*>(static_cast<const T*>(a.v_new) + skv * D)[lane];
          const uint32_t off = (lane / 8) * Cfg::BOX_BYTES + sw128_off(new_row, lane % 8);
          *reinterpret_cast<uint4*>(ktile + off) = kn;
          *reinterpret_cast<uint4*>(vtile + off) = vn;
          const int64_t row_off = (int64_t)tbl[jb + i] * block_bytes + (int64_t)new_row * Cfg::ROW_BYTES;
          reinterpret_cast<uint4*>(kbase + row_off)[lane] = kn;
          reinterpret_cast<uint4*>(vbase + row_off)[lane] = vn;
        }
        __syncwarp();  // zeroed and appended rows are visible to every lane

        // S = Q K^T: sc[0] tokens 0-7, sc[1] tokens 8-15 (rows 0-7 in c0,c1)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int row = (lane & 7) + ((lane >> 4) << 3);
          const int half = (lane >> 3) & 1;  // which 8-element half of the k-step
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            uint32_t b[4];
            const int c = ks * 2 + half;  // 16-byte chunk of the row
            ldmatrix_x4(b, smem_addr(ktile + (c / 8) * Cfg::BOX_BYTES + sw128_off(row, c % 8)));
            mma16816<T>(sc[0], qa[ks], b[0], b[1]);
            mma16816<T>(sc[1], qa[ks], b[2], b[3]);
          }
        }
        const int t0 = (lane & 3) * 2;  // token of c0 within each 8-token half
        float x0 = t0 < valid ? sc[0][0] * a.scale_log2 : -INFINITY;
        float x1 = t0 + 1 < valid ? sc[0][1] * a.scale_log2 : -INFINITY;
        float x2 = t0 + 8 < valid ? sc[1][0] * a.scale_log2 : -INFINITY;
        float x3 = t0 + 9 < valid ? sc[1][1] * a.scale_log2 : -INFINITY;
        float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
        // the reference max moves only when a weight would pass 2^8 (the four
        // lanes of a query row agree: mx is their common maximum)
        const bool move = mx > m_run + 8.f;
        float alpha = 1.f;
        if (move) {
          alpha = exp2f(m_run - mx);  // 0 on the first move
          m_run = mx;
        }
        const float mb = m_run == -INFINITY ? 0.f : m_run;
        const float p0 = exp2f(x0 - mb), p1 = exp2f(x1 - mb);
        const float p2 = exp2f(x2 - mb), p3 = exp2f(x3 - mb);
        float sum = (p0 + p1) + (p2 + p3);
        sum += __shfl_xor_sync(kFullMask, sum, 1);
        sum += __shfl_xor_sync(kFullMask, sum, 2);
        l_run = fmaf(l_run, alpha, sum);
        if (__any_sync(kFullMask, move)) {
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            o[j][0] *= alpha;
            o[j][1] *= alpha;
          }
        }
        constexpr bool kSplit = std::is_same<T, __nv_bfloat16>::value;
        uint32_t pa_[4] = {0u, 0u, 0u, 0u}, pl_[4] = {0u, 0u, 0u, 0u};
        if constexpr (kSplit) {
          pack_split<T>(p0, p1, pa_[0], pl_[0]);
          pack_split<T>(p2, p3, pa_[2], pl_[2]);
        } else {
          pa_[0] = MmaType<T>::pack(p0, p1);
          pa_[2] = MmaType<T>::pack(p2, p3);
        }
        {
          const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
          const int hi = lane >> 4;  // which of the two 8-wide column tiles
#pragma unroll
          for (int j = 0; j < NT; j += 2) {
            uint32_t b[4];
            const int c = j + hi;  // 16-byte chunk of the row
            ldmatrix_x4_trans(b, smem_addr(vtile + (c / 8) * Cfg::BOX_BYTES + sw128_off(row, c % 8)));
            float d0[4] = {o[j][0], o[j][1], 0.f, 0.f};
            float d1[4] = {o[j + 1][0], o[j + 1][1], 0.f, 0.f};
            mma16816<T>(d0, pa_, b[0], b[1]);
            mma16816<T>(d1, pa_, b[2], b[3]);
            if constexpr (kSplit) {
              mma16816<T>(d0, pl_, b[0], b[1]);
              mma16816<T>(d1, pl_, b[2], b[3]);
            }
            o[j][0] = d0[0];
            o[j][1] = d0[1];
            o[j + 1][0] = d1[0];
            o[j + 1][1] = d1[1];
          }
        }
        __syncwarp();  // every lane is done with this stage
        if (lane == 0 && i + NSTAGE < my_n) issue(k + NSTAGE, jb + i + NSTAGE);
        // as in the MHA kernel: the next item is reserved a few tiles before this one ends
        if (threadIdx.x == 0 && i == max(my_n - 3, 0)) next = atomicAdd(&a.plan->work_counter, 1);
      }
      if (!ok) {
        if (lane == 0) {  // as in the MHA kernel: report, stop, and poison the plan
          atomicOr(a.err, PA_DEVERR_TIMEOUT);
          s_abort = 1;
          a.plan->poisoned = 1;
          __threadfence();
        }
        const int issued = min(my_n, i + NSTAGE);
        for (int j = i; j < issued; ++j) {
          const uint32_t k = k0 + j;
          mbar_wait_bounded(smem_addr(&my_bars[k % NSTAGE]), (k / NSTAGE) & 1u);
        }
      } else {
        fills = k0 + my_n;
        if (half) {  // this half's state, for the other warp of the KV head (its stages are drained)
          float* xs = reinterpret_cast<float*>(my_stages);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            xs[(2 * j) * 32 + lane] = o[j][0];
            xs[(2 * j + 1) * 32 + lane] = o[j][1];
          }
          xs[2 * NT * 32 + lane] = m_run;
          xs[(2 * NT + 1) * 32 + lane] = l_run;
          fence_proxy_async_shared();  // before the ring's next bulk copies into the same bytes
        }
      }
    }
    __syncthreads();  // both halves of every KV head are done
    if (kvh < HK && half == 0 && !s_abort) {
      {  // fold in the second half (log-sum-exp rescale of both to the larger reference max)
        const float* xs = reinterpret_cast<const float*>(my_stages + NSTAGE * Cfg::STAGE_BYTES);
        const float mb = xs[2 * NT * 32 + lane], lb = xs[(2 * NT + 1) * 32 + lane];
        const float M = fmaxf(m_run, mb);
        const float sa = m_run == -INFINITY ? 0.f : exp2f(m_run - M);
        const float sb = mb == -INFINITY ? 0.f : exp2f(mb - M);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          o[j][0] = o[j][0] * sa + xs[(2 * j) * 32 + lane] * sb;
          o[j][1] = o[j][1] * sa + xs[(2 * j + 1) * 32 + lane] * sb;
        }
        l_run = l_run * sa + lb * sb;
        m_run = M;
        fence_proxy_async_shared();  // the other warp's ring is refilled after the loop's barrier
      }
      if (row_ok) {  // the output rows, or the partition's partials
        const int64_t sh = (int64_t)s * HQ + kvh * G + qrow;
        const int d0 = (lane & 3) * 2;
        if (!split) {
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
          T* dst = static_cast<T*>(a.out) + sh * D + d0;
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const uint32_t v = MmaType<T>::pack(o[j][0] * inv, o[j][1] * inv);
            *reinterpret_cast<uint32_t*>(dst + j * 8) = v;
          }
        } else {
          float* dst = a.part_acc + (sh * a.max_parts + p) * D + d0;
#pragma unroll
          for (int j = 0; j < NT; ++j) *reinterpret_cast<float2*>(dst + j * 8) = make_float2(o[j][0], o[j][1]);
          if ((lane & 3) == 0) a.part_ml[sh * a.max_parts + p] = make_float2(m_run, l_run);
        }
      }
    }
    if (split) {
      __syncthreads();
      if (threadIdx.x == 0) {
        int32_t* cnt = a.merge_cnt + (int64_t)s * a.head_groups + g;
        __threadfence();
        const int arrived = atomicAdd(cnt, 1) + 1;
        __threadfence();
        s_merge = arrived == ni && !s_abort && *(volatile int32_t*)&a.plan->poisoned == 0;
        if (arrived == ni) *cnt = 0;
      }
      __syncthreads();
      if (s_merge && kvh < HK && half == 0) {
        if (np > ni) grid_dependency_wait();  // shared-prefix partials: see the MHA kernel
        __threadfence();
        constexpr int BUF = NSTAGE * Cfg::STAGE_BYTES;
        const bool merged =
            G == 8   ? merge_group<T, D, 8, NSTAGE, BUF>(a, (int64_t)s * HQ + kvh * G, np, lane,
                                                         my_stages, my_bars, fills)
            : G == 4 ? merge_group<T, D, 4, NSTAGE, BUF>(a, (int64_t)s * HQ + kvh * G, np, lane,
                                                         my_stages, my_bars, fills)
                     : merge_group<T, D, 2, NSTAGE, BUF>(a, (int64_t)s * HQ + kvh * G, np, lane,
                                                         my_stages, my_bars, fills);
        if (!merged && lane == 0) {  // as for a copy of the item: report, stop, poison the plan
          atomicOr(a.err, PA_DEVERR_TIMEOUT);
          s_abort = 1;
          a.plan->poisoned = 1;
          __threadfence();
        }
      }
    }
    __syncthreads();
  }

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
