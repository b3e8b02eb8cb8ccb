// Decode over a shared prefix: the K/V blocks a group of sequences holds in
// common are read once and attended to by every member's query, on tensor
// cores (mma.sync m16n8k16, fp32 accumulation).
//
// "Atención paginada en modelos de lenguaje grandes (LLM)" (7minutos.es),
// section 3: requests with the same system prompt point their block tables
// at the same physical pages.  "PagedAttention" (wiki mirror), "Descripció":
// blocks are shared between requests or branches (prefix sharing, parallel
// sampling, beam search).  Attention over a set of tokens can be computed on
// any split of the set and merged by log-sum-exp, so the shared blocks are
// one partial result per member and the member's own blocks another.
//
// Design (ours): one CTA = (group, KV head, chunk of shared blocks, tile of
// 64 query rows).  A query row is (member, query head of this KV head).  Each
// warp owns 16 rows: S = Q.K^T for a 16-token block is 16 mma (8 k-steps x 2
// token halves), P.V another 16; the online softmax runs on the mma
// accumulator fragments (a row's 16 scores live in one lane quad).  K/V tiles
// arrive by cp.async into rows padded to D*2+16 bytes, so the ldmatrix reads
// are bank-conflict free.  The partial (m, l, unnormalised acc) of each row
// goes to the member's split-K slots after its own partitions; the decode
// kernel's merge folds them in.
#pragma once

#include <stdint.h>

#include "decode.cuh"
#include "device_utils.cuh"
#include "mma_utils.cuh"

namespace pa {

struct SharedPrefixArgs {
  const int32_t* group_offsets;  // [G+1] CSR offsets into group_members
  const int32_t* group_members;  // sequence ids
  int32_t num_members;           // entries of group_members
  const int32_t* group_blocks;   // [G] shared leading blocks of each group
  int32_t num_groups;
  int32_t row_tiles;   // 64-row tiles per group (from the largest group)
  int32_t chunk_blocks;
};

template <int D>
struct SharedPrefixConfig {
  static constexpr int WARPS = 4;
  static constexpr int ROWS = 16 * WARPS;         // query rows per CTA
  static constexpr int PITCH = D * 2 + 16;        // padded bytes per token row in shared memory
  static constexpr int TILE_BYTES = kBlock * PITCH;
  static constexpr int STAGES = 4;
  static constexpr size_t smem_bytes() { return (size_t)STAGES * 2 * TILE_BYTES; }
};

template <typename T, int D>
__global__ void __launch_bounds__(128) shared_prefix_kernel(SharedPrefixArgs sp, DecodeArgs a) {
  using Cfg = SharedPrefixConfig<D>;
  constexpr int KSTEPS = D / 16;   // k-steps of the score product
  constexpr int NT = D / 8;        // 8-column output tiles
  constexpr int CHUNKS = D * 2 / 16;  // 16-byte chunks per token row
  extern __shared__ __align__(128) uint8_t smem[];
  // the decode launch that follows may start now: it reads this kernel's
  // partials only after waiting for it to complete
  grid_dependents_launch();
  if (!plan_header_ok(a)) {  // not the plan this call wrote: touch nothing
    if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_PLAN);
    return;
  }

  const int G = a.q_per_kv;
  const int g = blockIdx.x / sp.row_tiles;
  const int row_tile = blockIdx.x % sp.row_tiles;
  const int kvh = blockIdx.y;
  const int chunk = blockIdx.z;
  if (g >= sp.num_groups) return;
  const int m0 = sp.group_offsets[g], m1 = sp.group_offsets[g + 1];
  const int nblocks = sp.group_blocks[g];
  const int blk_lo = chunk * sp.chunk_blocks;
  const int blk_hi = min(nblocks, blk_lo + sp.chunk_blocks);
  const int rows_in_group = (m1 - m0) * G;
  if (m1 <= m0 || blk_lo >= blk_hi || row_tile * Cfg::ROWS >= rows_in_group) return;
  // groups the plan could not have accepted are skipped (their members attend alone)
  if (m0 < 0 || m1 > sp.num_members || m1 - m0 > a.max_group_size ||
      nblocks > a.max_shared_blocks || nblocks > a.max_blocks_per_seq)
    return;
  const int rep = sp.group_members[m0];  // any member's table names the shared blocks
  if (rep < 0 || rep >= a.num_seqs) return;
  const int HK = a.heads, HQ = a.heads * G;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the two rows this lane's accumulator fragments cover, and whether they count
  int row_s[2], row_hq[2];
  bool row_ok[2];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = row_tile * Cfg::ROWS + warp * 16 + (lane >> 2) + 8 * h2;
    row_ok[h2] = r < rows_in_group;
    int member = row_ok[h2] ? sp.group_members[m0 + r / G] : rep;
    if (member < 0 || member >= a.num_seqs) {
      member = rep;
      row_ok[h2] = false;
    }
    row_s[h2] = member;
    row_hq[h2] = kvh * G + r % G;
    // a member the plan did not attach to this group (bad group data) is skipped
    if (row_ok[h2] && a.shared_of[member] != g) row_ok[h2] = false;
  }

  // Q fragments: rows (lane/4, +8), k = (lane%4)*2 (+8) within each 16-wide k-step
  uint32_t qa[KSTEPS][4];
  {
    const T* q0 = static_cast<const T*>(a.q) + ((int64_t)row_s[0] * HQ + row_hq[0]) * D;
    const T* q1 = static_cast<const T*>(a.q) + ((int64_t)row_s[1] * HQ + row_hq[1]) * D;
    const int kc = (lane & 3) * 2;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      const uint32_t z = 0;
      qa[ks][0] = row_ok[0] ? *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + kc) : z;
      qa[ks][1] = row_ok[1] ? *reinterpret_cast<const uint32_t*>(q1 + ks * 16 + kc) : z;
      qa[ks][2] = row_ok[0] ? *reinterpret_cast<const uint32_t*>(q0 + ks * 16 + kc + 8) : z;
      qa[ks][3] = row_ok[1] ? *reinterpret_cast<const uint32_t*>(q1 + ks * 16 + kc + 8) : z;
    }
  }

  const int32_t* table = a.block_tables + (int64_t)rep * a.max_blocks_per_seq;
  const int64_t tile_elems = (int64_t)kBlock * D;
  const int64_t block_elems = (int64_t)HK * tile_elems;
  auto load_stage = [&](int stage, int bi) {
    int32_t blk = table[bi];
    if (blk < 0 || blk >= a.num_blocks) {
      if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_BLOCK_ID);
      blk = 0;
    }
    const T* ksrc = static_cast<const T*>(a.k_pool) + blk * block_elems + kvh * tile_elems;
    const T* vsrc = static_cast<const T*>(a.v_pool) + blk * block_elems + kvh * tile_elems;
    uint8_t* kdst = smem + (size_t)stage * 2 * Cfg::TILE_BYTES;
    uint8_t* vdst = kdst + Cfg::TILE_BYTES;
    for (int i = threadIdx.x; i < kBlock * CHUNKS; i += blockDim.x) {
      const int row = i / CHUNKS, c = i % CHUNKS;
      cp_async16(smem_addr(kdst + row * Cfg::PITCH + c * 16), ksrc + row * D + c * 8);
      cp_async16(smem_addr(vdst + row * Cfg::PITCH + c * 16), vsrc + row * D + c * 8);
    }
  };

  const int nb = blk_hi - blk_lo;
#pragma unroll
  for (int st = 0; st < Cfg::STAGES - 1; ++st) {
    if (st < nb) load_stage(st, blk_lo + st);
    cp_async_commit();
  }

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  for (int i = 0; i < nb; ++i) {
    cp_async_wait<Cfg::STAGES - 2>();
    __syncthreads();
    // refill the stage freed by the previous iteration
    {
      const int nxt = i + Cfg::STAGES - 1;
      if (nxt < nb) load_stage(nxt % Cfg::STAGES, blk_lo + nxt);
      cp_async_commit();
    }
    const uint8_t* ktile = smem + (size_t)(i % Cfg::STAGES) * 2 * Cfg::TILE_BYTES;
    const uint8_t* vtile = ktile + Cfg::TILE_BYTES;

    // S = Q K^T for 16 tokens: s[0] tokens 0-7, s[1] tokens 8-15
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int row = (lane & 7) + ((lane >> 4) << 3);  // token row this lane addresses
      const int col8 = ((lane >> 3) & 1) * 8;           // k half within the 16-wide step
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        uint32_t b[4];
        ldmatrix_x4(b, smem_addr(ktile + row * Cfg::PITCH + (ks * 16 + col8) * 2));
        mma16816<T>(s[0], qa[ks], b[0], b[1]);
        mma16816<T>(s[1], qa[ks], b[2], b[3]);
      }
    }
    // online softmax on the fragments: c0,c1 -> row lane/4, c2,c3 -> row lane/4 + 8
    uint32_t pa_[4], pl_[4];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float x0 = s[0][2 * h2] * a.scale_log2, x1 = s[0][2 * h2 + 1] * a.scale_log2;
      float x2 = s[1][2 * h2] * a.scale_log2, x3 = s[1][2 * h2 + 1] * a.scale_log2;
      float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
      mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
      const float m_new = fmaxf(m_run[h2], mx);
      const float alpha = exp2f(m_run[h2] - m_new);
      const float p0 = exp2f(x0 - m_new), p1 = exp2f(x1 - m_new);
      const float p2 = exp2f(x2 - m_new), p3 = exp2f(x3 - m_new);
      float sum = (p0 + p1) + (p2 + p3);
      sum += __shfl_xor_sync(kFullMask, sum, 1);
      sum += __shfl_xor_sync(kFullMask, sum, 2);
      l_run[h2] = fmaf(l_run[h2], alpha, sum);
      m_run[h2] = m_new;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        o[j][2 * h2] *= alpha;
        o[j][2 * h2 + 1] *= alpha;
      }
      // P as the A fragment of the P.V product (k = tokens), as a high part
      // plus its rounding residual so bf16 operands keep the weights accurate
      pack_split<T>(p0, p1, pa_[h2], pl_[h2]);          // row, tokens (lane%4)*2..+1
      pack_split<T>(p2, p3, pa_[2 + h2], pl_[2 + h2]);  // row, tokens 8 + (lane%4)*2..+1
    }
    // O += P V: B fragments from V rows (tokens) by transposed ldmatrix
    {
      const int row = (lane & 7) + (((lane >> 3) & 1) << 3);  // token row
      const int col = (lane >> 4) * 8;                         // which of two 8-wide dim tiles
#pragma unroll
      for (int j = 0; j < NT; j += 2) {
        uint32_t b[4];
        ldmatrix_x4_trans(b, smem_addr(vtile + row * Cfg::PITCH + (j * 8 + col) * 2));
        mma16816<T>(o[j], pa_, b[0], b[1]);
        mma16816<T>(o[j], pl_, b[0], b[1]);
        mma16816<T>(o[j + 1], pa_, b[2], b[3]);
        mma16816<T>(o[j + 1], pl_, b[2], b[3]);
      }
    }
  }
  cp_async_wait<0>();

  // partial results go to each member's slot nitems + chunk
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    if (!row_ok[h2]) continue;
    const int s = row_s[h2];
    const int64_t sh = (int64_t)s * HQ + row_hq[h2];
    const int slot = a.nitems[s] + chunk;
    if (a.nitems[s] < 1 || slot >= a.max_parts) {  // a damaged plan entry
      atomicOr(a.err, PA_DEVERR_PLAN);
      continue;
    }
    float* dst = a.part_acc + (sh * a.max_parts + slot) * D + (lane & 3) * 2;
#pragma unroll
    for (int j = 0; j < NT; ++j)
      *reinterpret_cast<float2*>(dst + j * 8) = make_float2(o[j][2 * h2], o[j][2 * h2 + 1]);
    if ((lane & 3) == 0) a.part_ml[sh * a.max_parts + slot] = make_float2(m_run[h2], l_run[h2]);
  }
}

}  // namespace pa
