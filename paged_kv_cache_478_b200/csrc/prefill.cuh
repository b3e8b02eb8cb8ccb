// Paged prefill on 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Many new query tokens per sequence attend causally to the sequence's paged
// cache: query i at absolute position pos_i sees tokens 0..pos_i.  The
// block-wise form of "PagedAttention" (wiki mirror, "Formulació matemàtica")
// applies to every query; with 128 queries a tile the two products are dense
// contractions, S = Q.K^T and O = P.V.
//
// One CTA = (sequence, query head, tile of 128 new queries); 4 warps, thread
// r owns query row r.  Per 64-key tile:
//   * all threads stage K and V rows from their physical blocks with cp.async
//     into 128-byte-swizzled tiles (two stages), rows past the context are
//     zeroed;
//   * thread 0 issues S = Q.K^T (M=128, N=64, K=head_dim in steps of 16) into
//     TMEM and commits to an mbarrier;
//   * each thread reads its row of S from TMEM, applies the causal mask and
//     the online softmax in fp32 (log2 domain), rescales its row of O in TMEM
//     when the running max moved, and writes its row of P (fp16/bf16) into a
//     swizzled shared tile;
//   * thread 0 issues O += P.V (M=128, N=head_dim, K=64) into TMEM.
// Shared-memory operands are described by SW128 matrix descriptors (K-major
// for Q, K and P; MN-major for V).  TMEM holds S (64 columns) and O
// (head_dim columns); the CTA allocates 256 columns and frees them on every
// exit path.  Every wait is bounded.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "device_utils.cuh"
#include "mma_utils.cuh"
#include "pagedattn.h"

namespace pa {

struct PrefillArgs {
  const void* q;            // [T][HQ][D]
  const void* k_pool;
  const void* v_pool;
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
  float scale_log2;
};

// SPLIT_P: the softmax weights go to the tensor core as a high part plus its
// rounding residual (two P tiles, two P.V chains).  bf16 needs it (8-bit
// significand); fp16's 11 bits keep the result inside the parity gate alone.
template <int D, bool SPLIT_P>
struct PrefillConfig {
  static constexpr int BM = 128;  // queries per CTA (TMEM lanes)
  static constexpr int BN = 64;   // keys per tile
  static constexpr int KB = D / 64;                 // 128-byte K-blocks across head_dim
  static constexpr int Q_BYTES = KB * BM * 128;
  static constexpr int KV_BYTES = KB * BN * 128;    // one of K or V
  static constexpr int P_BYTES = BM * 128;          // BM rows x 64 keys
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;    // [stage][K|V]
  static constexpr int OFF_P = OFF_KV + 2 * 2 * KV_BYTES;      // P (high part)
  static constexpr int OFF_PL = OFF_P + P_BYTES;               // P residual (SPLIT_P)
  static constexpr int OFF_BAR = OFF_PL + (SPLIT_P ? P_BYTES : 0);  // 2 mbarriers + TMEM address
  // The dynamic window starts 1024-byte aligned when the kernel has no static
  // shared variables (checked at run time), so two CTAs fit per SM.
  static constexpr size_t SMEM = OFF_BAR + 64;
  static constexpr int TMEM_COLS = 256;             // S: 64 columns, O: D columns
  static constexpr int S_COL = 0;
  static constexpr int O_COL = 64;
  static_assert(D == 64 || D == 128, "head_dim");
};

// ---- tcgen05 / descriptor helpers ------------------------------------------------

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

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
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

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile whose
// rows are 128 bytes (one K-block).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

template <typename T>
constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;

template <typename T, int D>
__global__ void __launch_bounds__(128) paged_prefill_kernel(PrefillArgs a) {
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  using Cfg = PrefillConfig<D, kSplitP<T>>;
  constexpr int BM = Cfg::BM, BN = Cfg::BN;
  constexpr uint32_t IDESC_S = f16_idesc(BM, BN, kBf16, false);
  constexpr uint32_t IDESC_PV = f16_idesc(BM, D, kBf16, true);

  extern __shared__ __align__(1024) uint8_t prefill_smem[];
  uint8_t* smem = prefill_smem;

  const int qt = blockIdx.x, hq = blockIdx.y, s = blockIdx.z;
  if (smem_addr(smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_TIMEOUT);
    return;
  }
  const int q0 = a.query_start[s];
  const int n = a.query_start[s + 1] - q0;
  if (n <= 0 || qt * BM >= n) return;
  const int cap = min(a.max_context_len, a.max_blocks_per_seq * kBlock);
  const int L = a.context_lens[s];
  if (L < n || L > cap) {  // the new tokens must be in the cache
    if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
    return;
  }
  const int G = a.q_per_kv, HQ = a.heads * G, kvh = hq / G;
  const int row = threadIdx.x, warp = row >> 5;
  const int qi = qt * BM + row;
  const bool row_valid = qi < n;
  const int pos = L - n + qi;                               // this query's position
  const int last_pos = L - n + min(n, (qt + 1) * BM) - 1;  // last query of the tile
  const int nkt = (last_pos + BN) / BN;                     // key tiles to visit

  uint8_t* sQ = smem + Cfg::OFF_Q;
  uint8_t* sP = smem + Cfg::OFF_P;
  uint8_t* sPL = smem + Cfg::OFF_PL;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_BAR + 16);
  const uint32_t bar_s = smem_addr(&bars[0]), bar_pv = smem_addr(&bars[1]);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_pv, 1);
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes

  // ---- Q tile: row r = query qt*BM + r, zero past the new tokens -------------
  {
    constexpr int CH = D / 8;  // 16-byte chunks per row
    for (int idx = threadIdx.x; idx < BM * CH; idx += blockDim.x) {
      const int r = idx / CH, c = idx % CH;
      uint8_t* dst = sQ + (c >> 3) * (BM * 128) + sw128_off(r, c & 7);
      if (qt * BM + r < n) {
        const T* src = static_cast<const T*>(a.q) + ((int64_t)(q0 + qt * BM + r) * HQ + hq) * D + c * 8;
        cp_async16(smem_addr(dst), src);
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
  }
  const int32_t* table = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
  const int64_t tile_elems = (int64_t)kBlock * D;
  const int64_t block_elems = (int64_t)a.heads * tile_elems;
  // stage K/V rows of key tile j (tokens j*BN ..): rows at or past L are zeroed
  auto load_kv = [&](int j, int stage) {
    uint8_t* sK = smem + Cfg::OFF_KV + stage * 2 * Cfg::KV_BYTES;
    uint8_t* sV = sK + Cfg::KV_BYTES;
    constexpr int CH = D / 8;
    for (int idx = threadIdx.x; idx < BN * CH; idx += blockDim.x) {
      const int r = idx / CH, c = idx % CH;
      const int t = j * BN + r;
      const uint32_t off = (c >> 3) * (BN * 128) + sw128_off(r, c & 7);
      if (t < L) {
        int32_t blk = table[t / kBlock];
        if (blk < 0 || blk >= a.num_blocks) {
          atomicOr(a.err, PA_DEVERR_BLOCK_ID);
          blk = 0;
        }
        const int64_t e = blk * block_elems + kvh * tile_elems + (int64_t)(t % kBlock) * D + c * 8;
        cp_async16(smem_addr(sK + off), static_cast<const T*>(a.k_pool) + e);
        cp_async16(smem_addr(sV + off), static_cast<const T*>(a.v_pool) + e);
      } else {
        *reinterpret_cast<uint4*>(sK + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sV + off) = make_uint4(0, 0, 0, 0);
      }
    }
  };
  load_kv(0, 0);
  cp_async_commit();  // group 0: Q + key tile 0

  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;
  int last_s = -1, last_pv = -1;  // last tiles whose products were issued (uniform)
  for (int j = 0; j < nkt; ++j) {
    const int stage = j & 1;
    if (j >= 1) {
      // O += P.V of tile j-1 done: O is stable, P and stage (j+1)&1 are free
      ok = mbar_wait_bounded(bar_pv, (j - 1) & 1);
      if (!__syncthreads_and(ok)) break;
      tc_fence_after();
    }
    if (j + 1 < nkt) load_kv(j + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();          // this thread's copies of tile j have landed
    fence_proxy_async_shared();  // ... and are visible to the tensor core
    __syncthreads();

    uint8_t* sK = smem + Cfg::OFF_KV + stage * 2 * Cfg::KV_BYTES;
    uint8_t* sV = sK + Cfg::KV_BYTES;
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t kofs = (kk & 3) * 32;  // 16 elements further along the 128-byte row
        const uint64_t ad = sw128_desc(smem_addr(sQ + (kk >> 2) * (BM * 128)) + kofs, 16, 1024);
        const uint64_t bd = sw128_desc(smem_addr(sK + (kk >> 2) * (BN * 128)) + kofs, 16, 1024);
        umma_f16(tmem + Cfg::S_COL, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
      }
      umma_commit(bar_s);
    }
    last_s = j;
    ok = mbar_wait_bounded(bar_s, j & 1);
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();

    // ---- this row's scores, causal mask, online softmax -----------------------
    float sc[BN];
    tmem_ld32(tmem + lane_base + Cfg::S_COL, sc);
    tmem_ld32(tmem + lane_base + Cfg::S_COL + 32, sc + 32);
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      const int t = j * BN + c;
      sc[c] = (row_valid && t <= pos) ? sc[c] * a.scale_log2 : -INFINITY;
      mx = fmaxf(mx, sc[c]);
    }
    const float m_new = fmaxf(m_run, mx);
    const float alpha = m_new == -INFINITY ? 1.f : exp2f(m_run - m_new);
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < BN; ++c) {
      sc[c] = m_new == -INFINITY ? 0.f : exp2f(sc[c] - m_new);
      sum += sc[c];
    }
    l_run = fmaf(l_run, alpha, sum);
    m_run = m_new;
    // rescale this row of O when the running max moved (the whole warp takes
    // part in the TMEM access if any of its rows needs it)
    if (j >= 1 && __any_sync(kFullMask, alpha != 1.f)) {
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + Cfg::O_COL + c0, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= alpha;
        tmem_st32(tmem + lane_base + Cfg::O_COL + c0, o);
      }
    }
    // this row of P into the swizzled A tile (64 keys = 8 chunks of 16 bytes)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 v, r;
      if constexpr (Cfg::OFF_PL != Cfg::OFF_BAR) {  // SPLIT_P
        pack_split<T>(sc[8 * c + 0], sc[8 * c + 1], v.x, r.x);
        pack_split<T>(sc[8 * c + 2], sc[8 * c + 3], v.y, r.y);
        pack_split<T>(sc[8 * c + 4], sc[8 * c + 5], v.z, r.z);
        pack_split<T>(sc[8 * c + 6], sc[8 * c + 7], v.w, r.w);
        *reinterpret_cast<uint4*>(sPL + sw128_off(row, c)) = r;
      } else {
        v.x = MmaType<T>::pack(sc[8 * c + 0], sc[8 * c + 1]);
        v.y = MmaType<T>::pack(sc[8 * c + 2], sc[8 * c + 3]);
        v.z = MmaType<T>::pack(sc[8 * c + 4], sc[8 * c + 5]);
        v.w = MmaType<T>::pack(sc[8 * c + 6], sc[8 * c + 7]);
      }
      *reinterpret_cast<uint4*>(sP + sw128_off(row, c)) = v;
    }
    fence_proxy_async_shared();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const uint64_t ad = sw128_desc(smem_addr(sP) + kk * 32, 16, 1024);
        // V is MN-major: 64-dim blocks LBO apart, 8-key groups 1024 bytes apart
        const uint64_t bd = sw128_desc(smem_addr(sV) + kk * 2048, BN * 128, 1024);
        umma_f16(tmem + Cfg::O_COL, ad, bd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        if constexpr (Cfg::OFF_PL != Cfg::OFF_BAR) {
          const uint64_t adl = sw128_desc(smem_addr(sPL) + kk * 32, 16, 1024);
          umma_f16(tmem + Cfg::O_COL, adl, bd, IDESC_PV, 1u);
        }
      }
      umma_commit(bar_pv);
    }
    last_pv = j;
  }
  if (ok) ok = mbar_wait_bounded(bar_pv, (nkt - 1) & 1);
  ok = __syncthreads_and(ok);
  if (!ok) {
    // a wait gave up: let the products already issued land (bounded) before
    // the shared memory and TMEM are released
    if (last_s >= 0) mbar_wait_bounded(bar_s, last_s & 1);
    if (last_pv >= 0) mbar_wait_bounded(bar_pv, last_pv & 1);
  }
  tc_fence_after();

  if (ok) {
    // ---- O / l for this row -------------------------------------------------
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    T* dst = static_cast<T*>(a.out) + ((int64_t)(q0 + qi) * HQ + hq) * D;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      float o[32];
      tmem_ld32(tmem + lane_base + Cfg::O_COL + c0, o);
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
  } else if (threadIdx.x == 0) {
    atomicOr(a.err, PA_DEVERR_TIMEOUT);
  }
  // let any copies still in flight land, then free TMEM
  cp_async_wait<0>();
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
