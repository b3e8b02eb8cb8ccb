// Arguments of the paged decode path and its work plan.
//
// The plan kernel (one CTA per call, or once per step with the planned API)
// validates context lengths and shared-prefix groups and orders the work
// items the decode kernels take from an atomic queue: the ragged last
// partitions of split sequences first (by decreasing size), then the full
// partitions, then the sequences that fit one partition (by decreasing
// size).  A split sequence is merged when its last partition arrives, so
// this puts the merges in the middle of the launch instead of at its end,
// and leaves the tail to unsplit items, which merge nothing.  It lives apart from
// the decode kernel so that the decode kernel's source (whose DRAM traffic
// profiles record) changes only with the kernel.
#pragma once

#include <math.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "pagedattn.h"

namespace pa {

constexpr int kBlock = 16;  // tokens per physical block

struct PlanHeader {
  int32_t num_pairs;     // (sequence, partition) pairs
  int32_t num_items;     // num_pairs * head_groups
  int32_t work_counter;  // next item index to hand out
  int32_t done_counter;  // CTAs that have left the work loop
  uint64_t stamp;        // the host's number for this plan; a launch runs only on its own plan
  int32_t poisoned;      // a launch on this plan gave up on a wait: refused until re-planned
  int32_t reserved;
};

struct DecodeArgs {
  const void* q;
  const void* k_pool;
  const void* v_pool;
  const int32_t* block_tables;
  const int32_t* context_lens;
  void* out;
  PlanHeader* plan;
  int32_t* lens;    // [S] clamped context lengths
  int32_t* nparts;  // [S] partial results per sequence (>= 1): own partitions + shared chunks
  int32_t* nitems;  // [S] own partitions (work items whose arrival triggers the merge)
  int32_t* base;    // [S] first token of the sequence's own part (after its shared prefix)
  int32_t* shared_of;  // [S] shared-prefix group of the sequence, or -1
  // shared-prefix groups (null when there are none): CSR members, shared leading blocks
  const int32_t* group_offsets;
  const int32_t* group_members;
  int32_t num_members;     // entries of group_members
  const int32_t* group_blocks;
  int32_t num_groups;
  int32_t max_shared_blocks;
  int32_t max_group_size;  // members per group the shared-prefix launch covers
  int32_t shared_chunk;  // shared blocks per partial result
  int2* pairs;      // [S * max_parts] work pairs (s, p)
  float2* part_ml;  // [S][H][max_parts] (running max in log2 units, sum of weights)
  float* part_acc;  // [S][H][max_parts][D] unnormalised partial outputs
  int32_t* merge_cnt;  // [S][head_groups] partitions finished (re-armed to 0 by the merger)
  const void* k_new;   // [S][H][D] token appended at position L-1, or null (no append)
  const void* v_new;
  uint32_t* err;
  int64_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int32_t heads;        // KV heads in the pool
  int32_t q_per_kv;     // query heads per KV head (1 = MHA; GQA/MQA otherwise)
  int32_t head_groups;  // work items per (sequence, partition)
  int32_t partition_size;
  int32_t max_parts;
  int32_t max_context_len;
  float scale_log2;  // scale * log2(e)
  uint64_t stamp;    // number of the plan the host expects in the workspace
  int32_t after_plan;  // launched as a programmatic dependent of the plan kernel: wait for it first
};

// Checks a CTA makes before it trusts the plan in the workspace: the header
// carries the stamp this launch was given, no earlier launch on the plan gave
// up, and the item count is within what the workspace can hold.  Any failure
// raises PA_DEVERR_PLAN and the launch touches nothing in the workspace.
__device__ __forceinline__ bool plan_header_ok(const DecodeArgs& a) {
  const PlanHeader* h = a.plan;
  const int64_t cap = (int64_t)a.num_seqs * a.max_parts * a.head_groups;
  return h->stamp == a.stamp && h->poisoned == 0 && h->num_items >= 0 && h->num_items <= cap;
}

// One work item's view of the plan, bounds-checked so that a damaged
// workspace can cost the result but never an access outside the caller's
// buffers: the sequence is in range, its clamped length within the table
// and max_context_len, its own part starts on a block boundary inside the
// context, and the partition index and partial counts fit the workspace.
struct PlanItem {
  int s, p, L, np, ni, base;
};

__device__ __forceinline__ bool plan_item(const DecodeArgs& a, int item, PlanItem* it) {
  const int2 pr = a.pairs[item / a.head_groups];
  it->s = pr.x;
  it->p = pr.y;
  if (pr.x < 0 || pr.x >= a.num_seqs) return false;
  it->L = a.lens[pr.x];
  it->np = a.nparts[pr.x];
  it->ni = a.nitems[pr.x];
  it->base = a.base[pr.x];
  const int64_t cap = min((int64_t)a.max_context_len, (int64_t)a.max_blocks_per_seq * kBlock);
  return it->L >= 0 && it->L <= cap && it->base >= 0 && it->base <= it->L &&
         it->base % kBlock == 0 && it->ni >= 1 && it->np >= it->ni && it->np <= a.max_parts &&
         pr.y >= 0 && pr.y < it->ni &&
         (int64_t)it->base + (int64_t)pr.y * a.partition_size <= it->L;
}

// ---- plan: one CTA orders the work ------------------------------------------------

__global__ void __launch_bounds__(1024) decode_plan_kernel(DecodeArgs a) {
  // a decode launch that follows as a programmatic dependent may start its
  // CTAs now; they wait for this grid to complete before reading the plan
  grid_dependents_launch();
  // bucket[0..nb]: ragged last partitions of split sequences by block count;
  // bucket[nb+1..2nb+1]: unsplit sequences by block count (nb+1: no own tokens)
  extern __shared__ int32_t bucket[];
  __shared__ int32_t n_full, n_full2, full_base;  // full partitions: count, placed, first slot
  const int PS = a.partition_size;
  const int nb = PS / kBlock;
  for (int i = threadIdx.x; i <= 2 * nb + 1; i += blockDim.x) bucket[i] = 0;
  if (threadIdx.x == 0) {
    n_full = 0;
    n_full2 = 0;
  }
  const int cap = (int)min((int64_t)a.max_context_len, (int64_t)a.max_blocks_per_seq * kBlock);
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    int L = a.context_lens[s];
    if (L < 0 || L > cap) {
      atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
      L = L < 0 ? 0 : cap;
    }
    a.lens[s] = L;
    a.shared_of[s] = -1;
    for (int g = 0; g < a.head_groups; ++g) a.merge_cnt[(int64_t)s * a.head_groups + g] = 0;
  }
  __syncthreads();
  // shared-prefix groups: a member joins if its table starts with the first
  // member's blocks and it is long enough; anything else is reported and the
  // sequence attends to its whole context on its own
  if (a.group_offsets != nullptr) {
    // groups in turn, their members spread over the CTA's threads
    for (int g = 0; g < a.num_groups; ++g) {
      const int m0 = a.group_offsets[g], m1 = a.group_offsets[g + 1];
      const int nbk = a.group_blocks[g];
      if (m1 <= m0 || nbk <= 0) continue;
      // a group beyond the launch's bounds would be covered only in part
      if (nbk > a.max_shared_blocks || nbk > a.max_blocks_per_seq || m0 < 0 ||
          m1 > a.num_members || m1 - m0 > a.max_group_size) {
        if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      const int rep = a.group_members[m0];
      if (rep < 0 || rep >= a.num_seqs || a.lens[rep] < nbk * kBlock) {
        if (threadIdx.x == 0) atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
        continue;
      }
      const int32_t* rt = a.block_tables + (int64_t)rep * a.max_blocks_per_seq;
      // each warp takes MPW members at a time, their lanes comparing 32 table
      // entries per step, with the loads of all MPW members in flight together
      constexpr int MPW = 4;
      const int lane = threadIdx.x & 31;
      for (int mb = m0 + (threadIdx.x >> 5) * MPW; mb < m1; mb += (blockDim.x >> 5) * MPW) {
        int sv[MPW], diff[MPW];
        bool ok[MPW];
#pragma unroll
        for (int u = 0; u < MPW; ++u) sv[u] = mb + u < m1 ? a.group_members[mb + u] : -1;
#pragma unroll
        for (int u = 0; u < MPW; ++u) {
          ok[u] = sv[u] >= 0 && sv[u] < a.num_seqs && a.lens[sv[u]] >= nbk * kBlock;
          diff[u] = 0;
        }
        for (int j = lane; j < nbk; j += 32) {
          const int32_t r = rt[j];
#pragma unroll
          for (int u = 0; u < MPW; ++u)
            if (ok[u]) diff[u] |= a.block_tables[(int64_t)sv[u] * a.max_blocks_per_seq + j] ^ r;
        }
#pragma unroll
        for (int u = 0; u < MPW; ++u) {
          if (mb + u >= m1) break;  // the same for the whole warp
          const bool good = ok[u] && !__any_sync(kFullMask, diff[u] != 0);
          if (lane == 0) {
            if (!good) {
              atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);
            } else if (atomicCAS(&a.shared_of[sv[u]], -1, g) != -1) {
              atomicOr(a.err, PA_DEVERR_CONTEXT_LEN);  // already in another group
            }
          }
        }
      }
    }
  }
  __syncthreads();
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int L = a.lens[s];
    const int g = a.shared_of[s];
    const int sb = g >= 0 ? a.group_blocks[g] : 0;
    const int base = sb * kBlock;
    const int U = L - base;  // the sequence's own tokens
    const int full = U / PS, rem = U % PS;
    const int ni = max(1, full + (rem > 0 ? 1 : 0));
    a.base[s] = base;
    a.nitems[s] = ni;
    a.nparts[s] = ni + (sb > 0 ? (sb + a.shared_chunk - 1) / a.shared_chunk : 0);
    if (full > 0) atomicAdd(&n_full, full);
    if (U == 0 || rem > 0)  // a ragged last partition, or the whole (possibly empty) sequence
      atomicAdd(&bucket[(full > 0 ? 0 : nb + 1) + (U == 0 ? 0 : (rem + kBlock - 1) / kBlock)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int b = nb; b >= 0; --b) {  // remainders of split sequences, biggest first
      const int c = bucket[b];
      bucket[b] = run;
      run += c;
    }
    full_base = run;  // then the full partitions
    run += n_full;
    for (int b = 2 * nb + 1; b > nb; --b) {  // then the unsplit sequences, biggest first
      const int c = bucket[b];
      bucket[b] = run;
      run += c;
    }
    a.plan->num_pairs = run;
    a.plan->num_items = run * a.head_groups;
    a.plan->work_counter = 0;
    a.plan->done_counter = 0;
    a.plan->stamp = a.stamp;
    a.plan->poisoned = 0;
  }
  __syncthreads();
  for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
    const int U = a.lens[s] - a.base[s];
    const int rem = U % PS, full = U / PS;
    if (full > 0) {
      const int pos = full_base + atomicAdd(&n_full2, full);
      for (int p = 0; p < full; ++p) a.pairs[pos + p] = make_int2(s, p);
    }
    if (U == 0 || rem > 0) {
      const int b = (full > 0 ? 0 : nb + 1) + (U == 0 ? 0 : (rem + kBlock - 1) / kBlock);
      const int pos = atomicAdd(&bucket[b], 1);
      a.pairs[pos] = make_int2(s, full);
    }
  }
}

}  // namespace pa
