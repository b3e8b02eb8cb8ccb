// C ABI of libpagedattn.so: host-side validation, per-device set-up and
// kernel launches.  Declarations and argument contracts: include/pagedattn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <random>
#include <unordered_map>

#include "cache_ops.cuh"
#include "decode.cuh"
#include "shared_prefix.cuh"
#include "decode_gqa.cuh"
#include "prefill.cuh"
#include "pagedattn.h"
#include "status.h"

namespace pa {

// Per-device error word raised by the kernels (PA_DEVERR_* bits).
__device__ uint32_t g_device_errors;

namespace {

constexpr int kMaxDevices = 64;
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 4
#endif
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 2
#endif
constexpr int kDecodeWarps = PA_DECODE_WARPS;    // heads per CTA (one warp each)
constexpr int kDecodeStages = PA_DECODE_STAGES;  // per-warp ring depth
constexpr int kMinAutoPartition = 256;    // smallest partition the automatic choice makes
constexpr int kFullBatchPartition = 512;  // partition when the batch alone fills the GPU
constexpr int kMaxPartition = 4096;

struct DeviceState {
  bool ready = false;
  uint32_t* err = nullptr;  // device address of g_device_errors
  int num_sms = 0;
  int decode_ctas_per_sm = 1;  // resident decode CTAs per SM (fp16, head_dim 128 kernel)
  // driver's tensor-map encoder, resolved through the runtime (no libcuda link)
  PFN_cuTensorMapEncodeTiled_v12000 encode_tiled = nullptr;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];

// One NVTX range per C-ABI call that launches work, named after the call, so
// a timeline profiler shows each call around its kernels.  Header-only NVTX:
// without an attached tool the push and pop cost a few nanoseconds.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

pa_status cuda_fail(cudaError_t e, const char* what) {
  char buf[256];
  std::snprintf(buf, sizeof buf, "%s: %s", what, cudaGetErrorString(e));
  return fail(PA_ERR_CUDA, buf);
}

// Warps per CTA for G query heads per KV head: G warps share one ring, and
// a CTA keeps at least kDecodeWarps warps.
constexpr int warps_for(int G) { return G > kDecodeWarps ? G : kDecodeWarps; }

// Ring depth: the CTA keeps kDecodeWarps * kDecodeStages stages in flight
// whatever the grouping (at most 8 per ring), reduced until the stages fit
// the 227 KB a CTA may use (fp32 tiles at head_dim 128 are 8 KB).
constexpr int stages_for(int tile_bytes, int G) {
  const int rings = warps_for(G) / G;
  int s = kDecodeWarps * kDecodeStages / rings;
  if (s > 8) s = 8;
  if (s < 1) s = 1;
  while (s > 1 && rings * s * 2 * tile_bytes + 4096 > 227 * 1024) --s;
  return s;
}

template <typename T, int D, int G>
using DecodeKernelCfg =
    DecodeConfig<T, D, warps_for(G), stages_for(kBlock * D * (int)sizeof(T), G), G>;

template <typename T, int D, int G>
constexpr auto decode_kernel_ptr() {
  return paged_decode_kernel<T, D, warps_for(G), stages_for(kBlock * D * (int)sizeof(T), G), G>;
}

template <typename T, int D, int G>
cudaError_t set_decode_attrs() {
  const size_t smem = DecodeKernelCfg<T, D, G>::smem_bytes(kMaxPartition);
  return cudaFuncSetAttribute(decode_kernel_ptr<T, D, G>(),
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

template <typename T, int D>
cudaError_t set_decode_attrs_all_groups() {
  cudaError_t e = set_decode_attrs<T, D, 1>();
  if (e == cudaSuccess) e = set_decode_attrs<T, D, 2>();
  if (e == cudaSuccess) e = set_decode_attrs<T, D, 4>();
  if (e == cudaSuccess) e = set_decode_attrs<T, D, 8>();
  return e;
}

// KV heads one work item covers, for G query heads per KV head.
int rings_for(int G) { return warps_for(G) / G; }

// Groups of 2, 4 or 8 query heads on fp16/bf16 pools take the tensor-core
// kernel (two warps per KV head); MHA and fp32 pools take the CUDA-core
// kernel.  (Pairs once ran faster on CUDA cores; since the tensor-core
// kernel stages whole tiles and merges all heads of a KV head at once it
// is faster for them too: 106 -> 89 us on 200 requests x 8 KV heads.)
bool use_gqa_mma(const pa_pool* pool) { return pool->q_per_kv >= 2 && pool->dtype != PA_F32; }
#ifndef PA_GQA_STAGES
#define PA_GQA_STAGES 2
#endif
constexpr int kGqaStages = PA_GQA_STAGES;  // per-warp ring depth of the tensor-core kernel

int kv_heads_per_item(const pa_pool* pool) {
  return use_gqa_mma(pool) ? GqaConfig<__half, 128, kGqaStages>::KVPI : rings_for(pool->q_per_kv);
}

template <typename T, int D>
size_t prefill_smem() {
  return PrefillConfig<D, kSplitP<T>>::SMEM;
}

// K or V pool as a 2-D tensor [num_blocks * heads * 16 rows][head_dim] with a
// {64, 16} box (one physical block, one 64-wide slice of head_dim) and
// 128-byte swizzle: the tile layout of the prefill and grouped-query decode
// kernels.
pa_status encode_pool_map(const DeviceState& dev, CUtensorMap* map, const void* base,
                          const pa_pool* pool) {
  const cuuint64_t dims[2] = {(cuuint64_t)pool->head_dim,
                              (cuuint64_t)pool->num_blocks * pool->heads * kBlock};
  const cuuint64_t strides[1] = {(cuuint64_t)pool->head_dim * pool->elem_bytes};
  const cuuint32_t box[2] = {64u, (cuuint32_t)kBlock};
  const cuuint32_t elem_strides[2] = {1u, 1u};
  const CUresult r = dev.encode_tiled(
      map, pool->dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
      2, const_cast<void*>(base), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    std::snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled (pool) failed (%d)", (int)r);
    return fail(PA_ERR_CUDA, buf);
  }
  return PA_OK;
}

// q as a 3-D tensor [num_tokens][query heads][head_dim] with a {64, 1, 128} box
// (128 query rows of one head, one 64-wide slice) and 128-byte swizzle.
pa_status encode_q_map(const DeviceState& dev, CUtensorMap* map, const void* q, const pa_pool* pool,
                       int32_t num_tokens) {
  const cuuint64_t hq = (cuuint64_t)pool->heads * pool->q_per_kv;
  const cuuint64_t dims[3] = {(cuuint64_t)pool->head_dim, hq, (cuuint64_t)num_tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)pool->head_dim * pool->elem_bytes,
                                 hq * pool->head_dim * pool->elem_bytes};
  const cuuint32_t box[3] = {64u, 1u, 128u};
  const cuuint32_t elem_strides[3] = {1u, 1u, 1u};
  const CUresult r = dev.encode_tiled(
      map, pool->dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
      3, const_cast<void*>(q), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    std::snprintf(buf, sizeof buf, "prefill: cuTensorMapEncodeTiled (q) failed (%d)", (int)r);
    return fail(PA_ERR_CUDA, buf);
  }
  return PA_OK;
}

template <typename T, int D>
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                           const CUtensorMap& q, int grid, cudaStream_t s) {
  paged_prefill_kernel<T, D><<<grid, PrefillConfig<D, kSplitP<T>>::THREADS, prefill_smem<T, D>(),
                               s>>>(a, k, v, q);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t set_prefill_attrs() {
  return cudaFuncSetAttribute(paged_prefill_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)prefill_smem<T, D>());
}

// The shared-prefix kernel runs beside the decode kernel that follows it (a
// programmatic dependent launch); with the shared-memory carveout at its
// maximum, an SM running shared-prefix CTAs can also take decode CTAs.
template <typename T, int D>
cudaError_t set_shared_prefix_attrs() {
  return cudaFuncSetAttribute(shared_prefix_kernel<T, D>,
                              cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}

template <typename T, int D>
cudaError_t set_gqa_attrs() {
  return cudaFuncSetAttribute(paged_decode_gqa_kernel<T, D, kGqaStages>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)GqaConfig<T, D, kGqaStages>::smem_bytes(kMaxPartition));
}

// Launch a persistent decode kernel.  With `overlap`, it is a programmatic
// dependent launch on the preceding kernel of the stream: the shared-prefix
// kernel (the decode CTAs wait for it only before merging a sequence that
// has shared-prefix partials) or the plan kernel (a.after_plan: they wait for
// it before reading the plan).
template <typename K, typename... Extra>
cudaError_t launch_decode_grid(K kernel, int grid, int threads, size_t smem, cudaStream_t stream,
                               const DecodeArgs& a, bool overlap, const Extra&... extra) {
  if (!overlap) {
    kernel<<<grid, threads, smem, stream>>>(a, extra...);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, extra...);
}

template <typename T, int D>
cudaError_t launch_gqa(const DecodeArgs& a, const DeviceState& dev, cudaStream_t stream,
                       const CUtensorMap& tm_k, const CUtensorMap& tm_v, bool overlap = false) {
  using Cfg = GqaConfig<T, D, kGqaStages>;
  auto kernel = paged_decode_gqa_kernel<T, D, kGqaStages>;
  const size_t smem = Cfg::smem_bytes(a.partition_size);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, Cfg::THREADS, smem);
  if (e != cudaSuccess) return e;
  per_sm = std::max(per_sm, 1);
  const int64_t upper = (int64_t)a.num_seqs * a.max_parts * a.head_groups;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(upper, (int64_t)dev.num_sms * per_sm));
  return launch_decode_grid(kernel, grid, Cfg::THREADS, smem, stream, a, overlap, tm_k, tm_v);
}

// Once per device, with that device current: resolve the error word's device
// address and raise the shared-memory limit of the decode kernels.
pa_status device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_errors);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_device_errors)");
    st.err = static_cast<uint32_t*>(p);
    e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDriverEntryPointByVersion");
    if (q != cudaDriverEntryPointSuccess || !fn)
      return fail(PA_ERR_CUDA, "driver has no cuTensorMapEncodeTiled");
    st.encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cudaError_t attrs[] = {set_decode_attrs_all_groups<float, 64>(),
                           set_decode_attrs_all_groups<float, 128>(),
                           set_decode_attrs_all_groups<__half, 64>(),
                           set_decode_attrs_all_groups<__half, 128>(),
                           set_decode_attrs_all_groups<__nv_bfloat16, 64>(),
                           set_decode_attrs_all_groups<__nv_bfloat16, 128>(),
                           set_gqa_attrs<__half, 64>(),
                           set_gqa_attrs<__half, 128>(),
                           set_gqa_attrs<__nv_bfloat16, 64>(),
                           set_gqa_attrs<__nv_bfloat16, 128>(),
                           set_prefill_attrs<__half, 64>(),
                           set_prefill_attrs<__half, 128>(),
                           set_prefill_attrs<__nv_bfloat16, 64>(),
                           set_prefill_attrs<__nv_bfloat16, 128>(),
                           set_shared_prefix_attrs<__half, 64>(),
                           set_shared_prefix_attrs<__half, 128>(),
                           set_shared_prefix_attrs<__nv_bfloat16, 64>(),
                           set_shared_prefix_attrs<__nv_bfloat16, 128>()};
    for (cudaError_t a : attrs)
      if (a != cudaSuccess) return cuda_fail(a, "cudaFuncSetAttribute");
    using Cfg = DecodeKernelCfg<__half, 128, 1>;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&st.decode_ctas_per_sm,
                                                      decode_kernel_ptr<__half, 128, 1>(),
                                                      Cfg::THREADS, Cfg::smem_bytes(512));
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    st.decode_ctas_per_sm = std::max(1, st.decode_ctas_per_sm);
    st.ready = true;
  }
  *out = &st;
  return PA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status check_pool(const pa_pool* pool) {
  if (!pool) return fail(PA_ERR_INVALID_ARG, "pool descriptor is null");
  if (pool->block_size != kBlock) return fail(PA_ERR_UNSUPPORTED, "block_size must be 16");
  if (pool->head_dim != 64 && pool->head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (pool->dtype < PA_F32 || pool->dtype > PA_BF16) return fail(PA_ERR_UNSUPPORTED, "unknown dtype");
  if (pool->q_per_kv != 1 && pool->q_per_kv != 2 && pool->q_per_kv != 4 && pool->q_per_kv != 8)
    return fail(PA_ERR_UNSUPPORTED, "query heads per KV head must be 1, 2, 4 or 8");
  if (pool->num_blocks <= 0 || pool->heads <= 0) return fail(PA_ERR_INVALID_ARG, "empty pool");
  if (pool->num_blocks * pool->block_size > INT32_MAX)
    return fail(PA_ERR_INVALID_ARG, "num_blocks * block_size must fit int32");
  return PA_OK;
}

struct WorkspaceLayout {
  size_t header = 0, lens = 0, nparts = 0, nitems = 0, base = 0, shared_of = 0, merge_cnt = 0,
         pairs = 0, part_ml = 0, part_acc = 0, total = 0;
};

constexpr int kSharedChunk = 16;  // shared-prefix blocks per partial result

// Partial-result slots per (sequence, head): own partitions + shared chunks.
int total_parts(int maxL, int ps, int max_shared_blocks) {
  return std::max(1, (maxL + ps - 1) / ps) + (max_shared_blocks + kSharedChunk - 1) / kSharedChunk;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// H = query heads (partials are per query head); G = query heads per KV head.
WorkspaceLayout layout_for(int64_t S, int64_t H, int64_t max_parts, int64_t D, int G,
                           int kv_per_item) {
  WorkspaceLayout w;
  size_t off = 0;
  w.header = off;
  off = align256(off + sizeof(PlanHeader));
  w.lens = off;
  off = align256(off + S * 4);
  w.nparts = off;
  off = align256(off + S * 4);
  w.nitems = off;
  off = align256(off + S * 4);
  w.base = off;
  off = align256(off + S * 4);
  w.shared_of = off;
  off = align256(off + S * 4);
  w.merge_cnt = off;
  off = align256(off + S * ((H / G + kv_per_item - 1) / kv_per_item) * 4);
  w.pairs = off;
  off = align256(off + S * max_parts * 8);
  w.part_ml = off;
  off = align256(off + S * H * max_parts * 8);
  w.part_acc = off;
  off = align256(off + S * H * max_parts * D * 4);
  w.total = off;
  return w;
}

int round_up16(int64_t x) { return (int)std::min<int64_t>(kMaxPartition, (x + 15) / 16 * 16); }

// Automatic partition size.  Every work item pays a pipeline ramp and a
// split costs partial results and a merge, while one long item is streamed
// by a single CTA at a fraction of the chip's bandwidth and can become the
// critical path.  Measured on B200: when (sequences x head groups) already
// gives `full_items` items per resident CTA, 512-token partitions are best
// (2 for the CUDA-core kernel; 1 for the tensor-core GQA kernel, whose items
// of 2 KV heads are streamed by 4 warps: 200 requests x 8 KV heads took
// 84.7 us at 512 tokens against 88.5 at the 352 the rule below gives); with
// few sequences, aim for about four items per resident CTA (never below 256).
int auto_partition(int num_seqs, int head_groups, int max_context_len, int slots, int full_items) {
  const int64_t whole = (int64_t)num_seqs * head_groups;
  const int64_t maxL = std::max(16, max_context_len);
  if (whole >= (int64_t)full_items * slots) return std::min(kFullBatchPartition, round_up16(maxL));
  // About 4 work items per resident CTA.  Only the longest context is known
  // here; a ragged batch averages about half of it, so the partitions are
  // sized for maxL / 2 (sizing them for maxL left items too long to balance).
  const int64_t want_parts = (4LL * slots + whole - 1) / std::max<int64_t>(whole, 1);
  const int64_t ps = (maxL / 2 + want_parts - 1) / want_parts;
  return std::max(kMinAutoPartition, round_up16(ps));
}

int resolve_max_context(const pa_pool* pool, int32_t max_blocks_per_seq, int32_t max_context_len) {
  const int64_t cap = (int64_t)max_blocks_per_seq * pool->block_size;
  const int64_t m = max_context_len == 0 ? cap : std::min<int64_t>(cap, max_context_len);
  return (int)std::min<int64_t>(m, INT32_MAX);
}

template <typename T, int D, int G>
cudaError_t launch_decode(const DecodeArgs& a, const DeviceState& dev, cudaStream_t stream,
                          bool overlap = false) {
  using Cfg = DecodeKernelCfg<T, D, G>;
  auto kernel = decode_kernel_ptr<T, D, G>();
  const size_t smem = Cfg::smem_bytes(a.partition_size);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, Cfg::THREADS, smem);
  if (e != cudaSuccess) return e;
  per_sm = std::max(per_sm, 1);
  const int64_t upper = (int64_t)a.num_seqs * a.max_parts * a.head_groups;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(upper, (int64_t)dev.num_sms * per_sm));
  return launch_decode_grid(kernel, grid, Cfg::THREADS, smem, stream, a, overlap);
}

template <typename T, int D>
cudaError_t launch_grouped(int G, const DecodeArgs& a, const DeviceState& dev, cudaStream_t s,
                           bool overlap = false) {
  switch (G) {
    case 1: return launch_decode<T, D, 1>(a, dev, s, overlap);
    case 2: return launch_decode<T, D, 2>(a, dev, s, overlap);
    case 4: return launch_decode<T, D, 4>(a, dev, s, overlap);
    default: return launch_decode<T, D, 8>(a, dev, s, overlap);
  }
}

// One warp waits on a barrier that expects two arrivals but gets one.
__global__ void wait_timeout_selftest_kernel(uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 2);
    mbar_init_fence();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&bar)) : "memory");
  }
  __syncwarp();
  const bool done = mbar_wait_bounded(smem_addr(&bar), 0);
  if (!__all_sync(kFullMask, done) && threadIdx.x == 0) atomicOr(err, PA_DEVERR_TIMEOUT);
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

pa_status pa_pool_create(int64_t num_blocks, int32_t block_size, int32_t heads, int32_t head_dim,
                         int32_t dtype, pa_pool* out) {
  if (!out) return fail(PA_ERR_INVALID_ARG, "pa_pool_create: out is null");
  if (num_blocks <= 0 || block_size <= 0 || heads <= 0 || head_dim <= 0)
    return fail(PA_ERR_INVALID_ARG, "pa_pool_create: sizes must be positive");
  pa_pool p{};
  p.num_blocks = num_blocks;
  p.block_size = block_size;
  p.heads = heads;
  p.head_dim = head_dim;
  p.dtype = dtype;
  p.q_per_kv = 1;
  p.elem_bytes = dtype == PA_F32 ? 4 : 2;
  p.token_stride = head_dim;
  p.head_stride = (int64_t)block_size * head_dim;
  p.block_stride = (int64_t)heads * block_size * head_dim;
  p.bytes_per_pool = num_blocks * p.block_stride * p.elem_bytes;
  pa_status st = check_pool(&p);
  if (st != PA_OK) return st;
  *out = p;
  return PA_OK;
}

pa_status pa_pool_set_query_heads(pa_pool* pool, int32_t num_q_heads) {
  if (!pool) return fail(PA_ERR_INVALID_ARG, "pa_pool_set_query_heads: pool is null");
  if (num_q_heads <= 0 || num_q_heads % pool->heads != 0)
    return fail(PA_ERR_INVALID_ARG,
                "pa_pool_set_query_heads: query heads must be a positive multiple of KV heads");
  const int32_t g = num_q_heads / pool->heads;
  if (g != 1 && g != 2 && g != 4 && g != 8)
    return fail(PA_ERR_UNSUPPORTED, "query heads per KV head must be 1, 2, 4 or 8");
  pool->q_per_kv = g;
  return PA_OK;
}

pa_status pa_reshape_and_cache(const pa_pool* pool, const void* k_new, const void* v_new,
                               const int32_t* slot_mapping, int32_t num_tokens, void* k_pool,
                               void* v_pool, void* stream) {
  CallRange range("pa_reshape_and_cache");
  pa_status st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: num_tokens < 0");
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool)
    return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: null pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return fail(PA_ERR_INVALID_ARG, "pa_reshape_and_cache: buffers must be 16-byte aligned");
  DeviceState* dev;
  if ((st = device_state(&dev)) != PA_OK) return st;
  const int row_chunks = pool->head_dim * pool->elem_bytes / 16;
  const int64_t total = (int64_t)num_tokens * pool->heads * row_chunks;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)dev->num_sms * 16);
  reshape_and_cache_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping,
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), pool->heads, row_chunks,
      num_tokens, pool->num_blocks * pool->block_size, dev->err);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "reshape_and_cache launch");
}

pa_status pa_decode_shared_prefix_workspace_bytes(const pa_pool* pool, int32_t num_seqs,
                                                  int32_t max_blocks_per_seq,
                                                  int32_t max_context_len, int32_t partition_size,
                                                  int32_t max_shared_blocks, size_t* bytes) {
  pa_status st = check_pool(pool);
  if (st != PA_OK) return st;
  if (!bytes) return fail(PA_ERR_INVALID_ARG, "workspace bytes: bytes is null");
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || max_shared_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "workspace bytes: bad size");
  // partition_size 0: the automatic choice is never below kMinAutoPartition
  const int ps = partition_size == 0 ? kMinAutoPartition : partition_size;
  if (ps < kBlock || ps % kBlock != 0 || ps > kMaxPartition)
    return fail(PA_ERR_INVALID_ARG, "partition_size must be a multiple of 16 in [16, 4096]");
  const int maxL = resolve_max_context(pool, max_blocks_per_seq, max_context_len);
  *bytes = layout_for(num_seqs, (int64_t)pool->heads * pool->q_per_kv,
                      total_parts(maxL, ps, max_shared_blocks), pool->head_dim, pool->q_per_kv,
                      kv_heads_per_item(pool))
               .total;
  return PA_OK;
}

pa_status pa_decode_workspace_bytes(const pa_pool* pool, int32_t num_seqs,
                                    int32_t max_blocks_per_seq, int32_t max_context_len,
                                    int32_t partition_size, size_t* bytes) {
  return pa_decode_shared_prefix_workspace_bytes(pool, num_seqs, max_blocks_per_seq,
                                                 max_context_len, partition_size, 0, bytes);
}

}  // extern "C"

namespace {

// Validate the sizes shared by the plan and run halves and fill the
// workspace pointers of a.
pa_status prepare_decode(const pa_pool* pool, int32_t num_seqs, int32_t max_blocks_per_seq,
                         int32_t max_context_len, int32_t partition_size, void* workspace,
                         size_t workspace_bytes, DecodeArgs* a, DeviceState** dev,
                         int32_t max_shared_blocks = 0) {
  pa_status st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
    return fail(PA_ERR_INVALID_ARG, "decode: bad size");
  if (partition_size != 0 &&
      (partition_size < kBlock || partition_size % kBlock != 0 || partition_size > kMaxPartition))
    return fail(PA_ERR_INVALID_ARG, "partition_size must be a multiple of 16 in [16, 4096]");
  if ((st = device_state(dev)) != PA_OK) return st;
  const int maxL = resolve_max_context(pool, max_blocks_per_seq, max_context_len);
  const int G = pool->q_per_kv;
  const int head_groups = (pool->heads + kv_heads_per_item(pool) - 1) / kv_heads_per_item(pool);
  // With shared prefixes the decode kernel attends only each sequence's own
  // tokens, which are typically far shorter than max_context_len: the
  // smallest automatic partition keeps its items fine enough to balance
  // (128 sequences sharing a 1000-token prompt: 132 us at 256 tokens against
  // 138 us at the 512 the rule below picks from the full lengths).
  const int ps = partition_size != 0 ? partition_size
                 : max_shared_blocks > 0
                     ? kMinAutoPartition
                     : auto_partition(num_seqs, head_groups, maxL,
                                      (*dev)->num_sms * (*dev)->decode_ctas_per_sm,
                                      use_gqa_mma(pool) ? 1 : 2);
  const int max_parts = total_parts(maxL, ps, max_shared_blocks);
  const WorkspaceLayout w = layout_for(num_seqs, (int64_t)pool->heads * G, max_parts,
                                       pool->head_dim, G, kv_heads_per_item(pool));
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(PA_ERR_WORKSPACE, "decode: workspace missing, not 256-byte aligned or too small");
  char* ws = static_cast<char*>(workspace);
  *a = DecodeArgs{};
  a->plan = reinterpret_cast<PlanHeader*>(ws + w.header);
  a->lens = reinterpret_cast<int32_t*>(ws + w.lens);
  a->nparts = reinterpret_cast<int32_t*>(ws + w.nparts);
  a->nitems = reinterpret_cast<int32_t*>(ws + w.nitems);
  a->base = reinterpret_cast<int32_t*>(ws + w.base);
  a->shared_of = reinterpret_cast<int32_t*>(ws + w.shared_of);
  a->max_shared_blocks = max_shared_blocks;
  a->shared_chunk = kSharedChunk;
  a->pairs = reinterpret_cast<int2*>(ws + w.pairs);
  a->part_ml = reinterpret_cast<float2*>(ws + w.part_ml);
  a->part_acc = reinterpret_cast<float*>(ws + w.part_acc);
  a->merge_cnt = reinterpret_cast<int32_t*>(ws + w.merge_cnt);
  a->err = (*dev)->err;
  a->num_blocks = pool->num_blocks;
  a->max_blocks_per_seq = max_blocks_per_seq;
  a->num_seqs = num_seqs;
  a->heads = pool->heads;
  a->q_per_kv = G;
  a->head_groups = head_groups;
  a->partition_size = ps;
  a->max_parts = max_parts;
  a->max_context_len = maxL;
  return PA_OK;
}

// ---- plans recorded per workspace ------------------------------------------------
// The work items, partial slots and merge counters a planned call reads were
// laid out by the plan in its workspace.  Every plan the library writes is
// recorded under the workspace's plan address with the parameters it was made
// with, and a planned call that resolves to other parameters, or finds no
// plan there, is refused rather than run on a layout it does not match.
struct PlanKey {
  int32_t num_seqs, max_blocks_per_seq, max_context_len, partition_size, max_parts, head_groups,
      heads, q_per_kv, head_dim, dtype, device;
};

PlanKey plan_key(const pa_pool* pool, const DecodeArgs& a) {
  int dev = -1;
  cudaGetDevice(&dev);
  return PlanKey{a.num_seqs,   a.max_blocks_per_seq, a.max_context_len, a.partition_size,
                 a.max_parts,  a.head_groups,        pool->heads,       pool->q_per_kv,
                 pool->head_dim, (int32_t)pool->dtype, dev};
}

struct PlanRecord {
  PlanKey key;
  uint64_t stamp;  // written into the plan's header; the kernels run only on a matching one
};

std::mutex g_plan_mutex;
std::unordered_map<const void*, PlanRecord>& plan_registry() {
  static std::unordered_map<const void*, PlanRecord> plans;
  return plans;
}

// A fresh number for every plan: a random per-process high half (so a stale
// plan left in reused memory by another process does not match) and a
// counter that never yields zero (so a zeroed workspace does not match).
uint64_t next_plan_stamp() {
  static const uint64_t salt = [] {
    std::random_device rd;
    return (uint64_t)rd() << 32;
  }();
  static std::atomic<uint32_t> counter{0};
  uint32_t n = ++counter;
  if (n == 0) n = ++counter;
  return salt | n;
}

// On success a->stamp is the stamp of the plan recorded for a's workspace.
pa_status check_plan(const pa_pool* pool, DecodeArgs* a, const char* who) {
  const PlanKey want = plan_key(pool, *a);
  std::lock_guard<std::mutex> lock(g_plan_mutex);
  const auto it = plan_registry().find(a->plan);
  char buf[200];
  if (it == plan_registry().end()) {
    std::snprintf(buf, sizeof buf, "%s: no plan was written to this workspace (pa_decode_plan)",
                  who);
    return fail(PA_ERR_INVALID_ARG, buf);
  }
  if (std::memcmp(&it->second.key, &want, sizeof want) != 0) {
    std::snprintf(buf, sizeof buf,
                  "%s: the arguments differ from the plan's in this workspace (sequences, "
                  "table width, max_context_len, partition_size and pool must match)",
                  who);
    return fail(PA_ERR_INVALID_ARG, buf);
  }
  a->stamp = it->second.stamp;
  return PA_OK;
}

// Write a plan under a fresh stamp (left in a->stamp for the launches that
// follow in the same call) and record it for the workspace.
pa_status launch_plan(const pa_pool* pool, DecodeArgs* a, cudaStream_t s) {
  a->stamp = next_plan_stamp();
  decode_plan_kernel<<<1, 1024, 2 * (a->partition_size / kBlock + 1) * sizeof(int32_t), s>>>(*a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode plan launch");
  const PlanKey k = plan_key(pool, *a);
  std::lock_guard<std::mutex> lock(g_plan_mutex);
  plan_registry()[a->plan] = PlanRecord{k, a->stamp};
  return PA_OK;
}

pa_status launch_run(const pa_pool* pool, const DecodeArgs& a, const DeviceState& dev,
                     cudaStream_t s, bool overlap = false) {
  cudaError_t e;
  if (use_gqa_mma(pool)) {
    // the tensor-core kernel stages tiles by tensor copies whose row
    // coordinate (block * heads + head) * 16 must fit int32; a pool past that
    // would not fit in device memory at these head sizes anyway
    if ((int64_t)pool->num_blocks * pool->heads * kBlock > INT32_MAX)
      return fail(PA_ERR_UNSUPPORTED, "decode: pool rows exceed the tensor-copy coordinate range");
    CUtensorMap tk, tv;
    pa_status st;
    if ((st = encode_pool_map(dev, &tk, a.k_pool, pool)) != PA_OK ||
        (st = encode_pool_map(dev, &tv, a.v_pool, pool)) != PA_OK)
      return st;
    switch (pool->dtype * 1000 + pool->head_dim) {
      case PA_F16 * 1000 + 64: e = launch_gqa<__half, 64>(a, dev, s, tk, tv, overlap); break;
      case PA_F16 * 1000 + 128: e = launch_gqa<__half, 128>(a, dev, s, tk, tv, overlap); break;
      case PA_BF16 * 1000 + 64: e = launch_gqa<__nv_bfloat16, 64>(a, dev, s, tk, tv, overlap); break;
      case PA_BF16 * 1000 + 128:
        e = launch_gqa<__nv_bfloat16, 128>(a, dev, s, tk, tv, overlap);
        break;
      default: return fail(PA_ERR_UNSUPPORTED, "decode: dtype/head_dim not built");
    }
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "decode launch");
  }
  switch (pool->dtype * 1000 + pool->head_dim) {
    case PA_F32 * 1000 + 64: e = launch_grouped<float, 64>(pool->q_per_kv, a, dev, s, overlap); break;
    case PA_F32 * 1000 + 128: e = launch_grouped<float, 128>(pool->q_per_kv, a, dev, s, overlap); break;
    case PA_F16 * 1000 + 64: e = launch_grouped<__half, 64>(pool->q_per_kv, a, dev, s, overlap); break;
    case PA_F16 * 1000 + 128: e = launch_grouped<__half, 128>(pool->q_per_kv, a, dev, s, overlap); break;
    case PA_BF16 * 1000 + 64: e = launch_grouped<__nv_bfloat16, 64>(pool->q_per_kv, a, dev, s, overlap); break;
    case PA_BF16 * 1000 + 128:
      e = launch_grouped<__nv_bfloat16, 128>(pool->q_per_kv, a, dev, s, overlap);
      break;
    default: return fail(PA_ERR_UNSUPPORTED, "decode: dtype/head_dim not built");
  }
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "decode launch");
}

pa_status check_run_pointers(const void* q, const void* k_pool, const void* v_pool,
                             const int32_t* block_tables, const void* out, float scale) {
  if (!q || !k_pool || !v_pool || !block_tables || !out)
    return fail(PA_ERR_INVALID_ARG, "decode: null pointer");
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return fail(PA_ERR_INVALID_ARG, "decode: q, pools and out must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "decode: scale not finite");
  return PA_OK;
}

void set_run_args(DecodeArgs* a, const void* q, const void* k_pool, const void* v_pool,
                  const int32_t* block_tables, void* out, float scale) {
  a->q = q;
  a->k_pool = k_pool;
  a->v_pool = v_pool;
  a->block_tables = block_tables;
  a->out = out;
  a->scale_log2 = scale * 1.4426950408889634f;  // log2(e)
}

}  // namespace

extern "C" {

pa_status pa_decode_plan(const pa_pool* pool, const int32_t* context_lens, int32_t num_seqs,
                         int32_t max_blocks_per_seq, int32_t max_context_len,
                         int32_t partition_size, void* workspace, size_t workspace_bytes,
                         void* stream) {
  CallRange range("pa_decode_plan");
  if (num_seqs == 0) return check_pool(pool);
  if (!context_lens) return fail(PA_ERR_INVALID_ARG, "pa_decode_plan: context_lens is null");
  DecodeArgs a;
  DeviceState* dev;
  pa_status st = prepare_decode(pool, num_seqs, max_blocks_per_seq, max_context_len,
                                partition_size, workspace, workspace_bytes, &a, &dev);
  if (st != PA_OK) return st;
  a.context_lens = context_lens;
  return launch_plan(pool, &a, static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_attention_planned(const pa_pool* pool, const void* q, const void* k_pool,
                                      const void* v_pool, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, int32_t num_seqs,
                                      int32_t max_context_len, float scale, void* out,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t partition_size, void* stream) {
  CallRange range("pa_decode_attention_planned");
  if (num_seqs == 0) return check_pool(pool);
  pa_status st = check_run_pointers(q, k_pool, v_pool, block_tables, out, scale);
  if (st != PA_OK) return st;
  DecodeArgs a;
  DeviceState* dev;
  st = prepare_decode(pool, num_seqs, max_blocks_per_seq, max_context_len, partition_size,
                      workspace, workspace_bytes, &a, &dev);
  if (st != PA_OK) return st;
  if ((st = check_plan(pool, &a, "pa_decode_attention_planned")) != PA_OK) return st;
  set_run_args(&a, q, k_pool, v_pool, block_tables, out, scale);
  return launch_run(pool, a, *dev, static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_attention(const pa_pool* pool, const void* q, const void* k_pool,
                              const void* v_pool, const int32_t* block_tables,
                              int32_t max_blocks_per_seq, const int32_t* context_lens,
                              int32_t num_seqs, int32_t max_context_len, float scale, void* out,
                              void* workspace, size_t workspace_bytes, int32_t partition_size,
                              void* stream) {
  CallRange range("pa_decode_attention");
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: num_seqs < 0");
  if (num_seqs == 0) return check_pool(pool);
  pa_status st = check_run_pointers(q, k_pool, v_pool, block_tables, out, scale);
  if (st != PA_OK) return st;
  if (!context_lens) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention: null pointer");
  DecodeArgs a;
  DeviceState* dev;
  st = prepare_decode(pool, num_seqs, max_blocks_per_seq, max_context_len, partition_size,
                      workspace, workspace_bytes, &a, &dev);
  if (st != PA_OK) return st;
  a.context_lens = context_lens;
  set_run_args(&a, q, k_pool, v_pool, block_tables, out, scale);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = launch_plan(pool, &a, s)) != PA_OK) return st;
  a.after_plan = 1;  // the decode launch overlaps the plan kernel's run
  return launch_run(pool, a, *dev, s, true);
}

pa_status pa_decode_append_attention_planned(const pa_pool* pool, const void* q,
                                             const void* k_new, const void* v_new, void* k_pool,
                                             void* v_pool, const int32_t* block_tables,
                                             int32_t max_blocks_per_seq, int32_t num_seqs,
                                             int32_t max_context_len, float scale, void* out,
                                             void* workspace, size_t workspace_bytes,
                                             int32_t partition_size, void* stream) {
  CallRange range("pa_decode_append_attention_planned");
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "decode append: num_seqs < 0");
  if (num_seqs == 0) return check_pool(pool);
  pa_status st = check_run_pointers(q, k_pool, v_pool, block_tables, out, scale);
  if (st != PA_OK) return st;
  if (!k_new || !v_new) return fail(PA_ERR_INVALID_ARG, "decode append: k_new/v_new is null");
  if (!aligned16(k_new) || !aligned16(v_new))
    return fail(PA_ERR_INVALID_ARG, "decode append: k_new/v_new must be 16-byte aligned");
  DecodeArgs a;
  DeviceState* dev;
  st = prepare_decode(pool, num_seqs, max_blocks_per_seq, max_context_len, partition_size,
                      workspace, workspace_bytes, &a, &dev);
  if (st != PA_OK) return st;
  if ((st = check_plan(pool, &a, "pa_decode_append_attention_planned")) != PA_OK) return st;
  set_run_args(&a, q, k_pool, v_pool, block_tables, out, scale);
  a.k_new = k_new;
  a.v_new = v_new;
  return launch_run(pool, a, *dev, static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_append_attention(const pa_pool* pool, const void* q, const void* k_new,
                                     const void* v_new, void* k_pool, void* v_pool,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t num_seqs,
                                     int32_t max_context_len, float scale, void* out,
                                     void* workspace, size_t workspace_bytes,
                                     int32_t partition_size, void* stream) {
  CallRange range("pa_decode_append_attention");
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "decode append: num_seqs < 0");
  if (num_seqs == 0) return check_pool(pool);
  pa_status st = check_run_pointers(q, k_pool, v_pool, block_tables, out, scale);
  if (st != PA_OK) return st;
  if (!context_lens) return fail(PA_ERR_INVALID_ARG, "decode append: context_lens is null");
  if (!k_new || !v_new) return fail(PA_ERR_INVALID_ARG, "decode append: k_new/v_new is null");
  if (!aligned16(k_new) || !aligned16(v_new))
    return fail(PA_ERR_INVALID_ARG, "decode append: k_new/v_new must be 16-byte aligned");
  DecodeArgs a;
  DeviceState* dev;
  st = prepare_decode(pool, num_seqs, max_blocks_per_seq, max_context_len, partition_size,
                      workspace, workspace_bytes, &a, &dev);
  if (st != PA_OK) return st;
  a.context_lens = context_lens;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = launch_plan(pool, &a, s)) != PA_OK) return st;
  set_run_args(&a, q, k_pool, v_pool, block_tables, out, scale);
  a.k_new = k_new;
  a.v_new = v_new;
  a.after_plan = 1;  // the decode launch overlaps the plan kernel's run
  return launch_run(pool, a, *dev, s, true);
}

pa_status pa_decode_attention_shared_prefix(
    const pa_pool* pool, const void* q, const void* k_pool, const void* v_pool,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
    int32_t num_seqs, const int32_t* group_offsets, const int32_t* group_members,
    int32_t num_members, const int32_t* group_blocks, int32_t num_groups, int32_t max_group_size,
    int32_t max_shared_blocks, int32_t max_context_len, float scale, void* out, void* workspace,
    size_t workspace_bytes, int32_t partition_size, void* stream) {
  CallRange range("pa_decode_attention_shared_prefix");
  if (num_seqs < 0 || num_groups < 0 || num_members < 0 || max_group_size < 0 ||
      max_shared_blocks < 0)
    return fail(PA_ERR_INVALID_ARG, "shared prefix: negative size");
  if (num_seqs == 0) return check_pool(pool);
  pa_status st = check_pool(pool);
  if (st != PA_OK) return st;
  if (pool->dtype == PA_F32)
    return fail(PA_ERR_UNSUPPORTED, "shared prefix: fp16 or bf16 pools only (tensor-core path)");
  st = check_run_pointers(q, k_pool, v_pool, block_tables, out, scale);
  if (st != PA_OK) return st;
  if (!context_lens) return fail(PA_ERR_INVALID_ARG, "shared prefix: context_lens is null");
  if (num_groups > 0 && (!group_offsets || !group_members || !group_blocks))
    return fail(PA_ERR_INVALID_ARG, "shared prefix: group arrays are null");
  DecodeArgs a;
  DeviceState* dev;
  st = prepare_decode(pool, num_seqs, max_blocks_per_seq, max_context_len, partition_size,
                      workspace, workspace_bytes, &a, &dev, max_shared_blocks);
  if (st != PA_OK) return st;
  a.context_lens = context_lens;
  if (num_groups > 0 && max_shared_blocks > 0 && max_group_size > 0) {
    a.group_offsets = group_offsets;
    a.group_members = group_members;
    a.group_blocks = group_blocks;
    a.num_groups = num_groups;
    a.num_members = num_members;
    a.max_group_size = max_group_size;
  }
  set_run_args(&a, q, k_pool, v_pool, block_tables, out, scale);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = launch_plan(pool, &a, s)) != PA_OK) return st;
  if (a.group_offsets != nullptr) {
    SharedPrefixArgs sp;
    sp.group_offsets = group_offsets;
    sp.group_members = group_members;
    sp.num_members = num_members;
    sp.group_blocks = group_blocks;
    sp.num_groups = num_groups;
    const int rows = max_group_size * pool->q_per_kv;
    sp.row_tiles = (rows + 63) / 64;
    sp.chunk_blocks = kSharedChunk;
    const dim3 grid((unsigned)((int64_t)num_groups * sp.row_tiles), (unsigned)pool->heads,
                    (unsigned)((max_shared_blocks + kSharedChunk - 1) / kSharedChunk));
    if ((int64_t)num_groups * sp.row_tiles > INT32_MAX || grid.z > 65535 || grid.y > 65535)
      return fail(PA_ERR_INVALID_ARG, "shared prefix: too many groups or blocks");
    const bool bf16 = pool->dtype == PA_BF16;
    if (pool->head_dim == 128) {
      if (bf16)
        shared_prefix_kernel<__nv_bfloat16, 128>
            <<<grid, 128, SharedPrefixConfig<128>::smem_bytes(), s>>>(sp, a);
      else
        shared_prefix_kernel<__half, 128><<<grid, 128, SharedPrefixConfig<128>::smem_bytes(), s>>>(sp, a);
    } else {
      if (bf16)
        shared_prefix_kernel<__nv_bfloat16, 64>
            <<<grid, 128, SharedPrefixConfig<64>::smem_bytes(), s>>>(sp, a);
      else
        shared_prefix_kernel<__half, 64><<<grid, 128, SharedPrefixConfig<64>::smem_bytes(), s>>>(sp, a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "shared prefix launch");
  }
  // the decode launch overlaps the shared-prefix kernel (it needs its
  // partials only to merge)
  return launch_run(pool, a, *dev, s, a.group_offsets != nullptr);
}

pa_status pa_prefill_attention(const pa_pool* pool, const void* q, const void* k_pool,
                               const void* v_pool, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* context_lens,
                               const int32_t* query_start, int32_t num_seqs, int32_t num_tokens,
                               int32_t max_new_tokens, int32_t max_context_len, float scale,
                               void* out, void* stream) {
  CallRange range("pa_prefill_attention");
  pa_status st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_tokens < 0 || max_new_tokens < 0 || max_blocks_per_seq <= 0 ||
      max_context_len < 0)
    return fail(PA_ERR_INVALID_ARG, "prefill: bad size");
  if (num_seqs == 0 || max_new_tokens == 0 || num_tokens == 0) return PA_OK;
  if (pool->dtype == PA_F32)
    return fail(PA_ERR_UNSUPPORTED, "prefill: fp16 or bf16 pools only (tcgen05 kind::f16)");
  st = check_run_pointers(q, k_pool, v_pool, block_tables, out, scale);
  if (st != PA_OK) return st;
  if (!context_lens || !query_start) return fail(PA_ERR_INVALID_ARG, "prefill: null pointer");
  DeviceState* dev;
  if ((st = device_state(&dev)) != PA_OK) return st;
  PrefillArgs a{};
  a.q = q;
  a.v_pool = v_pool;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start = query_start;
  a.out = out;
  a.err = dev->err;
  a.num_blocks = pool->num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.heads = pool->heads;
  a.q_per_kv = pool->q_per_kv;
  a.max_context_len = resolve_max_context(pool, max_blocks_per_seq, max_context_len);
  a.scale_log2 = scale * 1.4426950408889634f;
  const int64_t pairs = (max_new_tokens + 255) / 256;  // two 128-query tiles per item
  const int64_t hq = (int64_t)pool->heads * pool->q_per_kv;
  const int64_t items = hq * num_seqs * pairs;
  if (items > INT32_MAX) return fail(PA_ERR_INVALID_ARG, "prefill: too many work items");
  if ((int64_t)pool->num_blocks * pool->heads * kBlock > INT32_MAX)
    return fail(PA_ERR_INVALID_ARG, "prefill: pool rows exceed the tensor-copy coordinate range");
  a.q_pairs = (int32_t)pairs;
  a.max_new_tokens = max_new_tokens;
  a.num_tokens = num_tokens;
  CUtensorMap tk, tv, tq;
  if ((st = encode_pool_map(*dev, &tk, k_pool, pool)) != PA_OK ||
      (st = encode_pool_map(*dev, &tv, v_pool, pool)) != PA_OK ||
      (st = encode_q_map(*dev, &tq, q, pool, num_tokens)) != PA_OK)
    return st;
  // fp16: persistent, one CTA per SM walking the items (shared memory admits
  // one).  bf16: one CTA per item, so the hardware hands items out as CTAs
  // finish.  Measured on 2048- and 4096-token prompts: persistence saves each
  // item's start-up (+1-8 % for fp16), while the fixed item-to-CTA assignment
  // loses the hardware's balancing, which costs the longer bf16 items more
  // than the start-up they save (-6 % persistent vs -1.5 % one per item).
  const bool bf16 = pool->dtype == PA_BF16;
  const int grid = bf16 ? (int)items : (int)std::min<int64_t>(items, dev->num_sms);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (pool->head_dim == 128)
    e = bf16 ? launch_prefill<__nv_bfloat16, 128>(a, tk, tv, tq, grid, s)
             : launch_prefill<__half, 128>(a, tk, tv, tq, grid, s);
  else
    e = bf16 ? launch_prefill<__nv_bfloat16, 64>(a, tk, tv, tq, grid, s)
             : launch_prefill<__half, 64>(a, tk, tv, tq, grid, s);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "prefill launch");
}

pa_status pa_copy_blocks(const pa_pool* pool, void* k_pool, void* v_pool, const int32_t* pairs,
                         int32_t num_pairs, void* stream) {
  CallRange range("pa_copy_blocks");
  pa_status st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: num_pairs < 0");
  if (num_pairs == 0) return PA_OK;
  if (!k_pool || !v_pool || !pairs) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: null pointer");
  if (!aligned16(k_pool) || !aligned16(v_pool))
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: pools must be 16-byte aligned");
  DeviceState* dev;
  if ((st = device_state(&dev)) != PA_OK) return st;
  const int64_t block_chunks = pool->block_stride * pool->elem_bytes / 16;
  const int64_t total = (int64_t)num_pairs * block_chunks;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)dev->num_sms * 16);
  copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), pairs, num_pairs,
      pool->num_blocks, block_chunks, dev->err);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks launch");
}

pa_status pa_selftest_wait_timeout(void* stream) {
  DeviceState* dev;
  pa_status st = device_state(&dev);
  if (st != PA_OK) return st;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev->err);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "selftest launch");
}

}  // extern "C"

// ---- decode with a static scratch buffer (no allocation by anyone) ----------------------
// For callers that may not call cudaMalloc: plugins whose host runtime owns
// all device memory, and loops that cannot pay cudaMalloc's implicit device
// synchronisation.  The plan and the split-K partials live in this buffer.
// Every call shares it, so calls that overlap on the GPU race; the plan
// kernel rewrites the header and counters it needs at the start of each call.
static __device__ __align__(256) uint8_t g_static_scratch[PA_STATIC_SCRATCH_BYTES];

namespace {

// Device address of g_static_scratch, resolved once per device with that
// device current (the host-side symbol is only a stand-in, never a device
// address).
void* g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_static_mutex;

pa_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_static_scratch)");
    g_static_scratch_ptr[dev] = ptr;
  }
  *out = g_static_scratch_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode_attention_static(const pa_pool* pool, const void* q, const void* k_pool,
                                     const void* v_pool, const int32_t* block_tables,
                                     int32_t max_blocks_per_seq, const int32_t* context_lens,
                                     int32_t num_seqs, int32_t max_context_len, float scale,
                                     void* out, int32_t partition_size, void* stream) {
  CallRange range("pa_decode_attention_static");
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "pa_decode_attention_static: num_seqs < 0");
  if (num_seqs == 0) return check_pool(pool);  // as pa_decode_attention: nothing to launch
  size_t need = 0;
  pa_status st = pa_decode_workspace_bytes(pool, num_seqs, max_blocks_per_seq, max_context_len,
                                           partition_size, &need);
  if (st != PA_OK) return st;
  if (need > PA_STATIC_SCRATCH_BYTES) {
    char buf[256];
    std::snprintf(buf, sizeof buf,
                  "pa_decode_attention_static: these sizes need %zu bytes of scratch; the static "
                  "buffer holds %u (use fewer sequences or a larger partition_size, or "
                  "pa_decode_attention with a caller workspace)",
                  need, PA_STATIC_SCRATCH_BYTES);
    return fail(PA_ERR_WORKSPACE, buf);
  }
  void* scratch = nullptr;
  if ((st = static_scratch(&scratch)) != PA_OK) return st;
  return pa_decode_attention(pool, q, k_pool, v_pool, block_tables, max_blocks_per_seq,
                             context_lens, num_seqs, max_context_len, scale, out, scratch,
                             PA_STATIC_SCRATCH_BYTES, partition_size, stream);
}

pa_status pa_device_errors(void* stream, uint32_t* flags) {
  if (!flags) return fail(PA_ERR_INVALID_ARG, "pa_device_errors: flags is null");
  *flags = 0;
  DeviceState* dev;
  pa_status st = device_state(&dev);
  if (st != PA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, dev->err, sizeof v, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dev->err, 0, sizeof v, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "pa_device_errors");
  *flags = v;
  if (v & PA_DEVERR_TIMEOUT) return fail(PA_ERR_TIMEOUT, "a device-side wait timed out");
  if (v & PA_DEVERR_PLAN)
    return fail(PA_ERR_OUT_OF_BOUNDS,
                "a planned launch found no valid plan in its workspace, or a damaged entry");
  if (v) return fail(PA_ERR_OUT_OF_BOUNDS, "a device-side bounds check fired");
  return PA_OK;
}

}  // extern "C"
