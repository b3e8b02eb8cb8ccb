/*
 * pagedattn.h: C ABI of the paged decode-attention library (libpagedattn.so).
 *
 * What it computes (sources are web pages on PagedAttention):
 *   - "Atención paginada en modelos de lenguaje grandes (LLM)" (7minutos.es),
 *     section 2: the KV cache lives in a flat pool of equal physical pages of
 *     16 tokens; a request's block_table maps logical page i to a physical
 *     page id, and a new page is claimed only when the token count crosses a
 *     page boundary.  Section 3: pages are reference-counted and shared by
 *     requests with a common prefix; share() raises the count, cow_copy()
 *     gives a writer a private copy and lowers the original's count.
 *   - "PagedAttention" (e-fortepiano.pl wiki mirror), "Descripció": logical
 *     blocks need not be physically contiguous; "Formulació matemàtica": the
 *     attention of one query token is computed block by block over the KV
 *     blocks and equals the ordinary softmax(q.K^T * scale).V.
 *
 * Data layout (all device buffers are owned by the caller):
 *   k_pool, v_pool   [num_blocks][heads][block_size][head_dim], dtype elements,
 *                    16-byte aligned base.  Physical slot of a token =
 *                    block_id * block_size + in-block offset.
 *   q, out           [num_seqs][heads * q_per_kv][head_dim], same dtype as
 *                    the pool (q_per_kv = 1 unless pa_pool_set_query_heads).
 *   k_new, v_new of the fused append: [num_seqs][heads][head_dim].
 *   k_new, v_new     [num_tokens][heads][head_dim], same dtype as the pool.
 *   block_tables     int32 [num_seqs][max_blocks_per_seq]; entries past a
 *                    sequence's last block are never read.
 *   context_lens     int32 [num_seqs]: tokens cached per sequence, counting
 *                    the token appended this step.
 *   slot_mapping     int32 [num_tokens]; a negative slot is skipped (padding).
 *   pairs            int32 [num_pairs][2] = (src_block, dst_block).
 *
 * Errors: every call returns a pa_status; PA_OK means the arguments passed
 * host-side validation and the kernels were enqueued on `stream` (a
 * cudaStream_t; NULL is the legacy default stream).  Launches are
 * asynchronous.  Values that only the device sees (block ids, slots, context
 * lengths) are bounds-checked in the kernels: a bad value is skipped or
 * clamped, never dereferenced, and raises a bit in a per-device error word
 * that pa_device_errors() returns and clears.  pa_last_error() gives a
 * message for the last failing call on the calling thread.
 *
 * Supported: block_size 16; head_dim 64 or 128; dtype fp32, fp16, bf16.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned buffer */
  PA_ERR_UNSUPPORTED = 2,   /* dtype / head_dim / block_size not built */
  PA_ERR_CUDA = 3,          /* a CUDA runtime call failed; see pa_last_error() */
  PA_ERR_OUT_OF_BOUNDS = 4, /* device-side bounds check fired */
  PA_ERR_NO_FREE_BLOCKS = 5,/* block manager: pool exhausted */
  PA_ERR_WORKSPACE = 6,     /* workspace missing or too small */
  PA_ERR_TIMEOUT = 7        /* a device-side wait gave up */
} pa_status;

/* Bits of the device error word (pa_device_errors). */
#define PA_DEVERR_BLOCK_ID 0x1u    /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_SLOT 0x2u        /* slot outside [0, num_blocks * block_size) */
#define PA_DEVERR_CONTEXT_LEN 0x4u /* context_len < 0 or above the table / max bound */
#define PA_DEVERR_PAIR 0x8u        /* copy_blocks pair outside the pool */
#define PA_DEVERR_TIMEOUT 0x10u    /* an mbarrier wait ran past its limit */
#define PA_DEVERR_PLAN 0x20u       /* the workspace holds no plan this launch may run, or a
                                      damaged entry of one (the launch skips what it cannot
                                      trust) */

/* Plain value descriptor of one K or V pool (the two share it). */
typedef struct pa_pool {
  int64_t num_blocks;
  int32_t block_size;
  int32_t heads;
  int32_t head_dim;
  int32_t dtype;       /* pa_dtype */
  int32_t elem_bytes;
  int32_t q_per_kv;     /* query heads per KV head: 1 (MHA), 2, 4 or 8 (GQA/MQA) */
  int64_t token_stride; /* elements between consecutive slots of a block: head_dim */
  int64_t head_stride;  /* elements between heads of a block: block_size * head_dim */
  int64_t block_stride; /* elements between blocks: heads * block_size * head_dim */
  int64_t bytes_per_pool; /* bytes of ONE of k_pool / v_pool */
} pa_pool;

/*
 * Describe a pool (section 2 of the 7minutos.es article: a flat array of
 * equal pages).  Allocates nothing; fills *out.  num_blocks * block_size must
 * stay below 2^31 so that slots fit int32.
 * Errors: PA_ERR_INVALID_ARG (non-positive sizes, null out, slot overflow),
 *         PA_ERR_UNSUPPORTED (block_size != 16, head_dim not 64/128, dtype).
 */
pa_status pa_pool_create(int64_t num_blocks, int32_t block_size, int32_t heads,
                         int32_t head_dim, int32_t dtype, pa_pool* out);

/*
 * Grouped-query attention (no counterpart on the pages, which use one query
 * head per KV head): declare that q and out carry num_q_heads heads, a
 * multiple (1, 2, 4 or 8) of the pool's KV heads.  Query head h reads KV
 * head h / (num_q_heads / heads).  The pool itself (and reshape_and_cache,
 * copy_blocks, k_new and v_new) keeps the KV head count.  The KV tile is read
 * once per KV head and shared by its query heads.
 */
pa_status pa_pool_set_query_heads(pa_pool* pool, int32_t num_q_heads);

/*
 * Write each new token's K and V rows into the slot slot_mapping names:
 * k_pool[slot / bs][h][slot % bs][:] = k_new[t][h][:] for every head, the
 * same for V (7minutos.es section 2: the new token goes into the tail page).
 * Bit copy.  A negative slot is skipped; a slot >= num_blocks * block_size
 * sets PA_DEVERR_SLOT and is skipped.  num_tokens == 0 is a no-op.
 */
pa_status pa_reshape_and_cache(const pa_pool* pool, const void* k_new, const void* v_new,
                               const int32_t* slot_mapping, int32_t num_tokens, void* k_pool,
                               void* v_pool, void* stream);

/*
 * Bytes of device workspace pa_decode_attention needs for these sizes
 * (work plan + split-K partial results).  With partition_size 0 the result
 * covers every automatic choice.  max_context_len 0 = max_blocks_per_seq *
 * block_size.
 */
pa_status pa_decode_workspace_bytes(const pa_pool* pool, int32_t num_seqs,
                                    int32_t max_blocks_per_seq, int32_t max_context_len,
                                    int32_t partition_size, size_t* bytes);

/*
 * Single-query decode attention over the paged cache ("PagedAttention" wiki
 * mirror, "Formulació matemàtica"): for every sequence s and head h,
 *   out[s][h] = sum_t softmax_t(scale * q[s][h] . K_t) V_t,  t < context_lens[s],
 * with K_t, V_t read through block_tables[s].  fp32 accumulation, online
 * softmax; the result is rounded to the pool dtype.  A sequence of length 0
 * gets zeros.
 * Long contexts are split into partitions of partition_size tokens (a
 * multiple of 16 up to 4096) whose partial results are merged by
 * log-sum-exp, in partition order, by the last CTA to finish a sequence.
 * partition_size 0 chooses automatically: 512-token partitions while
 * sequences x head groups already give two work items per resident CTA
 * (one with 2-8 query heads per KV head on fp16/bf16 pools), otherwise
 * about four items per resident CTA (never below 256 tokens).  The work
 * order is planned on the device from context_lens (longest partitions
 * first).
 * max_context_len bounds every context_lens[s] (0 = max_blocks_per_seq *
 * block_size); a length above it or above the table width sets
 * PA_DEVERR_CONTEXT_LEN and is clamped.  Block ids outside the pool set
 * PA_DEVERR_BLOCK_ID and are replaced by block 0.
 * workspace: device buffer of at least pa_decode_workspace_bytes(); its
 * contents on entry do not matter.  Calls that share a workspace must be
 * ordered on one stream.
 * Errors: PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA.
 */
pa_status pa_decode_attention(const pa_pool* pool, const void* q, const void* k_pool,
                              const void* v_pool, const int32_t* block_tables,
                              int32_t max_blocks_per_seq, const int32_t* context_lens,
                              int32_t num_seqs, int32_t max_context_len, float scale, void* out,
                              void* workspace, size_t workspace_bytes, int32_t partition_size,
                              void* stream);

/*
 * The two halves of pa_decode_attention, for callers that run many layers
 * over the same context lengths in one step (every layer of a model shares
 * the step's block tables and lengths):
 *   pa_decode_plan writes the work plan (clamped lengths, partitions per
 *   sequence, work items ordered longest first) into the workspace;
 *   pa_decode_attention_planned runs the partition and merge kernels from it.
 * A plan stays valid for any number of planned calls with the same pool
 * geometry (heads, head_dim, dtype), num_seqs, max_blocks_per_seq,
 * max_context_len and partition_size, issued in stream order on the same
 * workspace; each planned call leaves the plan ready for the next.  The
 * library records the parameters of every plan it writes, per workspace: a
 * planned call whose arguments resolve to others, or that finds no plan in
 * its workspace, returns PA_ERR_INVALID_ARG without launching.
 * Each plan also carries a stamp, a number the host draws for it, in the
 * workspace header.  The kernels check it on the device: a launch that
 * finds another stamp (the workspace was freed and reused, overwritten or
 * zeroed since the plan was written, or holds an older plan) raises
 * PA_DEVERR_PLAN and touches neither the workspace nor out.  Every plan
 * entry a launch uses is bounds-checked before it indexes anything; a
 * damaged entry raises PA_DEVERR_PLAN and its work item is skipped.
 * After PA_DEVERR_TIMEOUT the outputs of that launch are undefined, and the
 * plan is marked so that later planned launches on it are refused
 * (PA_DEVERR_PLAN) until pa_decode_plan rewrites it: a launch that gave up
 * may leave the split-K merge counters mid-count.
 */
pa_status pa_decode_plan(const pa_pool* pool, const int32_t* context_lens, int32_t num_seqs,
                         int32_t max_blocks_per_seq, int32_t max_context_len,
                         int32_t partition_size, void* workspace, size_t workspace_bytes,
                         void* stream);

pa_status pa_decode_attention_planned(const pa_pool* pool, const void* q, const void* k_pool,
                                      const void* v_pool, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, int32_t num_seqs,
                                      int32_t max_context_len, float scale, void* out,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t partition_size, void* stream);

/*
 * Fused append + attend: pa_reshape_and_cache of each sequence's new token
 * followed by pa_decode_attention, in one pass.  k_new, v_new are
 * [num_seqs][heads][head_dim] (pool dtype, 16-byte aligned): the token of
 * sequence s is written at its position context_lens[s] - 1, i.e. slot
 * block_tables[s][(L-1)/bs] * bs + (L-1) % bs, and attended to with the rest.
 * The pools after the call, and the output, are bit-identical to the two
 * separate calls.  Sequences of length 0 append nothing.  The block holding
 * the new token must be private to its sequence (copy it on write first, as
 * for pa_reshape_and_cache).  The planned form takes a plan written by
 * pa_decode_plan, with the same rules as pa_decode_attention_planned.
 */
pa_status pa_decode_append_attention(const pa_pool* pool, const void* q, const void* k_new,
                                     const void* v_new, void* k_pool, void* v_pool,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t num_seqs,
                                     int32_t max_context_len, float scale, void* out,
                                     void* workspace, size_t workspace_bytes,
                                     int32_t partition_size, void* stream);

pa_status pa_decode_append_attention_planned(const pa_pool* pool, const void* q,
                                             const void* k_new, const void* v_new, void* k_pool,
                                             void* v_pool, const int32_t* block_tables,
                                             int32_t max_blocks_per_seq, int32_t num_seqs,
                                             int32_t max_context_len, float scale, void* out,
                                             void* workspace, size_t workspace_bytes,
                                             int32_t partition_size, void* stream);

/*
 * Decode over shared prefixes ("Atención paginada en modelos de lenguaje
 * grandes (LLM)", 7minutos.es, section 3: requests with the same system
 * prompt point at the same physical pages; "PagedAttention" wiki mirror,
 * "Descripció": blocks shared across requests and branches).  Same result as
 * pa_decode_attention, computed so that each shared block is read once for
 * all the sequences holding it.
 * Groups (device int32 arrays, CSR): members of group g are
 * group_members[group_offsets[g] .. group_offsets[g+1]) (num_members entries
 * in all; offsets outside them reject the group); they all hold the
 * same physical blocks as the group's first member in their first
 * group_blocks[g] table entries, and those blocks are full (16 tokens).
 * A tensor-core kernel attends every member's query heads to the shared
 * blocks (one partial result per 16-block chunk); the decode kernel attends
 * each sequence to the rest of its context and merges everything by
 * log-sum-exp.  Three launches on `stream`: the plan, the shared-prefix
 * kernel, and the decode kernel as a programmatic dependent launch that may
 * run alongside the shared-prefix kernel and waits for it before any merge
 * that reads its partials.  fp16/bf16 pools only (PA_ERR_UNSUPPORTED for
 * fp32).
 * max_group_size and max_shared_blocks bound the group sizes and
 * group_blocks (launch sizing); a group beyond either bound is reported
 * (PA_DEVERR_CONTEXT_LEN) and its members attend alone.  A member that is
 * too short, holds different blocks or belongs to two groups raises
 * PA_DEVERR_CONTEXT_LEN and attends to its whole context on its own, so the
 * result stays correct.
 * Workspace: pa_decode_shared_prefix_workspace_bytes (max_shared_blocks
 * extra slots per head).  pa_find_shared_prefixes builds groups from host
 * block tables.  partition_size 0 here means 256-token partitions: the
 * decode kernel attends only each sequence's own tokens, typically far
 * fewer than max_context_len.
 */
pa_status pa_decode_shared_prefix_workspace_bytes(const pa_pool* pool, int32_t num_seqs,
                                                  int32_t max_blocks_per_seq,
                                                  int32_t max_context_len, int32_t partition_size,
                                                  int32_t max_shared_blocks, size_t* bytes);

pa_status pa_decode_attention_shared_prefix(
    const pa_pool* pool, const void* q, const void* k_pool, const void* v_pool,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
    int32_t num_seqs, const int32_t* group_offsets, const int32_t* group_members,
    int32_t num_members, const int32_t* group_blocks, int32_t num_groups, int32_t max_group_size,
    int32_t max_shared_blocks, int32_t max_context_len, float scale, void* out, void* workspace,
    size_t workspace_bytes, int32_t partition_size, void* stream);

/*
 * Paged prefill: many new query tokens per sequence attend causally to the
 * sequence's paged cache ("PagedAttention" wiki mirror, "Formulació
 * matemàtica": the block-wise form holds for every query token).  Sequence s
 * has n_s = query_start[s+1] - query_start[s] new tokens, rows
 * query_start[s].. of q and out ([T][heads * q_per_kv][head_dim]); they sit
 * at positions context_lens[s] - n_s .. context_lens[s] - 1 and their K/V
 * must already be in the pool (pa_reshape_and_cache).  Query i sees tokens
 * 0..its position.  max_new_tokens bounds every n_s (launch sizing).
 * Runs on tcgen05 tensor cores with TMEM accumulators; fp16/bf16 pools,
 * head_dim 64 or 128.  num_tokens is the number of rows q and out hold.  A
 * context length below n_s or above the table, n_s above max_new_tokens, or
 * rows outside [0, num_tokens) raise PA_DEVERR_CONTEXT_LEN and that sequence
 * is skipped (its rows of out are not written).
 */
pa_status pa_prefill_attention(const pa_pool* pool, const void* q, const void* k_pool,
                               const void* v_pool, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* context_lens,
                               const int32_t* query_start, int32_t num_seqs, int32_t num_tokens,
                               int32_t max_new_tokens, int32_t max_context_len, float scale,
                               void* out, void* stream);

/*
 * Decode attention that allocates nothing.  Same computation, arguments and
 * errors as pa_decode_attention, minus the workspace: the plan and split-K
 * partials live in a static device buffer inside the library of
 * PA_STATIC_SCRATCH_BYTES (32 MiB), which every GPU that loads the library
 * holds until the process exits.  No counterpart on the pages: it exists for
 * callers that may not call cudaMalloc, such as plugins hosted by a runtime
 * that owns all device memory through its own pool, or latency-bound loops
 * that cannot afford cudaMalloc's implicit device synchronisation.
 * Sizes whose workspace (pa_decode_workspace_bytes) exceeds the buffer are
 * rejected with PA_ERR_WORKSPACE before anything is launched.
 * The first call on each device resolves the buffer's device address (with
 * that device current); make that first call before any stream capture.
 * All calls share the one buffer: calls that overlap on the GPU (different
 * streams, or different threads without ordering) race and corrupt each
 * other's results; order them on one stream.  The buffer keeps the last
 * call's contents; each call rewrites every part it reads.
 */
#define PA_STATIC_SCRATCH_BYTES (32u << 20)
pa_status pa_decode_attention_static(const pa_pool* pool, const void* q, const void* k_pool,
                                     const void* v_pool, const int32_t* block_tables,
                                     int32_t max_blocks_per_seq, const int32_t* context_lens,
                                     int32_t num_seqs, int32_t max_context_len, float scale,
                                     void* out, int32_t partition_size, void* stream);

/*
 * Block-granular copy-on-write, device half ("PagedAttention" wiki mirror,
 * "Descripció"; 7minutos.es section 3, cow_copy): for each (src, dst) row of
 * pairs (device int32 [num_pairs][2]) copy the whole physical block, every
 * head and slot, of K and of V.  Bit copy.  No dst may be another pair's src
 * or dst (the block manager hands out fresh destinations).  Ids outside the
 * pool set PA_DEVERR_PAIR and the pair is skipped.
 */
pa_status pa_copy_blocks(const pa_pool* pool, void* k_pool, void* v_pool, const int32_t* pairs,
                         int32_t num_pairs, void* stream);

/*
 * Synchronise `stream`, then return in *flags the PA_DEVERR_* bits raised on
 * the current device since the last call, and clear them.  Returns
 * PA_ERR_OUT_OF_BOUNDS / PA_ERR_TIMEOUT when a bit is set, else PA_OK.
 */
pa_status pa_device_errors(void* stream, uint32_t* flags);

/*
 * Self-test of the device-side wait limit: launches one warp that waits on
 * an mbarrier nothing will complete, so the bounded wait used by the decode
 * pipeline runs out (about one second), raises PA_DEVERR_TIMEOUT and returns.
 * Nothing faults and the context stays usable; read the bit with
 * pa_device_errors().  No counterpart on the pages: it exists to test the
 * failure path without a GPU fault.
 */
pa_status pa_selftest_wait_timeout(void* stream);

/* Message of the last failing call on this thread ("" if none). */
const char* pa_last_error(void);
/* Fixed name of a status code. */
const char* pa_status_string(int32_t status);

/* ---- host block manager (reference counts and free list stay on the host) ----
 * 7minutos.es, sections 2 and 3: a pool of pages with a free list and a
 * reference count per page; a page returns to the free list as soon as its
 * count reaches zero.  The lowest free id is handed out first.  Not
 * thread-safe: one manager per thread, or lock around it. */
typedef struct pa_allocator pa_allocator;

pa_status pa_alloc_create(int64_t num_blocks, pa_allocator** out);
void pa_alloc_destroy(pa_allocator* a);
/* Take the lowest free block (refcount becomes 1); PA_ERR_NO_FREE_BLOCKS if none. */
pa_status pa_alloc_block(pa_allocator* a, int32_t* block_id);
/* share(): one more holder of a live block; allocates nothing. */
pa_status pa_share_block(pa_allocator* a, int32_t block_id);
/* Drop one holder; at zero the block goes back to the free list. */
pa_status pa_free_block(pa_allocator* a, int32_t block_id);
/* cow_copy(): allocate a private block for one holder of a live block and
 * drop that holder's reference to the original.  The caller copies the data
 * (pa_copy_blocks). */
pa_status pa_cow_block(pa_allocator* a, int32_t block_id, int32_t* new_block_id);
pa_status pa_refcount(const pa_allocator* a, int32_t block_id, int32_t* refcount);
int64_t pa_num_free(const pa_allocator* a);

/*
 * Append num_new tokens to one sequence (generate_token() of section 2).
 * block_table holds ceil(*context_len / block_size) live block ids and has
 * room for max_blocks.  For each new token at position p: a fresh block is
 * taken when p is a multiple of block_size; otherwise, if the tail block is
 * shared (refcount > 1), it is copied on write (section 3) and the
 * (src, dst) pair is appended to cow_pairs (room for num_new pairs).
 * slots[i] receives the physical slot of the i-th new token.  On error the
 * tokens appended before it stay appended (*context_len and *num_cow say how
 * far it got).
 */
pa_status pa_append_tokens(pa_allocator* a, int32_t block_size, int32_t* block_table,
                           int32_t max_blocks, int32_t* context_len, int32_t num_new,
                           int32_t* slots, int32_t* cow_pairs, int32_t* num_cow);

/* Give dst_table the same blocks as src_table (prefix sharing: one share()
 * per block). */
pa_status pa_fork_table(pa_allocator* a, const int32_t* src_table, int32_t num_blocks,
                        int32_t* dst_table);

/* Drop the sequence's reference to each of its blocks (request finished). */
pa_status pa_release_table(pa_allocator* a, const int32_t* block_table, int32_t num_blocks);

/*
 * Host helper: find shared prefixes in host block tables.  Sequences whose
 * first table entries name the same block are candidates; a candidate set of
 * two or more becomes a group whose shared length is the longest run of
 * leading full blocks every member has in common (at least
 * min_shared_blocks, else no group).  Outputs (host arrays sized num_seqs + 1,
 * num_seqs, num_seqs): CSR offsets, members in table order, shared blocks;
 * *num_groups, *max_group_size, *max_shared_blocks.
 */
pa_status pa_find_shared_prefixes(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t num_seqs,
                                  int32_t block_size, int32_t min_shared_blocks,
                                  int32_t* group_offsets, int32_t* group_members,
                                  int32_t* group_blocks, int32_t* num_groups,
                                  int32_t* max_group_size, int32_t* max_shared_blocks);

/* Host helper for tables built elsewhere: slot of the last token of each
 * sequence, block_tables[s][(L-1)/bs] * bs + (L-1) % bs, or -1 when L == 0.
 * All pointers are host memory. */
pa_status pa_decode_slots(const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t num_seqs, int32_t block_size,
                          int32_t* slots);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
