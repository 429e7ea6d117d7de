/*
 * pa.h - C ABI of the B200 paged KV-cache library (libpa_b200.so): cache
 * writes (pa_reshape_and_cache), decode attention (pa_decode,
 * pa_decode_static), prefill-chunk attention (pa_prefill), copy-on-write
 * copies (pa_copy_blocks) and the host block allocator / manager.
 *
 * PagedAttention keeps each request's K/V cache in fixed-size physical blocks
 * that a per-request block table maps from logical order; attention reads the
 * scattered blocks through that table.  Sources, by page title and section:
 *   [KVC]  "KV Cache & PagedAttention" studynote (agnusdei1207), II
 *          (block table, copy-on-write) and III (attention kernel modified);
 *   [VLLM] "vLLM PagedAttention" studynote (agnusdei1207), II (fixed-size
 *          blocks, e.g. 16 tokens; logical -> physical block table);
 *   [119]  "09. PagedAttention" (119-ai-studio), 해법 (logical / physical
 *          blocks, block table; only the last block is partly filled);
 *   [VEL]  "Paged Attention" (velog @junegood), 작동 예시 (on-demand block
 *          growth), 메모리 공유 (copy-on-write for beams), 구현 세부사항
 *          (BlockAllocator.allocate_block / free_block).
 *
 * Conventions for every call:
 *  - Return value: a pa_status (0 = PA_OK).  Host-side argument checks run
 *    before anything is launched; a failed check launches nothing.
 *  - Device pointers are caller-owned (e.g. PyTorch tensors).  The library
 *    never allocates or frees device memory and never synchronises; it
 *    launches only on `stream` (a cudaStream_t; NULL = legacy default stream).
 *  - `err_flag` (nullable) is a device int32 that kernels set to a
 *    PA_DEV_* code when they meet bad data (first code wins; 0 is never
 *    written).  The bad access is skipped; no kernel traps.  The caller
 *    clears and reads it.
 *  - Cache layout (part of this ABI): key_cache and value_cache are each
 *    [num_blocks][num_kv_heads][block_size][head_dim] elements of `dtype`,
 *    row-major, 16-byte aligned.  One (block, KV head) tile is
 *    block_size*head_dim contiguous elements; slot = block*block_size + offset.
 *  - Supported: head_dim 64 or 128; block_size 8, 16, 32, 64 or 128;
 *    dtype f32, f16, bf16 (pa_prefill: f16, bf16); num_q_heads =
 *    G * num_kv_heads with G in 1,2,4,8.
 *  - Host objects (allocator, manager) are not thread-safe.
 */
#ifndef PA_B200_H
#define PA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID = -1,      /* bad argument (null pointer, size, range) */
    PA_ERR_UNSUPPORTED = -2,  /* valid but not built (head_dim, dtype, G)  */
    PA_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed      */
    PA_ERR_OOM = -4,          /* the block pool is empty                   */
    PA_ERR_STATE = -5         /* refcount / sequence state violated        */
} pa_status;

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/* Codes written to *err_flag by kernels. */
enum {
    PA_DEV_BAD_SLOT = 1,      /* slot_mapping entry >= num_blocks*block_size */
    PA_DEV_BAD_BLOCK = 2,     /* block table entry outside [0, num_blocks)   */
    PA_DEV_BAD_LEN = 3,       /* context_len < 0, > max_context_len, or
                                 > max_blocks_per_seq*block_size (clamped)  */
    PA_DEV_BAD_PAIR = 4,      /* copy pair id outside [0, num_blocks)        */
    PA_DEV_TIMEOUT = 5        /* a pipeline wait exceeded its time limit     */
};

/* Human-readable name of a pa_status. */
const char* pa_status_string(int status);
/* ABI version (major*100 + minor). */
int pa_version(void);

/* --------------------------------------------------------------------------
 * pa_reshape_and_cache - write each new token's K and V rows into its slot.
 *
 * [119] 해법 / [VEL] 작동 예시: a token's K/V goes into the physical block the
 * table assigns to its logical position.  For t < num_tokens and every KV
 * head h:  key_cache[s / bs][h][s % bs][:] = key[t][h][:]  (same for value),
 * s = slot_mapping[t].  s < 0 marks padding: skipped.  s >= num_blocks*bs sets
 * PA_DEV_BAD_SLOT and is skipped.
 *   key, value    device [num_tokens][num_kv_heads][head_dim] dtype, contiguous
 *   slot_mapping  device int64 [num_tokens]; distinct non-negative entries
 * Bit copy: the cache holds exactly the input bits.  The kernel is a
 * programmatic dependent of the kernel before it in the stream and touches
 * memory only after that kernel has completed; it lets the kernel after it
 * (pa_decode, pa_prefill) start early.
 */
int pa_reshape_and_cache(const void* key, const void* value, void* key_cache,
                         void* value_cache, const int64_t* slot_mapping,
                         int num_tokens, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* err_flag, void* stream);

/* --------------------------------------------------------------------------
 * pa_decode - one decode step of paged attention.
 *
 * [KVC] II-III / [119] 해법: attention reads K/V through the block table.  For
 * sequence s, query head h, KV head j = h / G (G = num_q_heads/num_kv_heads),
 * tokens t < L = context_lens[s] (L counts the token written this step):
 *   K_t = key_cache[block_tables[s][t / bs]][j][t % bs][:],  V_t likewise,
 *   x_t = scale * <query[s][h], K_t>,  w = softmax(x),  out[s][h] = sum_t w_t V_t
 * fp32 accumulation; out is rounded to nearest even in dtype.  L = 0 gives 0.
 * Long contexts are split into partitions of `partition_size` tokens
 * (a positive multiple of 16; 0 = one partition per sequence) whose partial
 * results are merged with their log-sum-exp weights.  With the tensor-core
 * engine and ceil(max_context_len / partition_size) <= 4 the work unit that
 * completes a split sequence merges it inside the decode kernel (one launch
 * per call); otherwise, when ceil(max_context_len / partition_size) > 1, a
 * second kernel on the same stream merges (two launches).
 *   out           device [num_seqs][num_q_heads][head_dim] dtype
 *   query         device [num_seqs][num_q_heads][head_dim] dtype, 16-B aligned
 *   block_tables  device int32 [num_seqs][max_blocks_per_seq]; entries past
 *                 ceil(L/bs) are ignored (conventionally -1)
 *   context_lens  device int32 [num_seqs]
 *   max_context_len  host upper bound of context_lens (sizes the workspace)
 *   workspace     device, >= pa_decode_workspace_size() bytes, 256-B aligned;
 *                 must be zero-filled before its first use (see
 *                 pa_decode_workspace_init); every call leaves its scheduler
 *                 words and split counters zero again, also after a
 *                 PA_DEV_TIMEOUT.  Calls sharing one workspace must not
 *                 overlap on the GPU.
 * The physical placement of blocks does not change the result: summation
 * order depends only on logical token positions.
 * Launch order: the decode kernel is a programmatic dependent of the kernel
 * before it in the stream.  It may read context_lens and block_tables before
 * that kernel has completed if that kernel lets dependents start early
 * (griddepcontrol.launch_dependents); everything else (queries, cache,
 * workspace, every write) waits for its completion.  Of this library's
 * kernels pa_reshape_and_cache and the tensor-core decode kernel let their
 * dependents start early (the decode from its start when no merge kernel
 * follows it, so the next step's decode sets up during this one's tail);
 * none writes lengths or tables.
 * A kernel launched after pa_decode with programmatic stream serialization
 * must wait (griddepcontrol.wait) before it reads what the call writes.
 */
int pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads,
                             int head_dim, int max_context_len,
                             int partition_size, size_t* bytes);
int pa_decode_workspace_init(void* workspace, size_t workspace_bytes, void* stream);
int pa_decode(void* out, const void* query, const void* key_cache,
              const void* value_cache, const int32_t* block_tables,
              int max_blocks_per_seq, const int32_t* context_lens,
              int max_context_len, int num_seqs, int num_q_heads,
              int num_kv_heads, int head_dim, int block_size, int num_blocks,
              float scale, int partition_size, void* workspace,
              size_t workspace_bytes, pa_dtype dtype, int32_t* err_flag,
              void* stream);

/* pa_decode_static - pa_decode without a caller-provided workspace, for
 * callers that cannot allocate device memory (a plugin inside a host that
 * owns every device allocation, a fixed memory budget, or a latency-critical
 * path where cudaMalloc's possible device synchronisation is not acceptable).
 * The pages have no counterpart: this is an interface convenience.
 * The workspace is a fixed array of PA_DECODE_STATIC_WORKSPACE_BYTES that the
 * library keeps in device memory on every GPU that loads it, until exit.
 * Arguments and results are those of pa_decode.  A call whose workspace
 * (pa_decode_workspace_size) exceeds the array returns PA_ERR_INVALID and
 * launches nothing, and so does a call that fails any other of pa_decode's
 * host checks.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current, and looks it up
 * again when the current context changes (e.g. after cudaDeviceReset); make
 * that first call before any stream capture.  Each call clears the scheduler
 * words on `stream` and then runs the decode with pa_decode's defaults.  All
 * calls on a device share the one array and it keeps the last call's
 * contents: calls that overlap on the GPU race and must be serialised by the
 * caller (e.g. one stream).  Allocates nothing. */
#define PA_DECODE_STATIC_WORKSPACE_BYTES (16u << 20)
int pa_decode_static(void* out, const void* query, const void* key_cache,
                     const void* value_cache, const int32_t* block_tables,
                     int max_blocks_per_seq, const int32_t* context_lens,
                     int max_context_len, int num_seqs, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     float scale, int partition_size, pa_dtype dtype,
                     int32_t* err_flag, void* stream);

/* pa_decode_ex - pa_decode with per-call options; options = NULL is exactly
 * pa_decode.  The options apply to this call only (no process-wide state).
 *   struct_size  sizeof(pa_decode_options) as the caller was compiled; at
 *                least the size of the first three fields (a smaller value
 *                returns PA_ERR_INVALID).  Fields past struct_size read as
 *                zero / NULL, so callers built against an older header keep
 *                working.
 *   engine       PA_ENGINE_AUTO (pa_decode's choice): tcgen05 tensor-core
 *                MMAs with accumulators in tensor memory for f16/bf16 (the
 *                CUDA-core engine when its shared-memory ring does not fit,
 *                i.e. several thousand sequences), CUDA cores for f32.
 *                PA_ENGINE_CUDA_CORE: fp32 dot products on CUDA cores, any
 *                dtype.  PA_ENGINE_TENSOR: the tensor-core engine, f16/bf16
 *                only (f32 returns PA_ERR_UNSUPPORTED).
 *   test_withhold_stage  failure-detection test aid, -1 = off.  With s >= 0
 *                the producer that takes the first work unit of this call
 *                withholds that unit's stage s (no copies, no arrival on the
 *                stage's barrier), so the warps that need it give up after
 *                the 2 s wait limit, set PA_DEV_TIMEOUT in err_flag and
 *                return; the context and the workspace stay usable.  No GPU
 *                fault is involved.  The pages have no counterpart.
 *   key_new, value_new, slot_mapping  the step's cache write, done by this
 *                call ([VEL] 작동 예시 / [119] 해법: the new token's K/V goes
 *                into the slot its table assigns, then attention reads it).
 *                All NULL (the default): no write.  All set: the result is
 *                that of pa_reshape_and_cache(key_new, value_new, ...,
 *                slot_mapping, num_tokens = num_seqs) on the same stream
 *                followed by this decode, with one difference in launches:
 *                the tensor-core engine writes each sequence's token from
 *                inside the decode kernel, just before the copy of the block
 *                that holds it (one launch fewer per step); the CUDA-core
 *                engine launches the cache write first.
 *                  key_new, value_new  device [num_seqs][num_kv_heads][head_dim]
 *                    dtype, contiguous, 16-B aligned: row s is sequence s's
 *                    new token (the one at position context_lens[s] - 1)
 *                  slot_mapping  device int64 [num_seqs]: slot_mapping[s] <
 *                    0 skips sequence s's write; otherwise it must be the
 *                    slot of position context_lens[s] - 1 through
 *                    block_tables[s], else PA_DEV_BAD_SLOT is set and that
 *                    token is not written (any engine).
 *                The block holding a written slot must not be read by another
 *                sequence of this call (a block manager's copy-on-write
 *                before the write guarantees it); otherwise what that other
 *                sequence reads of the written row is unspecified.
 *                Only some of the three set: PA_ERR_INVALID.
 * Out-of-range option values return PA_ERR_INVALID before any launch. */
enum { PA_ENGINE_AUTO = 0, PA_ENGINE_CUDA_CORE = 1, PA_ENGINE_TENSOR = 2 };
typedef struct pa_decode_options {
    int struct_size;
    int engine;
    int test_withhold_stage;
    const void* key_new;
    const void* value_new;
    const int64_t* slot_mapping;
} pa_decode_options;
int pa_decode_ex(void* out, const void* query, const void* key_cache,
                 const void* value_cache, const int32_t* block_tables,
                 int max_blocks_per_seq, const int32_t* context_lens,
                 int max_context_len, int num_seqs, int num_q_heads,
                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                 float scale, int partition_size, void* workspace,
                 size_t workspace_bytes, pa_dtype dtype, int32_t* err_flag,
                 void* stream, const pa_decode_options* options);

/* --------------------------------------------------------------------------
 * pa_prefill - causal multi-query attention of prefill chunks over the paged
 * cache (tiled attention over paged K/V: "KV Cache & PagedAttention"
 * studynote, section III, where the serving stack pairs FlashAttention with
 * PagedAttention; the pages give no formula, the chunk reading is the plain
 * causal one).
 *
 * Sequence s holds context_lens[s] tokens in the cache; its chunk is its last
 * n_s = cu_seqlens_q[s+1] - cu_seqlens_q[s] tokens, whose K/V must already be
 * written (pa_reshape_and_cache).  Chunk row i, packed row cu_seqlens_q[s] + i
 * of `query`, sits at position p = context_lens[s] - n_s + i and attends to
 * the sequence's tokens 0..p:
 *   out[row][h] = sum_{t<=p} softmax_t(scale * <query[row][h], K_t>) V_t,
 * query head h reading KV head h / (num_q_heads / num_kv_heads).  n_s = 1 is
 * a decode step; n_s = context_lens[s] a whole prompt.
 *
 *   out          [total_q][num_q_heads][head_dim]  device, written
 *   query        [total_q][num_q_heads][head_dim]  device
 *   key_cache, value_cache, block_tables, num_blocks: as pa_decode
 *   context_lens [num_seqs] int32 device (they count the chunk)
 *   cu_seqlens_q [num_seqs + 1] int32 device, 0 = cu[0] <= ... <= cu[num_seqs]
 *                = total_q
 *   max_query_len  an upper bound of every n_s (it sizes the launch)
 *   workspace    device, >= PA_PREFILL_WORKSPACE_BYTES, 16-byte aligned, owned
 *                by the caller: the work-item counter of the persistent launch
 *                (one CTA per SM takes pairs of query tiles until none is
 *                left).  Zero-filled before its first use; every call leaves
 *                it zeroed again (also after a timeout), so it is reused as is.
 *                Calls that may run at the same time need distinct workspaces.
 *   dtype        PA_F16 or PA_BF16 (tensor cores); PA_F32 -> PA_ERR_UNSUPPORTED
 * head_dim 64 or 128; num_q_heads / num_kv_heads in {1, 2, 4, 8}; block_size
 * 8, 16, 32, 64 or 128; every pointer 16-byte aligned.  Nothing is allocated;
 * asynchronous on `stream`.  Device-side errors (err_flag, first code wins):
 * PA_DEV_BAD_LEN when context_lens[s] < 0 or > max_blocks_per_seq *
 * block_size, n_s > context_lens[s] or > max_query_len, or cu_seqlens_q
 * leaves [0, total_q] (rows of that sequence may then be left unwritten);
 * PA_DEV_BAD_BLOCK for a table entry outside [0, num_blocks) that a chunk
 * reads (those tokens are skipped); PA_DEV_TIMEOUT as pa_decode.
 * Returns PA_OK, PA_ERR_INVALID (a null or short workspace included),
 * PA_ERR_UNSUPPORTED or PA_ERR_CUDA. */
#define PA_PREFILL_WORKSPACE_BYTES 64u
int pa_prefill(void* out, const void* query, const void* key_cache, const void* value_cache,
               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
               const int32_t* cu_seqlens_q, int num_seqs, int total_q, int max_query_len,
               int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
               float scale, void* workspace, size_t workspace_bytes, pa_dtype dtype,
               int32_t* err_flag, void* stream);

/* --------------------------------------------------------------------------
 * pa_copy_blocks - copy-on-write block copies.
 *
 * [KVC] II (copy-on-write) / [VEL] 메모리 공유: before a sharer writes into a
 * shared block, the block is copied to a fresh one.  For each pair p:
 * key_cache[dst] = key_cache[src] (all KV heads and offsets), same for value.
 *   block_pairs  device int64 [num_pairs][2] = (src, dst); dsts distinct and
 *                disjoint from srcs.  An id outside [0, num_blocks) sets
 *                PA_DEV_BAD_PAIR and that pair is skipped.
 */
int pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs,
                   int num_pairs, int num_kv_heads, int head_dim, int block_size,
                   int num_blocks, pa_dtype dtype, int32_t* err_flag, void* stream);

/* --------------------------------------------------------------------------
 * Host block allocator ([VEL] 구현 세부사항: allocate_block / free_block).
 *
 * A first-in-first-out pool of free physical block ids with a reference
 * count per block.  create: `free_order` (nullable) lists the ids handed out
 * first, `num_free` of them; ids not listed start held (count 1) by an outside
 * owner, which models a pool other requests have fragmented.  NULL = all ids
 * free in ascending order.  allocate: pops the front (count 1), PA_ERR_OOM
 * when empty.  incref: shares an allocated block (PA_ERR_STATE if free).
 * free: drops one reference; at zero the id joins the back of the pool;
 * PA_ERR_STATE on a free block (double free).
 */
typedef struct pa_allocator pa_allocator;
int pa_allocator_create(int num_blocks, const int32_t* free_order, int num_free,
                        pa_allocator** out);
void pa_allocator_destroy(pa_allocator* a);
int pa_allocator_allocate(pa_allocator* a, int32_t* block_id);
int pa_allocator_incref(pa_allocator* a, int32_t block_id);
int pa_allocator_free(pa_allocator* a, int32_t block_id);
int pa_allocator_refcount(const pa_allocator* a, int32_t block_id, int32_t* refcount);
int pa_allocator_num_free(const pa_allocator* a, int32_t* num_free);

/* --------------------------------------------------------------------------
 * Host block-table manager: per-sequence logical -> physical tables over an
 * allocator ([119] 해법; [VEL] 작동 예시, 메모리 공유).
 *
 * append (one token at position p = current length): if p % bs == 0 a new
 * block is taken; otherwise the token goes into the last block, and if that
 * block is shared (count > 1) it is first replaced by a fresh block, the pair
 * (old, new) is reported for pa_copy_blocks and the old block loses one
 * reference.  slot = table[p / bs] * bs + p % bs.  Appends are all-or-nothing:
 * PA_ERR_OOM leaves every table and count unchanged, except that with the
 * prefix cache on, cached blocks that the call evicted to find room stay
 * evicted (they are back in the free pool; their cache entries are gone).
 *   pa_manager_append       num_tokens tokens to one sequence; slots[num_tokens];
 *                           cow_pairs int64 [>=1][2], *num_cow in {0,1}
 *   pa_manager_append_step  one token to each of seq_ids[0..n); slots[n];
 *                           cow_pairs int64 [n][2]; *num_cow <= n
 *   pa_manager_fork         child shares every block of parent (incref)
 *   pa_manager_free_seq     drops the sequence's references
 *   pa_manager_block_tables rows [n][max_blocks] padded with -1, lengths [n];
 *                           PA_ERR_INVALID if a table is longer than max_blocks
 * The manager borrows the allocator, which must outlive it.
 */
typedef struct pa_manager pa_manager;
int pa_manager_create(pa_allocator* alloc, int block_size, pa_manager** out);
void pa_manager_destroy(pa_manager* m);
int pa_manager_add_seq(pa_manager* m, int64_t seq_id);
int pa_manager_fork(pa_manager* m, int64_t parent, int64_t child);
int pa_manager_free_seq(pa_manager* m, int64_t seq_id);
int pa_manager_append(pa_manager* m, int64_t seq_id, int num_tokens,
                      int64_t* slots, int64_t* cow_pairs, int* num_cow);
int pa_manager_append_step(pa_manager* m, const int64_t* seq_ids, int num_seqs,
                           int64_t* slots, int64_t* cow_pairs, int* num_cow);
int pa_manager_seq_len(const pa_manager* m, int64_t seq_id, int32_t* len);
int pa_manager_block_tables(const pa_manager* m, const int64_t* seq_ids,
                            int num_seqs, int32_t* block_tables, int max_blocks,
                            int32_t* context_lens);

/* --------------------------------------------------------------------------
 * Prefix caching - [VLLM] prefix caching, [119] 다음 장: a prompt that starts
 * with the same tokens as an earlier one maps the same physical blocks
 * (reference counted) instead of storing them again.
 *   pa_manager_enable_prefix_cache  switch the cache on; PA_ERR_STATE once
 *                    the manager holds sequences.
 *   pa_manager_add_seq_prompt  new sequence whose first num_tokens tokens
 *                    have ids tokens[0..n).  Its leading full blocks are
 *                    looked up block by block (a block matches when the whole
 *                    token prefix up to its end matches: a 64-bit fingerprint
 *                    chained over the blocks, plus an exact comparison of the
 *                    block's own ids) until the first miss; hits are shared
 *                    (incref).  The block holding the prompt's last token is
 *                    never served from the cache (a prompt of whole blocks
 *                    looks up all but its last), so *num_cached < num_tokens
 *                    for any non-empty prompt and at least the last token is
 *                    left to compute.  The remaining tokens are appended as usual and
 *                    every full block they fill is cached.  slots[n]: -1 for
 *                    the *num_cached leading tokens served from the cache
 *                    (pa_reshape_and_cache skips them), the slot otherwise; so
 *                    the caller writes K/V through the same array.  A cached
 *                    block must hold its K/V before any sequence that hit it
 *                    is decoded (write this call's slots first).  PA_ERR_OOM
 *                    undoes the call except for evictions it made.
 *   pa_manager_prefix_cache_stats  stats int64 [4]: cached blocks, block
 *                    hits, block misses, evictions (cumulative).
 * The cache keeps one reference per cached block, so a cached block outlives
 * the sequences that used it.  When the free pool is empty, the least recently
 * used cached block that nothing else references is evicted (freed) first.
 * Appends of generated tokens (pa_manager_append*) are not cached.
 */
int pa_manager_enable_prefix_cache(pa_manager* m);
int pa_manager_add_seq_prompt(pa_manager* m, int64_t seq_id, const int32_t* tokens,
                              int num_tokens, int64_t* slots, int* num_cached);
int pa_manager_prefix_cache_stats(const pa_manager* m, int64_t* stats);

#ifdef __cplusplus
}
#endif
#endif /* PA_B200_H */
