/*
 * pa.h -- C ABI of libpa: the paged-KV-cache decode hot path on B200 (sm_100a).
 *
 * The operations of PagedAttention's decode path, as the pages describe them
 * (the first three are the hot path; the rest follow below):
 *
 *   pa_write_kv     store this step's new K/V rows in their cache slots
 *                   ("Optimizing LLM Inference: From PagedAttention to AI
 *                   Infra", section "Understanding KV Cache ...": K and V of
 *                   every token are kept at every layer so later steps read
 *                   them instead of recomputing them).
 *   pa_decode       single-token decode attention over a paged cache, walking
 *                   each sequence's block table in logical order (same page,
 *                   "PagedAttention: Decoupling Logical Context from
 *                   Contiguous GPU Memory", Figure 2; "The Memory Wall ...",
 *                   "How it Works Under the Hood" and "Show Me The Code").
 *                   Long contexts are cut into fixed token partitions whose
 *                   partial results a log-sum-exp reduce combines (the
 *                   "sequence splits" of "PagedAttention in Action ...",
 *                   section "New Developments in 2026").
 *   pa_copy_blocks  whole-block copies that fork a shared block on
 *                   copy-on-write ("Optimizing LLM Inference ...",
 *                   "Copy-on-Write"; "PagedAttention", "KV Cache Sharing
 *                   (Copy-on-Write)").
 *   pa_decode_persistent  pa_decode scheduled as a device-planned work queue.
 *   pa_prefill_chunk      attention of several query tokens per sequence
 *                         (chunked prefill, speculative verification).
 *   pa_swap_blocks        blocks between a device pool and a pinned host pool.
 *   pa_bm_*               host block manager: refcounted blocks, on-demand
 *                         allocation, copy-on-write decisions.
 *   pa_decode_static      pa_decode with a scratch array compiled into libpa.
 *   pa_read_probe         measurement utility: the streaming-read ceiling.
 *
 * Memory layout (all device memory, row-major, no padding):
 *   k_cache, v_cache : [num_blocks][num_kv_heads][PA_BLOCK_SIZE][head_dim]
 *                      16-bit elements (fp16 or bf16), 16-byte aligned base.
 *   q, out           : [num_seqs][num_q_heads][head_dim]
 *   k, v (new rows)  : [num_tokens][num_kv_heads][head_dim]
 *   block_tables     : int32 [num_seqs][block_table_stride]; entry j is the
 *                      physical block of logical block j (tokens 16j..16j+15).
 *                      Entries at or past ceil(context_len / 16) are not read.
 *   context_lens     : int32 [num_seqs], tokens to attend to, including the
 *                      token written by this step's pa_write_kv.
 *   slot_mapping     : int64 [num_tokens]; slot = physical_block * 16 + offset;
 *                      a negative slot marks a padding token and is skipped.
 *   GQA              : query head h reads KV head h / group_size.
 *
 * Ownership: the caller allocates and owns every buffer, the workspace and the
 * stream. The library borrows the pointers for the duration of the
 * asynchronous call, allocates no device memory, keeps no per-call state and
 * never synchronises the stream (exceptions, each documented below: the
 * scratch array of pa_decode_static and the host object a pa_bm handle owns).
 * Every call is stream-ordered on `stream` (a cudaStream_t; NULL is the legacy
 * default stream).
 *
 * Errors: problems visible on the host (a NULL pointer, an unsupported shape,
 * a too-small workspace, an out-of-range argument) return a status and launch
 * nothing. A failed launch returns PA_ERR_CUDA (pa_last_cuda_error() gives
 * the CUDA error string). Problems only visible in device data (a slot past
 * the pool, a table entry outside [0, num_blocks), a context length above
 * max_context_len) never fault and never trap: the offending token or block
 * is skipped (the context length is clamped to max_context_len) and one is
 * added to *dev_error when dev_error is not NULL. Device waits are bounded;
 * a wait that gives up adds PA_DEV_ERR_TIMEOUT to *dev_error.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_BLOCK_SIZE 16
#define PA_MAX_LAYERS 256
#define PA_DEV_ERR_TIMEOUT (1 << 24)

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,
  PA_ERR_UNSUPPORTED = 2,
  PA_ERR_WORKSPACE_TOO_SMALL = 3,
  PA_ERR_CUDA = 4,
  PA_ERR_OUT_OF_BLOCKS = 5 /* block manager: not enough free blocks; nothing changed */
} pa_status;

typedef enum { PA_DTYPE_F16 = 0, PA_DTYPE_BF16 = 1 } pa_dtype;

/*
 * Store num_tokens new K/V rows in the caches: token t goes to slot
 * slot_mapping[t] of every KV head, i.e. k_cache[slot / 16][h][slot % 16][:]
 * = k[t][h][:], and the same for v. A bit copy.
 *   k, v            device, [num_tokens][num_kv_heads][head_dim]
 *   k_cache, v_cache device, [num_blocks][num_kv_heads][16][head_dim]
 *   slot_mapping    device int64 [num_tokens]
 *   block_size      must be 16; head_dim must be a multiple of 8, <= 1024
 *   dev_error       device int32 counter or NULL (slots >= num_blocks * 16)
 * num_tokens == 0 is a no-op. Two tokens with the same slot race.
 */
pa_status pa_write_kv(const void* k, const void* v, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int32_t num_tokens,
                      int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                      int64_t num_blocks, pa_dtype dtype, int32_t* dev_error,
                      void* stream);

/*
 * Bytes of workspace pa_decode needs for these sizes: fp32 partial outputs
 * and log-sum-exp values of every (sequence, query head, partition) when a
 * context spans more than one partition; 0 when no split can happen
 * (partition_tokens == 0 or max_context_len <= partition_tokens).
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_tokens);

/*
 * Decode attention of one query token per sequence over its paged context:
 *   out[s][h] = sum_t softmax_t(scale * <q[s][h], K_t>) V_t,
 * t over the context_lens[s] tokens the block table of s reaches, K_t and V_t
 * taken from KV head h / group_size. Accumulation is fp32; out is rounded to
 * the storage type (round-to-nearest-even). An empty context gives zeros.
 *   out, q          device, [num_seqs][num_q_heads][head_dim]
 *   k_cache,v_cache device, [num_blocks][num_q_heads/group_size][16][head_dim]
 *   block_tables    device int32 [num_seqs][block_table_stride]
 *   context_lens    device int32 [num_seqs]
 *   group_size      query heads per KV head: 1..16, divides num_q_heads
 *   head_dim        64 or 128; block_size must be 16
 *   max_context_len host upper bound of context_lens (sizes the launch)
 *   partition_tokens 0 = one partition per sequence; else a multiple of 16:
 *                   contexts longer than it are split into partitions of
 *                   that many tokens, reduced by log-sum-exp
 *   workspace       device, >= pa_decode_workspace_size(...) bytes, 256-byte
 *                   aligned; may be NULL when that size is 0
 *   dev_error       device int32 counter or NULL
 * Deterministic: no atomics in the arithmetic; the result depends only on the
 * logical order of tokens, not on which physical blocks hold them.
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t block_table_stride,
                    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                    int32_t group_size, int32_t head_dim, int32_t block_size,
                    int64_t num_blocks, int32_t max_context_len, float scale,
                    int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                    int32_t* dev_error, pa_dtype dtype, void* stream);

/*
 * Bytes of workspace pa_decode_persistent needs: pa_decode's partials (if
 * any), a work list of num_seqs * partitions 32-bit items, and 256 bytes of
 * plan state. Never 0 for num_seqs > 0.
 */
size_t pa_decode_persistent_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                           int32_t head_dim, int32_t max_context_len,
                                           int32_t partition_tokens);

/*
 * pa_decode scheduled as a work queue ("New Developments in 2026": PersistentKV
 * organises decode by pages, KV-head groups, sequence splits and work queues).
 * Same arguments, same result bit for bit as pa_decode with the same
 * partition_tokens: each (sequence, partition, KV head) item is computed the
 * same way; only which CTA computes it, and when, differ. A plan kernel lists
 * the sequences' non-empty partitions on the device, longest first (so the
 * host needs no copy of context_lens); one wave of CTAs (SMs x resident CTAs
 * per SM) then pulls (item, KV head) pairs from a counter until none are
 * left. On skewed context lengths this removes the empty CTAs a grid sized by
 * max_context_len launches and the tail of a long item started last.
 *   workspace  device, >= pa_decode_persistent_workspace_size(...) bytes,
 *              256-byte aligned; never NULL. It holds the plan between the
 *              kernels of one call, so concurrent calls need separate ones.
 * Errors: as pa_decode; PA_ERR_UNSUPPORTED also when a sequence may have more
 * than 65536 partitions or num_seqs * partitions * KV heads exceeds 2^31 - 1.
 */
pa_status pa_decode_persistent(void* out, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables,
                               int32_t block_table_stride, const int32_t* context_lens,
                               int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                               int32_t head_dim, int32_t block_size, int64_t num_blocks,
                               int32_t max_context_len, float scale, int32_t partition_tokens,
                               void* workspace, size_t workspace_bytes, int32_t* dev_error,
                               pa_dtype dtype, void* stream);

/*
 * pa_decode for a batch whose sequences all begin with the same
 * shared_prefix_tokens tokens in the same physical blocks: the pages' many
 * users of one prompt, whose copy-on-write forks share every full prefix
 * block ("PagedAttention" guide, "KV Cache Sharing (Copy-on-Write)"). Same
 * arguments and result as pa_decode (within the same tolerance of the exact
 * attention; not bitwise equal to it). The whole partitions inside the shared
 * prefix, if there are at least two and they are not all of the longest
 * context's, are computed once for all sequences: every sequence's query
 * rows against the prefix keys of sequence 0's table, a dense contraction on
 * the tcgen05 tensor cores (the chunk kernel, without a causal mask), written
 * as the decode's fp32 partials; the decode kernel then covers the partitions
 * after them and the log-sum-exp reduce merges both. Needs head_dim 128, a
 * power-of-two group_size, num_seqs * group_size >= 64 and partition_tokens a
 * multiple of 128; otherwise (or when the prefix spans fewer than two whole
 * partitions) it runs pa_decode.
 *   shared_prefix_tokens  host, 0 <= shared_prefix_tokens <= max_context_len:
 *                         tokens at the start of every sequence held in the
 *                         same blocks as sequence 0's (its first
 *                         shared_prefix_tokens / 16 table entries, each
 *                         sequence's context at least that long). A sequence
 *                         that breaks this over the partitions taken as shared
 *                         is counted once in dev_error, and its output row is
 *                         not its attention.
 *   workspace             >= pa_decode_workspace_size(...) bytes, as pa_decode.
 * Errors: as pa_decode; PA_ERR_INVALID_ARG also for shared_prefix_tokens
 * outside [0, max_context_len].
 */
pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  int32_t block_table_stride, const int32_t* context_lens,
                                  int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                                  int32_t head_dim, int32_t block_size, int64_t num_blocks,
                                  int32_t max_context_len, float scale,
                                  int32_t shared_prefix_tokens, int32_t partition_tokens,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_error,
                                  pa_dtype dtype, void* stream);

/*
 * Attention of several query tokens per sequence over the paged cache, causal
 * within the chunk: the query tokens of sequence s are q rows q_start[s] ..
 * q_start[s+1]-1 and are the LAST Tq = q_start[s+1] - q_start[s] tokens of its
 * context (their K/V already written with pa_write_kv); query token t (0-based
 * in the chunk) attends to context positions 0 .. context_lens[s] - Tq + t.
 * This is the attention of chunked prefill ("PagedAttention in Action ...",
 * "Chunked Prefill: Don't Let Long Prompts Consume the Entire Budget") and of
 * verifying speculative draft tokens ("The Memory Wall ...", "The Next
 * Frontier: Speculative Decoding and Beyond"). With one token per sequence it
 * equals pa_decode bit for bit.
 * Two implementations, chosen per call: when max_query_len * group_size >= 64,
 * head_dim is 128, group_size is a power of two and the context is not split
 * or partition_tokens is a multiple of 128, the chunk runs on the tcgen05
 * tensor cores (accumulators in tensor memory, one CTA per pair of 128-row
 * query tiles, 128 keys per step); otherwise on the 16-row mma.sync tiles of
 * pa_decode. Both are within the same tolerance of the exact result; they are
 * not bitwise equal to each other.
 *   out, q          device, [num_q_tokens][num_q_heads][head_dim]
 *   q_start         device int32 [num_seqs + 1], non-decreasing, q_start[0] = 0
 *   max_query_len   host upper bound of Tq (sizes the launch); Tq must also be
 *                   <= context_lens[s]
 *   workspace       >= pa_decode_workspace_size(num_q_tokens, num_q_heads,
 *                   head_dim, max_context_len, partition_tokens) bytes (the
 *                   split partials; NULL when that is 0). On the tcgen05 path,
 *                   with >= pa_prefill_chunk_workspace_size(...) bytes
 *                   (256-byte aligned), a plan kernel first lists the work
 *                   items by descending key count in the space after the
 *                   partials, with a work counter, and the chunk kernel runs
 *                   one CTA per SM, each taking the next item of that list
 *                   whenever it is ready for one (longest first; no per-item
 *                   launch and set-up cost, fewer idle SMs at the end); with
 *                   less it runs one CTA per item in grid order. Same result
 *                   either way, bit for bit.
 *   other arguments as for pa_decode. A sequence whose query range falls
 *   outside [0, num_q_tokens) is skipped, one whose Tq exceeds max_query_len
 *   or its context length is clamped; both are counted in dev_error. With a
 *   malformed q_start the output rows of the sequences involved are undefined
 *   (never written out of bounds).
 */
/* Workspace bytes for pa_prefill_chunk's longest-first order: the split
 * partials (pa_decode_workspace_size of num_q_tokens rows) plus, when the call
 * takes the tcgen05 path, 8 bytes per possible (sequence, query-tile pair,
 * partition) item and 256 bytes (item count and work counter). 0 if no
 * workspace is needed. */
size_t pa_prefill_chunk_workspace_size(int32_t num_q_tokens, int32_t num_seqs,
                                       int32_t num_q_heads, int32_t group_size, int32_t head_dim,
                                       int32_t max_query_len, int32_t max_context_len,
                                       int32_t partition_tokens);

pa_status pa_prefill_chunk(void* out, const void* q, const int32_t* q_start,
                           int32_t num_q_tokens, int32_t max_query_len, const void* k_cache,
                           const void* v_cache, const int32_t* block_tables,
                           int32_t block_table_stride, const int32_t* context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t group_size,
                           int32_t head_dim, int32_t block_size, int64_t num_blocks,
                           int32_t max_context_len, float scale, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, int32_t* dev_error,
                           pa_dtype dtype, void* stream);

/*
 * Copy-on-write block copies: for each pair p and each layer l,
 * k_caches[l][dst] = k_caches[l][src] and v_caches[l][dst] = v_caches[l][src]
 * (whole blocks: num_kv_heads * 16 * head_dim elements), src = mapping[2p],
 * dst = mapping[2p+1].
 *   k_caches, v_caches HOST arrays of num_layers DEVICE pointers
 *   block_mapping   device int64 [num_pairs][2]
 *   num_layers      1..PA_MAX_LAYERS
 *   dev_error       device int32 counter or NULL (pairs outside [0, num_blocks))
 * A dst that repeats, or that is also some pair's src, is undefined.
 */
pa_status pa_copy_blocks(void* const* k_caches, void* const* v_caches, int32_t num_layers,
                         const int64_t* block_mapping, int32_t num_pairs,
                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         int64_t num_blocks, pa_dtype dtype, int32_t* dev_error,
                         void* stream);

/*
 * Swap whole blocks between two pools for preemption: a request's blocks go
 * from GPU memory to CPU RAM and come back later ("PagedAttention",
 * "Managing Virtual Memory (Block Manager)": inactive KV blocks are swapped
 * to CPU RAM and brought back when needed; "The Memory Wall ...", "The Block
 * Manager": preempt a request, save its state, resume later). For each pair p
 * and layer l: dst_k[l][mapping[2p+1]] = src_k[l][mapping[2p]], same for V.
 *   src_k, src_v, dst_k, dst_v  HOST arrays of num_layers pool pointers; each
 *                   pool is device memory or pinned / registered host memory
 *                   ([num_blocks][num_kv_heads][16][head_dim], 16-byte aligned)
 *   block_mapping   int64 [num_pairs][2] (src, dst), device or pinned host
 *   src_num_blocks, dst_num_blocks  pool sizes in blocks (pairs outside them
 *                   are skipped and counted in dev_error)
 * Pageable host memory is refused with PA_ERR_INVALID_ARG before any launch.
 * The copy runs as one kernel on `stream` (host pools cross the host link).
 * A dst that repeats is undefined.
 */
pa_status pa_swap_blocks(void* const* src_k, void* const* src_v, void* const* dst_k,
                         void* const* dst_v, int32_t num_layers, const int64_t* block_mapping,
                         int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                         int32_t block_size, int64_t src_num_blocks, int64_t dst_num_blocks,
                         pa_dtype dtype, int32_t* dev_error, void* stream);

/*
 * pa_decode for callers that cannot allocate device memory -- for example a
 * plugin inside a host application that owns all device memory and forbids
 * its plugins from calling cudaMalloc, or a latency-critical decode loop that
 * cannot afford cudaMalloc/cudaFree (they may synchronise the whole device).
 * The pages have no counterpart to this call; it is a deployment convenience.
 *
 * Same arguments and result as pa_decode, without workspace arguments: the
 * split-K scratch is a fixed array of PA_STATIC_WORKSPACE_BYTES compiled into
 * the library, present in each GPU's memory once the library's device code is
 * loaded there and held until the process exits. The caller still provides
 * every input and output buffer. The call allocates nothing.
 *   - Sizes whose pa_decode_workspace_size(...) exceeds
 *     PA_STATIC_WORKSPACE_BYTES return PA_ERR_WORKSPACE_TOO_SMALL and launch
 *     nothing (use pa_decode with a caller workspace for those).
 *   - The first call on a device looks the array's address up on that device
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture on the device. The address is kept with the
 *     id of the device's CUDA context; after cudaDeviceReset (a new context,
 *     the library's device code loaded again) the next call looks it up
 *     again, and that call too should precede any stream capture.
 *   - All calls on a device share the array. Nothing in it needs to start at
 *     zero, but calls whose kernels overlap on the GPU race on it: order them
 *     on one stream or with events.
 */
#define PA_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

pa_status pa_decode_static(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int32_t block_table_stride,
                           const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                           int32_t group_size, int32_t head_dim, int32_t block_size,
                           int64_t num_blocks, int32_t max_context_len, float scale,
                           int32_t partition_tokens, int32_t* dev_error, pa_dtype dtype,
                           void* stream);

/*
 * Host block manager: the allocator that decides which physical block every
 * token goes to and when a copy-on-write copy is due ("Optimizing LLM
 * Inference ...", "On-Demand Allocation" and "Copy-on-Write"; "PagedAttention",
 * "KV Cache Sharing (Copy-on-Write)"; "PagedAttention in Action ...", "Fixed
 * Block Size, Mitigating External Fragmentation"; "The Memory Wall ...", "The
 * Block Manager"). Host memory only; it produces the slot_mapping, the
 * copy-on-write block_mapping, the block tables and the context lengths that
 * pa_write_kv, pa_copy_blocks and pa_decode consume.
 *
 * Rules: a sequence holds ceil(tokens / 16) blocks; a fork shares all of its
 * parent's blocks (reference count + 1 each); appending a token takes a new
 * block when the last one is full, and copies the last block first when other
 * sequences still hold it (the copy pair is reported; the last holder writes
 * in place); freeing drops one reference per block and returns unreferenced
 * blocks to the pool. Free blocks are handed out last-freed first, and
 * initially in increasing id order. Every call either succeeds completely or
 * changes nothing. A manager is not thread-safe.
 */
typedef struct pa_block_manager pa_block_manager;

typedef struct {
  int64_t num_blocks;     /* pool size */
  int64_t free_blocks;
  int64_t used_blocks;    /* num_blocks - free_blocks */
  int64_t shared_blocks;  /* blocks held by more than one sequence */
  int64_t sequences;
  int64_t tokens;         /* sum of the sequences' token counts */
  int64_t logical_blocks; /* sum of the sequences' table lengths */
} pa_bm_stats;

/* A manager of num_blocks blocks of block_size (must be 16) tokens; NULL on
 * bad arguments or no memory. Release with pa_bm_destroy. */
pa_block_manager* pa_bm_create(int64_t num_blocks, int32_t block_size);
void pa_bm_destroy(pa_block_manager* bm);
int64_t pa_bm_num_free_blocks(const pa_block_manager* bm);

/* A new sequence whose first num_tokens tokens (a prompt) take
 * ceil(num_tokens / 16) fresh blocks. PA_ERR_INVALID_ARG if seq_id exists. */
pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, int64_t num_tokens);

/* child_id shares every block of parent_id (parallel samples, beams, a shared
 * system prompt). */
pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id);

/* Drop the sequence; blocks no other sequence holds return to the pool. */
pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/* slots[t] = cache slot of logical position start + t of seq_id, for
 * writing a prompt's K/V with pa_write_kv (positions must be < its length). */
pa_status pa_bm_slots(const pa_block_manager* bm, int64_t seq_id, int64_t start, int64_t count,
                      int64_t* slots);

/* One decode step: reserve the slot of the next token of each of num_seqs
 * distinct sequences (slot_mapping[i], host int64). Copy-on-write pairs
 * (src, dst) go to cow_pairs (host int64, room for num_seqs pairs), their
 * count to *num_cow; issue pa_copy_blocks with them before pa_write_kv.
 * PA_ERR_OUT_OF_BLOCKS (nothing changed) when the pool cannot cover it. */
pa_status pa_bm_append_slots(pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                             int64_t* slot_mapping, int64_t* cow_pairs, int32_t* num_cow);

/* Decode inputs for num_seqs sequences: block_tables [num_seqs][stride]
 * (entries past each table = -1) and context_lens, both host int32. */
pa_status pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids,
                             int32_t num_seqs, int32_t* block_tables, int32_t stride,
                             int32_t* context_lens);

pa_status pa_bm_get_stats(const pa_block_manager* bm, pa_bm_stats* out);

/* Reference count of one physical block (-1 for a bad id). */
int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block);

/*
 * Measurement utility, with no counterpart on the pages: the streaming-read
 * ceiling of this GPU's memory, the roofline of the decode path (which only
 * reads the cache; a read+write copy benchmark is not its ceiling).
 * Reads `bytes` bytes at `buf` (device memory, 16-byte aligned, bytes a
 * multiple of 16) once with every SM and discards them:
 *   method 0: 128-bit loads that bypass L1, eight in flight per thread,
 *             every resident thread sweeping the buffer;
 *   method 1: bulk asynchronous copies (cp.async.bulk, 16 KiB, into the issuing CTA)
 *             into a shared-memory ring per CTA -- the engine the decode
 *             kernels read their tiles with;
 *   method 2: the paged decode's access pattern without its arithmetic: the
 *             buffer as 4 KiB tiles (one KV head of one cache block at
 *             D = 128), each read once in a scattered order by two 2 KiB TMA
 *             tensor boxes, in the decode kernel's CTA shape (reads
 *             floor(bytes / 8 KiB) * 8 KiB bytes) -- the paged-read ceiling.
 * Each CTA XORs a fold of what it read into *sink (device uint64, 8-byte
 * aligned; its value means nothing, it only keeps the loads alive). A bulk
 * wait that gives up adds PA_DEV_ERR_TIMEOUT to *dev_error (nullable). Time
 * it with events on `stream`; buffers larger than L2 measure HBM.
 * PA_ERR_INVALID_ARG for a bad method, pointer, alignment or size.
 */
pa_status pa_read_probe(const void* buf, size_t bytes, int32_t method, uint64_t* sink,
                        int32_t* dev_error, void* stream);

/* Static description of a status code. */
const char* pa_status_string(pa_status status);

/* The CUDA error string of the last PA_ERR_CUDA on this thread ("" if none). */
const char* pa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
