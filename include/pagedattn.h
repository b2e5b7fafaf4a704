/*
 * pagedattn.h -- C ABI of the paged KV-cache decode library (libpagedattn.so).
 *
 * Decode attention over a KV cache cut into fixed-size physical blocks that
 * are scattered through a pooled cache and reached through a per-sequence
 * block table (logical block i -> physical block id).  Sources, by page
 * title and section:
 *   [csdn-QA] "VLLM中PagedAttention如何降低显存碎片？" (ask.csdn.net), sections 二-四
 *   [tech]    "PagedAttention技术解析：优化Transformer显存管理", sections 2.1-4.2
 *   [course]  "vLLM内存管理与PagedAttention精讲", chapter 2, sections 2.2-2.5
 *
 * Conventions for every call below
 *   - Pointers named *_d are DEVICE pointers owned by the caller (for
 *     example PyTorch tensors).  Tensors are dense, row-major, with the
 *     shapes given.  Device pointers passed to the attention and cache
 *     calls must be 16-byte aligned.  The library never allocates device
 *     memory; split decode takes a caller-owned workspace.
 *   - Every device call is asynchronous on `stream` (NULL = legacy default
 *     stream) and returns a pa_status describing argument checks and the
 *     launch only.  Faults found by the kernels' own bounds checks or
 *     bounded waits are recorded in a device-side error word that
 *     pa_device_error() reads.
 *   - On any non-PA_OK status pa_last_error() returns a message (thread
 *     local, valid until the next call on that thread).
 *   - Cache layout: k_cache and v_cache are two tensors
 *     [num_blocks, block_size, num_kv_heads, head_dim]: a block holds
 *     block_size tokens, each with its key (value) for every kv head and
 *     every dimension ([course] 2.3; [csdn-QA] 三, separate K and V pages).
 *     Bytes per block, K plus V: block_size * num_kv_heads * head_dim * 2 *
 *     element size ([course] 2.3).
 *   - Supported: dtype f32 or bf16 (q, key/value rows, caches and outputs
 *     share one dtype; arithmetic is fp32), head_dim in {64, 128, 256},
 *     block_size in {8, 16, 32, 64, 128} ([course] 2.3 and 2.5: 16 by
 *     default, 8 and 32 tried; [tech] 4.1: 32..128 suggested by head_dim),
 *     num_heads / num_kv_heads in {1, 2, 4, 8}.
 *     Anything else returns PA_ERR_UNSUPPORTED.
 *   - Validation: with PA_VALIDATE=1 in the environment (or
 *     pa_set_option(PA_OPT_VALIDATE, 1)) the calls first copy the index
 *     arrays to the host (synchronising `stream`) and return
 *     PA_ERR_BAD_BLOCK_ID for a block id outside [0, num_blocks), a
 *     context length above max_blocks_per_seq * block_size, a slot outside
 *     the pool, or a repeated copy destination.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* pa_stream_t;

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, misalignment, Hq % Hk != 0 */
    PA_ERR_UNSUPPORTED = 2,     /* dtype / head_dim / block_size / group size not built */
    PA_ERR_OUT_OF_BLOCKS = 3,   /* allocator: free pool exhausted, state unchanged */
    PA_ERR_BAD_BLOCK_ID = 4,    /* validation: index outside the pool or table */
    PA_ERR_CUDA = 5,            /* a CUDA runtime / driver call failed */
    PA_ERR_DEVICE_CHECK = 6     /* pa_device_error(): a kernel's own check fired */
} pa_status;

typedef enum pa_dtype { PA_DTYPE_F32 = 0, PA_DTYPE_BF16 = 1 } pa_dtype;

/* Bits of the device-side error word (pa_device_error). */
enum {
    PA_DEVERR_BLOCK_ID = 1u,     /* decode met a table entry outside [0, num_blocks) */
    PA_DEVERR_CONTEXT_LEN = 2u,  /* context length beyond the table; clamped */
    PA_DEVERR_WAIT_TIMEOUT = 4u, /* a bounded pipeline wait gave up */
    PA_DEVERR_SLOT = 8u,         /* reshape_and_cache slot outside the pool; row skipped */
    PA_DEVERR_COPY_ID = 16u,     /* copy_blocks pair outside the pool; pair skipped */
    PA_DEVERR_WORKSPACE = 32u    /* split decode: more partitions than the workspace holds */
};

typedef enum pa_option {
    PA_OPT_VALIDATE = 0,         /* 0/1: host-side index validation before launch */
    PA_OPT_DECODE_SPLIT_CTAS = 1, /* pa_decode CTAs per (sequence, kv head): 0 = auto, 1, 2, 4, 8 */
    PA_OPT_PDL = 2,               /* 0/1 (default 1, or PA_PDL in the environment): launch with
                                     programmatic dependent launch.  A kernel may start during
                                     the tail of the grid before it on the stream, and waits
                                     for that grid to complete before it reads anything that
                                     grid may write.  Before that wait, pa_decode's grid (and
                                     pa_decode_append's, pa_decode_step's) reads context_lens,
                                     which no kernel of this library writes: a caller's kernel
                                     that writes it must not release its dependents early
                                     (griddepcontrol.launch_dependents), or this option must
                                     be 0.  It also reads a few block-table entries there, but
                                     only to prefetch their tiles into L2; the entries it
                                     decodes with are read after the wait.  The shared-prefix decode's
                                     own-token pass streams the cache behind the shared pass,
                                     which has waited for the grid before it */
    PA_OPT_WAIT_LIMIT_US = 3,     /* upper bound, in microseconds, on every pipeline wait inside
                                     the decode kernels (default 2000000 = 2 s; 100 .. 10000000).
                                     A wait that runs out sets PA_DEVERR_WAIT_TIMEOUT; the warp
                                     stops issuing, waits (bounded) for its own loads in flight
                                     and contributes nothing, so the kernel still ends */
    PA_OPT_TEST_UNDERFED_STAGES = 4 /* TEST ONLY, 0/1 (default 0): arm every pipeline stage's
                                     barrier for 16 bytes more than its loads deliver.  Every
                                     load still lands in the CTA's own shared memory, but no
                                     stage ever completes, so every wait runs out: this drives
                                     the timeout path above without a lost load.  Outputs are
                                     then meaningless (zeros where nothing was merged) */
} pa_option;

const char* pa_last_error(void);
const char* pa_status_string(pa_status status);
int         pa_version(void);
pa_status   pa_set_option(pa_option option, int value);
int         pa_get_option(pa_option option);

/* Synchronise `stream`, return the device error word in *flags (0 = none)
 * and clear it when `clear` is non-zero.  Returns PA_ERR_DEVICE_CHECK when
 * the word is non-zero. */
pa_status pa_device_error(pa_stream_t stream, uint32_t* flags, int clear);

/*
 * pa_reshape_and_cache -- write new tokens' keys and values into the cache.
 * A generated token's K/V rows go into the slot its sequence's newest block
 * assigns to it ([course] 2.4.2: a new block only when the current one is
 * full; [csdn-QA] 四 flow: allocate a free page, update the mapping).
 *   key_d, value_d   [num_tokens, num_kv_heads, head_dim], dtype
 *   k_cache_d, v_cache_d  [num_blocks, block_size, num_kv_heads, head_dim]
 *   slot_mapping_d   int64 [num_tokens]: slot = block * block_size + row;
 *                    -1 skips the token.  Duplicate slots race (undefined).
 * The copy is exact (no conversion).  A slot >= num_blocks * block_size is
 * skipped and sets PA_DEVERR_SLOT.
 */
pa_status pa_reshape_and_cache(const void* key_d, const void* value_d,
                               void* k_cache_d, void* v_cache_d,
                               const int64_t* slot_mapping_d, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode -- one decode step of attention over the paged cache.
 * For each sequence s and query head h (kv head h / (num_heads/num_kv_heads)):
 *   out[s,h] = sum_t softmax_t(scale * <q[s,h], K_s[t]>) V_s[t],
 * t over the sequence's context_lens[s] tokens, token t read from physical
 * block block_tables[s, t / block_size] at row t % block_size ([course] 2.2
 * mapping, 2.5 block-wise loop; [csdn-QA] 三 items 4, 9).  The kernel walks
 * the blocks with an online (running max / running sum) softmax, which
 * reaches the same result as the plain softmax.
 *   out_d            [num_seqs, num_heads, head_dim], dtype (written)
 *   q_d              [num_seqs, num_heads, head_dim], dtype
 *   block_tables_d   int32 [num_seqs, max_blocks_per_seq]; only the first
 *                    ceil(context_lens[s] / block_size) entries are read
 *   context_lens_d   int32 [num_seqs]; 0 gives a zero output row
 * No workspace: a (sequence, kv head) may be split over a cluster of CTAs
 * that merge through distributed shared memory.
 */
pa_status pa_decode(void* out_d, const void* q_d,
                    const void* k_cache_d, const void* v_cache_d,
                    const int32_t* block_tables_d, int max_blocks_per_seq,
                    const int32_t* context_lens_d, int num_seqs, int num_heads,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                    float scale, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_append -- pa_reshape_and_cache of one new token per sequence
 * followed by pa_decode, in one launch (the decode loop's step: the new
 * token is stored, then attended to along with the rest of its sequence;
 * [course] 2.4.2 and 2.5, [csdn-QA] 四 flow: update the mapping, then run
 * the attention kernel).
 *   key_d, value_d   [num_seqs, num_kv_heads, head_dim]: sequence s's new row
 *   slot_mapping_d   int64 [num_seqs]: its slot (-1: sequence s gains no token)
 *   k_cache_d, v_cache_d  written at those slots, then read
 * Other arguments as pa_decode; context_lens already count the new token.
 * Preconditions: each new slot is its sequence's last position (the slot of
 * token context_lens[s]-1) and lies in a block no other sequence reads --
 * the allocator's copy-on-write guarantees both.  Validate mode checks the
 * first.  Out-of-pool slots are skipped and set PA_DEVERR_SLOT.
 */
pa_status pa_decode_append(void* out_d, const void* q_d, const void* key_d,
                           const void* value_d, void* k_cache_d, void* v_cache_d,
                           const int64_t* slot_mapping_d, const int32_t* block_tables_d,
                           int max_blocks_per_seq, const int32_t* context_lens_d, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float scale, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_decode_step -- one whole decode step in one launch: the mapping update
 * of pa_update_block_tables, then pa_decode_append ([csdn-QA] 四 flow:
 * allocate a free page, update the mapping, run the attention kernel).
 * The block of each sequence's new token is taken from its slot
 * (slot_mapping[s] / block_size) rather than from the table, and written
 * into the table:
 *   block_tables[s, (context_lens[s] - 1) / block_size] = slot_mapping[s] / block_size
 * so the caller's device tables need not hold the new block (a fresh block
 * or a copy-on-write replacement) before the call, and hold it after.
 *   block_tables_d   int32 [num_seqs, max_blocks_per_seq]; the entries
 *                    before a sequence's last block are read, the last one
 *                    is written (for sequences with slot_mapping[s] >= 0)
 * Other arguments and preconditions as pa_decode_append, except that a new
 * slot need only lie on the new token's row (slot % block_size equal to
 * (context_lens[s] - 1) % block_size) of a block no other sequence reads;
 * validate mode checks that and the entries read.  Sequences without a new
 * token (-1), slots outside the pool (PA_DEVERR_SLOT) and empty sequences
 * keep their entry.  Results equal pa_update_block_tables followed by
 * pa_decode_append on the same stream, bit for bit.
 */
pa_status pa_decode_step(void* out_d, const void* q_d, const void* key_d,
                         const void* value_d, void* k_cache_d, void* v_cache_d,
                         const int64_t* slot_mapping_d, int32_t* block_tables_d,
                         int max_blocks_per_seq, const int32_t* context_lens_d, int num_seqs,
                         int num_heads, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, float scale, pa_dtype dtype, pa_stream_t stream);

/*
 * pa_update_block_tables -- the "update the mapping" step of a decode step
 * ([csdn-QA] 四 flow: allocate a free page, update the mapping, run the
 * attention kernel; [course] 2.4.2: a new block only when the last one is
 * full).  After the host allocator has appended one token to each sequence,
 * the device copy of the block tables needs at most one new entry per
 * sequence: the block holding the new token, which is a newly allocated
 * block, the copy-on-write replacement of a shared last block, or the entry
 * already there.  This call writes
 *   block_tables[s, (context_lens[s] - 1) / block_size] = slot_mapping[s] / block_size
 * for every s with slot_mapping[s] >= 0, so a serving loop keeps the tables
 * resident on the device and uploads only the lengths and slots it already
 * sends for the cache write, instead of the whole table.
 *   block_tables_d   int32 [num_seqs, max_blocks_per_seq] (updated in place)
 *   context_lens_d   int32 [num_seqs], counting the new token
 *   slot_mapping_d   int64 [num_seqs], the new token's slot (-1: no token)
 * Entries a kernel earlier on the stream reads may change (copy-on-write),
 * so the call belongs on the stream of the decode that follows.  A slot
 * outside the pool, or a position outside the table, is skipped and sets
 * PA_DEVERR_SLOT; validate mode also checks that the slot's row is the new
 * token's row in its block.
 */
pa_status pa_update_block_tables(int32_t* block_tables_d, int max_blocks_per_seq,
                                 const int32_t* context_lens_d, const int64_t* slot_mapping_d,
                                 int num_seqs, int block_size, int num_blocks,
                                 pa_stream_t stream);

/*
 * pa_decode_split -- long-context decode in fixed token partitions merged by
 * log-sum-exp ("PagedAttention V2 ... block-wise computation",
 * [csdn-QA] 四, last paragraph; sequences up to 1M tokens, [tech] 1).
 * Partition p of sequence s covers tokens [p*P, min((p+1)*P, L_s)) with
 * P = partition_size (a multiple of block_size).  A first kernel writes per
 * (sequence, head, partition) the running max, the sum of exponentials and
 * the unnormalised output into `workspace_d`; a second kernel merges them:
 *   out = sum_p exp(m_p - M) o_p / sum_p exp(m_p - M) l_p,  M = max_p m_p.
 * Sequences with a single partition are written directly by the first kernel.
 * When few (sequence, head) pairs have many partitions, the merge splits each
 * pair's partitions into chunks over several CTAs, which leave their sums in
 * the workspace; the last chunk adds them in chunk order, so the result does
 * not depend on timing.
 *   max_context_len  >= every context_lens[s]; sizes the workspace
 *   workspace_d      caller-owned device memory of at least
 *                    pa_decode_split_workspace_bytes(...) bytes, 16-byte aligned
 * Other arguments as pa_decode.
 */
size_t pa_decode_split_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                       int max_context_len, int partition_size);

pa_status pa_decode_split(void* out_d, const void* q_d,
                          const void* k_cache_d, const void* v_cache_d,
                          const int32_t* block_tables_d, int max_blocks_per_seq,
                          const int32_t* context_lens_d, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int num_blocks,
                          float scale, pa_dtype dtype, int max_context_len,
                          int partition_size, void* workspace_d, size_t workspace_bytes,
                          pa_stream_t stream);

/*
 * pa_decode_split_noalloc -- pa_decode_split without a caller workspace.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory where they decode: a plugin inside a host
 * framework that owns all device memory and gives plugins none, or a
 * serving process with a fixed memory budget that allows no allocation
 * after start-up.  It takes pa_decode_split's arguments minus the workspace
 * and uses a scratch array built into the library instead, so it allocates
 * nothing (no cudaMalloc, no allocating library call).
 *   Limit: a batch whose pa_decode_split_workspace_bytes(...) exceeds
 *   PA_NOALLOC_SCRATCH_BYTES (16 MiB) is rejected with PA_ERR_UNSUPPORTED
 *   before anything is launched.  Every GPU that loads the library holds
 *   the 16 MiB until the process exits.
 *   The first call on a device, with that device current, looks up the
 *   scratch array's device address; make that first call before any
 *   stream capture.
 *   All calls share the one scratch array, which keeps the last call's
 *   contents (nothing needs to start at zero).  Calls that overlap on the
 *   GPU -- on different streams or from different host threads -- race on
 *   it and corrupt each other's results: serialise them.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)

pa_status pa_decode_split_noalloc(void* out_d, const void* q_d,
                                  const void* k_cache_d, const void* v_cache_d,
                                  const int32_t* block_tables_d, int max_blocks_per_seq,
                                  const int32_t* context_lens_d, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                  float scale, pa_dtype dtype, int max_context_len,
                                  int partition_size, pa_stream_t stream);

/*
 * pa_decode_shared_prefix -- decode of a batch whose sequences come in groups
 * sharing a prefix: sequences [group_starts[g], group_starts[g+1]) all start
 * with the same prefix_lens[g] tokens in the same physical blocks (forks of
 * one prompt: [course] 2.4.3 block tables pointing at the same physical
 * blocks; [csdn-QA] 三 item 8 shared prefix pages).  Same result as
 * pa_decode.  First the members of a group attend over the shared prefix
 * together -- members x G query rows form one dense contraction per kv head,
 * so each prefix block comes from HBM once per kv head (once per 64 query
 * rows from L2) instead of once per sequence -- leaving per-chunk partial
 * results in the workspace; then
 * pa_decode's kernel covers each sequence's own tokens and merges those
 * partials (log-sum-exp) into the output.  Two launches.
 *   group_starts_d   int32 [num_groups + 1], ascending, 0 .. num_seqs (the
 *                    groups cover every sequence; a group of one with prefix
 *                    0 is a plain sequence)
 *   prefix_lens_d    int32 [num_groups]: shared tokens, whole blocks and a
 *                    multiple of 16, at most max_prefix_len; every member is
 *                    at least that long and has the same first
 *                    prefix_lens[g] / block_size table entries
 *   max_group_size   >= every group's size
 *   workspace_d      >= pa_decode_shared_prefix_workspace_bytes(...) bytes
 * bf16 only (else PA_ERR_UNSUPPORTED); any built block_size (with 8-token
 * blocks a 16-token unit spans two blocks).  Validate mode checks every
 * precondition above.
 */
size_t pa_decode_shared_prefix_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                               int max_prefix_len);

pa_status pa_decode_shared_prefix(void* out_d, const void* q_d, const void* k_cache_d,
                                  const void* v_cache_d, const int32_t* block_tables_d,
                                  int max_blocks_per_seq, const int32_t* context_lens_d,
                                  int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                  int block_size, int num_blocks, float scale, pa_dtype dtype,
                                  const int32_t* group_starts_d, const int32_t* prefix_lens_d,
                                  int num_groups, int max_group_size, int max_prefix_len,
                                  void* workspace_d, size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_shared_prefix_step -- pa_decode_shared_prefix as a whole decode
 * step, the shared-prefix counterpart of pa_decode_step: the own-token pass
 * also stores each sequence's new token (key_d/value_d rows at
 * slot_mapping_d, as pa_decode_append) and the mapping update
 * (block_tables[s, (context_lens[s] - 1) / block_size] = slot / block_size,
 * as pa_decode_step), so a step is the two launches of the cascade and no
 * cache-write or table-update launch.  Arguments as pa_decode_shared_prefix
 * plus those of pa_decode_step; context_lens count the new token, which must
 * lie past its group's prefix (in a block of its own, as the allocator's
 * copy-on-write guarantees).  block_tables_d is written (the last entry of
 * each sequence with a new token).  Validate mode checks the preconditions
 * of both.  Results equal pa_update_block_tables, pa_reshape_and_cache and
 * pa_decode_shared_prefix on the same stream, bit for bit.
 */
pa_status pa_decode_shared_prefix_step(void* out_d, const void* q_d, const void* key_d,
                                       const void* value_d, void* k_cache_d, void* v_cache_d,
                                       const int64_t* slot_mapping_d, int32_t* block_tables_d,
                                       int max_blocks_per_seq, const int32_t* context_lens_d,
                                       int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int block_size, int num_blocks, float scale,
                                       pa_dtype dtype, const int32_t* group_starts_d,
                                       const int32_t* prefix_lens_d, int num_groups,
                                       int max_group_size, int max_prefix_len,
                                       void* workspace_d, size_t workspace_bytes,
                                       pa_stream_t stream);

/*
 * pa_copy_blocks -- copy-on-write of shared blocks: for each pair
 * (src, dst) the whole key block and value block dst <- src ([course] 2.4.3:
 * a write to a block whose reference count exceeds one first copies it).
 *   block_mapping_d  int64 [num_pairs, 2] (src, dst), device memory.
 * Destinations must be distinct and must not be sources (else undefined).
 * An id outside the pool skips the pair and sets PA_DEVERR_COPY_ID.
 */
pa_status pa_copy_blocks(void* k_cache_d, void* v_cache_d,
                         const int64_t* block_mapping_d, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks,
                         pa_dtype dtype, pa_stream_t stream);

/*
 * pa_swap_blocks -- move whole blocks (keys and values) between two pools,
 * typically the device cache and a pinned host cache: swapping pages out of
 * HBM and back ([csdn-QA] 三 item 10: page migration through pinned memory
 * and asynchronous copies).  For each pair (src, dst) of block_mapping,
 * block dst of the destination pool <- block src of the source pool.
 *   dst_k, dst_v, src_k, src_v  [num_blocks, block_size, kv_heads, head_dim]
 *                    pools: device memory, or pinned host memory (device-
 *                    mapped under unified addressing, as cudaHostAlloc /
 *                    torch pin_memory give); pageable host memory returns
 *                    PA_ERR_UNSUPPORTED
 *   block_mapping    int64 [num_pairs, 2] (src, dst), device or pinned host
 * One kernel moves every pair, 16 bytes per thread access, over the GPU's
 * link for host pools.  Destinations must be distinct (validate mode checks);
 * an id outside its pool skips the pair and sets PA_DEVERR_COPY_ID.
 */
pa_status pa_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                         const int64_t* block_mapping, int num_pairs, int num_kv_heads,
                         int head_dim, int block_size, int src_num_blocks, int dst_num_blocks,
                         pa_dtype dtype, pa_stream_t stream);

/*
 * Host block allocator ([tech] 2.1 Block {ref_count, is_allocated} and the
 * pool descriptor, 4.2 immediate reclamation at ref_count 0 and a free pool;
 * [csdn-QA] 三 item 7 slab-style frames, item 8 shared prefix pages;
 * [course] 2.4 on-demand growth, sharing, copy-on-write).
 * Host memory only; not thread-safe; the caller owns the handle.
 * The free pool is a stack: it starts as initial_free_order (element 0 is
 * handed out first; NULL = 0, 1, ..., num_blocks-1) and a block whose
 * count reaches 0 is pushed on top.  Failing calls change nothing.
 */
typedef struct pa_allocator pa_allocator;

pa_allocator* pa_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order);
void      pa_alloc_destroy(pa_allocator* alloc);
pa_status pa_alloc_allocate(pa_allocator* alloc, int32_t* block_out);  /* ref := 1 */
pa_status pa_alloc_incref(pa_allocator* alloc, int32_t block);         /* block must be allocated */
pa_status pa_alloc_decref(pa_allocator* alloc, int32_t block);         /* 0 -> back on the stack */
int       pa_alloc_num_free(const pa_allocator* alloc);
int       pa_alloc_num_blocks(const pa_allocator* alloc);
int       pa_alloc_block_size(const pa_allocator* alloc);
int       pa_alloc_ref_count(const pa_allocator* alloc, int32_t block);  /* -1 if out of range */
/* Free stack from top to bottom into out[0..capacity); *count = its size. */
pa_status pa_alloc_free_order(const pa_allocator* alloc, int32_t* out, int capacity, int* count);

/*
 * Sequence helpers on caller-owned host tables.  A sequence of `length`
 * tokens holds exactly ceil(length / block_size) table entries.
 *
 * pa_seq_append_slot: make room for token `*length`: a fresh block when
 * the last one is full; otherwise, if the last block is shared
 * (ref_count > 1), copy-on-write -- a fresh block replaces it in the table,
 * the old block's count drops, and (*cow_src, *cow_dst) report the pair to
 * copy (both -1 when no copy is needed).  *slot = block * block_size + row;
 * *length is incremented.  `capacity` is the table's size.
 */
pa_status pa_seq_append_slot(pa_allocator* alloc, int32_t* table, int capacity, int* length,
                             int64_t* slot, int32_t* cow_src, int32_t* cow_dst);

/* One token for each of `num_seqs` sequences, in ascending index (the last
 * sharer of a partial block writes in place).  tables: [num_seqs, stride];
 * lengths [num_seqs] updated; slots [num_seqs]; cow_pairs [num_seqs, 2]
 * receives *num_cow (src, dst) pairs.  All-or-nothing on OUT_OF_BLOCKS. */
pa_status pa_seq_append_slots(pa_allocator* alloc, int32_t* tables, int stride, int* lengths,
                              int num_seqs, int64_t* slots, int32_t* cow_pairs, int* num_cow);

/* `num_tokens` successive appends to one sequence (a prompt).  slots may be
 * NULL; (*cow_src, *cow_dst) report the copy the first append needed, if
 * any.  All-or-nothing on OUT_OF_BLOCKS. */
pa_status pa_seq_extend(pa_allocator* alloc, int32_t* table, int capacity, int* length,
                        int num_tokens, int64_t* slots, int32_t* cow_src, int32_t* cow_dst);

/* The child shares every parent block; each block's count goes up by one. */
pa_status pa_seq_fork(pa_allocator* alloc, const int32_t* parent_table, int num_table_blocks,
                      int32_t* child_table);

/* Drop the sequence's reference on each of its blocks. */
pa_status pa_seq_free(pa_allocator* alloc, const int32_t* table, int num_table_blocks);

/*
 * Compaction (periodic defragmentation, [tech] 2.1 and 4.2 item 2).  With
 * fixed-size blocks a free block serves any request, so compaction packs the
 * live blocks below `target_num_blocks` so the pool's tail can be released:
 * every live block at or above the target (ascending id) moves to a free
 * block below it (ascending id), its reference count travels with it, and
 * the pool shrinks to the target (the free stack keeps its order).  The
 * (src, dst) pairs go to moves[0 .. 2 * *num_moves); the caller then copies
 * the data (pa_copy_blocks with those pairs, int64 on the device) and
 * rewrites every table (pa_seq_remap).  OUT_OF_BLOCKS (nothing changes)
 * when more blocks are live than the target holds.
 */
pa_status pa_alloc_compact(pa_allocator* alloc, int target_num_blocks, int32_t* moves,
                           int capacity, int* num_moves);

/* Replace every entry of a host table that is a move's src by its dst. */
pa_status pa_seq_remap(int32_t* table, int num_table_blocks, const int32_t* moves, int num_moves);

/* pa_seq_remap for a whole batch in one call ([tech] 2.1: defragmentation
 * rewrites the block pointers; 4.2 item 2).  tables: host int32
 * [num_seqs][stride], row s holding lengths_in_blocks[s] live entries (the
 * rest is left untouched); moves: the (src, dst) pairs pa_alloc_compact
 * returned.  Every live entry equal to a move's src becomes its dst.
 * INVALID_ARG (nothing changes) for null arrays, a negative count, a row
 * longer than stride or a negative block in moves. */
pa_status pa_seq_remap_batch(int32_t* tables, int stride, const int* lengths_in_blocks,
                             int num_seqs, const int32_t* moves, int num_moves);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
