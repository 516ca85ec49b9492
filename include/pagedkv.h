/*
 * pagedkv.h — C-ABI of libpagedkv.so: the paged KV-cache decode path on B200 (sm_100a).
 *
 * The KV cache of every layer is split into fixed-size physical blocks ("pages")
 * reached through a per-sequence block table; decode attention reads the pages
 * through the table, a cache write scatters each step's new K/V into slots, and a
 * block copy duplicates shared pages before they are written (copy-on-write).
 * Sources: "vLLM / PagedAttention — 分页 KV Cache 分析" §2.2 (pages + block table),
 * §2.3 (block manager, block table, copy-on-write), §3.1 (the attention kernel reads
 * non-contiguous KV; its simplified per-page loop), §3.2 (copy a shared page before
 * changing it); "vLLM" entity page, 是什么 (blocks on demand, refcount sharing).
 *
 * Conventions (every entry point):
 *  - returns int: PKV_OK (0) or a negative PKV_ERR_* code; nothing throws across the ABI.
 *  - device pointers are raw CUDA device addresses owned by the caller; the library
 *    keeps no reference to them after the call returns.
 *  - device work is enqueued on `stream` (NULL = legacy default stream) and is
 *    asynchronous: a PKV_OK return means "arguments valid and launched", not
 *    "finished". Only pkv_get_device_status synchronises.
 *  - arguments are checked on the host before any launch; a rejected call launches
 *    nothing and changes nothing.
 *  - device-side index errors (a block id or slot outside the pool, a context length
 *    above the stated maximum) never fault: the kernel skips the access (or reads
 *    zeros), sets a bit in a per-device status word and continues. Read it with
 *    pkv_get_device_status.
 *
 * Layouts (row-major, element = 2 bytes, fp16 or bf16 as `dtype`):
 *  - q, out        [num_seqs][num_heads][head_dim]
 *  - k_cache, v_cache (one layer) [num_blocks][num_kv_heads][block_size][head_dim]
 *    (one (block, kv head) tile is block_size*head_dim contiguous elements)
 *  - k_new, v_new  [num_tokens][num_kv_heads][head_dim]
 *  - block_tables  int32 [num_seqs][max_blocks_per_seq], unused entries ignored
 *  - context_lens  int32 [num_seqs]  (tokens attended, including the one written this step)
 *  - slot_mapping  int64 [num_tokens] (slot = block * block_size + row; < 0 = skip)
 *  - block_pairs   int32 [num_pairs][2] = (src, dst)
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *pkv_stream_t;

enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = -1,   /* a size, pointer or dtype outside the documented range */
    PKV_ERR_OUT_OF_BLOCKS = -2, /* allocator: too few free blocks; state unchanged        */
    PKV_ERR_UNKNOWN_SEQ = -3,   /* allocator: no sequence with that id                    */
    PKV_ERR_SEQ_EXISTS = -4,    /* allocator: fork target id already in use                */
    PKV_ERR_TABLE_FULL = -5,    /* allocator: table would exceed max_blocks_per_seq        */
    PKV_ERR_BAD_INDEX = -6,     /* for callers that turn status-word bits into codes: an   */
    PKV_ERR_TIMEOUT = -7,       /* out-of-pool index / a wait that gave up (not returned)  */
    PKV_ERR_CUDA = -8,          /* a CUDA runtime call failed                             */
    PKV_ERR_WORKSPACE = -9,     /* workspace pointer NULL or smaller than required        */
    PKV_ERR_HOST_MEMORY = -10   /* allocator: a host allocation failed; the call may have  */
                                /* been partly applied: destroy the manager               */
};

enum pkv_dtype { PKV_F16 = 0, PKV_BF16 = 1 };

/* Bits of the per-device status word (pkv_get_device_status). */
enum pkv_device_status_bits {
    PKV_STATUS_BAD_SLOT = 1u << 0,     /* reshape_and_cache: slot >= num_blocks*block_size      */
    PKV_STATUS_BAD_PAIR = 1u << 1,     /* copy_blocks / swap_blocks: block id outside the pool  */
    PKV_STATUS_BAD_BLOCK = 1u << 2,    /* decode: block id outside [0, num_blocks) (read as 0)  */
    PKV_STATUS_BAD_LEN = 1u << 3,      /* decode: context_len < 0 or above its bound (clamped)  */
    PKV_STATUS_WAIT_TIMEOUT = 1u << 4, /* decode: a pipeline wait exceeded its iteration limit  */
    PKV_STATUS_NO_BLOCKS = 1u << 5,    /* device append: step refused, nothing changed          */
    PKV_STATUS_WORKSPACE = 1u << 6,    /* workspace not prepared for the call (step, planned)   */
    PKV_STATUS_SHARED_BLOCK = 1u << 7  /* device append refused: a sequence would write into a  */
                                       /* shared, partly filled block (copy-on-write needed)    */
};

/* Human-readable name of a status code (static string). */
const char *pkv_status_string(int code);

/* ------------------------------------------------------------------------------
 * Paged single-query decode attention ("分页 KV Cache 分析" §3.1; its per-page loop
 * read as one softmax per (sequence, query head) over all context tokens).
 *
 *   out[s][h][:] = sum_t softmax_t(scale * q[s][h] . K_s[t]) * V_s[t],  t < context_lens[s]
 *   K_s[t] = k_cache[block_tables[s][t / block_size]][h / G][t % block_size][:]   (V alike)
 *   G = num_heads / num_kv_heads (query heads h*G .. h*G+G-1 share KV head h).
 *
 * fp16/bf16 inputs, fp32 accumulation, output rounded to nearest even into `dtype`.
 * A zero-length context gives out = 0. Slots past context_lens[s] in the last block
 * are never used (any bits, NaN included, are ignored).
 * Long contexts are split into partitions of `partition_size` tokens (a multiple of
 * 64, at most 256 blocks; 0 = automatic) whose partial results are merged exactly
 * (log-sum-exp) by a second kernel; that needs `workspace` of at least
 * pkv_decode_workspace_size(...) bytes of device memory (16-byte aligned), which the
 * caller owns and may reuse between calls that are ordered on one stream.
 *
 * Limits: head_dim in {64, 128}; block_size in {8, 16, 32}; 1 <= G <= 16;
 * num_kv_heads >= 1; num_seqs >= 0; max_context_len <= max_blocks_per_seq*block_size;
 * num_blocks*num_kv_heads*block_size < 2^31. context_lens[s] is clamped on the
 * device to [0, max_context_len] (PKV_STATUS_BAD_LEN if it had to be).
 * Errors: PKV_ERR_INVALID_ARG, PKV_ERR_WORKSPACE, PKV_ERR_CUDA (launch failure).
 * ---------------------------------------------------------------------------- */
int pkv_paged_attention_decode(void *out, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *block_tables,
                               const int32_t *context_lens, int num_seqs, int num_heads,
                               int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int num_blocks, int max_context_len,
                               float scale, int dtype, int partition_size, void *workspace,
                               size_t workspace_bytes, pkv_stream_t stream);

/* The two launches of pkv_paged_attention_decode as separate calls (the decode of each
 * partition, "分页 KV Cache 分析" §3.1's per-page loop in streaming form, and the exact
 * log-sum-exp merge of the partitions), for callers that put other work between them or
 * time each:
 *  - pkv_paged_attention_decode_partitions: arguments, checks and errors as
 *    pkv_paged_attention_decode; launches the decode kernel only. Sequences whose context
 *    is one partition get their output; the others leave fp32 partials in `workspace`.
 *  - pkv_paged_attention_merge: merges those partials into `out` (outputs of one-partition
 *    sequences are not touched). The sizes, partition_size, context_lens and workspace
 *    must be those of the partitions call it follows on the same stream; it launches
 *    nothing when every context is one partition. Errors: PKV_ERR_INVALID_ARG,
 *    PKV_ERR_WORKSPACE, PKV_ERR_CUDA.
 * The partitions call followed by the merge gives the bits of pkv_paged_attention_decode.
 * The partitions call may be repeated on the same workspace without a merge between. */
int pkv_paged_attention_decode_partitions(void *out, const void *q, const void *k_cache,
                                          const void *v_cache, const int32_t *block_tables,
                                          const int32_t *context_lens, int num_seqs,
                                          int num_heads, int num_kv_heads, int head_dim,
                                          int block_size, int max_blocks_per_seq, int num_blocks,
                                          int max_context_len, float scale, int dtype,
                                          int partition_size, void *workspace,
                                          size_t workspace_bytes, pkv_stream_t stream);

int pkv_paged_attention_merge(void *out, const int32_t *context_lens, int num_seqs, int num_heads,
                              int num_kv_heads, int head_dim, int block_size, int max_context_len,
                              int partition_size, int dtype, void *workspace,
                              size_t workspace_bytes, pkv_stream_t stream);

/* ------------------------------------------------------------------------------
 * pkv_paged_attention_decode for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a library convenience.
 *
 * Some callers may not call cudaMalloc at all: plugin code inside a host framework
 * that owns every device allocation and hands the plugin only its input and output
 * buffers, serving loops that reserve all HBM for the KV pool up front, and latency-
 * critical code where an allocation may synchronise the device. This entry point
 * takes the same arguments as pkv_paged_attention_decode minus the workspace; the
 * partition scratch is a fixed array inside the library of PKV_NOALLOC_SCRATCH_BYTES
 * per device (every GPU that loads the library holds it until the process exits).
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * - Sizes whose scratch (pkv_decode_workspace_size) exceeds PKV_NOALLOC_SCRATCH_BYTES
 *   are rejected with PKV_ERR_WORKSPACE before any device work; a larger
 *   partition_size needs less scratch.
 * - The first call on a device looks up the scratch array's device address (once per
 *   device, with that device current); make that first call before any stream capture.
 * - Every call on a device shares the one array, which keeps the last call's
 *   contents (nothing in it needs to start at zero). Calls that can overlap on the
 *   GPU (unordered streams, several host threads) race on it and corrupt each
 *   other's results: order them on one stream.
 * Errors: as pkv_paged_attention_decode, plus PKV_ERR_CUDA if the address lookup fails.
 * ---------------------------------------------------------------------------- */
#define PKV_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

int pkv_paged_attention_decode_noalloc(void *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       const int32_t *context_lens, int num_seqs, int num_heads,
                                       int num_kv_heads, int head_dim, int block_size,
                                       int max_blocks_per_seq, int num_blocks,
                                       int max_context_len, float scale, int dtype,
                                       int partition_size, pkv_stream_t stream);

/* ------------------------------------------------------------------------------
 * Shared-prefix-aware decode: the same result as pkv_paged_attention_decode, for
 * batches where groups of sequences share their first pages (parallel sampling, common
 * prompts: "vLLM" entity page, 是什么; "分页 KV Cache 分析" §3.2). Each shared prefix page
 * of a KV head is read once for up to 16 query rows (the G heads of up to 16/G member
 * sequences) instead of once per sequence; private suffixes are read per sequence, in the
 * same work item as the prefix where both fit in one partition (then written directly),
 * else as pieces merged exactly (log-sum-exp).
 *
 * group_start  device int32 [num_groups + 1]: sequences group_start[g] ..
 *              group_start[g+1]-1 form group g (0 = group_start[0] < ... <
 *              group_start[num_groups] = num_seqs). Unshared sequences are groups of one.
 * prefix_lens  device int32 [num_groups]: tokens the group's members share. Taken as a
 *              hint: it is cut to a multiple of block_size, to the shortest member, and at
 *              the first logical block where a member's table differs from the group's
 *              first member — a wrong value costs sharing, never correctness.
 * A malformed group_start is treated as one group per sequence and sets
 * PKV_STATUS_BAD_LEN. Workspace: pkv_decode_shared_prefix_workspace_size bytes of device
 * memory, 16-byte aligned, owned by the caller, no initial contents required (else
 * PKV_ERR_WORKSPACE). partition_size 0 selects this path's own automatic size
 * (pkv_decode_shared_prefix_partition_size: 2048 tokens, at most 256 blocks, smaller for
 * small batches). Other arguments, limits and errors as
 * pkv_paged_attention_decode (num_groups >= 1, <= num_seqs). Three kernel launches.
 * ---------------------------------------------------------------------------- */
int pkv_paged_attention_decode_shared_prefix(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, const int32_t *group_start,
    const int32_t *prefix_lens, int num_groups, int num_seqs, int num_heads, int num_kv_heads,
    int head_dim, int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len,
    float scale, int dtype, int partition_size, void *workspace, size_t workspace_bytes,
    pkv_stream_t stream);

/* The same call in two parts, so that one plan serves every layer of a step (the plan
 * depends only on the tables, lengths and groups, which the layers share):
 * pkv_shared_prefix_plan builds the item list in the workspace (one launch);
 * pkv_paged_attention_decode_shared_prefix_planned runs the decode and the merge over it
 * (two launches) and may be called any number of times on the same workspace, ordered on
 * one stream, while the tables and lengths stay as planned. A planned call whose sizes
 * (num_seqs, num_heads, num_kv_heads, partition size) differ from the plan's writes nothing
 * and sets PKV_STATUS_WORKSPACE. Arguments as pkv_paged_attention_decode_shared_prefix;
 * pkv_paged_attention_decode_shared_prefix is the plan followed by one planned call. */
int pkv_shared_prefix_plan(const int32_t *block_tables, const int32_t *context_lens,
                           const int32_t *group_start, const int32_t *prefix_lens, int num_groups,
                           int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                           int block_size, int max_blocks_per_seq, int max_context_len,
                           int partition_size, void *workspace, size_t workspace_bytes,
                           pkv_stream_t stream);

int pkv_paged_attention_decode_shared_prefix_planned(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
    int max_context_len, float scale, int dtype, int partition_size, void *workspace,
    size_t workspace_bytes, pkv_stream_t stream);

int pkv_decode_shared_prefix_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_context_len,
                                            int partition_size, size_t *bytes_out);

/* The partition size the shared-prefix calls use for these sizes (resolves 0 to the
 * shared path's automatic size). */
int pkv_decode_shared_prefix_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                            int head_dim, int block_size, int max_context_len,
                                            int partition_size, int *partition_out);

/* Workspace bytes pkv_paged_attention_decode needs for these sizes (0 when the
 * given partition size makes every context a single partition). Same argument
 * meaning as the decode call. */
int pkv_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_context_len, int partition_size,
                              size_t *bytes_out);

/* The partition size the decode call uses for these sizes (resolves 0 = automatic). */
int pkv_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int max_context_len, int partition_size,
                              int *partition_out);

/* ------------------------------------------------------------------------------
 * Cache write ("分页 KV Cache 分析" §3.2: a new token is written into its page).
 *   for t < num_tokens with slot = slot_mapping[t] >= 0:
 *     k_cache[slot / block_size][h][slot % block_size][:] = k_new[t][h][:]   (V alike)
 * Bit-exact copy. Slots must be distinct. A slot >= num_blocks*block_size is skipped
 * and sets PKV_STATUS_BAD_SLOT. Limits as for decode (head_dim, block_size).
 * ---------------------------------------------------------------------------- */
int pkv_reshape_and_cache(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                          const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int block_size, int num_blocks, int dtype,
                          pkv_stream_t stream);

/* ------------------------------------------------------------------------------
 * Copy-on-write block copy ("分页 KV Cache 分析" §3.2: copy first, then modify).
 *   for each layer l < num_layers and pair (src, dst) in block_pairs:
 *     k_caches[l][dst] = k_caches[l][src]; v_caches[l][dst] = v_caches[l][src]
 * (all KV heads). k_caches / v_caches are DEVICE arrays of num_layers device pointers,
 * each a cache in the layout above. block_pairs is a device array. Every dst must be
 * distinct and no dst may also be a src in the same call (then pair order does not
 * matter). A pair with src or dst outside [0, num_blocks) is skipped and sets
 * PKV_STATUS_BAD_PAIR.
 * ---------------------------------------------------------------------------- */
int pkv_copy_blocks(void *const *k_caches, void *const *v_caches, int num_layers,
                    const int32_t *block_pairs, int num_pairs, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, pkv_stream_t stream);

/* ------------------------------------------------------------------------------
 * Swap of whole blocks between the device caches and pinned host memory, for
 * preemption ("vLLM/PagedAttention — L3 Cross-Paper Synthesis" §3: eviction swaps every
 * block of a request out; "vLLM" entity page, observation 2: host transfers made of many
 * small copies leave the link mostly idle). One kernel moves every listed block of every
 * layer, K and V, through mapped host memory:
 *   to_host = 1: host_buffer[l][kv][i][:] = (kv ? v_caches : k_caches)[l][block_ids[i]]
 *   to_host = 0: the reverse (blocks are written back to the listed ids)
 * host_buffer: HOST pointer to pinned memory (cudaHostAlloc / a pinned torch tensor) that
 * the current device can address; layout [num_layers][2][num_ids][Hkv*BS*D] elements,
 * at least num_layers*2*num_ids*Hkv*BS*D*2 bytes, 16-byte aligned. Anything else
 * (pageable or device memory, too small) is rejected with PKV_ERR_INVALID_ARG before
 * launch. k_caches / v_caches / block_ids are device arrays as for pkv_copy_blocks; ids
 * outside [0, num_blocks) are skipped and set PKV_STATUS_BAD_PAIR. For to_host = 0 the
 * ids must be distinct. The copy is asynchronous on `stream`: the host buffer is
 * complete (or may be refilled) once the stream reaches this point.
 * ---------------------------------------------------------------------------- */
int pkv_swap_blocks(void *const *k_caches, void *const *v_caches, int num_layers,
                    const int32_t *block_ids, int num_ids, void *host_buffer,
                    size_t host_buffer_bytes, int to_host, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, int dtype, pkv_stream_t stream);

/* The same swap (same arguments, same host buffer layout and contents) moved in large
 * copies: the listed tiles are gathered into (or scattered from) `staging`, a DEVICE buffer
 * of staging_bytes (16-byte aligned, at least two tiles of Hkv*BS*D*2 bytes), used as two
 * halves: each half, once full, crosses the host link as one cudaMemcpyAsync while the
 * other half is gathered (or scattered), so the link runs at the rate of its copy engine
 * rather than of the SMs' stores to mapped memory. The copies run on a stream of the
 * library's, ordered after the work `stream` holds at the call by an event, and `stream`
 * waits for the last of them: as for pkv_swap_blocks, the host buffer is complete (or may
 * be refilled) once `stream` reaches this point. Calls that use this path are serialised
 * on the host while they enqueue. host_buffer must be pinned host memory (the copies are
 * asynchronous only from it). Tiles of ids outside [0, num_blocks) set PKV_STATUS_BAD_PAIR
 * and are zero in the host buffer (to_host = 1) or not written (to_host = 0). Errors: as
 * pkv_swap_blocks; PKV_ERR_WORKSPACE (staging missing, misaligned or smaller than two
 * tiles); PKV_ERR_INVALID_ARG (staging not device memory); PKV_ERR_CUDA. */
int pkv_swap_blocks_staged(void *const *k_caches, void *const *v_caches, int num_layers,
                           const int32_t *block_ids, int num_ids, void *host_buffer,
                           size_t host_buffer_bytes, int to_host, int num_kv_heads,
                           int head_dim, int block_size, int num_blocks, int dtype,
                           void *staging, size_t staging_bytes, pkv_stream_t stream);

/* ------------------------------------------------------------------------------
 * Decode step on the device ("分页 KV Cache 分析" §3.1: each decode step writes the new
 * token's K/V into its page, then attention reads the pages; §2.3: the block manager
 * hands a sequence a new page when its last one is full; "vLLM" entity page, 关键观察:
 * a kernel launch costs a few microseconds, a visible share of a decode step). Two calls
 * replace, per step, the host table update + upload and, per layer, the cache write,
 * decode and merge launches:
 *
 * pkv_device_append (once per step, before the layers): appends one token to each of
 * num_seqs sequences, in place on device arrays.
 *   n = context_lens[s]; if n % block_size == 0 the sequence takes the next entry of
 *   free_blocks (entries free_blocks[*free_used], [*free_used + 1], ... go to the
 *   sequences that need one, in increasing s) into block_tables[s][n / block_size];
 *   slots_out[s] = block_tables[s][n / block_size] * block_size + n % block_size (or -1,
 *   with PKV_STATUS_BAD_BLOCK, if that entry is outside [0, num_blocks));
 *   context_lens[s] = n + 1; finally *free_used += blocks taken.
 * With free_blocks holding the host block manager's free blocks in the order it would
 * pop them, the result equals pkv_seq_append(.., 1, ..) on s = 0, 1, ... as long as no
 * sequence writes into a block it shares: copy-on-write ("分页 KV Cache 分析" §3.2, copy a
 * shared page before changing it) stays on the host. block_refcounts (device int32
 * [num_blocks], the host manager's counts from pkv_alloc_refcounts, uploaded after its
 * last fork or free; NULL = the caller guarantees that nothing is shared) lets the kernel
 * check this: a sequence with n % block_size != 0 whose block block_tables[s][n /
 * block_size] has a count above 1 refuses the step (PKV_STATUS_SHARED_BLOCK). Blocks the
 * device append itself took from free_blocks count 0 there: they are private.
 * All or nothing: if fewer than the needed entries remain (free_count - *free_used), an
 * entry is outside [0, num_blocks), some n < 0, n + 1 > max_context_len or
 * n / block_size >= max_blocks_per_seq, nothing is written and PKV_STATUS_NO_BLOCKS is
 * set; a shared block as above also writes nothing and sets PKV_STATUS_NO_BLOCKS |
 * PKV_STATUS_SHARED_BLOCK. block_tables int32 [num_seqs][max_blocks_per_seq],
 * context_lens int32 [num_seqs], free_blocks int32 [free_count], free_used int32 [1]
 * (all device), slots_out int64 [num_seqs] device or NULL. One CTA; asynchronous on
 * `stream`. Errors: PKV_ERR_INVALID_ARG, PKV_ERR_CUDA.
 * ---------------------------------------------------------------------------- */
int pkv_device_append(int32_t *block_tables, int32_t *context_lens, const int32_t *free_blocks,
                      int free_count, int32_t *free_used, const int32_t *block_refcounts,
                      int64_t *slots_out, int num_seqs, int max_blocks_per_seq, int block_size,
                      int num_blocks, int max_context_len, pkv_stream_t stream);

/* pkv_paged_decode_step (once per layer): one launch that writes every sequence's newest
 * token and computes the decode attention over it:
 *   for each s with len = context_lens[s] >= 1, slot = block_tables[s][(len-1)/bs]*bs +
 *   (len-1)%bs: k_cache[slot / bs][h][slot % bs][:] = k_new[s][h][:] (V alike), then
 *   out = pkv_paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens).
 * Same arguments, layouts, limits and results as pkv_reshape_and_cache with that slot
 * mapping followed by pkv_paged_attention_decode (same partition size: identical bits),
 * plus k_new / v_new [num_seqs][num_kv_heads][head_dim] device, 16-byte aligned.
 * Workspace: pkv_decode_step_workspace_size bytes (at least 256), 256-byte aligned, owned
 * by the caller, ZERO-FILLED before its first use and then reused only by this call on one
 * stream (each launch leaves it ready for the next). A workspace that
 * pkv_paged_attention_decode has used with several partitions (same layout; its merge
 * kernel re-arms the header) also serves. A launch that merges in the step kernel
 * refuses, on the device and before any write, a header that is none of these: zero
 * (with a zero barrier generation), or left by these kernels with a zero exit count
 * (PKV_STATUS_WORKSPACE, no output). A stale arrival count, which cannot be checked at
 * the start, is caught at the grid barrier (PKV_STATUS_WORKSPACE; do not use that
 * launch's output); the launch still leaves the header ready for the next one.
 * When some context spans several partitions they are merged either in the same launch
 * (cooperative, all CTAs resident: after a bounded grid barrier every warp merges
 * (sequence, head) pairs; PKV_STATUS_WAIT_TIMEOUT if the barrier gives up), chosen when
 * num_seqs * num_heads is at most the grid's warp count (2 CTAs of 5 warps per SM, at most
 * one CTA per work item), or else by the partition-merge kernel launched right after
 * (pkv_decode_step_launches tells which). Errors: as pkv_paged_attention_decode. */
int pkv_paged_decode_step(void *out, const void *q, const void *k_new, const void *v_new,
                          void *k_cache, void *v_cache, const int32_t *block_tables,
                          const int32_t *context_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                          int num_blocks, int max_context_len, float scale, int dtype,
                          int partition_size, void *workspace, size_t workspace_bytes,
                          pkv_stream_t stream);

/* The write-and-decode launch of pkv_paged_decode_step alone (never the in-launch merge):
 * every newest token written, one-partition sequences' outputs, the others' partials left
 * in `workspace` for pkv_paged_attention_merge (same sizes and workspace). Arguments,
 * workspace rules and errors as pkv_paged_decode_step; followed by the merge it gives the
 * bits of pkv_paged_decode_step. */
int pkv_paged_decode_step_partitions(void *out, const void *q, const void *k_new,
                                     const void *v_new, void *k_cache, void *v_cache,
                                     const int32_t *block_tables, const int32_t *context_lens,
                                     int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                     int block_size, int max_blocks_per_seq, int num_blocks,
                                     int max_context_len, float scale, int dtype,
                                     int partition_size, void *workspace, size_t workspace_bytes,
                                     pkv_stream_t stream);

int pkv_decode_step_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                   int block_size, int max_context_len, int partition_size,
                                   size_t *bytes_out);

/* Kernel launches one pkv_paged_decode_step call with these sizes makes (0, 1 or 2), into
 * *launches_out. Needs the current device (its SM count). */
int pkv_decode_step_launches(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                             int block_size, int max_context_len, int partition_size,
                             int *launches_out);

/* Synchronise `stream`, then read (and with clear != 0 reset) the status word of the
 * current device. *status_out gets the PKV_STATUS_* bits. Returns PKV_OK, or
 * PKV_ERR_CUDA if synchronisation or the read failed. */
int pkv_get_device_status(uint32_t *status_out, int clear, pkv_stream_t stream);

/* ------------------------------------------------------------------------------
 * Host block manager ("vLLM" entity page, 是什么; "分页 KV Cache 分析" §2.3, §3.2, §3.3).
 * Pure host code; no CUDA call. Not thread-safe: one handle per thread at a time.
 *
 * Rules (the pages fix no order; these are the library's readings):
 *  - free list: LIFO stack seeded so successive allocations return
 *    initial_order[0], initial_order[1], ... (NULL = 0, 1, 2, ...).
 *  - append of one token at length n: if n % block_size == 0 take a new block
 *    (refcount 1); else if the last block's refcount > 1 take a new block b', emit the
 *    copy-on-write pair (last, b'), drop one reference to `last`, put b' in the table.
 *    The token's slot is table[n / bs] * bs + n % bs; then n += 1.
 *  - append of k tokens is all-or-nothing (PKV_ERR_TABLE_FULL / PKV_ERR_OUT_OF_BLOCKS
 *    leave every state unchanged).
 *  - fork copies the parent's table and length, adding one reference per block.
 *  - free walks the table from the last logical block to the first, drops one
 *    reference each and returns blocks whose count reaches 0 to the free list.
 * ---------------------------------------------------------------------------- */
typedef struct pkv_alloc pkv_alloc;

/* Creates a manager of num_blocks blocks. initial_order: NULL or a host array that is a
 * permutation of 0..num_blocks-1 (copied). Errors: PKV_ERR_INVALID_ARG. */
int pkv_alloc_create(pkv_alloc **out, int num_blocks, int block_size, int max_blocks_per_seq,
                     const int32_t *initial_order);
int pkv_alloc_destroy(pkv_alloc *a);

/* Appends n_tokens tokens to seq_id (creating it on first use). slots_out: host int64
 * [n_tokens] (may be NULL when n_tokens == 0). cow_pairs_out: host int32 [n_tokens][2],
 * receives *n_cow_out (src, dst) pairs to copy before writing. */
int pkv_seq_append(pkv_alloc *a, int64_t seq_id, int n_tokens, int64_t *slots_out,
                   int32_t *cow_pairs_out, int *n_cow_out);
/* One decode step for a batch: pkv_seq_append(a, seq_ids[i], n_tokens, ...) for i = 0..n-1 in
 * order. Sequence i's slots go to slots_out[i*n_tokens .. i*n_tokens+n_tokens); all copy-on-write
 * pairs go to cow_pairs_out (host int32 [n*n_tokens][2]) in call order, *n_cow_out of them.
 * Stops at the first sequence whose append fails and returns its error; *n_done_out (may be
 * NULL) = sequences appended before it, whose results stand (the failing one changed nothing). */
int pkv_seq_append_batch(pkv_alloc *a, const int64_t *seq_ids, int n, int n_tokens,
                         int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out,
                         int *n_done_out);

/* A decode step's host work in one call: pkv_seq_append_batch (same arguments, same results)
 * and then, if every append succeeded, pkv_block_tables of the same sequences into host
 * tables_out [n][max_blocks_per_seq] (unused entries -1) and lens_out [n] (may be NULL).
 * "分页 KV Cache 分析" §2.3: each step the block manager extends every running sequence,
 * handing out a page when its last one is full, and the kernel reads the updated tables.
 * On a failed append the tables are not written. Errors: those of pkv_seq_append_batch;
 * PKV_ERR_INVALID_ARG (tables_out NULL with n > 0: nothing changes). */
int pkv_seq_append_tables(pkv_alloc *a, const int64_t *seq_ids, int n, int n_tokens,
                          int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out,
                          int *n_done_out, int32_t *tables_out, int32_t *lens_out);

/* Errors: PKV_ERR_UNKNOWN_SEQ (no parent), PKV_ERR_SEQ_EXISTS (child id in use). */
int pkv_seq_fork(pkv_alloc *a, int64_t parent, int64_t child);

/* pkv_seq_fork(parents[i], children[i]) and pkv_seq_free(seq_ids[i]) for i = 0, 1, ... in
 * one call each (host arrays of n ids), for parallel sampling and beam search, which fork
 * and retire many sequences per step. They stop at the first failing call and return its
 * status; *n_done_out (may be NULL) = calls that succeeded, whose effects stay. */
int pkv_seq_fork_batch(pkv_alloc *a, const int64_t *parents, const int64_t *children, int n,
                       int *n_done_out);
int pkv_seq_free_batch(pkv_alloc *a, const int64_t *seq_ids, int n, int *n_done_out);

/* The blocks the next allocations would take, in that order (free blocks, then cached
 * blocks nobody holds, least recently released first): at most max_out of them into
 * blocks_out, their count into *n_out. Uploaded to the device, this is the free list
 * pkv_device_append takes from. */
int pkv_alloc_free_list(const pkv_alloc *a, int32_t *blocks_out, int max_out, int *n_out);

/* The reference count of every block (sequences whose table holds it; 0 = free or cached
 * and unheld) into the host array refcounts_out [n], n >= num_blocks (entries past
 * num_blocks untouched). Uploaded to the device, it is the block_refcounts argument of
 * pkv_device_append. Errors: PKV_ERR_INVALID_ARG. */
int pkv_alloc_refcounts(const pkv_alloc *a, int32_t *refcounts_out, int n);

/* ------------------------------------------------------------------------------
 * Prefix caching ("分页 KV Cache 分析" §2.3 and §3.2: common prefixes such as a system
 * prompt or few-shot examples are found automatically and their pages reused across
 * requests; 五: only exactly identical token sequences share). Off by default; with it
 * off every call below behaves as if no block were ever cached.
 *
 * Readings (the pages fix no mechanism):
 *  - only full blocks are cached. A full block is identified by a 64-bit hash chained over
 *    all tokens up to its end (splitmix64 applied token by token, starting from the hash
 *    of the blocks before it, 0 for the first block); a match also compares the block's
 *    own tokens and its parent hash exactly.
 *  - a block becomes cached when a sequence whose every token came with its id (created
 *    by pkv_seq_append_tokens or pkv_seq_share_prefix) fills it, unless an identical block
 *    is already cached. Appending without ids stops that sequence from caching.
 *  - a cached block nobody holds is kept (evictable) instead of freed; allocation takes a
 *    free block first and otherwise reclaims the least recently released cached block.
 *    Evictable blocks count as free in pkv_stats.
 * ---------------------------------------------------------------------------- */
int pkv_alloc_set_prefix_cache(pkv_alloc *a, int enable);

/* pkv_seq_append with the appended tokens' ids (host int32 [n_tokens]). */
int pkv_seq_append_tokens(pkv_alloc *a, int64_t seq_id, const int32_t *tokens, int n_tokens,
                          int64_t *slots_out, int32_t *cow_pairs_out, int *n_cow_out);

/* Creates sequence seq_id holding the longest cached run of full blocks that matches
 * tokens[0..n_tokens) (one more reference each); *n_cached_out = tokens covered (a
 * multiple of block_size, 0 when the cache is off or nothing matches). The caller then
 * appends the remaining tokens with pkv_seq_append_tokens (to keep one token uncached,
 * pass n_tokens - 1). Errors: PKV_ERR_SEQ_EXISTS. */
int pkv_seq_share_prefix(pkv_alloc *a, int64_t seq_id, const int32_t *tokens, int n_tokens,
                         int *n_cached_out);

/* Groups for the shared-prefix-aware decode, read from the tables ("分页 KV Cache 分析" §3.2:
 * requests with a common prompt share its pages; "vLLM" entity page, 是什么: parallel samples
 * share their prompt's blocks). Sequences whose first full block is the same physical block
 * form a group (in the order of their first member in seq_ids, members in seq_ids order); a
 * sequence with no full block is a group of one. order_out [n]: the sequence ids, grouped;
 * group_start_out [n + 1]: the first num_groups + 1 entries are the group boundaries in that
 * order (0 = group_start[0] < ... = n); prefix_lens_out [n]: the first num_groups entries
 * are block_size x the leading blocks every member's table holds in common, counting only
 * each member's full blocks (0 for a group of one). Build the block tables, lengths and
 * queries in order_out's order and pass these as group_start / prefix_lens to
 * pkv_paged_attention_decode_shared_prefix. Errors: PKV_ERR_UNKNOWN_SEQ; PKV_ERR_INVALID_ARG
 * (an id listed twice, a NULL output with n > 0); nothing is written past the check. */
int pkv_prefix_groups(const pkv_alloc *a, const int64_t *seq_ids, int n, int64_t *order_out,
                      int32_t *group_start_out, int32_t *prefix_lens_out, int *num_groups_out);

/* Blocks in the cache, of which evictable; tokens queried by pkv_seq_share_prefix and
 * tokens it found cached. Any output pointer may be NULL. */
int pkv_prefix_cache_stats(const pkv_alloc *a, int *cached_blocks, int *evictable_blocks,
                           int64_t *query_tokens, int64_t *hit_tokens);
/* Errors: PKV_ERR_UNKNOWN_SEQ. */
int pkv_seq_free(pkv_alloc *a, int64_t seq_id);

/* Writes the block tables of n sequences into host tables_out [n][max_blocks_per_seq]
 * (unused entries -1) and their lengths into lens_out [n] (may be NULL).
 * Errors: PKV_ERR_UNKNOWN_SEQ (nothing written past the first unknown id). */
int pkv_block_tables(const pkv_alloc *a, const int64_t *seq_ids, int n, int32_t *tables_out,
                     int32_t *lens_out);

/* free + held = num_blocks; logical_tokens = sum of lengths; utilisation =
 * logical_tokens / (held * block_size) ("分页 KV Cache 分析" §4.2), 0 when nothing is
 * held. Any output pointer may be NULL. */
int pkv_stats(const pkv_alloc *a, int *free_blocks, int *held_blocks, int64_t *logical_tokens,
              double *utilisation);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
