/*
 * pa.h -- C ABI of the paged KV-cache decode library (NVIDIA B200, sm_100a).
 *
 * The library implements the data-parallel hot path of PagedAttention:
 *
 *   - a shared pool of fixed-size KV blocks addressed through per-request
 *     block tables ("PagedAttention & vLLM" (fp-ai-systems.pages.dev),
 *     section "The insight: KV cache as virtual memory"),
 *   - the cache-append write through a slot mapping ("Walk through paged
 *     attention end to end" (zenaique.com), conceptual
 *     paged_attention_decode, append step),
 *   - single-query decode attention that looks up each token's block
 *     through the table (same page, attention step; "What is
 *     PagedAttention and how does it manage KV cache" (n4n.ai), section
 *     "How PagedAttention works": two-level indirection, tokens contiguous
 *     inside a block),
 *   - the copy-on-write block copy ("PagedAttention & vLLM", section
 *     "Copy-on-write sharing"),
 *   - a host-side refcounted block allocator with fork and copy-on-write.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every function returns an int status (pa_status).  Argument errors are
 *    detected on the host, before any launch, and nothing is launched.
 *    A failed launch returns PA_ERR_CUDA.
 *  - Device pointers are caller-owned device memory of the current CUDA
 *    device.  The library allocates no device memory at run time; the
 *    caller provides the decode workspace (size from
 *    pa_decode_workspace_size).  The one exception is
 *    pa_decode_builtin_scratch, whose scratch is a static device array.
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Device work is asynchronous on that stream.
 *  - Data-dependent index errors (a slot, block id or copy pair out of range,
 *    a sequence longer than its table) never fault: the offending access is
 *    skipped and a PA_FLAG_* bit is OR-ed into *err_flag (an int32 in device
 *    memory; may be NULL to skip reporting).  The caller reads it when it
 *    chooses to.  Bounded waits inside kernels that run out set
 *    PA_FLAG_TIMEOUT the same way.  Kernels never trap.
 *  - Pool layout (both K and V, separate allocations):
 *        bf16 [num_blocks, num_kv_heads, block_size, head_dim], row-major,
 *    base address 16-byte aligned.  One (block, kv head) tile of
 *    block_size x head_dim values is contiguous.
 *  - Supported shapes: bf16 only; head_dim in {64, 128}; block_size in
 *    {8, 16, 32, 64}; num_q_heads / num_kv_heads in {1, 2, 4, 8}.
 *  - A slot is physical_block * block_size + row_in_block.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer, ... */
    PA_ERR_UNSUPPORTED = 2, /* shape outside the supported set */
    PA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    PA_ERR_BAD_INDEX = 4,   /* host allocator: unknown sequence / block id */
    PA_ERR_TIMEOUT = 5,     /* reserved for host-side waits */
    PA_ERR_OOM = 6,         /* host allocator: pool exhausted (state unchanged) */
    PA_ERR_STATE = 7        /* operation not valid in the current state */
} pa_status;

/* Bits OR-ed into the device error flag by kernels. */
#define PA_FLAG_BAD_SLOT 0x1    /* reshape: slot outside [0, num_blocks*block_size), not -1 */
#define PA_FLAG_BAD_BLOCK 0x2   /* decode: block id outside [0, num_blocks) */
#define PA_FLAG_BAD_PAIR 0x4    /* copy: src or dst outside [0, num_blocks) */
#define PA_FLAG_BAD_LEN 0x8     /* decode: seq_len < 0, > max_seq_len, or > table capacity */
#define PA_FLAG_TIMEOUT 0x10    /* a bounded in-kernel wait ran out */

/* Human-readable name of a status code (static string, never NULL). */
const char *pa_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int pa_version(void);

/* Number of kernels this library has launched in the process so far. */
uint64_t pa_launch_count(void);

/* ------------------------------------------------------------------------
 * Cache write ("Walk through paged attention end to end", conceptual
 * paged_attention_decode: the new token's K and V go to block
 * table[-1] at offset next_pos % block_size).
 *
 *   k_cache[s / bs, h, s % bs, :] = k_new[t, h, :]   for s = slot_mapping[t]
 *   v_cache[s / bs, h, s % bs, :] = v_new[t, h, :]
 *
 * k_new, v_new   : device bf16 [num_tokens, num_kv_heads, head_dim], 16-byte aligned
 * k_cache,v_cache: device bf16 pools (layout above)
 * slot_mapping   : device int32 [num_tokens]; -1 = skip (padding token);
 *                  other values outside [0, num_blocks*block_size) set
 *                  PA_FLAG_BAD_SLOT and are skipped.
 * Distinct tokens must name distinct slots (otherwise the winner is
 * unspecified).  num_tokens == 0 launches nothing.  Bit-exact copy.
 * ---------------------------------------------------------------------- */
int pa_reshape_and_cache(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                         const int32_t *slot_mapping, int num_tokens, int64_t num_blocks,
                         int num_kv_heads, int block_size, int head_dim, int32_t *err_flag,
                         void *stream);

/* ------------------------------------------------------------------------
 * Copy-on-write block copy ("PagedAttention & vLLM", Copy-on-write sharing:
 * a sequence about to change a shared block first gets a private copy).
 *
 * For each pair i: block pairs[2i+1] of both pools becomes a bit copy of
 * block pairs[2i] (all heads, rows and dims).
 *
 * pairs : device int32 [num_pairs, 2] = (src, dst).  Destinations must be
 *         distinct and must not appear as sources in the same call (a source
 *         may repeat).  Ids outside [0, num_blocks) set PA_FLAG_BAD_PAIR and
 *         the pair is skipped.  num_pairs == 0 launches nothing.
 * ---------------------------------------------------------------------- */
int pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *pairs, int num_pairs,
                   int64_t num_blocks, int num_kv_heads, int block_size, int head_dim,
                   int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Block swap between two pools ("What is PagedAttention and how does it
 * manage KV cache", Swapping and preemption: under memory pressure a
 * request's blocks move out to host memory and come back when it resumes).
 *
 * For each pair i: block pairs[2i+1] of the destination pools becomes a bit
 * copy of block pairs[2i] of the source pools (K and V, all heads, rows and
 * dims).  Either side may be device memory or page-locked host memory that
 * the device can address (pinned with cudaHostAlloc / cudaHostRegister on a
 * system with unified addressing): swap-out is device -> host, swap-in is
 * host -> device.  Both sides use the pool layout above with the same
 * num_kv_heads, block_size and head_dim; they may differ in block count.
 * pairs: int32 [num_pairs, 2] = (src block, dst block), device-addressable.
 * Every pointer is checked with cudaPointerGetAttributes before the launch:
 * one the device cannot reach (pageable host memory, another GPU's memory,
 * an address CUDA does not know) gives PA_ERR_INVALID_ARG and nothing runs.
 * Destinations must be distinct.  Ids out of range set PA_FLAG_BAD_PAIR and
 * the pair is skipped.  Bandwidth is that of the slower side (PCIe or
 * NVLink-C2C for host memory).
 * ---------------------------------------------------------------------- */
int pa_swap_blocks(void *dst_k_cache, void *dst_v_cache, int64_t dst_num_blocks, const void *src_k_cache,
                   const void *src_v_cache, int64_t src_num_blocks, const int32_t *pairs, int num_pairs,
                   int num_kv_heads, int block_size, int head_dim, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Paged decode attention.  For every sequence b and query head g, with
 * kv head h = g / (num_q_heads / num_kv_heads) and L = seq_lens[b]:
 *
 *   s_p   = scale * q[b,g,:] . K_h[p,:]          p = 0 .. L-1
 *   out   = sum_p exp(s_p - max s) V_h[p,:] / sum_p exp(s_p - max s)
 *
 * where row p of sequence b is pool[block_tables[b, p / bs], h, p % bs, :]
 * ("Walk through paged attention end to end", attention step; the math is
 * standard attention, only the addressing changes).  L = 0 yields zeros.
 * seq_lens counts the token appended in this step (append, then attend).
 *
 * out           : device fp32 [batch, num_q_heads, head_dim]
 * q             : device bf16 [batch, num_q_heads, head_dim], 16-byte aligned
 * block_tables  : device int32 [batch, max_blocks_per_seq]; only entries
 *                 j < ceil(L/bs) are read (padding may hold anything)
 * seq_lens      : device int32 [batch]
 * max_seq_len   : host-side upper bound of seq_lens (sizes the split grid);
 *                 longer sequences set PA_FLAG_BAD_LEN and are truncated.
 * scale         : softmax scale (usually 1/sqrt(head_dim))
 * partition_tokens : 0 = library default for this shape, -1 = one pass per
 *                 (sequence, kv head), > 0 = split each sequence into
 *                 partitions of this many tokens (a multiple of block_size).
 *                 Each partition stores its partial softmax state (max, sum,
 *                 normalised output) in the workspace, and a second kernel,
 *                 launched as a programmatic dependent, merges them
 *                 (log-sum-exp).  A sequence that fits one partition is
 *                 written by the decode directly.
 * workspace     : device scratch of at least pa_decode_workspace_size(...)
 *                 bytes, 16-byte aligned (may be NULL if that size is 0).
 *                 Its contents need no initialisation: every partial state
 *                 the merge reads is written earlier in the same call.  Calls
 *                 that run at the same time need separate workspaces.
 * Each (sequence, kv head) is processed by one CTA (per partition) that
 * serves all query heads of the group, so every K/V byte is read once.
 * Launches one kernel, two when it splits (none when batch == 0).  Shared-prefix
 * locality: the grid runs the kv heads and partitions of a sequence next to
 * each other with the sequence index slowest, so sequences that follow each
 * other in the batch and share blocks (forks) re-read those blocks from L2.
 * ---------------------------------------------------------------------- */
size_t pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int max_seq_len, int partition_tokens);

/* The partition size pa_decode will use for these arguments (-1 = one pass). */
int pa_decode_partition_tokens(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_seq_len, int partition_tokens);

int pa_decode(float *out, const void *q, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens,
              int batch, int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, int64_t num_blocks, float scale, int partition_tokens,
              void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Fused decode step: each sequence's new token is written to the cache and
 * attended in the same launch ("Walk through paged attention end to end",
 * conceptual paged_attention_decode: append the new K/V to the block of
 * position next_pos, then attend over every position).
 *
 * Equivalent to pa_reshape_and_cache with
 *     slot_mapping[b] = block_tables[b][(L-1)/bs] * bs + (L-1) % bs,  L = seq_lens[b]
 * followed by pa_decode, but in one decode launch (plus the reduce when the
 * call splits).  k_new, v_new: device bf16 [batch, num_kv_heads, head_dim],
 * 16-byte aligned; row b is the token at position seq_lens[b] - 1 (seq_lens
 * counts it).  Sequences with seq_lens[b] == 0, or longer than max_seq_len
 * or their table (PA_FLAG_BAD_LEN), write nothing.  The block that receives
 * the new token must belong to this sequence alone (the allocator's
 * copy-on-write guarantees that; apply its copy pairs first).  Other
 * arguments, layouts and errors: as pa_decode (the same workspace size).
 * ---------------------------------------------------------------------- */
int pa_decode_append(float *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
                     void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                     int partition_tokens, void *workspace, size_t workspace_bytes, int32_t *err_flag,
                     void *stream);

/* ------------------------------------------------------------------------
 * Shared-prefix decode.  "PagedAttention & vLLM", Copy-on-write sharing:
 * n samples of one prompt keep the prompt's KV in one set of physical
 * blocks ("one copy, not four"); "What is PagedAttention and how does it
 * manage KV cache", Concrete example: requests sharing a system prompt
 * allocate its blocks once.  This call turns that shared storage into shared
 * reads: the shared tokens of a group are read from HBM once per kv head for
 * all of its members, instead of once per member.
 *
 * Computes exactly what pa_decode computes (pa_decode_append when k_new and
 * v_new are given), for batches laid out in groups: sequences
 * [g*group_size, (g+1)*group_size) form group g (the last group may be
 * shorter), and for every member b of group g the K/V rows of positions
 * p < prefix_lens[g] must equal those of the group's first member (the same
 * physical blocks, as after pa_seq_fork, or copies of them, as after a
 * copy-on-write).  Per group, the shared range actually used is
 *     S_g = min(prefix_lens[g], L_b - 1 over members b), rounded down to a
 *           multiple of 16 tokens (0 for groups of one sequence),
 * so the token appended in this step is never read through another member's
 * table.  The rows of [0, S_g) are read once per kv head through the first
 * member's block table and combined with each member's query heads (up to
 * 8 / (num_q_heads / num_kv_heads) members per read); each member's own
 * rows [S_g, L_b) are read through its own table, and the two partial
 * softmax states are merged as in the split decode.  prefix_lens[g] = 0
 * means group g shares nothing; prefix_lens[g] < 0 sets PA_FLAG_BAD_LEN and
 * is read as 0.
 *
 * prefix_lens : device int32 [ceil(batch / group_size)]
 * group_size  : 1 .. 64
 * k_new, v_new: both NULL (no cache write) or both device bf16
 *               [batch, num_kv_heads, head_dim] as in pa_decode_append.
 * partition_tokens: as pa_decode, except that -1 (and a default that would
 *               not split) means one work item for the shared range and one
 *               for each member's own range.
 * workspace   : at least pa_decode_shared_prefix_workspace_size(...) bytes,
 *               16-byte aligned, no initialisation needed (as pa_decode).
 * Other arguments, layouts and errors: as pa_decode / pa_decode_append.
 * ---------------------------------------------------------------------- */
size_t pa_decode_shared_prefix_workspace_size(int batch, int group_size, int num_q_heads, int num_kv_heads,
                                              int head_dim, int block_size, int max_seq_len,
                                              int partition_tokens);

int pa_decode_shared_prefix(float *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
                            void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *seq_lens, const int32_t *prefix_lens, int group_size, int batch,
                            int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int64_t num_blocks, float scale, int partition_tokens, void *workspace,
                            size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * One decode step from host buffers.  Enqueues, in order:
 *   1. the upload of the copy pairs, the block tables, the sequence
 *      lengths, q, k_new and v_new into `staging`: one kernel reads every
 *      input that is page-locked and 16-byte aligned straight from host
 *      memory through its device mapping; any other input is copied with
 *      cudaMemcpyAsync,
 *   2. pa_copy_blocks of the copy pairs (if any),
 *   3. pa_decode_append (cache write of each sequence's new token + decode),
 *   4. the fp32 output into out_host.  When out_host is page-locked host
 *      memory the device can address (checked with cudaPointerGetAttributes),
 *      the decode kernels store the output into it directly, so the transfer
 *      overlaps the decode; otherwise the output is staged on the device and
 *      copied back with cudaMemcpyAsync.
 * The call returns once everything is enqueued; synchronise `stream` before
 * reading out_host.  Host buffers should be page-locked (pinned) for the
 * copies to be asynchronous, and must stay valid and unchanged until the
 * stream has passed them.
 *
 * num_chunks: 1 runs the four steps on `stream` alone.  n in 2..8 cuts the
 * batch into n chunks of consecutive sequences (the first about half the
 * size of the others) and pipelines them: chunk uploads and downloads run on library-owned
 * copy streams and chunk decodes alternate between `stream` and a
 * library-owned compute stream, so transfers of one chunk overlap the decode
 * of another.  All of them start after the work already enqueued on `stream`
 * and are joined back into `stream` before the call returns (on error paths
 * too), so synchronising `stream` covers the whole step.  0 picks the count
 * from the bytes crossing the host link: one chunk per 512 KiB, at most 4
 * (8 for a prepared step in shared-prefix mode), at most one per sequence
 * (measured on B200: a step moving 2.6 MB took 230, 213, 208 and 205 us end to
 * end with 1 to 4 chunks).  The output, the pools
 * and the error flag do not depend on the chunk count: the partitioning is resolved once for the whole
 * batch (as pa_decode_partition_tokens reports it) and each chunk decodes
 * its sequences exactly as an unchunked call would.  The side streams and
 * events of a device are created by its first chunked call and kept until
 * the process exits; calls on one device serialise their enqueueing on a
 * lock.  num_chunks < 0 or > 8: PA_ERR_INVALID_ARG.
 *
 * Host inputs: q_host bf16 [batch, Hq, d]; k_new_host, v_new_host bf16
 * [batch, Hkv, d] (the token at position seq_lens[b]-1); block_tables_host
 * int32 [batch, max_blocks_per_seq]; seq_lens_host int32 [batch];
 * copy_pairs_host int32 [num_pairs, 2] (may be NULL when num_pairs == 0).
 * Host output: out_host fp32 [batch, Hq, d].
 * staging: device memory of at least pa_decode_step_staging_size(...) bytes
 * (computed with the same batch, max_blocks_per_seq, max_copy_pairs and
 * shapes, and a max_seq_len at least this call's), 256-byte aligned; it
 * holds the uploaded inputs, the device output and the decode workspace
 * (with room for one slice per chunk).  A staging buffer may be reused by
 * the next call on the same stream.
 * Other arguments, layouts and errors: as pa_decode_append.
 * ---------------------------------------------------------------------- */
size_t pa_decode_step_staging_size(int batch, int max_blocks_per_seq, int max_copy_pairs, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size, int max_seq_len,
                                   int partition_tokens);

int pa_decode_step_host(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                        const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                        const int32_t *copy_pairs_host, int num_pairs, int max_copy_pairs, void *k_cache,
                        void *v_cache, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int64_t num_blocks, float scale, int partition_tokens,
                        int num_chunks, void *staging, size_t staging_bytes, int32_t *err_flag, void *stream);

/* The same step over fp8 (E4M3) pools (format and scales: see the fp8
 * section below).  The new rows arrive in bf16 and are quantised by the
 * fused write; copy pairs move E4M3 blocks (pa_copy_blocks_fp8); the decode
 * is pa_decode_append_fp8.  Staging is sized by pa_decode_step_staging_size
 * as for bf16 pools.  k_scale, v_scale not finite and > 0:
 * PA_ERR_INVALID_ARG, nothing enqueued.  Everything else: as
 * pa_decode_step_host. */
int pa_decode_step_host_fp8(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                            const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                            const int32_t *copy_pairs_host, int num_pairs, int max_copy_pairs, void *k_cache,
                            void *v_cache, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                            int head_dim, int block_size, int64_t num_blocks, float scale, float k_scale,
                            float v_scale, int partition_tokens, int num_chunks, void *staging,
                            size_t staging_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Prepared host step: pa_decode_step_host with everything that stays the same
 * from step to step resolved once -- argument checks, the staging layout,
 * the device view of each host buffer (cudaPointerGetAttributes: page-locked
 * buffers are read and written through their device mapping), the output
 * path and the chunk count.  A serving loop then pays one short call per
 * step.  No counterpart in the pages.
 *
 * pa_decode_step_plan_create takes the arguments of pa_decode_step_host
 * except the per-step ones (num_pairs, err_flag, stream) and with
 * max_seq_len_cap, the largest max_seq_len any run will pass (the staging
 * size must have been computed with it); kv_fp8 != 0 selects E4M3 pools
 * with k_scale / v_scale (ignored otherwise).  The plan keeps the pointers:
 * every buffer must stay allocated, at the same address and with the same
 * memory type (page-locked or not) until pa_decode_step_plan_destroy.  The
 * plan owns only host memory.  Errors: as pa_decode_step_host;
 * PA_ERR_OOM if the plan itself cannot be allocated.
 *
 * pa_decode_step_plan_run enqueues one step exactly as pa_decode_step_host
 * would with the same arguments: max_seq_len <= max_seq_len_cap and
 * num_pairs <= max_copy_pairs (else PA_ERR_INVALID_ARG, nothing enqueued).
 * The host buffers are read when the stream reaches the step, so fill them
 * (pa_alloc_step, the new rows) before the call and leave them unchanged
 * until the stream has passed it.
 * ---------------------------------------------------------------------- */
typedef struct pa_decode_step_plan pa_decode_step_plan;

int pa_decode_step_plan_create(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                               const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                               const int32_t *copy_pairs_host, int max_copy_pairs, void *k_cache, void *v_cache,
                               int batch, int max_seq_len_cap, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int64_t num_blocks, float scale, int partition_tokens, int num_chunks,
                               void *staging, size_t staging_bytes, int kv_fp8, float k_scale, float v_scale,
                               pa_decode_step_plan **plan);

int pa_decode_step_plan_run(const pa_decode_step_plan *plan, int max_seq_len, int num_pairs, int32_t *err_flag,
                            void *stream);

/* Makes a prepared step (bf16 pools) decode with pa_decode_shared_prefix:
 * sequences [g*group_size, (g+1)*group_size) share their first
 * prefix_lens_host[g] tokens (int32 [ceil(batch / group_size)], read on every
 * run like the other host inputs), under that call's contract ("PagedAttention
 * & vLLM", Copy-on-write sharing: the shared tokens sit in the same physical
 * blocks in every member's table).  Each run then gives the outputs and pools
 * of pa_decode_shared_prefix with the fused write (k_new, v_new) on the
 * uploaded inputs.  Chunks hold whole groups.  group_size 0 returns the plan
 * to the plain decode.
 * The staging buffer must hold pa_decode_step_staging_size_shared_prefix(...)
 * bytes (same arguments as at create, plus group_size): the prefix lengths
 * and that decode's larger workspace.
 * Errors (the plan is left unchanged): plan NULL, group_size < 0 or > 64,
 * prefix_lens_host NULL with group_size > 0, or staging smaller than that
 * size: PA_ERR_INVALID_ARG; a plan over fp8 pools: PA_ERR_UNSUPPORTED. */
int pa_decode_step_plan_set_shared_prefix(pa_decode_step_plan *plan, const int32_t *prefix_lens_host,
                                          int group_size);

size_t pa_decode_step_staging_size_shared_prefix(int batch, int group_size, int max_blocks_per_seq,
                                                 int max_copy_pairs, int num_q_heads, int num_kv_heads,
                                                 int head_dim, int block_size, int max_seq_len,
                                                 int partition_tokens);

void pa_decode_step_plan_destroy(pa_decode_step_plan *plan);

/* ------------------------------------------------------------------------
 * Decode with library-owned scratch (no workspace argument).
 *
 * The pages have no counterpart: this entry point is a convenience of this
 * library, not a step of PagedAttention.
 *
 * Some callers cannot allocate device memory at the moment they decode:
 * a plugin whose host program owns every device allocation through its own
 * pool and forbids direct cudaMalloc, a caller from another language
 * runtime that only hands over pointers to tensors it already owns, or a
 * latency-critical loop that must not pay for (or synchronise on)
 * cudaMalloc/cudaFree.  For them this call behaves exactly like pa_decode,
 * except that the partial softmax states of the split variant go to a
 * device array owned by the library instead of a caller workspace.
 *
 *  - The array is a file-scope device variable of
 *    PA_DECODE_BUILTIN_SCRATCH_BYTES bytes.  The CUDA driver reserves it
 *    when the library's decode module is loaded on a device, which (with
 *    lazy module loading, the CUDA 12 default) may be this entry point's
 *    first call there; if that reservation fails the call returns
 *    PA_ERR_CUDA.  The device then holds the array until the process exits.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress)
 *    with the current device, so a context that was reset and rebuilt gets
 *    the new address.  Make the first call on a device before any stream
 *    capture, since it may load the module.
 *  - If the split this call would use needs more scratch than
 *    PA_DECODE_BUILTIN_SCRATCH_BYTES (see pa_decode_workspace_size), the
 *    call returns PA_ERR_UNSUPPORTED and launches nothing.
 *  - No cudaMalloc, cudaFree or other allocating routine is called.
 *  - All calls share the one array, and it keeps whatever the last call
 *    wrote.  Nothing in it has to start at zero: each partition's state is
 *    written before it is read within the same call.  Calls queued one
 *    after another on one stream are safe.  Calls whose kernels can overlap on the GPU (different
 *    streams, or several host threads) race on the array; issue them on one
 *    stream.
 * Other arguments, layouts and errors: as pa_decode.
 * ---------------------------------------------------------------------- */
#define PA_DECODE_BUILTIN_SCRATCH_BYTES ((size_t)32 << 20)

int pa_decode_builtin_scratch(float *out, const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads,
                              int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                              float scale, int partition_tokens, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * fp8 KV pools.  "Walk through paged attention end to end" (summary) only
 * says paging composes with KV quantization; the format is this library's:
 *
 *   - Each pool holds OCP 8-bit E4M3 codes (no infinities, S.1111.111 is NaN,
 *     largest finite 448), 1 byte per value, same [num_blocks, num_kv_heads,
 *     block_size, head_dim] layout as the bf16 pools.
 *   - One scale per pool (k_scale, v_scale > 0): a code c stands for
 *     E4M3_value(c) * scale.
 *   - Writing quantises: c = E4M3(x * inv), x the bf16 input widened to fp32,
 *     inv = 1.0f / scale (fp32 division), the product an fp32 multiply,
 *     rounded to nearest with ties to even and saturated to +-448.
 *   - Decode computes exactly the pa_decode result on the dequantised rows.
 *     It runs its mma in f16: q is rescaled by a power of two so its largest
 *     entry lies in [2^13, 2^14); entries more than 2^37 below that largest
 *     one are flushed to zero.
 *
 * Entry points mirror their bf16 counterparts; copy and swap move bytes.
 * ---------------------------------------------------------------------- */

/* dst[i] = E4M3(bf16 src[i] * (1/scale)); num_values a multiple of 8;
 * src 16-byte aligned, dst 8-byte aligned (device memory). */
int pa_quantize_fp8(const void *src, void *dst, int64_t num_values, float scale, void *stream);

int pa_reshape_and_cache_fp8(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                             const int32_t *slot_mapping, int num_tokens, int64_t num_blocks, int num_kv_heads,
                             int block_size, int head_dim, float k_scale, float v_scale, int32_t *err_flag,
                             void *stream);

int pa_copy_blocks_fp8(void *k_cache, void *v_cache, const int32_t *pairs, int num_pairs, int64_t num_blocks,
                       int num_kv_heads, int block_size, int head_dim, int32_t *err_flag, void *stream);

int pa_swap_blocks_fp8(void *dst_k_cache, void *dst_v_cache, int64_t dst_num_blocks, const void *src_k_cache,
                       const void *src_v_cache, int64_t src_num_blocks, const int32_t *pairs, int num_pairs,
                       int num_kv_heads, int block_size, int head_dim, int32_t *err_flag, void *stream);

/* pa_decode over fp8 pools (same workspace size as pa_decode). */
int pa_decode_fp8(float *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int batch,
                  int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                  int64_t num_blocks, float scale, float k_scale, float v_scale, int partition_tokens,
                  void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream);

/* pa_decode_append over fp8 pools: the bf16 new token is quantised as it is written. */
int pa_decode_append_fp8(float *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
                         void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                         float k_scale, float v_scale, int partition_tokens, void *workspace,
                         size_t workspace_bytes, int32_t *err_flag, void *stream);

/* ------------------------------------------------------------------------
 * Host block allocator (owns host memory only; not thread-safe).
 *
 * append  : the token at position n of a sequence goes to logical block
 *           n / block_size, row n % block_size; a fresh block is taken from
 *           the free pool when n % block_size == 0 ("Walk through paged
 *           attention end to end", append step; "What is PagedAttention",
 *           BlockTable.append_token).  Writing into a block whose refcount
 *           is above one first moves the sequence to a fresh copy and
 *           reports the (src, dst) pair the caller must pass to
 *           pa_copy_blocks before the cache write ("PagedAttention & vLLM",
 *           Copy-on-write sharing).  The last owner writes in place.
 * fork    : the child references every block of the parent, the partially
 *           filled last one included; each refcount grows by one.
 * free    : refcounts drop; blocks that reach zero return to the pool at
 *           once, no compaction ("What is PagedAttention", chat workload
 *           example).
 * On PA_ERR_OOM the allocator state is unchanged.
 * ---------------------------------------------------------------------- */
typedef struct pa_allocator pa_allocator;

/* Pool of num_blocks blocks handed out in id order 0, 1, 2, ...
 * block_size must be one the kernels address (8, 16, 32 or 64; else
 * PA_ERR_UNSUPPORTED), and every slot id must fit int32:
 * num_blocks * block_size <= INT32_MAX (else PA_ERR_INVALID_ARG). */
int pa_alloc_create(int num_blocks, int block_size, pa_allocator **out);
/* Same, but fresh blocks are handed out in the order order[0], order[1], ...
 * (order must be a permutation of 0..num_blocks-1; host memory, copied). */
int pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t *order,
                            pa_allocator **out);
void pa_alloc_destroy(pa_allocator *alloc);

int pa_seq_create(pa_allocator *alloc, int *seq_id);
/* Append one token.  *slot_out = slot of the new token; (*cow_src, *cow_dst)
 * = the block copy required first, or (-1, -1).  cow_* may be NULL only if
 * the caller knows no copy can be needed (no forks). */
int pa_seq_append(pa_allocator *alloc, int seq_id, int32_t *slot_out, int32_t *cow_src,
                  int32_t *cow_dst);
/* Append one token to each of seq_ids[0..n) in order (a decode step).
 * slots_out[i] receives the slot of seq_ids[i]; cow_pairs_out (capacity n
 * pairs, int32 [n,2]) receives the required copies, *n_cow their count.
 * All-or-nothing: on PA_ERR_OOM nothing changed. */
int pa_seq_append_batch(pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *slots_out,
                        int32_t *cow_pairs_out, int *n_cow);
int pa_seq_fork(pa_allocator *alloc, int parent_id, int *child_id);
int pa_seq_free(pa_allocator *alloc, int seq_id);
/* Copy a sequence's block table into out[0..cap); *n_blocks and *n_tokens
 * receive its sizes.  PA_ERR_INVALID_ARG if cap < *n_blocks. */
int pa_seq_block_table(const pa_allocator *alloc, int seq_id, int32_t *out, int cap,
                       int *n_blocks, int *n_tokens);
/* Export tables of seq_ids[0..n) as a padded int32 [n, max_blocks] array
 * (unused entries = pad) plus int32 seq_lens[n]; host memory. */
int pa_alloc_export(const pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *tables,
                    int max_blocks, int32_t pad, int32_t *seq_lens);
/* The host side of one decode step in one call: pa_seq_append_batch on
 * seq_ids[0..n) (slots are not reported: the fused decode derives each new
 * token's slot from the table), then pa_alloc_export of the same sequences
 * into tables [n, max_blocks] / seq_lens [n].  cow_pairs_out (capacity n
 * pairs) receives the copies to apply before the decode, *n_cow their count,
 * *max_seq_len the longest length after the append.  All-or-nothing: on
 * PA_ERR_OOM, or PA_ERR_INVALID_ARG because a table would outgrow
 * max_blocks, the allocator is unchanged (the output arrays may have been
 * written).  Host memory throughout. */
int pa_alloc_step(pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *tables, int max_blocks,
                  int32_t pad, int32_t *seq_lens, int32_t *cow_pairs_out, int *n_cow, int *max_seq_len);
int pa_alloc_num_free(const pa_allocator *alloc);
/* Host-side check of decode inputs held in host memory, a debugging aid
 * (the kernels bounds-check the same things and report them through
 * err_flag).  For every sequence b: 0 <= seq_lens[b] <= max_blocks *
 * block_size, and the first ceil(seq_lens[b] / block_size) entries of row b
 * of tables [batch, max_blocks] are block ids in [0, num_blocks), none
 * repeated within the row (rows may share blocks with each other: forks).
 * Entries past those are not read.  Returns PA_OK with *bad_seq =
 * *bad_entry = -1, or PA_ERR_BAD_INDEX with the first offending sequence in
 * *bad_seq and table entry in *bad_entry (-1 when the length itself is out
 * of range).  Bad arguments: PA_ERR_INVALID_ARG. */
int pa_validate_tables(const int32_t *tables, int batch, int max_blocks, const int32_t *seq_lens,
                       int64_t num_blocks, int block_size, int *bad_seq, int *bad_entry);
/* Reference count of a block (0 = free), or -1 for an id out of range. */
int pa_block_refcount(const pa_allocator *alloc, int32_t block);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
