/* One decode step of a serving loop through the C ABI, as plain C99: the
 * allocator appends a token to every running sequence, then one call
 * uploads the step's inputs, applies copy-on-write copies, writes the new
 * tokens and decodes, with the output landing in pinned host memory.
 * Compiled and linked by the tests (it is not run: it needs a GPU and
 * buffers set up by the caller). */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>

#include "pa.h"

int decode_one_step(pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *tables_pinned, int max_blocks,
                    int32_t *lens_pinned, int32_t *pairs_pinned, const void *q_pinned, const void *k_new_pinned,
                    const void *v_new_pinned, float *out_pinned, void *k_pool, void *v_pool, int64_t num_blocks,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale, void *staging,
                    size_t staging_bytes, int32_t *err_flag_dev, void *stream) {
    int n_pairs = 0, max_len = 0;
    int st = pa_alloc_step(alloc, seq_ids, n, tables_pinned, max_blocks, -1, lens_pinned, pairs_pinned, &n_pairs,
                           &max_len);
    if (st != PA_OK) {
        fprintf(stderr, "pa_alloc_step: %s\n", pa_status_string(st));
        return st;
    }
    st = pa_decode_step_host(out_pinned, q_pinned, k_new_pinned, v_new_pinned, tables_pinned, max_blocks,
                             lens_pinned, pairs_pinned, n_pairs, n, k_pool, v_pool, n, max_len, num_q_heads,
                             num_kv_heads, head_dim, block_size, num_blocks, scale, /*partition_tokens=*/0,
                             /*num_chunks=*/0, staging, staging_bytes, err_flag_dev, stream);
    if (st != PA_OK) fprintf(stderr, "pa_decode_step_host: %s\n", pa_status_string(st));
    return st;  /* synchronise `stream` before reading out_pinned */
}

int main(void) { return pa_version() > 0 ? 0 : 1; }
