// One decode step from host buffers: upload the step's inputs, apply the
// copy-on-write block copies, run the fused cache write + decode, and copy
// the output back -- all enqueued on one stream by one call.
#include "pa_common.cuh"

namespace pa {
namespace {

constexpr size_t kAlign = 256;

inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Device staging of one step, each section 256-byte aligned.
struct StagingLayout {
    size_t q, k_new, v_new, tables, lens, pairs, out, workspace, workspace_bytes, total;
};

StagingLayout staging_layout(int batch, int max_blocks_per_seq, int max_copy_pairs, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, int max_seq_len,
                             int partition_tokens) {
    StagingLayout l{};
    size_t off = 0;
    l.q = off;
    off += round_up((size_t)batch * num_q_heads * head_dim * 2);
    l.k_new = off;
    off += round_up((size_t)batch * num_kv_heads * head_dim * 2);
    l.v_new = off;
    off += round_up((size_t)batch * num_kv_heads * head_dim * 2);
    l.tables = off;
    off += round_up((size_t)batch * max_blocks_per_seq * 4);
    l.lens = off;
    off += round_up((size_t)batch * 4);
    l.pairs = off;
    off += round_up((size_t)(max_copy_pairs > 0 ? max_copy_pairs : 0) * 8);
    l.out = off;
    off += round_up((size_t)batch * num_q_heads * head_dim * 4);
    l.workspace = off;
    l.workspace_bytes = pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                                 max_seq_len, partition_tokens);
    off += round_up(l.workspace_bytes);
    l.total = off;
    return l;
}

int h2d(void *dst, const void *src, size_t bytes, cudaStream_t s) {
    if (bytes == 0) return PA_OK;
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace
}  // namespace pa

extern "C" {

size_t pa_decode_step_staging_size(int batch, int max_blocks_per_seq, int max_copy_pairs, int num_q_heads,
                                   int num_kv_heads, int head_dim, int block_size, int max_seq_len,
                                   int partition_tokens) {
    if (batch <= 0 || max_blocks_per_seq < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return 0;
    return pa::staging_layout(batch, max_blocks_per_seq, max_copy_pairs, num_q_heads, num_kv_heads, head_dim,
                              block_size, max_seq_len, partition_tokens)
        .total;
}

int pa_decode_step_host(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                        const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                        const int32_t *copy_pairs_host, int num_pairs, int max_copy_pairs, void *k_cache,
                        void *v_cache, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int64_t num_blocks, float scale, int partition_tokens,
                        void *staging, size_t staging_bytes, int32_t *err_flag, void *stream) {
    if (batch < 0 || num_pairs < 0 || max_copy_pairs < 0 || max_blocks_per_seq < 0 || max_seq_len < 0)
        return PA_ERR_INVALID_ARG;
    if (!pa::supported_shape(num_q_heads, num_kv_heads, head_dim, block_size)) return PA_ERR_UNSUPPORTED;
    if (batch == 0) return PA_OK;
    if (!out_host || !q_host || !k_new_host || !v_new_host || !block_tables_host || !seq_lens_host || !staging ||
        !k_cache || !v_cache)
        return PA_ERR_INVALID_ARG;
    if (num_pairs > max_copy_pairs || (num_pairs > 0 && !copy_pairs_host)) return PA_ERR_INVALID_ARG;
    const pa::StagingLayout l = pa::staging_layout(batch, max_blocks_per_seq, max_copy_pairs, num_q_heads,
                                                   num_kv_heads, head_dim, block_size, max_seq_len,
                                                   partition_tokens);
    if (staging_bytes < l.total || (reinterpret_cast<uintptr_t>(staging) & (pa::kAlign - 1)))
        return PA_ERR_INVALID_ARG;
    char *st = static_cast<char *>(staging);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t q_bytes = (size_t)batch * num_q_heads * head_dim * 2;
    const size_t kv_bytes = (size_t)batch * num_kv_heads * head_dim * 2;
    int rc = pa::h2d(st + l.q, q_host, q_bytes, s);
    if (rc == PA_OK) rc = pa::h2d(st + l.k_new, k_new_host, kv_bytes, s);
    if (rc == PA_OK) rc = pa::h2d(st + l.v_new, v_new_host, kv_bytes, s);
    if (rc == PA_OK) rc = pa::h2d(st + l.tables, block_tables_host, (size_t)batch * max_blocks_per_seq * 4, s);
    if (rc == PA_OK) rc = pa::h2d(st + l.lens, seq_lens_host, (size_t)batch * 4, s);
    if (rc == PA_OK) rc = pa::h2d(st + l.pairs, copy_pairs_host, (size_t)num_pairs * 8, s);
    if (rc != PA_OK) return rc;
    if (num_pairs > 0) {
        rc = pa_copy_blocks(k_cache, v_cache, reinterpret_cast<const int32_t *>(st + l.pairs), num_pairs,
                            num_blocks, num_kv_heads, block_size, head_dim, err_flag, stream);
        if (rc != PA_OK) return rc;
    }
    float *out_dev = reinterpret_cast<float *>(st + l.out);
    rc = pa::decode_impl(out_dev, st + l.q, st + l.k_new, st + l.v_new, k_cache, v_cache,
                         reinterpret_cast<const int32_t *>(st + l.tables), max_blocks_per_seq,
                         reinterpret_cast<const int32_t *>(st + l.lens), batch, max_seq_len, num_q_heads,
                         num_kv_heads, head_dim, block_size, num_blocks, scale, partition_tokens,
                         l.workspace_bytes ? st + l.workspace : nullptr, l.workspace_bytes, err_flag, stream,
                         false, 1.f, 1.f);
    if (rc != PA_OK) return rc;
    if (cudaMemcpyAsync(out_host, out_dev, (size_t)batch * num_q_heads * head_dim * 4, cudaMemcpyDeviceToHost,
                        s) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

}  // extern "C"
