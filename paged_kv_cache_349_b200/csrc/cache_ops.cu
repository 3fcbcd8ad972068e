// Cache write (slot mapping) and copy-on-write block copy.
//
// Both are pure data movement and HBM-bound: 16-byte vector loads and
// stores, several in flight per thread, grids sized from the work.
#include "pa_common.cuh"

namespace pa {
namespace {

// One thread moves one 16-byte chunk of one (token, kv head) row of K and of V
// to slot_mapping[token] ("Walk through paged attention end to end", append
// step: write_kv_to_pool(last_block, offset)).
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, uint4 *__restrict__ k_cache,
    uint4 *__restrict__ v_cache, const int32_t *__restrict__ slot_mapping, int num_tokens,
    int64_t num_slots, int num_kv_heads, int block_size, int chunks_per_row,
    int32_t *__restrict__ err_flag) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_token = (int64_t)num_kv_heads * chunks_per_row;
    if (idx >= (int64_t)num_tokens * per_token) return;
    const int t = (int)(idx / per_token);
    const int rem = (int)(idx - (int64_t)t * per_token);
    const int h = rem / chunks_per_row;
    const int c = rem - h * chunks_per_row;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot == -1) return;
    if (slot < 0 || slot >= num_slots) {
        if (rem == 0) raise_flag(err_flag, PA_FLAG_BAD_SLOT);
        return;
    }
    const int64_t blk = slot / block_size;
    const int64_t row = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + row) * chunks_per_row + c;
    const uint4 kv = __ldg(k_new + idx);
    const uint4 vv = __ldg(v_new + idx);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
}

// fp8 pools: one thread quantises one 8-value chunk of one (token, kv head) row
// of K and of V into the slot: code = E4M3(x * (1/scale)), nearest even,
// saturating (the library's fp8 format; the pages do not fix one).
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new, uint2 *__restrict__ k_cache,
    uint2 *__restrict__ v_cache, const int32_t *__restrict__ slot_mapping, int num_tokens, int64_t num_slots,
    int num_kv_heads, int block_size, int chunks_per_row, float k_inv_scale, float v_inv_scale,
    int32_t *__restrict__ err_flag) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_token = (int64_t)num_kv_heads * chunks_per_row;
    if (idx >= (int64_t)num_tokens * per_token) return;
    const int t = (int)(idx / per_token);
    const int rem = (int)(idx - (int64_t)t * per_token);
    const int h = rem / chunks_per_row;
    const int c = rem - h * chunks_per_row;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot == -1) return;
    if (slot < 0 || slot >= num_slots) {
        if (rem == 0) raise_flag(err_flag, PA_FLAG_BAD_SLOT);
        return;
    }
    const int64_t blk = slot / block_size;
    const int64_t row = slot - blk * block_size;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + row) * chunks_per_row + c;
    k_cache[dst] = bf16x8_to_e4m3x8(__ldg(k_new + idx), k_inv_scale);
    v_cache[dst] = bf16x8_to_e4m3x8(__ldg(v_new + idx), v_inv_scale);
}

// Bulk conversion of bf16 values to E4M3 codes (8 values per thread).
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const uint4 *__restrict__ src, uint2 *__restrict__ dst,
                                                           int64_t chunks, float inv_scale) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = bf16x8_to_e4m3x8(__ldcs(src + i), inv_scale);
}

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;  // 16-byte chunks in flight per thread

// grid.x: pair * groups_per_block + chunk group, grid.y: 0 = K pool, 1 = V pool.
// Copies block src of the source pools to block dst of the destination pools
// ("PagedAttention & vLLM", Copy-on-write sharing, when both are the same pools;
// "What is PagedAttention...", swapping to CPU memory, when one side is pinned
// host memory mapped into the device address space).
__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(
    uint4 *__restrict__ dst_k, uint4 *__restrict__ dst_v, const uint4 *src_k, const uint4 *src_v,
    const int32_t *__restrict__ pairs, int64_t src_blocks, int64_t dst_blocks, int64_t chunks_per_block,
    int groups_per_block, int flag_bit, int32_t *__restrict__ err_flag) {
    const int pair = blockIdx.x / groups_per_block;
    const int group = blockIdx.x - pair * groups_per_block;
    const int64_t src = __ldg(pairs + 2 * pair);
    const int64_t dst = __ldg(pairs + 2 * pair + 1);
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (group == 0 && blockIdx.y == 0 && threadIdx.x == 0) raise_flag(err_flag, flag_bit);
        return;
    }
    const uint4 *from = (blockIdx.y == 0 ? src_k : src_v) + src * chunks_per_block;
    uint4 *to = (blockIdx.y == 0 ? dst_k : dst_v) + dst * chunks_per_block;
    const int64_t base = (int64_t)group * (kCopyThreads * kCopyUnroll) + threadIdx.x;
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = base + (int64_t)u * kCopyThreads;
        if (i < chunks_per_block) buf[u] = __ldcs(from + i);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = base + (int64_t)u * kCopyThreads;
        if (i < chunks_per_block) __stcs(to + i, buf[u]);
    }
}

int launch_block_copy(void *dst_k, void *dst_v, const void *src_k, const void *src_v, const int32_t *pairs,
                      int num_pairs, int64_t src_blocks, int64_t dst_blocks, int num_kv_heads, int block_size,
                      int head_dim, int elem_bytes, int flag_bit, int32_t *err_flag, void *stream) {
    const int64_t chunks = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes / 16;
    const int64_t per_cta = kCopyThreads * kCopyUnroll;
    const int64_t groups = (chunks + per_cta - 1) / per_cta;
    if (groups * num_pairs > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
    dim3 grid((unsigned)(groups * num_pairs), 2);
    copy_blocks_kernel<<<grid, kCopyThreads, 0, (cudaStream_t)stream>>>(
        (uint4 *)dst_k, (uint4 *)dst_v, (const uint4 *)src_k, (const uint4 *)src_v, pairs, src_blocks,
        dst_blocks, chunks, (int)groups, flag_bit, err_flag);
    count_launch();
    return launch_status();
}

}  // namespace
}  // namespace pa

extern "C" {

int pa_reshape_and_cache(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                         const int32_t *slot_mapping, int num_tokens, int64_t num_blocks,
                         int num_kv_heads, int block_size, int head_dim, int32_t *err_flag,
                         void *stream) {
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pa::supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(k_new) || !pa::aligned16(v_new) || !pa::aligned16(k_cache) ||
        !pa::aligned16(v_cache))
        return PA_ERR_INVALID_ARG;
    const int chunks = head_dim / 8;
    const int64_t total = (int64_t)num_tokens * num_kv_heads * chunks;
    const int threads = 256;
    const int64_t grid = (total + threads - 1) / threads;
    if (grid > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
    pa::reshape_and_cache_kernel<<<(unsigned)grid, threads, 0, (cudaStream_t)stream>>>(
        (const uint4 *)k_new, (const uint4 *)v_new, (uint4 *)k_cache, (uint4 *)v_cache,
        slot_mapping, num_tokens, num_blocks * block_size, num_kv_heads, block_size, chunks,
        err_flag);
    pa::count_launch();
    return pa::launch_status();
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *pairs, int num_pairs,
                   int64_t num_blocks, int num_kv_heads, int block_size, int head_dim,
                   int32_t *err_flag, void *stream) {
    if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pa::supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !pairs) return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(k_cache) || !pa::aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    return pa::launch_block_copy(k_cache, v_cache, k_cache, v_cache, pairs, num_pairs, num_blocks, num_blocks,
                                 num_kv_heads, block_size, head_dim, 2, PA_FLAG_BAD_PAIR, err_flag, stream);
}

int pa_swap_blocks(void *dst_k_cache, void *dst_v_cache, int64_t dst_num_blocks, const void *src_k_cache,
                   const void *src_v_cache, int64_t src_num_blocks, const int32_t *pairs, int num_pairs,
                   int num_kv_heads, int block_size, int head_dim, int32_t *err_flag, void *stream) {
    if (num_pairs < 0 || dst_num_blocks <= 0 || src_num_blocks <= 0 || num_kv_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pa::supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !pairs) return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(dst_k_cache) || !pa::aligned16(dst_v_cache) || !pa::aligned16(src_k_cache) ||
        !pa::aligned16(src_v_cache))
        return PA_ERR_INVALID_ARG;
    // Each side must be reachable from the device: device memory, or host memory
    // that is page-locked (pageable host memory is an argument error, not a fault).
    void *dk = nullptr, *dv = nullptr, *sk = nullptr, *sv = nullptr;
    int rc = pa::device_address(dst_k_cache, &dk);
    if (rc == PA_OK) rc = pa::device_address(dst_v_cache, &dv);
    if (rc == PA_OK) rc = pa::device_address(src_k_cache, &sk);
    if (rc == PA_OK) rc = pa::device_address(src_v_cache, &sv);
    void *pp = nullptr;
    if (rc == PA_OK) rc = pa::device_address(pairs, &pp);
    if (rc != PA_OK) return rc;
    return pa::launch_block_copy(dk, dv, sk, sv, static_cast<const int32_t *>(pp), num_pairs, src_num_blocks,
                                 dst_num_blocks, num_kv_heads, block_size, head_dim, 2, PA_FLAG_BAD_PAIR,
                                 err_flag, stream);
}

int pa_reshape_and_cache_fp8(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                             const int32_t *slot_mapping, int num_tokens, int64_t num_blocks, int num_kv_heads,
                             int block_size, int head_dim, float k_scale, float v_scale, int32_t *err_flag,
                             void *stream) {
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pa::supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (!(k_scale > 0.f && v_scale > 0.f && k_scale < 3.0e38f && v_scale < 3.0e38f)) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(k_new) || !pa::aligned16(v_new) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache))
        return PA_ERR_INVALID_ARG;
    const int chunks = head_dim / 8;
    const int64_t total = (int64_t)num_tokens * num_kv_heads * chunks;
    const int64_t grid = (total + 255) / 256;
    if (grid > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
    pa::reshape_and_cache_fp8_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(
        (const uint4 *)k_new, (const uint4 *)v_new, (uint2 *)k_cache, (uint2 *)v_cache, slot_mapping, num_tokens,
        num_blocks * block_size, num_kv_heads, block_size, chunks, 1.0f / k_scale, 1.0f / v_scale, err_flag);
    pa::count_launch();
    return pa::launch_status();
}

int pa_quantize_fp8(const void *src, void *dst, int64_t num_values, float scale, void *stream) {
    if (num_values < 0 || num_values % 8 || !(scale > 0.f && scale < 3.0e38f)) return PA_ERR_INVALID_ARG;
    if (num_values == 0) return PA_OK;
    if (!src || !dst || !pa::aligned16(src) || (reinterpret_cast<uintptr_t>(dst) & 7u)) return PA_ERR_INVALID_ARG;
    const int64_t chunks = num_values / 8;
    const int64_t want = (chunks + 255) / 256;
    const unsigned grid = (unsigned)(want < 148LL * 16 ? want : 148LL * 16);
    pa::quantize_fp8_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>((const uint4 *)src, (uint2 *)dst, chunks,
                                                                     1.0f / scale);
    pa::count_launch();
    return pa::launch_status();
}

int pa_copy_blocks_fp8(void *k_cache, void *v_cache, const int32_t *pairs, int num_pairs, int64_t num_blocks,
                       int num_kv_heads, int block_size, int head_dim, int32_t *err_flag, void *stream) {
    if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pa::supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !pairs) return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(k_cache) || !pa::aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    return pa::launch_block_copy(k_cache, v_cache, k_cache, v_cache, pairs, num_pairs, num_blocks, num_blocks,
                                 num_kv_heads, block_size, head_dim, 1, PA_FLAG_BAD_PAIR, err_flag, stream);
}

int pa_swap_blocks_fp8(void *dst_k_cache, void *dst_v_cache, int64_t dst_num_blocks, const void *src_k_cache,
                       const void *src_v_cache, int64_t src_num_blocks, const int32_t *pairs, int num_pairs,
                       int num_kv_heads, int block_size, int head_dim, int32_t *err_flag, void *stream) {
    if (num_pairs < 0 || dst_num_blocks <= 0 || src_num_blocks <= 0 || num_kv_heads <= 0)
        return PA_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (!pa::supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !pairs) return PA_ERR_INVALID_ARG;
    if (!pa::aligned16(dst_k_cache) || !pa::aligned16(dst_v_cache) || !pa::aligned16(src_k_cache) ||
        !pa::aligned16(src_v_cache))
        return PA_ERR_INVALID_ARG;
    // Each side must be reachable from the device: device memory, or host memory
    // that is page-locked (pageable host memory is an argument error, not a fault).
    void *dk = nullptr, *dv = nullptr, *sk = nullptr, *sv = nullptr;
    int rc = pa::device_address(dst_k_cache, &dk);
    if (rc == PA_OK) rc = pa::device_address(dst_v_cache, &dv);
    if (rc == PA_OK) rc = pa::device_address(src_k_cache, &sk);
    if (rc == PA_OK) rc = pa::device_address(src_v_cache, &sv);
    void *pp = nullptr;
    if (rc == PA_OK) rc = pa::device_address(pairs, &pp);
    if (rc != PA_OK) return rc;
    return pa::launch_block_copy(dk, dv, sk, sv, static_cast<const int32_t *>(pp), num_pairs, src_num_blocks,
                                 dst_num_blocks, num_kv_heads, block_size, head_dim, 1, PA_FLAG_BAD_PAIR,
                                 err_flag, stream);
}

}  // extern "C"
