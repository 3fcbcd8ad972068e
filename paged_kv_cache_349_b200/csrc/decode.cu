// Host side of the paged decode: tensor maps of the pools, the choice of
// partitioning, the split workspace layout, the decode launches (the device
// code is in decode_kernels.cuh) and the C entry points.
#include <mutex>

#include "decode_kernels.cuh"

namespace pa {
namespace {

// ---------------------------------------------------------------------------
// Host helpers
// ---------------------------------------------------------------------------

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

struct MapKey {
    const void *ptr;
    uint64_t rows;
    int head_dim;
    int box_rows;
    bool fp8;
    int device;
};

// Small cache of pool tensor maps: a decode step re-uses the same pools.
// bf16 pools: 64-column boxes with the 128-byte swizzle; fp8 pools: one box
// spanning the row, 128-byte swizzled for head_dim 128 and unswizzled for 64.
bool pool_tensor_map(const void *pool, uint64_t rows, int head_dim, int box_rows, bool fp8, CUtensorMap *out) {
    static std::mutex mu;
    static MapKey keys[8];
    static CUtensorMap maps[8];
    static int used = 0, next = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
        if (keys[i].ptr == pool && keys[i].rows == rows && keys[i].head_dim == head_dim &&
            keys[i].box_rows == box_rows && keys[i].fp8 == fp8 && keys[i].device == dev) {
            *out = maps[i];
            return true;
        }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    CUtensorMap m;
    cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)head_dim * (fp8 ? 1 : 2)};
    cuuint32_t box[2] = {(cuuint32_t)(fp8 ? head_dim : 64), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void *>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     (fp8 && head_dim != 128) ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    const int slot = used < 8 ? used++ : (next++ & 7);
    keys[slot] = MapKey{pool, rows, head_dim, box_rows, fp8, dev};
    maps[slot] = m;
    *out = m;
    return true;
}

// Resolve the partition size: -1 = single pass, else tokens per partition.
//
// Default (measured on B200, decode of bf16 d=128 pools): one CTA per
// (sequence, kv head) is best when there are enough of them to fill the GPU
// several times over and no sequence can be much longer than the rest;
// otherwise 1024-token partitions keep the CTAs short enough that the last
// wave does not leave SMs idle (long-tailed length mixes, few sequences).
int resolve_partition(int batch, int num_kv_heads, int block_size, int max_seq_len, int requested) {
    (void)block_size;
    if (requested < 0) return -1;
    if (requested > 0) return requested >= max_seq_len ? -1 : requested;
    constexpr int kDefaultPartition = 1024;
    if (max_seq_len <= kDefaultPartition) return -1;
    const int64_t units = (int64_t)batch * num_kv_heads;
    const int64_t resident = 3LL * device_sm_count();  // CTAs resident at once
    if (units >= 2 * resident && max_seq_len < 3 * kDefaultPartition) return -1;
    return kDefaultPartition;
}

template <int HEAD_DIM, bool SPLIT, bool APPEND, bool FP8, bool PREFIX>
int launch_decode(const CUtensorMap &km, const CUtensorMap &vm, const DecodeParams &p, int grid_z,
                  cudaStream_t stream) {
    using C = Cfg<HEAD_DIM, FP8>;
    auto kern = paged_decode_kernel<HEAD_DIM, SPLIT, APPEND, FP8, PREFIX>;
    {
        // The shared-memory opt-in belongs to the kernel as loaded on one device:
        // set it once per device.
        static std::mutex mu;
        static bool done[64] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
                cudaSuccess)
                return PA_ERR_CUDA;
            done[dev] = true;
        }
    }
    // B (or the item index) is the slowest grid dimension: the kv heads and
    // partitions of one sequence -- and with prefix groups the shared items and
    // then the members of a group -- are launched next to each other, so rows
    // several CTAs read (shared prefix blocks) are still in L2 when the later
    // ones reach them.
    dim3 grid((unsigned)p.num_parts, (unsigned)p.num_kv_heads, (unsigned)grid_z);
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(km, vm, p);
    count_launch();
    int st = launch_status();
    if (st != PA_OK || !SPLIT) return st;
    // The reduce, one CTA per (query head, sequence), launched as a programmatic
    // dependent: it is scheduled while the decode's last wave runs and waits
    // (griddepcontrol.wait) for the decode grid's results.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_q_heads, (unsigned)p.batch);
    cfg.blockDim = dim3(kReduceThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, lse_reduce_kernel<HEAD_DIM, PREFIX>, p);
    count_launch();
    return e == cudaSuccess ? launch_status() : PA_ERR_CUDA;
}

// Split workspace: partial states part_o [B, Hq, slots, d], then part_ml
// [B, Hq, slots, 2] (fp32) 256-byte aligned.
struct SplitLayout {
    size_t o, ml, total;
};

SplitLayout split_layout(int64_t batch, int num_q_heads, int head_dim, int64_t slots) {
    const int64_t rows = batch * num_q_heads * slots;
    SplitLayout l{};
    l.o = 0;
    l.ml = (size_t)((rows * head_dim * 4 + 255) / 256 * 256);
    l.total = l.ml + (size_t)(rows * 2 * 4);
    return l;
}

// Partial-state slots per row: one per partition, twice that with prefix groups
// (the shared items' partitions, then the sequence's own).  pt = -1: one each.
int64_t split_slots(int max_seq_len, int pt, bool prefix) {
    const int64_t parts = pt > 0 ? ((int64_t)max_seq_len + pt - 1) / pt : 1;
    return prefix ? 2 * parts : parts;
}

}  // namespace

// Scratch for pa_decode_builtin_scratch, for callers that cannot allocate a
// workspace.  In host code the name is only a stand-in: kernels receive the
// device address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_builtin_scratch[PA_DECODE_BUILTIN_SCRATCH_BYTES];

// Device address of the scratch array in the current device's context.  It is
// looked up on every call (a host-side lookup once the module is loaded), so a
// context that was torn down and rebuilt never gets a stale address.
int builtin_scratch_address(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_builtin_scratch) != cudaSuccess || p == nullptr) return PA_ERR_CUDA;
    *out = p;
    return PA_OK;
}

template <bool SPLIT, bool APPEND, bool FP8, bool PREFIX = false>
int launch_decode_d(int head_dim, const CUtensorMap &km, const CUtensorMap &vm, const DecodeParams &p, int grid_z,
                    cudaStream_t s) {
    return head_dim == 128 ? launch_decode<128, SPLIT, APPEND, FP8, PREFIX>(km, vm, p, grid_z, s)
                           : launch_decode<64, SPLIT, APPEND, FP8, PREFIX>(km, vm, p, grid_z, s);
}

// Shared body of every decode entry point (k_new == nullptr: no cache write;
// fp8: E4M3 pools dequantised with k_scale / v_scale; prefix_lens != nullptr:
// groups of group_size sequences read their shared prefix once).
int decode_impl(float *out, const void *q, const void *k_new, const void *v_new, const void *k_cache,
                const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                int head_dim, int block_size, int64_t num_blocks, float scale, int partition_tokens,
                void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream, bool fp8,
                float k_scale, float v_scale, const int32_t *prefix_lens, int group_size) {
    const bool append = k_new != nullptr;
    const bool prefix = prefix_lens != nullptr;
    if (fp8 && !(k_scale > 0.f && v_scale > 0.f && k_scale < 3.0e38f && v_scale < 3.0e38f))
        return PA_ERR_INVALID_ARG;
    if (batch < 0 || max_seq_len < 0 || num_blocks <= 0 || max_blocks_per_seq < 0)
        return PA_ERR_INVALID_ARG;
    if (prefix && (group_size < 1 || group_size > kMaxGroupSize)) return PA_ERR_INVALID_ARG;
    if (!supported_shape(num_q_heads, num_kv_heads, head_dim, block_size)) return PA_ERR_UNSUPPORTED;
    if (batch == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return PA_ERR_INVALID_ARG;
    if (append && (!v_new || !aligned16(k_new) || !aligned16(v_new))) return PA_ERR_INVALID_ARG;
    if (partition_tokens > 0 && partition_tokens % block_size) return PA_ERR_INVALID_ARG;
    if (batch > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    const uint64_t rows = (uint64_t)num_blocks * (uint64_t)num_kv_heads * (uint64_t)block_size;
    if (rows >= (1ull << 31)) return PA_ERR_UNSUPPORTED;  // TMA row coordinate is int32

    DecodeParams p{};
    p.out = out;
    p.q = static_cast<const uint16_t *>(q);
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err_flag = err_flag;
    p.num_blocks = num_blocks;
    p.max_blocks = max_blocks_per_seq;
    p.max_seq_len = max_seq_len;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = num_q_heads / num_kv_heads;
    p.block_size = block_size;
    p.scale_log2 = scale * kLog2e;
    p.k_new = static_cast<const uint16_t *>(k_new);
    p.v_new = static_cast<const uint16_t *>(v_new);
    p.k_pool = static_cast<uint16_t *>(const_cast<void *>(k_cache));
    p.v_pool = static_cast<uint16_t *>(const_cast<void *>(v_cache));
    p.k_scale = fp8 ? k_scale : 1.f;
    p.v_scale = fp8 ? v_scale : 1.f;
    p.k_inv_scale = fp8 ? 1.0f / k_scale : 1.f;
    p.v_inv_scale = fp8 ? 1.0f / v_scale : 1.f;
    p.batch = batch;

    int pt = max_seq_len > 0
                 ? resolve_partition(batch, num_kv_heads, block_size, max_seq_len, partition_tokens)
                 : -1;
    // With prefix groups every call merges partial states (the shared items'
    // and each sequence's own); "one pass" then means one item of each kind.
    if (prefix && max_seq_len > 0 && pt <= 0) pt = max_seq_len;
    const bool split = pt > 0;
    int grid_z = batch;
    if (split) {
        const size_t need = prefix ? pa_decode_shared_prefix_workspace_size(batch, group_size, num_q_heads,
                                                                            num_kv_heads, head_dim, block_size,
                                                                            max_seq_len, partition_tokens)
                                   : pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                              block_size, max_seq_len, partition_tokens);
        if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_INVALID_ARG;
        p.part_tokens = pt;
        p.num_parts = (max_seq_len + pt - 1) / pt;
        const int64_t slots = split_slots(max_seq_len, pt, prefix);
        p.num_slots = (int)slots;
        const SplitLayout l = split_layout(batch, num_q_heads, head_dim, slots);
        char *ws = static_cast<char *>(workspace);
        p.part_o = reinterpret_cast<float *>(ws + l.o);
        p.part_ml = reinterpret_cast<float *>(ws + l.ml);
        if (prefix) {
            p.prefix_lens = prefix_lens;
            p.group_size = group_size;
            p.num_groups = (batch + group_size - 1) / group_size;
            p.members_per_item = 8 / p.group;
            p.items_per_group = (group_size + p.members_per_item - 1) / p.members_per_item;
            const int64_t z = (int64_t)p.num_groups * p.items_per_group + batch;
            if (z > 65535) return PA_ERR_UNSUPPORTED;
            grid_z = (int)z;
        }
        if (p.num_parts > 65535) return PA_ERR_UNSUPPORTED;
    } else {
        p.part_tokens = max_seq_len > 0 ? max_seq_len : 1;
        p.num_parts = 1;
        p.num_slots = 1;
    }

    CUtensorMap km, vm;
    const int box_rows = block_size < kTileTokens ? block_size : kTileTokens;
    if (!pool_tensor_map(k_cache, rows, head_dim, box_rows, fp8, &km) ||
        !pool_tensor_map(v_cache, rows, head_dim, box_rows, fp8, &vm))
        return PA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (prefix && split) {
        if (fp8)
            return append ? launch_decode_d<true, true, true, true>(head_dim, km, vm, p, grid_z, s)
                          : launch_decode_d<true, false, true, true>(head_dim, km, vm, p, grid_z, s);
        return append ? launch_decode_d<true, true, false, true>(head_dim, km, vm, p, grid_z, s)
                      : launch_decode_d<true, false, false, true>(head_dim, km, vm, p, grid_z, s);
    }
    if (!split) {
        if (fp8)
            return append ? launch_decode_d<false, true, true>(head_dim, km, vm, p, grid_z, s)
                          : launch_decode_d<false, false, true>(head_dim, km, vm, p, grid_z, s);
        return append ? launch_decode_d<false, true, false>(head_dim, km, vm, p, grid_z, s)
                      : launch_decode_d<false, false, false>(head_dim, km, vm, p, grid_z, s);
    }
    if (fp8)
        return append ? launch_decode_d<true, true, true>(head_dim, km, vm, p, grid_z, s)
                      : launch_decode_d<true, false, true>(head_dim, km, vm, p, grid_z, s);
    return append ? launch_decode_d<true, true, false>(head_dim, km, vm, p, grid_z, s)
                  : launch_decode_d<true, false, false>(head_dim, km, vm, p, grid_z, s);
}

}  // namespace pa

extern "C" {

int pa_decode_partition_tokens(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_seq_len, int partition_tokens) {
    (void)num_q_heads;
    (void)head_dim;
    if (batch <= 0 || max_seq_len <= 0) return -1;
    return pa::resolve_partition(batch, num_kv_heads, block_size, max_seq_len, partition_tokens);
}

size_t pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                int block_size, int max_seq_len, int partition_tokens) {
    if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_seq_len <= 0) return 0;
    const int pt = pa::resolve_partition(batch, num_kv_heads, block_size, max_seq_len, partition_tokens);
    if (pt <= 0) return 0;
    return pa::split_layout(batch, num_q_heads, head_dim, pa::split_slots(max_seq_len, pt, false)).total;
}

size_t pa_decode_shared_prefix_workspace_size(int batch, int group_size, int num_q_heads, int num_kv_heads,
                                              int head_dim, int block_size, int max_seq_len,
                                              int partition_tokens) {
    if (batch <= 0 || group_size <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_seq_len <= 0) return 0;
    int pt = pa::resolve_partition(batch, num_kv_heads, block_size, max_seq_len, partition_tokens);
    if (pt <= 0) pt = max_seq_len;
    return pa::split_layout(batch, num_q_heads, head_dim, pa::split_slots(max_seq_len, pt, true)).total;
}

int pa_decode(float *out, const void *q, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens,
              int batch, int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, int64_t num_blocks, float scale, int partition_tokens,
              void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream) {
    return pa::decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           seq_lens, batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size,
                           num_blocks, scale, partition_tokens, workspace, workspace_bytes, err_flag, stream,
                           false, 1.f, 1.f, nullptr, 0);
}

int pa_decode_append(float *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
                     void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                     int partition_tokens, void *workspace, size_t workspace_bytes, int32_t *err_flag,
                     void *stream) {
    if (batch > 0 && (!k_new || !v_new)) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           seq_lens, batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size,
                           num_blocks, scale, partition_tokens, workspace, workspace_bytes, err_flag, stream,
                           false, 1.f, 1.f, nullptr, 0);
}

int pa_decode_fp8(float *out, const void *q, const void *k_cache, const void *v_cache,
                  const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int batch,
                  int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                  int64_t num_blocks, float scale, float k_scale, float v_scale, int partition_tokens,
                  void *workspace, size_t workspace_bytes, int32_t *err_flag, void *stream) {
    return pa::decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           seq_lens, batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size,
                           num_blocks, scale, partition_tokens, workspace, workspace_bytes, err_flag, stream,
                           true, k_scale, v_scale, nullptr, 0);
}

int pa_decode_append_fp8(float *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
                         void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                         float k_scale, float v_scale, int partition_tokens, void *workspace,
                         size_t workspace_bytes, int32_t *err_flag, void *stream) {
    if (batch > 0 && (!k_new || !v_new)) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           seq_lens, batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size,
                           num_blocks, scale, partition_tokens, workspace, workspace_bytes, err_flag, stream,
                           true, k_scale, v_scale, nullptr, 0);
}

int pa_decode_shared_prefix(float *out, const void *q, const void *k_new, const void *v_new, void *k_cache,
                            void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *seq_lens, const int32_t *prefix_lens, int group_size, int batch,
                            int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int64_t num_blocks, float scale, int partition_tokens, void *workspace,
                            size_t workspace_bytes, int32_t *err_flag, void *stream) {
    if (batch > 0 && (!prefix_lens || (k_new == nullptr) != (v_new == nullptr))) return PA_ERR_INVALID_ARG;
    if (batch > 0 && max_seq_len > 0 && !prefix_lens) return PA_ERR_INVALID_ARG;
    return pa::decode_impl(out, q, k_new, v_new, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                           batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                           partition_tokens, workspace, workspace_bytes, err_flag, stream, false, 1.f, 1.f,
                           batch > 0 ? prefix_lens : nullptr, group_size);
}

int pa_decode_builtin_scratch(float *out, const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *seq_lens, int batch, int max_seq_len, int num_q_heads,
                              int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                              float scale, int partition_tokens, int32_t *err_flag, void *stream) {
    if (batch < 0 || max_seq_len < 0) return PA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    const int st = pa::builtin_scratch_address(&scratch);
    if (st != PA_OK) return st;
    const size_t need = batch > 0 ? pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                             block_size, max_seq_len, partition_tokens)
                                  : 0;
    if (need > PA_DECODE_BUILTIN_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
    return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, batch,
                     max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                     partition_tokens, scratch, PA_DECODE_BUILTIN_SCRATCH_BYTES, err_flag, stream);
}

}  // extern "C"
