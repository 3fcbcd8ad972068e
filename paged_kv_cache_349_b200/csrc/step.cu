// One decode step from host buffers: upload the step's inputs, apply the
// copy-on-write block copies, run the fused cache write + decode, and copy
// the output back -- all enqueued by one call.
//
// A page-locked output buffer is written by the kernels directly; any other
// is staged on the device and copied back.  A large step is cut into chunks
// of whole sequences and pipelined over streams owned by the library: while
// chunk c decodes, chunk c+1 is uploaded (and, for a staged output, chunk c-1
// downloaded).  Chunk decodes alternate between the caller's stream and a
// second compute stream, so one chunk's last wave of CTAs overlaps the next
// chunk's first.  Every side stream is joined back
// into the caller's stream before the call returns, so synchronising that
// stream covers the whole step.
#include <algorithm>
#include <mutex>
#include <new>

#include "pa_common.cuh"

namespace pa {
namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxChunks = 8;
constexpr int kMaxDevices = 64;
// Auto chunking: one chunk per this many bytes crossing the host link, at most
// 4, or 8 in shared-prefix mode.  Enqueueing costs ~10 us of host time per chunk,
// which a short step cannot hide; the shared-prefix decode writes its output at
// each chunk's end, so it gains from more, smaller chunks.  (Measured on B200,
// end to end: the Llama-2-7B-shaped step, 2.6 MB over the link, 230, 213, 208,
// 205 us with 1, 2, 3, 4 chunks; the Llama-3-8B one, 7.5 MB, 0.29 ms with 4
// chunks and 0.31-0.33 with 8; the chat mix in shared-prefix mode 0.46-0.47 ms
// with 4 and 0.43-0.44 with 8.)
constexpr size_t kAutoChunkBytes = (size_t)1 << 19;
constexpr int kAutoMaxChunks = 4;
constexpr int kAutoMaxChunksShared = 8;

inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Device staging of one step, each section 256-byte aligned.  The workspace
// section leaves room for every chunk to have a 256-byte aligned slice of its own.
// group_size > 0: the step runs the shared-prefix decode, with one prefix length
// per group of group_size sequences and that decode's partial-state workspace.
struct StagingLayout {
    size_t q, k_new, v_new, tables, lens, pairs, prefix, out, workspace, workspace_bytes, total;
};

StagingLayout staging_layout(int batch, int max_blocks_per_seq, int max_copy_pairs, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, int max_seq_len,
                             int partition_tokens, int group_size = 0) {
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
    l.prefix = off;
    if (group_size > 0) off += round_up((size_t)((batch + group_size - 1) / group_size) * 4);
    l.out = off;
    off += round_up((size_t)batch * num_q_heads * head_dim * 4);
    l.workspace = off;
    l.workspace_bytes = group_size > 0
                            ? pa_decode_shared_prefix_workspace_size(batch, group_size, num_q_heads, num_kv_heads,
                                                                     head_dim, block_size, max_seq_len,
                                                                     partition_tokens)
                            : pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                                       max_seq_len, partition_tokens);
    // Each chunk's slice rounds its partial states and itself up to kAlign.
    if (l.workspace_bytes) l.workspace_bytes += 2 * kAlign * kMaxChunks;
    off += round_up(l.workspace_bytes);
    l.total = off;
    return l;
}

int h2d(void *dst, const void *src, size_t bytes, cudaStream_t s) {
    if (bytes == 0) return PA_OK;
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Upload of a step's inputs by the SMs.  A copy engine pays a fixed latency of
// several microseconds per copy and moves the step's sub-megabyte inputs far
// below the link rate; SM loads from page-locked host memory (through its
// device mapping), four 16-byte loads in flight per thread, fill the link with
// one launch for all of them.
// ---------------------------------------------------------------------------
constexpr int kMaxSegs = 8;  // copy pairs, tables, lengths, prefix lengths, q, k_new, v_new (+1 spare)
constexpr int kUploadThreads = 256;
constexpr int kUploadInFlight = 4;

struct UploadSeg {
    const uint4 *src;          // device address of page-locked host memory, 16-byte aligned
    uint4 *dst;                // device memory, 16-byte aligned
    unsigned long long n16;    // whole 16-byte units
    unsigned long long tail;   // bytes after them (< 16)
};

struct UploadArgs {
    UploadSeg seg[kMaxSegs];
    int n;
};

__global__ void __launch_bounds__(kUploadThreads) upload_kernel(const __grid_constant__ UploadArgs a) {
    // end[i]: units of segments 0..i together
    unsigned long long end[kMaxSegs];
    unsigned long long total = 0;
#pragma unroll
    for (int i = 0; i < kMaxSegs; ++i) {
        total += i < a.n ? a.seg[i].n16 : 0ull;
        end[i] = total;
    }
    const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
    for (unsigned long long x0 = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; x0 < total;
         x0 += kUploadInFlight * stride) {
        uint4 v[kUploadInFlight];
        uint4 *d[kUploadInFlight];
#pragma unroll
        for (int j = 0; j < kUploadInFlight; ++j) {
            const unsigned long long x = x0 + j * stride;
            d[j] = nullptr;
            if (x < total) {
                const uint4 *src = a.seg[0].src;
                uint4 *dst = a.seg[0].dst;
                unsigned long long base = 0;
#pragma unroll
                for (int i = 1; i < kMaxSegs; ++i)
                    if (i < a.n && x >= end[i - 1]) {
                        src = a.seg[i].src;
                        dst = a.seg[i].dst;
                        base = end[i - 1];
                    }
                v[j] = src[x - base];
                d[j] = dst + (x - base);
            }
        }
#pragma unroll
        for (int j = 0; j < kUploadInFlight; ++j)
            if (d[j]) *d[j] = v[j];
    }
    if (blockIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < kMaxSegs; ++i)
            if (i < a.n && threadIdx.x == (unsigned)i && a.seg[i].tail) {
                const unsigned char *s8 = reinterpret_cast<const unsigned char *>(a.seg[i].src + a.seg[i].n16);
                unsigned char *d8 = reinterpret_cast<unsigned char *>(a.seg[i].dst + a.seg[i].n16);
                for (unsigned long long k = 0; k < a.seg[i].tail; ++k) d8[k] = s8[k];
            }
    }
}

// A host buffer as the device sees it: `mapped` is its device address when it is
// page-locked and 16-byte aligned (the upload kernel reads it), else null (it
// is copied with cudaMemcpyAsync).
struct HostSrc {
    const char *host = nullptr;
    const char *mapped = nullptr;
};

HostSrc host_src(const void *p) {
    HostSrc h;
    h.host = static_cast<const char *>(p);
    void *m = nullptr;
    if (p && device_address(p, &m) == PA_OK && aligned16(m)) h.mapped = static_cast<const char *>(m);
    return h;
}

// Collects the segments of one upload; copies what the kernel cannot read at once.
struct Upload {
    UploadArgs args{};

    int add(void *dst, const HostSrc &src, size_t offset, size_t bytes, cudaStream_t s) {
        if (bytes == 0) return PA_OK;
        if (!src.mapped || !aligned16(static_cast<char *>(dst)) || !aligned16(src.mapped + offset) ||
            args.n == kMaxSegs)
            return h2d(dst, src.host + offset, bytes, s);
        UploadSeg &g = args.seg[args.n++];
        g.src = reinterpret_cast<const uint4 *>(src.mapped + offset);
        g.dst = static_cast<uint4 *>(dst);
        g.n16 = bytes / 16;
        g.tail = bytes % 16;
        return PA_OK;
    }

    int launch(cudaStream_t s) {
        if (args.n == 0) return PA_OK;
        unsigned long long units = 0;
        for (int i = 0; i < args.n; ++i) units += args.seg[i].n16;
        const unsigned long long per_cta = (unsigned long long)kUploadThreads * kUploadInFlight;
        unsigned long long grid = (units + per_cta - 1) / per_cta;
        const unsigned long long cap = 2ull * device_sm_count();
        if (grid > cap) grid = cap;
        if (grid == 0) grid = 1;  // tails only
        upload_kernel<<<(unsigned)grid, kUploadThreads, 0, s>>>(args);
        count_launch();
        args.n = 0;
        return launch_status();
    }
};

int d2h(void *dst, const void *src, size_t bytes, cudaStream_t s) {
    if (bytes == 0) return PA_OK;
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Side streams and events of one device, created on first use.  The events are
// reused by every call, so one call's enqueue sequence holds `mu` throughout.
struct Pipes {
    std::mutex mu;
    bool ready = false;
    cudaStream_t up = nullptr, down = nullptr, comp = nullptr;
    cudaEvent_t start = nullptr, copied = nullptr, up_done = nullptr, comp_done = nullptr, down_done = nullptr;
    cudaEvent_t in[kMaxChunks] = {}, dec[kMaxChunks] = {};
};

Pipes g_pipes[kMaxDevices];

bool make_pipes(Pipes &p) {
    if (p.ready) return true;
    const unsigned sf = cudaStreamNonBlocking;
    const unsigned ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&p.up, sf) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.down, sf) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p.comp, sf) == cudaSuccess;
    for (cudaEvent_t *e : {&p.start, &p.copied, &p.up_done, &p.comp_done, &p.down_done})
        ok = ok && cudaEventCreateWithFlags(e, ef) == cudaSuccess;
    for (int c = 0; c < kMaxChunks; ++c)
        ok = ok && cudaEventCreateWithFlags(&p.in[c], ef) == cudaSuccess &&
             cudaEventCreateWithFlags(&p.dec[c], ef) == cudaSuccess;
    p.ready = ok;  // on failure the handles made so far are kept and reused by the next attempt
    return ok;
}

// Makes `waiter` wait for everything enqueued on `s` so far.
int after(cudaStream_t waiter, cudaStream_t s, cudaEvent_t e) {
    if (cudaEventRecord(e, s) != cudaSuccess) return PA_ERR_CUDA;
    return cudaStreamWaitEvent(waiter, e, 0) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int auto_chunks(int batch, size_t link_bytes, int max_chunks) {
    const size_t n = link_bytes / kAutoChunkBytes;
    int c = n < 1 ? 1 : (n > (size_t)max_chunks ? max_chunks : (int)n);
    return c > batch ? batch : c;
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

size_t pa_decode_step_staging_size_shared_prefix(int batch, int group_size, int max_blocks_per_seq,
                                                 int max_copy_pairs, int num_q_heads, int num_kv_heads,
                                                 int head_dim, int block_size, int max_seq_len,
                                                 int partition_tokens) {
    if (batch <= 0 || group_size < 1 || group_size > pa::kMaxGroupSize || max_blocks_per_seq < 0 ||
        num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return 0;
    return pa::staging_layout(batch, max_blocks_per_seq, max_copy_pairs, num_q_heads, num_kv_heads, head_dim,
                              block_size, max_seq_len, partition_tokens, group_size)
        .total;
}

}  // extern "C"

// A host step with everything that does not change from step to step resolved
// once: argument checks, the staging layout, the device view of each host
// buffer (page-locked memory read through its mapping), the output path and
// the chunk count.  pa_decode_step_host builds one per call; a
// pa_decode_step_plan keeps one for many steps.
struct pa_decode_step_plan {
    float *out_host;
    const int32_t *copy_pairs_host;
    void *k_cache, *v_cache;
    int batch, max_blocks_per_seq, max_copy_pairs, max_seq_len_cap;
    int num_q_heads, num_kv_heads, head_dim, block_size;
    int64_t num_blocks;
    float scale;
    int partition_tokens;
    int chunks;
    bool fp8;
    float k_scale, v_scale;
    char *st;                      // staging
    size_t staging_bytes;
    pa::StagingLayout l;
    pa::HostSrc hq, hk, hv, ht, hl, hp, hx;
    bool direct;                   // the kernels store the output into out_host
    char *out_base;
    int group_size;                // > 0: shared-prefix decode over groups of this many sequences
    const int32_t *prefix_lens_host;
    bool auto_chunks;              // the chunk count is the library's choice
    size_t link_bytes;             // bytes per step crossing the host link
};

namespace pa {
namespace {

int plan_init(pa_decode_step_plan &P, float *out_host, const void *q_host, const void *k_new_host,
              const void *v_new_host, const int32_t *block_tables_host, int max_blocks_per_seq,
              const int32_t *seq_lens_host, const int32_t *copy_pairs_host, int max_copy_pairs, void *k_cache,
              void *v_cache, int batch, int max_seq_len_cap, int num_q_heads, int num_kv_heads, int head_dim,
              int block_size, int64_t num_blocks, float scale, int partition_tokens, int num_chunks, void *staging,
              size_t staging_bytes, bool fp8, float k_scale, float v_scale) {
    if (fp8 && !(k_scale > 0.f && v_scale > 0.f && k_scale < 3.0e38f && v_scale < 3.0e38f))
        return PA_ERR_INVALID_ARG;
    if (batch < 0 || max_copy_pairs < 0 || max_blocks_per_seq < 0 || max_seq_len_cap < 0 || num_chunks < 0 ||
        num_chunks > kMaxChunks)
        return PA_ERR_INVALID_ARG;
    if (!supported_shape(num_q_heads, num_kv_heads, head_dim, block_size)) return PA_ERR_UNSUPPORTED;
    P = pa_decode_step_plan{};
    P.batch = batch;
    if (batch == 0) return PA_OK;
    if (!out_host || !q_host || !k_new_host || !v_new_host || !block_tables_host || !seq_lens_host || !staging ||
        !k_cache || !v_cache)
        return PA_ERR_INVALID_ARG;
    if (partition_tokens > 0 && partition_tokens % block_size) return PA_ERR_INVALID_ARG;  // as pa_decode
    P.l = staging_layout(batch, max_blocks_per_seq, max_copy_pairs, num_q_heads, num_kv_heads, head_dim,
                         block_size, max_seq_len_cap, partition_tokens);
    if (staging_bytes < P.l.total || (reinterpret_cast<uintptr_t>(staging) & (kAlign - 1))) return PA_ERR_INVALID_ARG;
    P.out_host = out_host;
    P.copy_pairs_host = copy_pairs_host;
    P.k_cache = k_cache;
    P.v_cache = v_cache;
    P.max_blocks_per_seq = max_blocks_per_seq;
    P.max_copy_pairs = max_copy_pairs;
    P.max_seq_len_cap = max_seq_len_cap;
    P.num_q_heads = num_q_heads;
    P.num_kv_heads = num_kv_heads;
    P.head_dim = head_dim;
    P.block_size = block_size;
    P.num_blocks = num_blocks;
    P.scale = scale;
    P.partition_tokens = partition_tokens;
    P.fp8 = fp8;
    P.k_scale = k_scale;
    P.v_scale = v_scale;
    P.st = static_cast<char *>(staging);
    P.staging_bytes = staging_bytes;
    // bytes per sequence crossing the host link: inputs and the fp32 output
    const size_t link_bytes = (size_t)batch * ((size_t)num_q_heads * head_dim * 6 + (size_t)num_kv_heads * head_dim * 4 +
                                               (size_t)max_blocks_per_seq * 4 + 4);
    P.auto_chunks = num_chunks == 0;
    P.link_bytes = link_bytes;
    P.chunks = num_chunks ? (num_chunks > batch ? batch : num_chunks) : auto_chunks(batch, link_bytes, kAutoMaxChunks);
    // Host inputs as the device sees them.
    P.hq = host_src(q_host);
    P.hk = host_src(k_new_host);
    P.hv = host_src(v_new_host);
    P.ht = host_src(block_tables_host);
    P.hl = host_src(seq_lens_host);
    P.hp = host_src(copy_pairs_host);
    // The output goes straight into out_host when the device can address it
    // (page-locked host memory): the kernels' stores cross the host link while
    // the decode runs, and no copy stage follows.  Otherwise it is staged on the
    // device and copied back.
    void *out_mapped = nullptr;
    P.direct = device_address(out_host, &out_mapped) == PA_OK;
    P.out_base = P.direct ? static_cast<char *>(out_mapped) : P.st + P.l.out;
    return PA_OK;
}

int plan_run(const pa_decode_step_plan &P, int max_seq_len, int num_pairs, int32_t *err_flag, cudaStream_t s) {
    if (P.batch == 0) return PA_OK;
    if (max_seq_len < 0 || max_seq_len > P.max_seq_len_cap || num_pairs < 0 || num_pairs > P.max_copy_pairs ||
        (num_pairs > 0 && !P.copy_pairs_host))
        return PA_ERR_INVALID_ARG;
    const int batch = P.batch;
    const StagingLayout &l = P.l;
    char *st = P.st;
    // Resolve the partitioning once for the whole batch, so that every chunk
    // splits its sequences exactly as an unchunked call would.
    const int pt = pa_decode_partition_tokens(batch, P.num_q_heads, P.num_kv_heads, P.head_dim, P.block_size,
                                              max_seq_len, P.partition_tokens);
    // bytes per sequence of each input and of the output
    const size_t q_row = (size_t)P.num_q_heads * P.head_dim * 2;
    const size_t kv_row = (size_t)P.num_kv_heads * P.head_dim * 2;
    const size_t tab_row = (size_t)P.max_blocks_per_seq * 4;
    const size_t out_row = (size_t)P.num_q_heads * P.head_dim * 4;
    const int chunks = P.group_size > 0 ? std::min(P.chunks, (batch + P.group_size - 1) / P.group_size) : P.chunks;

    // decode of sequences [b0, b0 + nb) with inputs in staging, on stream cs, workspace slice ws
    auto decode_rows = [&](int b0, int nb, char *ws, size_t ws_bytes, cudaStream_t cs) {
        // shared-prefix decode: b0 starts a group, so the chunk's groups are b0 / gs on
        const int32_t *prefix =
            P.group_size > 0 ? reinterpret_cast<const int32_t *>(st + l.prefix) + b0 / P.group_size : nullptr;
        return decode_impl(reinterpret_cast<float *>(P.out_base + b0 * out_row), st + l.q + b0 * q_row,
                           st + l.k_new + b0 * kv_row, st + l.v_new + b0 * kv_row, P.k_cache, P.v_cache,
                           reinterpret_cast<const int32_t *>(st + l.tables + b0 * tab_row), P.max_blocks_per_seq,
                           reinterpret_cast<const int32_t *>(st + l.lens) + b0, nb, max_seq_len, P.num_q_heads,
                           P.num_kv_heads, P.head_dim, P.block_size, P.num_blocks, P.scale, pt, ws, ws_bytes,
                           err_flag, cs, P.fp8, P.k_scale, P.v_scale, prefix, P.group_size);
    };
    // q, k_new and v_new of sequences [b0, b0 + nb); with `meta`, also the copy
    // pairs, block tables and lengths of the whole batch.  One kernel launch.
    auto upload = [&](int b0, int nb, bool meta, cudaStream_t cs) {
        Upload up;
        int rc = PA_OK;
        if (meta) {
            rc = up.add(st + l.pairs, P.hp, 0, (size_t)num_pairs * 8, cs);
            if (rc == PA_OK) rc = up.add(st + l.tables, P.ht, 0, batch * tab_row, cs);
            if (rc == PA_OK) rc = up.add(st + l.lens, P.hl, 0, (size_t)batch * 4, cs);
            if (rc == PA_OK && P.group_size > 0)
                rc = up.add(st + l.prefix, P.hx, 0, (size_t)((batch + P.group_size - 1) / P.group_size) * 4, cs);
        }
        if (rc == PA_OK) rc = up.add(st + l.q + b0 * q_row, P.hq, b0 * q_row, nb * q_row, cs);
        if (rc == PA_OK) rc = up.add(st + l.k_new + b0 * kv_row, P.hk, b0 * kv_row, nb * kv_row, cs);
        if (rc == PA_OK) rc = up.add(st + l.v_new + b0 * kv_row, P.hv, b0 * kv_row, nb * kv_row, cs);
        if (rc == PA_OK) rc = up.launch(cs);
        return rc;
    };
    auto copy_pairs = [&](cudaStream_t cs) {
        if (num_pairs == 0) return (int)PA_OK;
        const int32_t *pairs = reinterpret_cast<const int32_t *>(st + l.pairs);
        return P.fp8 ? pa_copy_blocks_fp8(P.k_cache, P.v_cache, pairs, num_pairs, P.num_blocks, P.num_kv_heads,
                                          P.block_size, P.head_dim, err_flag, cs)
                     : pa_copy_blocks(P.k_cache, P.v_cache, pairs, num_pairs, P.num_blocks, P.num_kv_heads,
                                      P.block_size, P.head_dim, err_flag, cs);
    };

    if (chunks <= 1) {
        int rc = upload(0, batch, true, s);
        if (rc == PA_OK) rc = copy_pairs(s);
        if (rc == PA_OK)
            rc = decode_rows(0, batch, l.workspace_bytes ? st + l.workspace : nullptr, l.workspace_bytes, s);
        if (rc == PA_OK && !P.direct) rc = d2h(P.out_host, st + l.out, batch * out_row, s);
        return rc;
    }

    // Chunk 0 has half the weight of the others: the first decode waits for its
    // upload alone, while every later upload runs ahead of the decodes (the link
    // delivers inputs faster than decode consumes them).  Chunks hold whole
    // groups of the shared-prefix decode (single sequences otherwise).  That
    // decode writes every output row from its reduce, after the chunk's decode,
    // so the last chunk's output crossing the link is not overlapped: its last
    // chunk is half-size too (chat mix, 8 chunks: 0.437 against 0.460 ms a step).
    const int gs = P.group_size > 0 ? P.group_size : 1;
    const int groups = (batch + gs - 1) / gs;
    const bool taper = P.group_size > 0 && chunks >= 3;
    const int64_t units = 2LL * chunks - 1 - (taper ? 1 : 0);
    auto chunk_start = [&](int c) {  // at least one group per chunk (chunks <= groups)
        int g = c == 0 ? 0 : (int)((int64_t)groups * (2LL * c - 1) / units);
        if (g < c) g = c;
        const int b = g * gs;
        return b < batch ? b : batch;
    };
    // Without copy pairs, chunk 0's upload goes first, on the caller's stream
    // (where chunk 0 decodes): the GPU starts while the rest is enqueued.
    const bool early = num_pairs == 0;
    if (early) {
        const int rc0 = upload(0, chunk_start(1), true, s);
        if (rc0 != PA_OK) return rc0;
    }

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    Pipes &p = g_pipes[dev];
    std::lock_guard<std::mutex> lock(p.mu);
    if (!make_pipes(p)) return PA_ERR_CUDA;

    // Fork: the side streams start after everything already on the caller's stream
    // (the previous step, which may still read this staging).
    if (cudaEventRecord(p.start, s) != cudaSuccess) return PA_ERR_CUDA;
    for (cudaStream_t side : {p.up, p.down, p.comp})
        if (cudaStreamWaitEvent(side, p.start, 0) != cudaSuccess) return PA_ERR_CUDA;

    // Block copies first, on the caller's stream; every chunk's decode comes after them.
    int rc = PA_OK;
    if (num_pairs > 0) {
        rc = upload(0, 0, true, p.up);
        if (rc == PA_OK) rc = after(s, p.up, p.copied);
        if (rc == PA_OK) rc = copy_pairs(s);
        if (rc == PA_OK) rc = after(p.comp, s, p.copied);
    }
    char *ws = l.workspace_bytes ? st + l.workspace : nullptr;
    size_t ws_left = l.workspace_bytes;
    for (int c = 0; c < chunks && rc == PA_OK; ++c) {
        const int b0 = chunk_start(c);
        const int nb = (c + 1 < chunks ? chunk_start(c + 1) : batch) - b0;
        if (nb == 0) continue;
        cudaStream_t cs = (c & 1) ? p.comp : s;
        if (!(c == 0 && early)) {  // (chunk 0's early upload is already on its stream)
            rc = upload(b0, nb, false, p.up);
            if (rc == PA_OK) rc = after(cs, p.up, p.in[c]);
        }
        size_t ws_bytes = 0;
        if (rc == PA_OK && ws) {
            ws_bytes = P.group_size > 0
                           ? pa_decode_shared_prefix_workspace_size(nb, P.group_size, P.num_q_heads, P.num_kv_heads,
                                                                    P.head_dim, P.block_size, max_seq_len, pt)
                           : pa_decode_workspace_size(nb, P.num_q_heads, P.num_kv_heads, P.head_dim, P.block_size,
                                                      max_seq_len, pt);
            if (round_up(ws_bytes) > ws_left) rc = PA_ERR_INVALID_ARG;
        }
        if (rc == PA_OK) rc = decode_rows(b0, nb, ws_bytes ? ws : nullptr, ws_bytes, cs);
        if (rc == PA_OK && ws_bytes) {
            ws += round_up(ws_bytes);
            ws_left -= round_up(ws_bytes);
        }
        if (rc == PA_OK && !P.direct) {
            rc = after(p.down, cs, p.dec[c]);
            if (rc == PA_OK)
                rc = d2h(reinterpret_cast<char *>(P.out_host) + b0 * out_row, st + l.out + b0 * out_row,
                         nb * out_row, p.down);
        }
    }
    // Join every side stream back into the caller's stream, on error paths too.
    const int jc = after(s, p.up, p.up_done);
    const int jp = after(s, p.comp, p.comp_done);
    const int jd = after(s, p.down, p.down_done);
    if (rc == PA_OK) rc = jc != PA_OK ? jc : (jp != PA_OK ? jp : jd);
    return rc;
}

// The host step for either pool type: bf16 pools, or E4M3 pools with their scales.
int step_host(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
              const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
              const int32_t *copy_pairs_host, int num_pairs, int max_copy_pairs, void *k_cache, void *v_cache,
              int batch, int max_seq_len, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
              int64_t num_blocks, float scale, int partition_tokens, int num_chunks, void *staging,
              size_t staging_bytes, int32_t *err_flag, void *stream, bool fp8, float k_scale, float v_scale) {
    if (num_pairs < 0 || max_seq_len < 0) return PA_ERR_INVALID_ARG;
    pa_decode_step_plan P;
    const int rc = plan_init(P, out_host, q_host, k_new_host, v_new_host, block_tables_host, max_blocks_per_seq,
                             seq_lens_host, num_pairs ? copy_pairs_host : nullptr, max_copy_pairs, k_cache, v_cache,
                             batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                             partition_tokens, num_chunks, staging, staging_bytes, fp8, k_scale, v_scale);
    if (rc != PA_OK) return rc;
    return plan_run(P, max_seq_len, num_pairs, err_flag, static_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace pa

extern "C" {

int pa_decode_step_host(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                        const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                        const int32_t *copy_pairs_host, int num_pairs, int max_copy_pairs, void *k_cache,
                        void *v_cache, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int64_t num_blocks, float scale, int partition_tokens,
                        int num_chunks, void *staging, size_t staging_bytes, int32_t *err_flag, void *stream) {
    return pa::step_host(out_host, q_host, k_new_host, v_new_host, block_tables_host, max_blocks_per_seq,
                     seq_lens_host, copy_pairs_host, num_pairs, max_copy_pairs, k_cache, v_cache, batch,
                     max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                     partition_tokens, num_chunks, staging, staging_bytes, err_flag, stream, false, 1.f, 1.f);
}

int pa_decode_step_host_fp8(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                            const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                            const int32_t *copy_pairs_host, int num_pairs, int max_copy_pairs, void *k_cache,
                            void *v_cache, int batch, int max_seq_len, int num_q_heads, int num_kv_heads,
                            int head_dim, int block_size, int64_t num_blocks, float scale, float k_scale,
                            float v_scale, int partition_tokens, int num_chunks, void *staging,
                            size_t staging_bytes, int32_t *err_flag, void *stream) {
    return pa::step_host(out_host, q_host, k_new_host, v_new_host, block_tables_host, max_blocks_per_seq,
                     seq_lens_host, copy_pairs_host, num_pairs, max_copy_pairs, k_cache, v_cache, batch,
                     max_seq_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                     partition_tokens, num_chunks, staging, staging_bytes, err_flag, stream, true, k_scale, v_scale);
}

int pa_decode_step_plan_create(float *out_host, const void *q_host, const void *k_new_host, const void *v_new_host,
                               const int32_t *block_tables_host, int max_blocks_per_seq, const int32_t *seq_lens_host,
                               const int32_t *copy_pairs_host, int max_copy_pairs, void *k_cache, void *v_cache,
                               int batch, int max_seq_len_cap, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int64_t num_blocks, float scale, int partition_tokens, int num_chunks,
                               void *staging, size_t staging_bytes, int kv_fp8, float k_scale, float v_scale,
                               pa_decode_step_plan **plan) {
    if (!plan) return PA_ERR_INVALID_ARG;
    *plan = nullptr;
    pa_decode_step_plan *P = new (std::nothrow) pa_decode_step_plan();
    if (!P) return PA_ERR_OOM;
    const int rc = pa::plan_init(*P, out_host, q_host, k_new_host, v_new_host, block_tables_host, max_blocks_per_seq,
                                 seq_lens_host, copy_pairs_host, max_copy_pairs, k_cache, v_cache, batch,
                                 max_seq_len_cap, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                                 partition_tokens, num_chunks, staging, staging_bytes, kv_fp8 != 0,
                                 kv_fp8 ? k_scale : 1.f, kv_fp8 ? v_scale : 1.f);
    if (rc != PA_OK) {
        delete P;
        return rc;
    }
    *plan = P;
    return PA_OK;
}

int pa_decode_step_plan_run(const pa_decode_step_plan *plan, int max_seq_len, int num_pairs, int32_t *err_flag,
                            void *stream) {
    if (!plan) return PA_ERR_INVALID_ARG;
    return pa::plan_run(*plan, max_seq_len, num_pairs, err_flag, static_cast<cudaStream_t>(stream));
}

int pa_decode_step_plan_set_shared_prefix(pa_decode_step_plan *plan, const int32_t *prefix_lens_host,
                                          int group_size) {
    if (!plan) return PA_ERR_INVALID_ARG;
    pa_decode_step_plan &P = *plan;
    if (group_size < 0 || group_size > pa::kMaxGroupSize) return PA_ERR_INVALID_ARG;
    if (group_size > 0 && P.fp8) return PA_ERR_UNSUPPORTED;
    if (P.batch == 0) {  // nothing to run: remember the mode only
        P.group_size = group_size;
        P.prefix_lens_host = prefix_lens_host;
        return PA_OK;
    }
    if (group_size > 0 && !prefix_lens_host) return PA_ERR_INVALID_ARG;
    const pa::StagingLayout l = pa::staging_layout(P.batch, P.max_blocks_per_seq, P.max_copy_pairs, P.num_q_heads,
                                                   P.num_kv_heads, P.head_dim, P.block_size, P.max_seq_len_cap,
                                                   P.partition_tokens, group_size);
    if (P.staging_bytes < l.total) return PA_ERR_INVALID_ARG;  // the plan is left as it was
    P.l = l;
    P.group_size = group_size;
    P.prefix_lens_host = group_size > 0 ? prefix_lens_host : nullptr;
    P.hx = group_size > 0 ? pa::host_src(prefix_lens_host) : pa::HostSrc{};
    if (!P.direct) P.out_base = P.st + P.l.out;  // the staged output section moves with the layout
    if (P.auto_chunks)
        P.chunks = pa::auto_chunks(P.batch, P.link_bytes,
                                   group_size > 0 ? pa::kAutoMaxChunksShared : pa::kAutoMaxChunks);
    return PA_OK;
}

void pa_decode_step_plan_destroy(pa_decode_step_plan *plan) { delete plan; }

}  // extern "C"
