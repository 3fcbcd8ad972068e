/*
 * Plain fp64 CPU oracle for paged decode -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the package's smoke check and the bench's CPU-baseline leg
 * may load this.  It shares no code with the CUDA library: the index
 * arithmetic, the bf16 decoding and the softmax below are written out
 * independently, slowly and in the order the definitions give them.
 *
 * What it computes:
 *  - gather: the K (or V) rows of one kv head for logical positions
 *    0..L-1 of one sequence, dereferencing the block table as
 *    phys = table[p / block_size], row = p % block_size
 *    ("Walk through paged attention end to end", conceptual
 *    paged_attention_decode, the attention loop; "What is PagedAttention"
 *    (n4n.ai), "How PagedAttention works": blocks hold tokens contiguously).
 *    Pool layout [num_blocks, num_kv_heads, block_size, head_dim].
 *  - attend: textbook softmax attention of one query over the gathered rows,
 *    s_p = scale * sum_i q_i k_p,i ; w_p = exp(s_p - max s) ;
 *    out = sum_p w_p v_p / sum_p w_p   -- paging leaves this math unchanged
 *    ("Walk through paged attention end to end", red flags: paging moves
 *    where K and V live, not what attention computes).  L = 0 gives a zero
 *    row.
 *  - decode: for every requested (sequence b, query head g) the kv head is
 *    h = g / (Hq / Hkv) (grouped-query sharing), gather + attend.
 *  - reshape_and_cache: write new K/V rows at slot s, i.e. block s / bs,
 *    row s % bs ("Walk through paged attention end to end", append step:
 *    last_block, offset); slot -1 is skipped.
 *  - copy_blocks: copy whole blocks src -> dst, K and V ("PagedAttention &
 *    vLLM", Copy-on-write sharing: the writer gets a private copy of the
 *    shared block).
 *  - swap_blocks: the same copy between two different pools (device pool
 *    and CPU-side pool), "What is PagedAttention and how does it manage KV
 *    cache", Swapping and preemption.
 *
 * All floating point is IEEE double (build without -ffast-math).  OpenMP
 * only spreads independent output rows over threads; each row's arithmetic
 * order is fixed, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the top half of an IEEE binary32; widening to double is exact. */
double oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Gather rows of kv head h of one sequence into dst[L][d] (double).
 * Returns 0, or -1 if a needed table entry is missing, -2 if a physical
 * block id is outside [0, num_blocks).
 */
int oracle_gather(const uint16_t *pool, int64_t num_blocks, int num_kv_heads,
                  int block_size, int head_dim, const int32_t *table,
                  int table_len, int seq_len, int h, double *dst)
{
    for (int p = 0; p < seq_len; ++p) {
        int j = p / block_size;
        int row = p % block_size;
        if (j >= table_len) return -1;
        int64_t phys = table[j];
        if (phys < 0 || phys >= num_blocks) return -2;
        int64_t base = ((phys * num_kv_heads + h) * (int64_t)block_size + row) * head_dim;
        for (int i = 0; i < head_dim; ++i)
            dst[(int64_t)p * head_dim + i] = oracle_bf16_to_f64(pool[base + i]);
    }
    return 0;
}

/* Softmax attention of one query q[d] over K[L][d], V[L][d]; writes out[d]. */
void oracle_attend(const double *q, const double *K, const double *V,
                   int seq_len, int head_dim, double scale, double *out)
{
    if (seq_len <= 0) {
        for (int i = 0; i < head_dim; ++i) out[i] = 0.0;
        return;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)seq_len);
    for (int p = 0; p < seq_len; ++p) {
        double dot = 0.0;
        for (int i = 0; i < head_dim; ++i) dot += q[i] * K[(int64_t)p * head_dim + i];
        s[p] = scale * dot;
    }
    double m = s[0];
    for (int p = 1; p < seq_len; ++p)
        if (s[p] > m) m = s[p];
    double z = 0.0;
    for (int p = 0; p < seq_len; ++p) {
        s[p] = exp(s[p] - m);
        z += s[p];
    }
    for (int i = 0; i < head_dim; ++i) {
        double acc = 0.0;
        for (int p = 0; p < seq_len; ++p) acc += s[p] * V[(int64_t)p * head_dim + i];
        out[i] = acc / z;
    }
    free(s);
}

/*
 * Decode the requested (b, g) rows.  rows[2r] = b, rows[2r+1] = g; out[r][d].
 * q is bf16 [B, Hq, d]; tables int32 [B, max_blocks]; seq_lens int32 [B].
 * Returns 0, or the first non-zero gather status.
 */
int oracle_decode_rows(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                       const int32_t *tables, int max_blocks, const int32_t *seq_lens,
                       int batch, int num_q_heads, int num_kv_heads, int head_dim,
                       int block_size, int64_t num_blocks, float scale,
                       const int32_t *rows, int n_rows, double *out)
{
    int status = 0;
    int group = num_q_heads / num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int b = rows[2 * r];
        int g = rows[2 * r + 1];
        int h = g / group;
        int L = (b >= 0 && b < batch) ? seq_lens[b] : 0;
        double *qd = (double *)malloc(sizeof(double) * (size_t)head_dim);
        double *K = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(L > 0 ? L : 1));
        double *V = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(L > 0 ? L : 1));
        for (int i = 0; i < head_dim; ++i)
            qd[i] = oracle_bf16_to_f64(q[((int64_t)b * num_q_heads + g) * head_dim + i]);
        const int32_t *table = tables + (int64_t)b * max_blocks;
        int st = oracle_gather(k_pool, num_blocks, num_kv_heads, block_size, head_dim,
                               table, max_blocks, L, h, K);
        if (st == 0)
            st = oracle_gather(v_pool, num_blocks, num_kv_heads, block_size, head_dim,
                               table, max_blocks, L, h, V);
        if (st == 0) {
            oracle_attend(qd, K, V, L, head_dim, (double)scale, out + (int64_t)r * head_dim);
        } else {
#pragma omp critical
            { if (status == 0) status = st; }
        }
        free(qd);
        free(K);
        free(V);
    }
    return status;
}

/* All rows, out[B][Hq][d]. */
int oracle_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                  const int32_t *tables, int max_blocks, const int32_t *seq_lens,
                  int batch, int num_q_heads, int num_kv_heads, int head_dim,
                  int block_size, int64_t num_blocks, float scale, double *out)
{
    int n = batch * num_q_heads;
    int32_t *rows = (int32_t *)malloc(sizeof(int32_t) * 2 * (size_t)(n > 0 ? n : 1));
    for (int b = 0; b < batch; ++b)
        for (int g = 0; g < num_q_heads; ++g) {
            rows[2 * (b * num_q_heads + g)] = b;
            rows[2 * (b * num_q_heads + g) + 1] = g;
        }
    int st = oracle_decode_rows(q, k_pool, v_pool, tables, max_blocks, seq_lens, batch,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                scale, rows, n, out);
    free(rows);
    return st;
}

/*
 * Write k_new/v_new [T, Hkv, d] into the pools at slot_mapping[t].
 * Slot -1 is skipped.  Returns the number of slots outside [0, NB*bs)
 * (those tokens are skipped too).
 */
int oracle_reshape_and_cache(const uint16_t *k_new, const uint16_t *v_new,
                             uint16_t *k_pool, uint16_t *v_pool,
                             const int32_t *slot_mapping, int num_tokens,
                             int64_t num_blocks, int num_kv_heads, int block_size,
                             int head_dim)
{
    int bad = 0;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t s = slot_mapping[t];
        if (s == -1) continue;
        if (s < 0 || s >= num_blocks * block_size) {
            ++bad;
            continue;
        }
        int64_t blk = s / block_size;
        int64_t row = s % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t dst = ((blk * num_kv_heads + h) * block_size + row) * head_dim;
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            for (int i = 0; i < head_dim; ++i) {
                k_pool[dst + i] = k_new[src + i];
                v_pool[dst + i] = v_new[src + i];
            }
        }
    }
    return bad;
}

/*
 * For each (src, dst) pair in order, copy block src to block dst in both
 * pools.  Returns the number of pairs with an id outside [0, NB) (skipped).
 */
int oracle_copy_blocks(uint16_t *k_pool, uint16_t *v_pool, const int32_t *pairs,
                       int num_pairs, int64_t num_blocks, int num_kv_heads,
                       int block_size, int head_dim)
{
    int bad = 0;
    int64_t block_elems = (int64_t)num_kv_heads * block_size * head_dim;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = pairs[2 * i];
        int64_t dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            ++bad;
            continue;
        }
        for (int64_t e = 0; e < block_elems; ++e) {
            k_pool[dst * block_elems + e] = k_pool[src * block_elems + e];
            v_pool[dst * block_elems + e] = v_pool[src * block_elems + e];
        }
    }
    return bad;
}

/*
 * For each (src, dst) pair in order, copy block src of the source pools to
 * block dst of the destination pools.  Returns the number of pairs with an
 * id out of range (skipped).
 */
int oracle_swap_blocks(uint16_t *dst_k, uint16_t *dst_v, int64_t dst_num_blocks, const uint16_t *src_k,
                       const uint16_t *src_v, int64_t src_num_blocks, const int32_t *pairs, int num_pairs,
                       int num_kv_heads, int block_size, int head_dim)
{
    int bad = 0;
    int64_t block_elems = (int64_t)num_kv_heads * block_size * head_dim;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = pairs[2 * i];
        int64_t dst = pairs[2 * i + 1];
        if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
            ++bad;
            continue;
        }
        for (int64_t e = 0; e < block_elems; ++e) {
            dst_k[dst * block_elems + e] = src_k[src * block_elems + e];
            dst_v[dst * block_elems + e] = src_v[src * block_elems + e];
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------
 * fp8 pools: OCP 8-bit E4M3 ("FN": no infinities, S.1111.111 is NaN, largest
 * finite 448).  Values are stored as code = E4M3(x * inv_scale), rounded to
 * nearest with ties to even and saturated to +-448, where x is the bf16 input
 * widened to fp32 and the product is an fp32 multiply; the value a code
 * stands for is E4M3_value(code) * scale.  The pages only say paging
 * composes with KV quantization ("Walk through paged attention end to end",
 * summary); the format and per-tensor scaling are this library's choice.
 * ---------------------------------------------------------------------- */

/* Value of an E4M3 code: sign, 4 exponent bits (bias 7), 3 mantissa bits. */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);            /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);     /* normal */
    return sign ? -v : v;
}

/* Nearest E4M3 code to an fp32 value: ties to even, saturating at 448. */
uint8_t oracle_e4m3_encode(float x)
{
    double v = (double)x;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {                   /* subnormal range, steps of 2^-9 */
        double q = nearbyint(ldexp(a, 9));     /* ties to even (default rounding mode) */
        return (uint8_t)(sign | (uint8_t)q);    /* q == 8 is exactly the smallest normal */
    }
    int ex;
    double f = frexp(a, &ex);                   /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;                             /* a = (2f) * 2^e, 2f in [1, 2) */
    double q = nearbyint((2.0 * f - 1.0) * 8.0);
    if (q == 8.0) {
        q = 0.0;
        e += 1;
    }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | (int)q));
}

/* dst[i] = E4M3(bf16(src[i]) * inv_scale) for n elements. */
void oracle_quantize_e4m3(const uint16_t *src, uint8_t *dst, int64_t n, float inv_scale)
{
    for (int64_t i = 0; i < n; ++i) {
        float x = (float)oracle_bf16_to_f64(src[i]);
        float prod = x * inv_scale;
        dst[i] = oracle_e4m3_encode(prod);
    }
}

/* Cache write into fp8 pools: like oracle_reshape_and_cache, quantizing each value. */
int oracle_reshape_and_cache_fp8(const uint16_t *k_new, const uint16_t *v_new, uint8_t *k_pool,
                                 uint8_t *v_pool, const int32_t *slot_mapping, int num_tokens,
                                 int64_t num_blocks, int num_kv_heads, int block_size, int head_dim,
                                 float k_inv_scale, float v_inv_scale)
{
    int bad = 0;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t s = slot_mapping[t];
        if (s == -1) continue;
        if (s < 0 || s >= num_blocks * block_size) {
            ++bad;
            continue;
        }
        int64_t blk = s / block_size;
        int64_t row = s % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t dst = ((blk * num_kv_heads + h) * block_size + row) * head_dim;
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            oracle_quantize_e4m3(k_new + src, k_pool + dst, head_dim, k_inv_scale);
            oracle_quantize_e4m3(v_new + src, v_pool + dst, head_dim, v_inv_scale);
        }
    }
    return bad;
}

/* Gather of fp8 rows, dequantised: dst[p][i] = E4M3_value(code) * scale. */
static int gather_fp8(const uint8_t *pool, int64_t num_blocks, int num_kv_heads, int block_size,
                      int head_dim, const int32_t *table, int table_len, int seq_len, int h,
                      double scale, double *dst)
{
    for (int p = 0; p < seq_len; ++p) {
        int j = p / block_size;
        int row = p % block_size;
        if (j >= table_len) return -1;
        int64_t phys = table[j];
        if (phys < 0 || phys >= num_blocks) return -2;
        int64_t base = ((phys * num_kv_heads + h) * (int64_t)block_size + row) * head_dim;
        for (int i = 0; i < head_dim; ++i)
            dst[(int64_t)p * head_dim + i] = oracle_e4m3_decode(pool[base + i]) * scale;
    }
    return 0;
}

/* Decode over fp8 pools: textbook attention on the dequantised rows. */
int oracle_decode_rows_fp8(const uint16_t *q, const uint8_t *k_pool, const uint8_t *v_pool,
                           const int32_t *tables, int max_blocks, const int32_t *seq_lens,
                           int batch, int num_q_heads, int num_kv_heads, int head_dim,
                           int block_size, int64_t num_blocks, float scale, float k_scale,
                           float v_scale, const int32_t *rows, int n_rows, double *out)
{
    int status = 0;
    int group = num_q_heads / num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n_rows; ++r) {
        int b = rows[2 * r];
        int g = rows[2 * r + 1];
        int h = g / group;
        int L = (b >= 0 && b < batch) ? seq_lens[b] : 0;
        double *qd = (double *)malloc(sizeof(double) * (size_t)head_dim);
        double *K = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(L > 0 ? L : 1));
        double *V = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(L > 0 ? L : 1));
        for (int i = 0; i < head_dim; ++i)
            qd[i] = oracle_bf16_to_f64(q[((int64_t)b * num_q_heads + g) * head_dim + i]);
        const int32_t *table = tables + (int64_t)b * max_blocks;
        int st = gather_fp8(k_pool, num_blocks, num_kv_heads, block_size, head_dim, table, max_blocks,
                            L, h, (double)k_scale, K);
        if (st == 0)
            st = gather_fp8(v_pool, num_blocks, num_kv_heads, block_size, head_dim, table, max_blocks,
                            L, h, (double)v_scale, V);
        if (st == 0) {
            oracle_attend(qd, K, V, L, head_dim, (double)scale, out + (int64_t)r * head_dim);
        } else {
#pragma omp critical
            { if (status == 0) status = st; }
        }
        free(qd);
        free(K);
        free(V);
    }
    return status;
}
