/*
 * pkv_oracle.c -- CPU oracle for attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path never
 * calls it, and it shares no source, header, table or helper with the CUDA path.
 *
 * It is plain and slow on purpose: every attention value is computed in fp64
 * straight from its definition, one (sequence, query head) at a time, gathering
 * the sequence's keys and values through its block table.  Quantization follows
 * the symmetric shared-scale rule in IEEE fp32 with the operation order written
 * out below, because the stored codes must match bit for bit.
 *
 * Sources (web pages on paged KV caches):
 *   [KVB]  "KV cache, continuous batching and paged attention"
 *   [KVG]  "KV cache, GQA, paging and continuous batching"
 *   [INF]  inference guide "a2-inf-2" (sections on PagedAttention, prefix caching,
 *          chunked prefill and KV-cache quantization)
 *
 * Pool format (a data format, so it is the same one the library documents):
 *   K and V each hold [num_blocks][num_kv_heads][16][row_bytes] with
 *   row_bytes = 2*d (f16, bf16), d (int8, fp8 e4m3), d/2 (int4, two codes a byte,
 *   element 2j in the low nibble).  Quantized pools carry one fp32 scale per
 *   (block, kv head) for K and another for V: [num_blocks][num_kv_heads].
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - query head h reads KV head h / G, G = H_q / H_kv (contiguous groups);
 *   - a context length of 0 gives a zero output row;
 *   - quantization is symmetric with Q = 127 (int8), 7 (int4), 448 (fp8 e4m3),
 *     scale s = amax / Q, codes rounded half to even and clamped to [-Q, Q];
 *   - a call that writes offset 0 of a block starts that block afresh; otherwise
 *     the block's scale only grows, and when it grows the codes already in the
 *     block that this call does not overwrite are re-quantized once to it.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define ORC_BLOCK 16

enum { ORC_F16 = 0, ORC_BF16 = 1, ORC_INT8 = 2, ORC_INT4 = 3, ORC_FP8 = 4 };

enum {
    ORC_OK = 0,
    ORC_ERR_ARG = -2,
    ORC_ERR_DTYPE = -3,
    ORC_ERR_INDEX = -8,
    ORC_ERR_NOMEM = -10
};

/* ------------------------------------------------------------------ sizes --
 * [KVB] "The KV cache" and [KVG] "Mechanics", the memory equation:
 * bytes per token = 2 (K and V) x layers x KV heads x head dim x bytes per element.
 */
int64_t orc_kv_bytes_per_token(int layers, int kv_heads, int head_dim, int bytes_per_elem)
{
    return (int64_t)2 * layers * kv_heads * head_dim * bytes_per_elem;
}

/* The whole cache for S tokens of context and B sequences ([KVG] "Mechanics"). */
int64_t orc_kv_cache_bytes(int layers, int kv_heads, int head_dim, int bytes_per_elem,
                           int64_t seq_len, int64_t batch)
{
    return orc_kv_bytes_per_token(layers, kv_heads, head_dim, bytes_per_elem) * seq_len * batch;
}

/* Blocks a sequence of n tokens occupies, and the slots it leaves empty
 * ([KVB] "Paged attention": waste is at most one partly filled block). */
int64_t orc_blocks_for_tokens(int64_t n) { return (n + ORC_BLOCK - 1) / ORC_BLOCK; }
int64_t orc_waste_slots(int64_t n) { return orc_blocks_for_tokens(n) * ORC_BLOCK - n; }

/* -------------------------------------------------------- element codecs -- */

/* bfloat16 is the upper half of an IEEE binary32. */
float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* zero or subnormal */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp(1.0 + (double)m / 1024.0, e - 15);
    return sign ? -v : v;
}

/* OCP 8-bit floating point, E4M3 ("fn": no infinities): bias 7, 3 fraction bits,
 * S.1111.111 is NaN, largest finite 448 = 1.75 * 2^8, subnormals m * 2^-9. */
double orc_e4m3_to_f64(uint8_t c)
{
    int sign = c >> 7;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 0xf && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* binary32 -> E4M3, round to nearest even, saturating to +-448 (values whose
 * rounding would pass 448 become 448; NaN stays NaN).  Every step but the one
 * rounding is exact in double. */
uint8_t orc_e4m3_from_f32(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(x))
        return 0x7f;
    if (a >= 448.0)
        return sign | 0x7e;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: a = m * 2^-9 */
        double m = nearbyint(a * 512.0);           /* round half to even */
        if (m >= 8.0)
            return sign | 0x08;                    /* rounds up to the smallest normal */
        return sign | (uint8_t)m;
    }
    int e2;
    double fr = frexp(a, &e2);                     /* a = fr * 2^e2, fr in [0.5, 1) */
    int e = e2 - 1;                                /* a = (2 fr) * 2^e, 2 fr in [1, 2) */
    double m = nearbyint((2.0 * fr - 1.0) * 8.0);
    if (m >= 8.0) {
        m = 0.0;
        e += 1;
    }
    int field = e + 7;
    if (field > 15 || (field == 15 && m > 6.0))
        return sign | 0x7e;                        /* saturate instead of NaN */
    return sign | (uint8_t)((field << 3) | (int)m);
}

/* ------------------------------------------------------------- pool views -- */

static int row_bytes(int dtype, int d)
{
    switch (dtype) {
    case ORC_F16:
    case ORC_BF16: return 2 * d;
    case ORC_INT8:
    case ORC_FP8: return d;
    case ORC_INT4: return d / 2;
    default: return -1;
    }
}

static double quant_levels(int dtype)
{
    switch (dtype) {
    case ORC_INT8: return 127.0;
    case ORC_INT4: return 7.0;
    case ORC_FP8: return 448.0;
    default: return 0.0;
    }
}

static size_t tile_index(int blk, int g, int H_kv)
{
    return (size_t)blk * H_kv + g;
}

/* One stored code as an integer (int8 / int4) or raw byte (fp8). */
static int read_code(const uint8_t* pool, int dtype, int blk, int g, int off, int dd, int H_kv, int d)
{
    size_t row = (tile_index(blk, g, H_kv) * ORC_BLOCK + off) * (size_t)row_bytes(dtype, d);
    if (dtype == ORC_INT8)
        return (int)(int8_t)pool[row + dd];
    if (dtype == ORC_FP8)
        return (int)pool[row + dd];
    /* int4: element 2j in the low nibble, 2j+1 in the high nibble, two's complement */
    uint8_t byte = pool[row + dd / 2];
    int nib = (dd & 1) ? (byte >> 4) : (byte & 0xf);
    return nib >= 8 ? nib - 16 : nib;
}

static void write_code(uint8_t* pool, int dtype, int blk, int g, int off, int dd, int H_kv, int d, int code)
{
    size_t row = (tile_index(blk, g, H_kv) * ORC_BLOCK + off) * (size_t)row_bytes(dtype, d);
    if (dtype == ORC_INT8 || dtype == ORC_FP8) {
        pool[row + dd] = (uint8_t)code;
        return;
    }
    uint8_t* p = &pool[row + dd / 2];
    uint8_t nib = (uint8_t)(code & 0xf);
    if (dd & 1)
        *p = (uint8_t)((*p & 0x0f) | (nib << 4));
    else
        *p = (uint8_t)((*p & 0xf0) | nib);
}

/* Value of one cached element, widened to double.  Quantized codes are
 * dequantized as code * scale ([INF] "KV-cache quantization"). */
static double pool_value(const uint8_t* pool, const float* scale, int dtype,
                         int blk, int g, int off, int dd, int H_kv, int d)
{
    if (dtype == ORC_F16 || dtype == ORC_BF16) {
        size_t idx = (tile_index(blk, g, H_kv) * ORC_BLOCK + off) * (size_t)d + dd;
        uint16_t h;
        memcpy(&h, pool + 2 * idx, 2);
        return dtype == ORC_F16 ? orc_f16_to_f64(h) : (double)orc_bf16_to_f32(h);
    }
    int c = read_code(pool, dtype, blk, g, off, dd, H_kv, d);
    double s = (double)scale[tile_index(blk, g, H_kv)];
    if (dtype == ORC_FP8)
        return orc_e4m3_to_f64((uint8_t)c) * s;
    return (double)c * s;
}

static double src_value(const uint16_t* src, int src_dtype, size_t idx)
{
    return src_dtype == ORC_F16 ? orc_f16_to_f64(src[idx]) : (double)orc_bf16_to_f32(src[idx]);
}

/* ---------------------------------------------------------------- append --
 * [KVB] "The KV cache": the new token's K and V are cached; [KVG] "PagedAttention":
 * a per-sequence block table maps logical positions to physical blocks, so a token
 * at logical position t of a sequence lands in slot table[t/16]*16 + t%16.
 * The caller passes those slots; a negative slot is padding and is skipped.
 *
 * 16-bit pools: a byte copy of each (token, head) row into its slot.
 *
 * Quantized pools ([INF] "KV-cache quantization": integer codes sharing one scale),
 * per (block, kv head) this call touches, separately for K and V, all in fp32:
 *   A     = max |x| over the call's tokens in that block (x = bf16 value, exact in fp32)
 *   S_old = 0 if the call writes offset 0 of the block, else the stored scale
 *   s     = max(S_old, A / Q)
 *   if s > S_old > 0: every code of the block the call does not overwrite becomes
 *         int:  clamp(rint(((float)c * S_old) / s))
 *         fp8:  e4m3(((float)value(c) * S_old) / s)
 *   new codes: int: clamp(rint(x / s), -Q, Q); fp8: e4m3(x / s); all 0 when s == 0
 *   the stored scale becomes s.
 */
static int quantize_code(int dtype, float x, float s)
{
    if (s == 0.0f)
        return 0;
    float r = x / s;
    if (dtype == ORC_FP8)
        return orc_e4m3_from_f32(r);
    float Q = (float)quant_levels(dtype);
    float c = rintf(r);
    if (c > Q) c = Q;
    if (c < -Q) c = -Q;
    return (int)c;
}

static int requantize_code(int dtype, int c, float s_old, float s)
{
    if (dtype == ORC_FP8) {
        float v = (float)orc_e4m3_to_f64((uint8_t)c);
        float r = (v * s_old) / s;
        return orc_e4m3_from_f32(r);
    }
    float Q = (float)quant_levels(dtype);
    float r = ((float)c * s_old) / s;
    float q = rintf(r);
    if (q > Q) q = Q;
    if (q < -Q) q = -Q;
    return (int)q;
}

static int append_quantized(int N, int H_kv, int d, int dtype, uint8_t* pool, float* scales,
                            const uint16_t* src, int src_dtype, const int32_t* slots, int T)
{
    /* tokens of the call grouped by block: first_tok[blk] -> chain through next_tok */
    int32_t* first_tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
    int32_t* next_tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    int32_t* touched = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    if (!first_tok || !next_tok || !touched) {
        free(first_tok); free(next_tok); free(touched);
        return ORC_ERR_NOMEM;
    }
    for (int b = 0; b < N; ++b) first_tok[b] = -1;
    int n_touched = 0;
    for (int i = T - 1; i >= 0; --i) {
        if (slots[i] < 0) continue;
        int blk = slots[i] / ORC_BLOCK;
        if (first_tok[blk] < 0) touched[n_touched++] = blk;
        next_tok[i] = first_tok[blk];
        first_tok[blk] = i;
    }
    const float Q = (float)quant_levels(dtype);
    for (int u = 0; u < n_touched; ++u) {
        int blk = touched[u];
        unsigned mask = 0;
        for (int i = first_tok[blk]; i >= 0; i = next_tok[i]) mask |= 1u << (slots[i] % ORC_BLOCK);
        int fresh = (mask & 1u) != 0;
        for (int g = 0; g < H_kv; ++g) {
            float A = 0.0f;
            for (int i = first_tok[blk]; i >= 0; i = next_tok[i])
                for (int dd = 0; dd < d; ++dd) {
                    float x = (float)src_value(src, src_dtype, ((size_t)i * H_kv + g) * d + dd);
                    float ax = fabsf(x);
                    if (ax > A) A = ax;
                }
            size_t si = tile_index(blk, g, H_kv);
            float s_old = fresh ? 0.0f : scales[si];
            float a_over_q = A / Q;
            float s = s_old > a_over_q ? s_old : a_over_q;
            if (s > s_old && s_old > 0.0f) {
                for (int off = 0; off < ORC_BLOCK; ++off) {
                    if (mask & (1u << off)) continue;
                    for (int dd = 0; dd < d; ++dd) {
                        int c = read_code(pool, dtype, blk, g, off, dd, H_kv, d);
                        write_code(pool, dtype, blk, g, off, dd, H_kv, d,
                                   requantize_code(dtype, c, s_old, s));
                    }
                }
            }
            for (int i = first_tok[blk]; i >= 0; i = next_tok[i]) {
                int off = slots[i] % ORC_BLOCK;
                for (int dd = 0; dd < d; ++dd) {
                    float x = (float)src_value(src, src_dtype, ((size_t)i * H_kv + g) * d + dd);
                    write_code(pool, dtype, blk, g, off, dd, H_kv, d, quantize_code(dtype, x, s));
                }
            }
            scales[si] = s;
        }
    }
    free(first_tok); free(next_tok); free(touched);
    return ORC_OK;
}

int orc_kv_append(int N, int H_kv, int d, int dtype,
                  uint8_t* k_pool, uint8_t* v_pool, float* k_scale, float* v_scale,
                  const uint16_t* k_src, const uint16_t* v_src, int src_dtype,
                  const int32_t* slots, int T)
{
    if (N <= 0 || H_kv <= 0 || d <= 0 || T < 0 || !k_pool || !v_pool || (T > 0 && (!k_src || !v_src || !slots)))
        return ORC_ERR_ARG;
    if (row_bytes(dtype, d) <= 0 || (dtype == ORC_INT4 && (d & 1)))
        return ORC_ERR_DTYPE;
    for (int i = 0; i < T; ++i)
        if (slots[i] >= (int64_t)N * ORC_BLOCK)
            return ORC_ERR_INDEX;
    if (dtype == ORC_F16 || dtype == ORC_BF16) {
        if (src_dtype != dtype)
            return ORC_ERR_DTYPE;
        size_t rb = (size_t)row_bytes(dtype, d);
        for (int i = 0; i < T; ++i) {
            if (slots[i] < 0) continue;
            int blk = slots[i] / ORC_BLOCK, off = slots[i] % ORC_BLOCK;
            for (int g = 0; g < H_kv; ++g) {
                size_t dst = (tile_index(blk, g, H_kv) * ORC_BLOCK + off) * rb;
                size_t srco = ((size_t)i * H_kv + g) * d;
                memcpy(k_pool + dst, k_src + srco, rb);
                memcpy(v_pool + dst, v_src + srco, rb);
            }
        }
        return ORC_OK;
    }
    if (src_dtype != ORC_BF16 || !k_scale || !v_scale)
        return ORC_ERR_DTYPE;
    int rc = append_quantized(N, H_kv, d, dtype, k_pool, k_scale, k_src, src_dtype, slots, T);
    if (rc != ORC_OK) return rc;
    return append_quantized(N, H_kv, d, dtype, v_pool, v_scale, v_src, src_dtype, slots, T);
}

/* ------------------------------------------------------------- attention --
 * Softmax attention of one query row over keys lo .. n-1 gathered through a block table
 * ([KVG] "What it is": the cache holds K and V of every earlier token; [KVB] "Paged
 * attention": the attention kernel follows the block table).  In fp64:
 *   s_t = scale * sum_j q_j K[t][j];  m = max_t s_t;  w_t = exp(s_t - m);
 *   out_j = sum_t w_t V[t][j] / sum_t w_t;   no keys give zeros.
 * lo > 0 only for sliding-window attention (see window_start).
 */
static int attend_one(int N, int H_kv, int d, int dtype,
                      const uint8_t* k_pool, const uint8_t* v_pool,
                      const float* k_scale, const float* v_scale,
                      const double* qrow, int g, const int32_t* table, int W, int lo, int n,
                      double scale, double* s_buf, double* out)
{
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (n <= lo) return ORC_OK;
    if ((n + ORC_BLOCK - 1) / ORC_BLOCK > W) return ORC_ERR_ARG;
    double m = -INFINITY;
    for (int t = lo; t < n; ++t) {
        int blk = table[t / ORC_BLOCK], off = t % ORC_BLOCK;
        if (blk < 0 || blk >= N) return ORC_ERR_INDEX;
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += qrow[j] * pool_value(k_pool, k_scale, dtype, blk, g, off, j, H_kv, d);
        s_buf[t] = scale * acc;
        if (s_buf[t] > m) m = s_buf[t];
    }
    double denom = 0.0;
    for (int t = lo; t < n; ++t) {
        int blk = table[t / ORC_BLOCK], off = t % ORC_BLOCK;
        double w = exp(s_buf[t] - m);
        denom += w;
        for (int j = 0; j < d; ++j)
            out[j] += w * pool_value(v_pool, v_scale, dtype, blk, g, off, j, H_kv, d);
    }
    for (int j = 0; j < d; ++j) out[j] /= denom;
    return ORC_OK;
}

/* Decode: one new query token per sequence attends to its whole cached context.
 * q is [B][H_q][d] (f16 or bf16), block_tables [B][W], ctx_lens [B], out [B][H_q][d].
 * [KVG] "Mechanics": GQA shares one KV head across G = H_q / H_kv query heads. */
/* Sliding-window attention ([KVB] "The KV cache": sliding-window or hybrid local/global
 * attention layers shrink what a query reads): a query at position pos sees the `window`
 * most recent positions pos - window + 1 .. pos; window 0 means no window.  For a query
 * whose keys end at n (exclusive), the first visible key is: */
static int window_start(int n, int window)
{
    return (window > 0 && n > window) ? n - window : 0;
}

int orc_paged_decode_window(int N, int H_kv, int d, int dtype,
                            const uint8_t* k_pool, const uint8_t* v_pool,
                            const float* k_scale, const float* v_scale,
                            const uint16_t* q, int q_dtype, int H_q,
                            const int32_t* block_tables, int W, const int32_t* ctx_lens, int B,
                            float scale, int window, double* out);

int orc_paged_decode(int N, int H_kv, int d, int dtype,
                     const uint8_t* k_pool, const uint8_t* v_pool,
                     const float* k_scale, const float* v_scale,
                     const uint16_t* q, int q_dtype, int H_q,
                     const int32_t* block_tables, int W, const int32_t* ctx_lens, int B,
                     float scale, double* out)
{
    return orc_paged_decode_window(N, H_kv, d, dtype, k_pool, v_pool, k_scale, v_scale, q, q_dtype, H_q,
                                   block_tables, W, ctx_lens, B, scale, 0, out);
}

/* Decode with an optional sliding window (window 0: the whole context). */
int orc_paged_decode_window(int N, int H_kv, int d, int dtype,
                            const uint8_t* k_pool, const uint8_t* v_pool,
                            const float* k_scale, const float* v_scale,
                            const uint16_t* q, int q_dtype, int H_q,
                            const int32_t* block_tables, int W, const int32_t* ctx_lens, int B,
                            float scale, int window, double* out)
{
    if (window < 0) return ORC_ERR_ARG;
    if (N <= 0 || H_kv <= 0 || d <= 0 || H_q <= 0 || B < 0 || W <= 0 || H_q % H_kv)
        return ORC_ERR_ARG;
    if (row_bytes(dtype, d) <= 0 || (q_dtype != ORC_F16 && q_dtype != ORC_BF16))
        return ORC_ERR_DTYPE;
    int max_n = 0;
    for (int b = 0; b < B; ++b) {
        if (ctx_lens[b] < 0) return ORC_ERR_ARG;
        if (ctx_lens[b] > max_n) max_n = ctx_lens[b];
    }
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_n > 0 ? max_n : 1));
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    if (!s_buf || !qrow) { free(s_buf); free(qrow); return ORC_ERR_NOMEM; }
    int G = H_q / H_kv, rc = ORC_OK;
    for (int b = 0; b < B && rc == ORC_OK; ++b)
        for (int h = 0; h < H_q && rc == ORC_OK; ++h) {
            size_t qo = ((size_t)b * H_q + h) * d;
            for (int j = 0; j < d; ++j) qrow[j] = src_value(q, q_dtype, qo + j);
            rc = attend_one(N, H_kv, d, dtype, k_pool, v_pool, k_scale, v_scale, qrow, h / G,
                            block_tables + (size_t)b * W, W, window_start(ctx_lens[b], window), ctx_lens[b],
                            (double)scale, s_buf, out + qo);
        }
    free(s_buf); free(qrow);
    return rc;
}

/* Chunked prefill ([INF] "Chunked prefill", [KVB] "Scheduling prefill and decode"):
 * C query positions P0 .. P0+C-1 of one sequence whose keys and values are already
 * in the pool.  Query row i attends causally to positions 0 .. P0+i, i.e. to the
 * earlier paged context and to its own chunk up to itself.
 * q is [C][H_q][d], block_table [W], out [C][H_q][d]. */
int orc_paged_prefill_chunk_window(int N, int H_kv, int d, int dtype,
                                   const uint8_t* k_pool, const uint8_t* v_pool,
                                   const float* k_scale, const float* v_scale,
                                   const uint16_t* q, int q_dtype, int H_q,
                                   const int32_t* block_table, int W, int ctx_before, int C,
                                   float scale, int window, double* out);

int orc_paged_prefill_chunk(int N, int H_kv, int d, int dtype,
                            const uint8_t* k_pool, const uint8_t* v_pool,
                            const float* k_scale, const float* v_scale,
                            const uint16_t* q, int q_dtype, int H_q,
                            const int32_t* block_table, int W, int ctx_before, int C,
                            float scale, double* out)
{
    return orc_paged_prefill_chunk_window(N, H_kv, d, dtype, k_pool, v_pool, k_scale, v_scale, q, q_dtype, H_q,
                                          block_table, W, ctx_before, C, scale, 0, out);
}

/* Chunked prefill with an optional sliding window: row i sees positions
 * max(0, ctx_before + i + 1 - window) .. ctx_before + i (window 0: all earlier ones). */
int orc_paged_prefill_chunk_window(int N, int H_kv, int d, int dtype,
                                   const uint8_t* k_pool, const uint8_t* v_pool,
                                   const float* k_scale, const float* v_scale,
                                   const uint16_t* q, int q_dtype, int H_q,
                                   const int32_t* block_table, int W, int ctx_before, int C,
                                   float scale, int window, double* out)
{
    if (window < 0) return ORC_ERR_ARG;
    if (N <= 0 || H_kv <= 0 || d <= 0 || H_q <= 0 || C < 0 || ctx_before < 0 || W <= 0 || H_q % H_kv)
        return ORC_ERR_ARG;
    if (row_bytes(dtype, d) <= 0 || (q_dtype != ORC_F16 && q_dtype != ORC_BF16))
        return ORC_ERR_DTYPE;
    int n_max = ctx_before + C;
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(n_max > 0 ? n_max : 1));
    double* qrow = (double*)malloc(sizeof(double) * (size_t)d);
    if (!s_buf || !qrow) { free(s_buf); free(qrow); return ORC_ERR_NOMEM; }
    int G = H_q / H_kv, rc = ORC_OK;
    for (int i = 0; i < C && rc == ORC_OK; ++i)
        for (int h = 0; h < H_q && rc == ORC_OK; ++h) {
            size_t qo = ((size_t)i * H_q + h) * d;
            for (int j = 0; j < d; ++j) qrow[j] = src_value(q, q_dtype, qo + j);
            rc = attend_one(N, H_kv, d, dtype, k_pool, v_pool, k_scale, v_scale, qrow, h / G,
                            block_table, W, window_start(ctx_before + i + 1, window), ctx_before + i + 1,
                            (double)scale, s_buf, out + qo);
        }
    free(s_buf); free(qrow);
    return rc;
}

/* ------------------------------------------------ array forms for testing -- */

void orc_e4m3_encode_array(const float* x, uint8_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_f32(x[i]);
}

void orc_e4m3_decode_array(const uint8_t* c, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_to_f64(c[i]);
}

void orc_f16_decode_array(const uint16_t* h, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f16_to_f64(h[i]);
}

void orc_bf16_decode_array(const uint16_t* h, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (double)orc_bf16_to_f32(h[i]);
}

/* Dequantized value of every element of a pool, [N][H_kv][16][d] in fp64. */
int orc_pool_dequant(int N, int H_kv, int d, int dtype, const uint8_t* pool, const float* scale, double* out)
{
    if (row_bytes(dtype, d) <= 0) return ORC_ERR_DTYPE;
    size_t o = 0;
    for (int blk = 0; blk < N; ++blk)
        for (int g = 0; g < H_kv; ++g)
            for (int off = 0; off < ORC_BLOCK; ++off)
                for (int j = 0; j < d; ++j)
                    out[o++] = pool_value(pool, scale, dtype, blk, g, off, j, H_kv, d);
    return ORC_OK;
}
