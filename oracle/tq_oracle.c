/*
 * TurboQuant paged KV cache -- CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, single-threaded
 * definition that the CUDA library is checked against.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load it; the
 * product path (libtq.so and its Python binding) never does, and the two
 * share no code, header, table or helper.
 *
 * Method source: "xInfer: Pure-Rust LLM Inference Without a Python Runtime",
 * section "What actually sits between the request and the tokens": the KV
 * cache is compressed by a Walsh-Hadamard rotation followed by per-head
 * absmax quantisation to a 2-4 bit cache; section "TurboQuant is a memory
 * trade": reading the cache dequantises on every attention step, and the
 * --kvcache-dtype flag selects turbo8 / turbo4 / turbo3 (no flag = BF16).
 * The paged layout follows "infero", section "Continuous batching"
 * (requests share the GPU over a paged KV cache).
 *
 * The pages leave the arithmetic open; this oracle fixes it as follows:
 *   rotation   y = H_d x / sqrt(d), H_d Sylvester-ordered, computed as fp32
 *              butterflies with strides h = 1, 2, 4, ..., d/2 (each butterfly
 *              (a, b) -> (a + b, a - b), lower index first), then ONE fp32
 *              multiply by c = fp32(1 / sqrt(d)).  Built with
 *              -ffp-contract=off, so no multiply-add is fused.
 *   scale      s = max_i |y_i| (fp32), stored as fp32.
 *   codes      L = 2^(b-1) - 1; t_i = fp32(y_i * L); code_i =
 *              clamp(roundf(t_i / s), -L, L) with an IEEE fp32 division and
 *              rounding half away from zero; s == 0 gives all codes 0.
 *   storage    u_i = code_i + L (offset binary), bit-packed LSB-first: u_i
 *              occupies bits [i*b, (i+1)*b) of a little-endian byte string.
 *   dequant    yhat_i = code_i * s / L in fp64.
 *   attention  qt = H q / sqrt(d); score_j = qt . yhat_k,j / sqrt(d);
 *              p = softmax over the visible keys (max-subtracted);
 *              out = H (sum_j p_j yhat_v,j) / sqrt(d); all in fp64.
 *   causality  query position t of q_len sees keys j <= seq_len - q_len + t.
 *   GQA        query head h reads kv head h / (num_q_heads / num_kv_heads).
 *
 * fp8 (format 17, the --kvcache-dtype fp8 choice of the xInfer page; the
 * pages give only "fp8", "2x" and "near-lossless", this oracle fixes it):
 *   codes      OCP E4M3 (1 sign, 4 exponent bits of bias 7, 3 mantissa bits,
 *              no infinities, largest finite 448); no rotation.
 *   scale      s = max_i |x_i| (fp32), stored as fp32; s == 0 gives codes 0.
 *   codes      y_i = fl(fl(x_i * 448) / s) (IEEE fp32), code_i = the E4M3
 *              value nearest y_i, ties to the even code, |y_i| > 448 to 448.
 *   storage    one byte per code (the E4M3 bit pattern), in the block layout
 *              of turbo8.
 *   dequant    xhat_i = value(code_i) * s / 448 in fp64; attention as for
 *              BF16 (no rotation) on the dequantised K and V.
 *
 * Cache layout (an interface, described in include/tq.h, implemented here
 * independently): blocks are ordered [page][kv_head].  For a turbo format
 * with b bits and page size P, a K block holds P token rows of d*b/8 code
 * bytes (row t = token t's packed vector as above) followed by P fp32
 * scales.  A V block holds the same codes dim-major: d rows of P*b/8 bytes,
 * row i packing the P tokens' codes of dimension i LSB-first (token t at
 * bits [t*b, (t+1)*b) of the row), followed by the P fp32 scales.  For BF16
 * each block holds P token rows of d bf16 values.  slot = page * P + offset.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

enum { OR_OK = 0, OR_BAD_ARG = -1, OR_BAD_PAGE = -2, OR_BAD_SLOT = -3 };

static float bf16_to_f32(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

enum { FORMAT_FP8 = 17 };

/* number of code bits of a turbo or fp8 format, 0 for bf16, -1 if unknown */
static int format_bits(int format)
{
    switch (format) {
    case 2: case 3: case 4: case 8: return format;
    case FORMAT_FP8: return 8;
    case 16: return 0;
    default: return -1;
    }
}

/* Value of an E4M3 code (OCP "e4m3fn": 0x7F and 0xFF are NaN). */
ORACLE_API double oracle_e4m3_value(uint8_t c)
{
    const int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* The E4M3 code nearest y, found by comparing y with every finite
 * non-negative code; a tie goes to the code with an even mantissa; |y|
 * above the largest finite value (448), infinity included, gives 448 (the
 * format saturates); NaN gives the NaN code 0x7F.  The sign of y is kept
 * (-0 gives 0x80). */
ORACLE_API uint8_t oracle_e4m3_encode(float y)
{
    const uint8_t sgn = signbit(y) ? 0x80 : 0x00;
    const double a = fabs((double)y);
    if (isnan(a)) return (uint8_t)(sgn | 0x7F);
    if (a > 448.0) return (uint8_t)(sgn | 0x7E);   /* every finite code is nearer than inf */
    int best = 0;
    double best_d = a;                          /* code 0: value 0 */
    for (int c = 1; c <= 0x7E; ++c) {
        const double dd = fabs(a - oracle_e4m3_value((uint8_t)c));
        if (dd < best_d || (dd == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = dd;
        }
    }
    return (uint8_t)(sgn | best);
}

/* fp8 codes and scale of one bf16 head vector (no rotation). */
ORACLE_API void oracle_fp8_quantize_vector(const uint16_t* x_bf16, int d, uint8_t* codes,
                                           float* scale)
{
    float s = 0.0f;
    for (int i = 0; i < d; ++i) {
        float a = fabsf(bf16_to_f32(x_bf16[i]));
        if (a > s) s = a;
    }
    for (int i = 0; i < d; ++i) {
        if (s == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float t = bf16_to_f32(x_bf16[i]) * 448.0f;
        codes[i] = oracle_e4m3_encode(t / s);
    }
    *scale = s;
}

static int64_t oracle_block_bytes_impl(int format, int d, int page_size)
{
    int b = format_bits(format);
    if (b < 0 || d <= 0 || page_size <= 0) return -1;
    if (b == 0) return (int64_t)page_size * d * 2;
    if ((d * b) % 8 != 0) return -1;
    return (int64_t)page_size * (d * b / 8 + 4);
}

ORACLE_API int64_t oracle_block_bytes(int format, int d, int page_size)
{
    return oracle_block_bytes_impl(format, d, page_size);
}

/* Unnormalised Sylvester Walsh-Hadamard transform, fp32, in place. */
ORACLE_API void oracle_fwht_f32(float* x, int d)
{
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = x[j];
                float b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
}

/* The same transform in fp64 (used by the attention side). */
ORACLE_API void oracle_fwht_f64(double* x, int d)
{
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = x[j];
                double b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
}

/* y = H x / sqrt(d) for one bf16 head vector, fp32 as described above. */
ORACLE_API void oracle_rotate_f32(const uint16_t* x_bf16, int d, float* y)
{
    for (int i = 0; i < d; ++i) y[i] = bf16_to_f32(x_bf16[i]);
    oracle_fwht_f32(y, d);
    const float c = (float)(1.0 / sqrt((double)d));
    for (int i = 0; i < d; ++i) y[i] = y[i] * c;
}

/* Absmax quantisation of an already rotated vector. */
ORACLE_API void oracle_quantize_rotated(const float* y, int d, int bits,
                                        int32_t* codes, float* scale)
{
    const int L = (1 << (bits - 1)) - 1;
    float s = 0.0f;
    for (int i = 0; i < d; ++i) {
        float a = fabsf(y[i]);
        if (a > s) s = a;
    }
    for (int i = 0; i < d; ++i) {
        if (s == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float t = y[i] * (float)L;
        float r = roundf(t / s);
        if (r > (float)L) r = (float)L;
        if (r < -(float)L) r = -(float)L;
        codes[i] = (int32_t)r;
    }
    *scale = s;
}

/* Offset-binary, LSB-first bit packing of d codes into d*bits/8 bytes. */
ORACLE_API void oracle_pack_codes(const int32_t* codes, int d, int bits,
                                  uint8_t* out)
{
    const int L = (1 << (bits - 1)) - 1;
    memset(out, 0, (size_t)(d * bits / 8));
    for (int i = 0; i < d; ++i) {
        uint32_t u = (uint32_t)(codes[i] + L);
        for (int k = 0; k < bits; ++k) {
            int bit = i * bits + k;
            if ((u >> k) & 1u) out[bit / 8] |= (uint8_t)(1u << (bit % 8));
        }
    }
}

ORACLE_API void oracle_unpack_codes(const uint8_t* in, int d, int bits,
                                    int32_t* codes)
{
    const int L = (1 << (bits - 1)) - 1;
    for (int i = 0; i < d; ++i) {
        uint32_t u = 0;
        for (int k = 0; k < bits; ++k) {
            int bit = i * bits + k;
            u |= (uint32_t)((in[bit / 8] >> (bit % 8)) & 1u) << k;
        }
        codes[i] = (int32_t)u - L;
    }
}

/* Write / read an nbits-wide unsigned field at bit position `bit` of a
 * little-endian byte string, one bit at a time. */
static void put_bits(uint8_t* base, int64_t bit, int nbits, uint32_t value)
{
    for (int k = 0; k < nbits; ++k) {
        int64_t b = bit + k;
        uint8_t m = (uint8_t)(1u << (b % 8));
        if ((value >> k) & 1u) base[b / 8] |= m;
        else base[b / 8] &= (uint8_t)~m;
    }
}

static uint32_t get_bits(const uint8_t* base, int64_t bit, int nbits)
{
    uint32_t v = 0;
    for (int k = 0; k < nbits; ++k) {
        int64_t b = bit + k;
        v |= (uint32_t)((base[b / 8] >> (b % 8)) & 1u) << k;
    }
    return v;
}

/* Rotate, quantise and pack one bf16 head vector. */
ORACLE_API void oracle_quantize_vector(const uint16_t* x_bf16, int d, int bits,
                                       uint8_t* packed, float* scale)
{
    float* y = (float*)malloc(sizeof(float) * (size_t)d);
    int32_t* codes = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
    oracle_rotate_f32(x_bf16, d, y);
    oracle_quantize_rotated(y, d, bits, codes, scale);
    oracle_pack_codes(codes, d, bits, packed);
    free(codes);
    free(y);
}

/*
 * Quantise and append num_tokens new K and V rows ([token][kv_head][d] bf16)
 * into the paged cache.  slot < 0 skips the token.
 */
ORACLE_API int oracle_quantize_append(const uint16_t* k, const uint16_t* v,
                                      const int64_t* slot_mapping,
                                      int num_tokens, int num_kv_heads, int d,
                                      int format, int page_size, int num_pages,
                                      uint8_t* k_pages, uint8_t* v_pages)
{
    if (format_bits(format) <= 0) return OR_BAD_ARG;
    int64_t bb = oracle_block_bytes_impl(format, d, page_size);
    if (bb < 0) return OR_BAD_ARG;
    const int bits = format_bits(format);
    const int fp8 = format == FORMAT_FP8;
    const int cb = d * bits / 8;
    float* y = (float*)malloc(sizeof(float) * (size_t)d);
    int32_t* codes = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);
    int rc = OR_OK;
    for (int t = 0; t < num_tokens && rc == OR_OK; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t page = slot / page_size;
        int64_t off = slot % page_size;
        if (page >= num_pages) { rc = OR_BAD_SLOT; break; }
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t blk = (size_t)((page * num_kv_heads + h) * bb);
            const uint16_t* kx = k + ((size_t)t * num_kv_heads + h) * d;
            const uint16_t* vx = v + ((size_t)t * num_kv_heads + h) * d;
            float ks, vs;
            if (fp8) {
                /* K: row `off` holds the token's d code bytes; V: byte `off`
                   of dimension row i holds code i */
                oracle_fp8_quantize_vector(kx, d, k_pages + blk + off * cb, &ks);
                uint8_t* vc = (uint8_t*)malloc((size_t)d);
                oracle_fp8_quantize_vector(vx, d, vc, &vs);
                for (int i = 0; i < d; ++i) v_pages[blk + (size_t)i * page_size + off] = vc[i];
                free(vc);
            } else {
                /* K: the token's packed vector is row `off` of the block */
                oracle_quantize_vector(kx, d, bits, k_pages + blk + off * cb, &ks);
                /* V: code i goes to row i (dim-major), field `off` */
                oracle_rotate_f32(vx, d, y);
                oracle_quantize_rotated(y, d, bits, codes, &vs);
                const int L = (1 << (bits - 1)) - 1;
                for (int i = 0; i < d; ++i)
                    put_bits(v_pages + blk, (int64_t)i * page_size * bits + (int64_t)off * bits,
                             bits, (uint32_t)(codes[i] + L));
            }
            memcpy(k_pages + blk + (size_t)page_size * cb + off * 4, &ks, 4);
            memcpy(v_pages + blk + (size_t)page_size * cb + off * 4, &vs, 4);
        }
    }
    free(codes);
    free(y);
    return rc;
}

/* Store bf16 rows unchanged into a BF16 paged cache. */
ORACLE_API int oracle_append_bf16(const uint16_t* k, const uint16_t* v,
                                  const int64_t* slot_mapping, int num_tokens,
                                  int num_kv_heads, int d, int page_size,
                                  int num_pages, uint16_t* k_pages,
                                  uint16_t* v_pages)
{
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t page = slot / page_size;
        int64_t off = slot % page_size;
        if (page >= num_pages) return OR_BAD_SLOT;
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t row = ((size_t)(page * num_kv_heads + h) * page_size + off) * d;
            memcpy(k_pages + row, k + ((size_t)t * num_kv_heads + h) * d, 2 * (size_t)d);
            memcpy(v_pages + row, v + ((size_t)t * num_kv_heads + h) * d, 2 * (size_t)d);
        }
    }
    return OR_OK;
}

/* Dequantised (still rotated) head vector of one cached token, fp64.
 * dim_major selects the V block layout (dimension rows of token fields). */
static void dequant_token(const uint8_t* pages, int64_t bb, int page, int kvh,
                          int num_kv_heads, int off, int page_size, int d,
                          int bits, int dim_major, int fp8, int32_t* codes, double* out)
{
    const int L = (1 << (bits - 1)) - 1;
    const int cb = d * bits / 8;
    const uint8_t* blk = pages + (size_t)(((int64_t)page * num_kv_heads + kvh) * bb);
    float s;
    memcpy(&s, blk + (size_t)page_size * cb + (size_t)off * 4, 4);
    if (fp8) {
        for (int i = 0; i < d; ++i) {
            const uint8_t c = dim_major ? blk[(size_t)i * page_size + off] : blk[(size_t)off * cb + i];
            out[i] = oracle_e4m3_value(c) * (double)s / 448.0;
        }
        return;
    }
    if (dim_major) {
        for (int i = 0; i < d; ++i)
            codes[i] = (int32_t)get_bits(blk, (int64_t)i * page_size * bits +
                                                  (int64_t)off * bits, bits) - L;
    } else {
        oracle_unpack_codes(blk + (size_t)off * cb, d, bits, codes);
    }
    for (int i = 0; i < d; ++i)
        out[i] = (double)codes[i] * (double)s / (double)L;
}

static void bf16_token(const uint16_t* pages, int page, int kvh,
                       int num_kv_heads, int off, int page_size, int d,
                       double* out)
{
    const uint16_t* row =
        pages + ((size_t)((int64_t)page * num_kv_heads + kvh) * page_size + off) * d;
    for (int i = 0; i < d; ++i) out[i] = (double)bf16_to_f32(row[i]);
}

static int check_decode_args(int format, int d, int num_kv_heads, int page_size,
                             int num_q_heads, int q_len, int batch)
{
    if (format_bits(format) < 0) return OR_BAD_ARG;
    if (d <= 0 || (d & (d - 1)) != 0) return OR_BAD_ARG;
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads)
        return OR_BAD_ARG;
    if (page_size <= 0 || q_len <= 0 || batch < 0) return OR_BAD_ARG;
    return OR_OK;
}

/*
 * Attention of one query row over n keys, fp64.
 *   rotated == 0: out = sum_j softmax_j(q . k_j / sqrt(d)) v_j.
 *   rotated == 1: K and V hold rotated vectors; qt = H q / sqrt(d),
 *                 score_j = qt . k_j / sqrt(d), out = H (sum_j p_j v_j) / sqrt(d).
 * K, V: [n][d] row-major.  n >= 1.
 */
ORACLE_API void oracle_attention_f64(const double* q, const double* K,
                                     const double* V, int n, int d,
                                     int rotated, double* out)
{
    const double rs = 1.0 / sqrt((double)d);
    double* qt = (double*)malloc(sizeof(double) * (size_t)d);
    double* w = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int i = 0; i < d; ++i) qt[i] = q[i];
    if (rotated) {
        oracle_fwht_f64(qt, d);
        for (int i = 0; i < d; ++i) qt[i] *= rs;
    }
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int i = 0; i < d; ++i) dot += qt[i] * K[(size_t)j * d + i];
        w[j] = dot * rs;
        if (w[j] > m) m = w[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        w[j] = exp(w[j] - m);
        l += w[j];
    }
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    for (int j = 0; j < n; ++j) {
        const double p = w[j] / l;
        for (int i = 0; i < d; ++i) out[i] += p * V[(size_t)j * d + i];
    }
    if (rotated) {
        oracle_fwht_f64(out, d);
        for (int i = 0; i < d; ++i) out[i] *= rs;
    }
    free(w);
    free(qt);
}

/*
 * Decode attention over the paged cache.  q: [batch][q_len][num_q_heads][d]
 * bf16.  seq_lens[b] counts the cached keys of sequence b, the q_len new
 * tokens included.  out: [batch][q_len][num_q_heads][d] fp64.
 * format 2/3/4/8 reads a turbo cache (dequantise, attend in the rotated
 * basis, rotate back); format 16 reads a BF16 cache with plain
 * softmax(q k / sqrt(d)) v attention.
 */
ORACLE_API int oracle_paged_decode(const uint16_t* q, int format, int d,
                                   int num_kv_heads, int page_size,
                                   int num_pages, const void* k_pages,
                                   const void* v_pages,
                                   const int32_t* page_table,
                                   int max_pages_per_seq,
                                   const int32_t* seq_lens, int batch,
                                   int q_len, int num_q_heads, double* out)
{
    int rc = check_decode_args(format, d, num_kv_heads, page_size, num_q_heads,
                               q_len, batch);
    if (rc) return rc;
    const int bits = format_bits(format);
    const int64_t bb = oracle_block_bytes_impl(format, d, page_size);
    const int group = num_q_heads / num_kv_heads;

    int max_len = 1;
    for (int b = 0; b < batch; ++b)
        if (seq_lens[b] > max_len) max_len = seq_lens[b];
    double* K = (double*)malloc(sizeof(double) * (size_t)max_len * d);
    double* V = (double*)malloc(sizeof(double) * (size_t)max_len * d);
    double* qx = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t* codes = (int32_t*)malloc(sizeof(int32_t) * (size_t)d);

    rc = OR_OK;
    for (int b = 0; b < batch && rc == OR_OK; ++b) {
        const int n = seq_lens[b];
        if (n < q_len || (n + page_size - 1) / page_size > max_pages_per_seq) {
            rc = OR_BAD_ARG;
            break;
        }
        for (int t = 0; t < q_len && rc == OR_OK; ++t) {
            const int visible = n - q_len + t + 1; /* keys 0 .. n-q_len+t */
            for (int h = 0; h < num_q_heads && rc == OR_OK; ++h) {
                const int kvh = h / group;
                for (int j = 0; j < visible; ++j) {
                    int page = page_table[(size_t)b * max_pages_per_seq + j / page_size];
                    if (page < 0 || page >= num_pages) { rc = OR_BAD_PAGE; break; }
                    double* kr = K + (size_t)j * d;
                    double* vr = V + (size_t)j * d;
                    if (bits > 0) {
                        dequant_token((const uint8_t*)k_pages, bb, page, kvh,
                                      num_kv_heads, j % page_size, page_size, d,
                                      bits, 0, format == FORMAT_FP8, codes, kr);
                        dequant_token((const uint8_t*)v_pages, bb, page, kvh,
                                      num_kv_heads, j % page_size, page_size, d,
                                      bits, 1, format == FORMAT_FP8, codes, vr);
                    } else {
                        bf16_token((const uint16_t*)k_pages, page, kvh,
                                   num_kv_heads, j % page_size, page_size, d, kr);
                        bf16_token((const uint16_t*)v_pages, page, kvh,
                                   num_kv_heads, j % page_size, page_size, d, vr);
                    }
                }
                if (rc != OR_OK) break;
                const uint16_t* qb = q + (((size_t)b * q_len + t) * num_q_heads + h) * d;
                for (int i = 0; i < d; ++i) qx[i] = (double)bf16_to_f32(qb[i]);
                double* dst = out + (((size_t)b * q_len + t) * num_q_heads + h) * d;
                /* turbo formats attend in the rotated basis; fp8 and bf16 do not */
                oracle_attention_f64(qx, K, V, visible, d, bits > 0 && format != FORMAT_FP8, dst);
            }
        }
    }
    free(codes);
    free(qx);
    free(V);
    free(K);
    return rc;
}
