/*
 * kvq_oracle.c -- plain, slow, float64 CPU oracle for the transformed-KV write path
 * (quantize-append) and read path (decode attention).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code, header,
 * table or constant with the CUDA library; the product never calls it.
 *
 * What it computes, and where the pages state it:
 *   - "WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms" (paperlayer
 *     summary), section 1 and section 4.2: one dense d x d key transform per KV head,
 *     applied after RoPE to every new key; the matching query-side compensation
 *     T^{-T} q; a per-KV-head value transform (folded into the weights on the real
 *     model, applied to the synthetic values here).
 *   - same page, section 5.3 and the abstract: OSCAR-style percentile-clipped affine
 *     quantization of the transformed cache at 2 bits (4 bits also supported).
 *   - same page, section 4.1: grouped-query attention, each KV head read by a group
 *     of query heads, over all cached positions.
 *   - "Spend Bits Where Queries Look" (NOVA-KV project page), "Three requirements",
 *     item 3: every token occupies the same number of bits (fixed-width layout).
 *   - WUSH-KV page, section 4.4: the full-precision window (first S_sink and newest
 *     S_keep positions kept in full precision, the middle quantized in batches of
 *     S_flush) -- the decode over such a sequence.
 *   - WUSH-KV page, section 4.3: the QuEST INT quantizer (RMS-based clipped levels).
 *   - "Spend Bits Where Queries Look" (NOVA-KV project page): the vector-quantized cache
 *     (codebook lookup plus one multiply on the read path).
 * Every step the pages leave open is stated next to the code that fixes it.
 *
 * Arithmetic: all transform and attention arithmetic is float64. Where the quantizer
 * prescribes float32 operations (the step size, the scaled value) each one is done
 * as the float64 operation on float32 operands rounded back to float32; because
 * 53 >= 2*24 + 2 this equals the IEEE float32 result for +, -, *, /. float16
 * conversion is round-to-nearest-even, written out below from the binary16 format.
 *
 * Pinned by tests/test_oracle.py (closed forms, brute force, invariants, hand-worked
 * fixtures under tests/golden/).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ scalar types */

/* binary32 -> binary16, round to nearest, ties to even; overflow -> inf; NaN kept. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t ex = (u >> 23) & 0xFFu;
    uint32_t man = u & 0x7FFFFFu;
    if (ex == 0xFFu)                                  /* inf or NaN */
        return (uint16_t)(sign | 0x7C00u | (man ? 0x200u : 0u));
    /* value = 1.man * 2^(ex-127) for normals, 0.man * 2^-126 for subnormals */
    int e = (int)ex - 127;
    if (ex == 0) {
        /* float32 subnormals are below 2^-126, far under half the smallest f16
         * subnormal (2^-25): they round to zero. */
        return sign;
    }
    uint32_t sig = man | 0x800000u;                   /* 24-bit significand, value sig*2^(e-23) */
    if (e > 15)
        return (uint16_t)(sign | 0x7C00u);            /* overflow */
    int shift;                                        /* bits of sig dropped */
    uint32_t base;                                    /* exponent field before rounding */
    if (e >= -14) {                                   /* f16 normal range */
        shift = 13;
        base = (uint32_t)(e + 15);
    } else {                                          /* f16 subnormal: units of 2^-24 */
        shift = 13 + (-14 - e);
        base = 0;
        if (shift > 24 + 1)                           /* below half of 2^-24 */
            return sign;
    }
    uint32_t kept = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (kept & 1u)))
        kept += 1;
    uint32_t h;
    if (base == 0) {
        h = kept;                                     /* may carry into the normal range */
    } else {
        /* kept holds the hidden bit at position 10; a carry to bit 11 bumps the exponent */
        h = (base << 10) + (kept - 0x400u);
        if (h >= 0x7C00u)
            h = 0x7C00u;
    }
    return (uint16_t)(sign | h);
}

double oracle_f16_to_f64(uint16_t h)
{
    int s = (h >> 15) & 1;
    int ex = (h >> 10) & 0x1F;
    int man = h & 0x3FF;
    double v;
    if (ex == 0)
        v = ldexp((double)man, -24);
    else if (ex == 31)
        v = man ? NAN : INFINITY;
    else
        v = ldexp((double)(man | 0x400), ex - 25);
    return s ? -v : v;
}

double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------------ clip index */

/* Order-statistic index kappa for "percentile clipping" with ratio alpha over a
 * group of g values: kappa = floor(alpha * (g - 1)), 0-indexed ascending, clip range
 * [x_(kappa), x_(g-1-kappa)] (WUSH-KV summary, section 5.3: percentile-clipped affine
 * quantizer; the pages give no formula, this is the plain "lower/higher" percentile). */
int oracle_kappa(float clip_alpha, int g)
{
    double k = floor((double)clip_alpha * (double)(g - 1));
    if (k < 0)
        k = 0;
    return (int)k;
}

/* ------------------------------------------------------------------ transform */

/* out_i = sum_j T[i][j] x_j in float64; T == NULL is the identity. */
void oracle_matvec(const double *T, const double *x, int d, double *out)
{
    for (int i = 0; i < d; ++i) {
        if (!T) {
            out[i] = x[i];
            continue;
        }
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += T[(size_t)i * d + j] * x[j];
        out[i] = acc;
    }
}

/* ------------------------------------------------------------------ quantizer */

static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

static float f32(double x) { return (float)x; }

/* Quantize one group of g float32 values (OSCAR-style percentile-clipped affine):
 *   lo = x_(kappa), hi = x_(g-1-kappa)           (sorted ascending, 0-indexed)
 *   s  = f32( f32(hi - lo) / (2^b - 1) )          IEEE float32 division
 *   s_h = f16(s), z_h = f16(lo)                   float16 scale and zero-point
 *   c  = clamp( rint( f32( f32(x - z) / s ) ), 0, 2^b - 1 )  with z, s read back from f16
 * rint is round-half-to-even. If s_h == 0 every code is 0 (the group dequantizes to z).
 * There is no separate pre-clip of x: the final integer clamp realises the clipping. */
void oracle_quantize_group(const float *x, int g, int bits, int kappa,
                           uint8_t *codes, uint16_t *s_h, uint16_t *z_h)
{
    double *sorted = (double *)malloc(sizeof(double) * (size_t)g);
    for (int i = 0; i < g; ++i)
        sorted[i] = (double)x[i];
    qsort(sorted, (size_t)g, sizeof(double), cmp_double);
    float lo = (float)sorted[kappa];
    float hi = (float)sorted[g - 1 - kappa];
    free(sorted);
    int qmax = (1 << bits) - 1;
    float range = f32((double)hi - (double)lo);
    float s = f32((double)range / (double)qmax);
    uint16_t sh = oracle_f32_to_f16(s);
    uint16_t zh = oracle_f32_to_f16(lo);
    double sf = oracle_f16_to_f64(sh), zf = oracle_f16_to_f64(zh);
    for (int i = 0; i < g; ++i) {
        int c = 0;
        if (sf != 0.0) {
            float diff = f32((double)x[i] - zf);
            float y = f32((double)diff / sf);
            double r = rint((double)y);
            if (r < 0)
                r = 0;
            if (r > qmax)
                r = qmax;
            c = (int)r;
        }
        codes[i] = (uint8_t)c;
    }
    *s_h = sh;
    *z_h = zh;
}

/*
 * QuEST INT quantizer ("WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms",
 * section 4.3 and the attention-stage comparison of section 5.1): each token's group of
 * channels is quantized with RMS-based clipped levels. The page gives no constants; the
 * reading here: a symmetric uniform grid of 2^b levels at (c - (2^b - 1)/2) * step,
 * c = 0 .. 2^b - 1, with step = delta_b * RMS(x), delta_b the uniform step that minimises
 * the mean squared error for a unit Gaussian (Max, 1960: 0.9957 for 4 levels, 0.3352 for
 * 16 levels); values beyond the outer levels clip to them. In the cache's affine form:
 *   ms  = sum_j x_j^2 / g                      (float64)
 *   rms = f32(sqrt(ms))
 *   s   = f32(rms * delta_b)                   (float32 product, delta_b a float32 constant)
 *   s_h = f16(s),  z_h = f16(-(2^b - 1)/2 * s_h)   (the product is exact in float32)
 *   c   = clamp(rint(f32(f32(x - z) / s)), 0, 2^b - 1) with z, s read back from f16, as
 *         the percentile quantizer; s_h == 0 gives all codes 0.
 * The decode is unchanged: x^ = z_h + c s_h.
 */
float oracle_quest_delta(int bits)
{
    return bits == 2 ? 0.9957f : bits == 4 ? 0.3352f : 0.0f;
}

void oracle_quantize_group_quest(const float *x, int g, int bits, uint8_t *codes, uint16_t *s_h,
                                 uint16_t *z_h)
{
    double ms = 0.0;
    for (int i = 0; i < g; ++i)
        ms += (double)x[i] * (double)x[i];
    ms /= (double)g;
    float rms = (float)sqrt(ms);
    int qmax = (1 << bits) - 1;
    float s = f32((double)rms * (double)oracle_quest_delta(bits));
    uint16_t sh = oracle_f32_to_f16(s);
    double sf = oracle_f16_to_f64(sh);
    float zq = f32(-0.5 * (double)qmax * sf);
    uint16_t zh = oracle_f32_to_f16(zq);
    double zf = oracle_f16_to_f64(zh);
    for (int i = 0; i < g; ++i) {
        int c = 0;
        if (sf != 0.0) {
            float diff = f32((double)x[i] - zf);
            float y = f32((double)diff / sf);
            double r = rint((double)y);
            if (r < 0)
                r = 0;
            if (r > qmax)
                r = qmax;
            c = (int)r;
        }
        codes[i] = (uint8_t)c;
    }
    *s_h = sh;
    *z_h = zh;
}

/* ------------------------------------------------------------------ cache layout */
/*
 * Fixed width per token ("Spend Bits Where Queries Look", Three requirements, item 3).
 * The pages fix no bit order; this library's cache format is:
 *
 * K codes plane, [B][Hkv][T_cap][d*bk/8] bytes: one row per token, element j at bit
 *   bk*j of the row (byte floor(bk*j/8), bit bk*j mod 8, little-endian).
 * V codes plane, [B][Hkv][T_cap/16][16*d*bv/8] bytes: tiles of 16 tokens. A tile is
 *   32 lane chunks of 2*d*bv/32 bytes. Lane L = 4*gq + tq holds tokens
 *   {tq, tq+4, tq+8, tq+12} x dims {8n + gq}. Inside a chunk, 32-bit little-endian
 *   words; with E = 16/bv codes per 16-bit half and W = d/(8E) words per token pair,
 *   word p*W + r holds, in its low half, token tq+4p and, in its high half, token
 *   tq+4p+8; half slot s (bits bv*s) holds dim 8*(E*r + s) + gq.
 * Scale/zero planes, [B][Hkv][T_cap][d/group] x 2 float16: (s, z) pairs, s first.
 */
size_t oracle_k_row_bytes(int d, int bits) { return (size_t)d * bits / 8; }

void oracle_k_code_pos(int d, int bits, int j, size_t *byte, int *bit)
{
    (void)d;
    size_t b = (size_t)bits * j;
    *byte = b / 8;
    *bit = (int)(b % 8);
}

void oracle_v_code_pos(int d, int bits, int tok, int j, size_t *byte, int *bit)
{
    int E = 16 / bits;
    int W = d / (8 * E);
    int chunk = 2 * d * bits / 32;                    /* bytes per lane chunk */
    int n = j / 8, gq = j % 8;
    int tq = tok % 4, p = (tok / 4) % 2, hi = tok / 8;
    int lane = 4 * gq + tq;
    int r = n / E, s = n % E;
    int word = p * W + r;
    int bitpos = 16 * hi + bits * s;
    *byte = (size_t)lane * chunk + (size_t)word * 4 + (size_t)(bitpos / 8);
    *bit = bitpos % 8;
}

static void put_code(uint8_t *base, size_t byte, int bit, int bits, int c)
{
    uint8_t m = (uint8_t)(((1 << bits) - 1) << bit);
    base[byte] = (uint8_t)((base[byte] & ~m) | ((c << bit) & m));
}

static int get_code(const uint8_t *base, size_t byte, int bit, int bits)
{
    return (base[byte] >> bit) & ((1 << bits) - 1);
}

/* Pack / unpack the d codes of one token into its K row. */
void oracle_pack_k_row(const uint8_t *codes, int d, int bits, uint8_t *row)
{
    for (int j = 0; j < d; ++j) {
        size_t by;
        int bi;
        oracle_k_code_pos(d, bits, j, &by, &bi);
        put_code(row, by, bi, bits, codes[j]);
    }
}

void oracle_unpack_k_row(const uint8_t *row, int d, int bits, uint8_t *codes)
{
    for (int j = 0; j < d; ++j) {
        size_t by;
        int bi;
        oracle_k_code_pos(d, bits, j, &by, &bi);
        codes[j] = (uint8_t)get_code(row, by, bi, bits);
    }
}

/* Pack / unpack the codes of token tok (0..15) of a 16-token V tile. */
void oracle_pack_v_token(const uint8_t *codes, int d, int bits, int tok, uint8_t *tile)
{
    for (int j = 0; j < d; ++j) {
        size_t by;
        int bi;
        oracle_v_code_pos(d, bits, tok, j, &by, &bi);
        put_code(tile, by, bi, bits, codes[j]);
    }
}

void oracle_unpack_v_token(const uint8_t *tile, int d, int bits, int tok, uint8_t *codes)
{
    for (int j = 0; j < d; ++j) {
        size_t by;
        int bi;
        oracle_v_code_pos(d, bits, tok, j, &by, &bi);
        codes[j] = (uint8_t)get_code(tile, by, bi, bits);
    }
}

typedef struct {
    int B, Hkv, T_cap, d, bits_k, bits_v, group;
    uint8_t *k_codes, *v_codes;      /* planes as laid out above */
    uint16_t *k_sz, *v_sz;
} oracle_cache;

static size_t kv_index(const oracle_cache *c, int b, int h)
{
    return (size_t)b * c->Hkv + h;
}

static uint8_t *k_row_ptr(const oracle_cache *c, int b, int h, int t)
{
    size_t rb = oracle_k_row_bytes(c->d, c->bits_k);
    return c->k_codes + (kv_index(c, b, h) * c->T_cap + t) * rb;
}

static uint8_t *v_tile_ptr(const oracle_cache *c, int b, int h, int t)
{
    size_t tile = (size_t)16 * c->d * c->bits_v / 8;
    return c->v_codes + (kv_index(c, b, h) * (c->T_cap / 16) + t / 16) * tile;
}

static uint16_t *sz_ptr(const oracle_cache *c, uint16_t *plane, int b, int h, int t)
{
    int ng = c->d / c->group;
    return plane + ((kv_index(c, b, h) * c->T_cap + t) * ng) * 2;
}

/* Write one quantized token (codes for d dims, ng (s,z) pairs) for K or V. */
static void store_token(const oracle_cache *c, int which_v, int b, int h, int t,
                        const uint8_t *codes, const uint16_t *sz)
{
    int ng = c->d / c->group;
    if (!which_v) {
        oracle_pack_k_row(codes, c->d, c->bits_k, k_row_ptr(c, b, h, t));
        memcpy(sz_ptr(c, c->k_sz, b, h, t), sz, sizeof(uint16_t) * 2 * ng);
    } else {
        oracle_pack_v_token(codes, c->d, c->bits_v, t % 16, v_tile_ptr(c, b, h, t));
        memcpy(sz_ptr(c, c->v_sz, b, h, t), sz, sizeof(uint16_t) * 2 * ng);
    }
}

/* Dequantized value of one cached token: xhat_j = z + c_j * s (exact in float64). */
static void load_token(const oracle_cache *c, int which_v, int b, int h, int t, double *xhat)
{
    int d = c->d, ng = d / c->group;
    uint8_t codes[1024];
    const uint16_t *sz;
    if (!which_v) {
        oracle_unpack_k_row(k_row_ptr(c, b, h, t), d, c->bits_k, codes);
        sz = sz_ptr(c, c->k_sz, b, h, t);
    } else {
        oracle_unpack_v_token(v_tile_ptr(c, b, h, t), d, c->bits_v, t % 16, codes);
        sz = sz_ptr(c, c->v_sz, b, h, t);
    }
    for (int gr = 0; gr < ng; ++gr) {
        double s = oracle_f16_to_f64(sz[2 * gr]);
        double z = oracle_f16_to_f64(sz[2 * gr + 1]);
        for (int j = gr * c->group; j < (gr + 1) * c->group; ++j)
            xhat[j] = z + (double)codes[j] * s;
    }
}

/* ------------------------------------------------------------------ write path */

static double load_in(const void *p, int dtype, size_t i)
{
    if (dtype == 0)
        return (double)((const float *)p)[i];
    return oracle_bf16_to_f64(((const uint16_t *)p)[i]);
}

/*
 * Quantize-append: for each sequence b, new tokens i = 0..n-1 go to positions
 * pos[b] + i. For every (b, token, KV head): x~ = f32(T x) in float64 (T_k for keys,
 * T_v for values; NULL = identity), then per group of `group` dims the clipped
 * affine quantizer above, then the fixed-width store.
 * Inputs k, v: [B][n][Hkv][d], dtype 0 = float32, 1 = bfloat16 bits.
 * T_k, T_v: [Hkv][d][d] float32 row-major (x~_i = sum_j T[i][j] x_j).
 * kt_out / vt_out (nullable): the float32 transformed inputs, [B][n][Hkv][d].
 * Returns 0, or -1 on an argument error.
 */
int oracle_quantize_append_q(const void *k, const void *v, int in_dtype,
                             const float *T_k, const float *T_v,
                             int B, int n, int Hkv, int d, int bits_k, int bits_v, int group,
                             float clip_alpha, int quantizer, int T_cap, const int32_t *pos,
                             uint8_t *k_codes, uint16_t *k_sz, uint8_t *v_codes, uint16_t *v_sz,
                             float *kt_out, float *vt_out);

/* The percentile-clipped quantizer (quantizer 0); see oracle_quantize_append_q. */
int oracle_quantize_append(const void *k, const void *v, int in_dtype,
                           const float *T_k, const float *T_v,
                           int B, int n, int Hkv, int d, int bits_k, int bits_v, int group,
                           float clip_alpha, int T_cap, const int32_t *pos,
                           uint8_t *k_codes, uint16_t *k_sz, uint8_t *v_codes, uint16_t *v_sz,
                           float *kt_out, float *vt_out)
{
    return oracle_quantize_append_q(k, v, in_dtype, T_k, T_v, B, n, Hkv, d, bits_k, bits_v,
                                    group, clip_alpha, 0, T_cap, pos, k_codes, k_sz, v_codes,
                                    v_sz, kt_out, vt_out);
}

/* quantizer: 0 = percentile-clipped affine (OSCAR-style, clip_alpha), 1 = QuEST INT
 * (RMS-based symmetric grid, clip_alpha unused). */
int oracle_quantize_append_q(const void *k, const void *v, int in_dtype,
                             const float *T_k, const float *T_v,
                             int B, int n, int Hkv, int d, int bits_k, int bits_v, int group,
                             float clip_alpha, int quantizer, int T_cap, const int32_t *pos,
                             uint8_t *k_codes, uint16_t *k_sz, uint8_t *v_codes, uint16_t *v_sz,
                             float *kt_out, float *vt_out)
{
    if (quantizer != 0 && quantizer != 1)
        return -1;
    if (d <= 0 || d > 1024 || group <= 0 || d % group || (bits_k != 2 && bits_k != 4) ||
        (bits_v != 2 && bits_v != 4) || T_cap % 16 || d % 64 ||
        2 * oracle_kappa(clip_alpha, group) >= group)
        return -1;
    for (int b = 0; b < B; ++b)
        if (pos[b] < 0 || pos[b] + n > T_cap)
            return -1;
    oracle_cache c = {B, Hkv, T_cap, d, bits_k, bits_v, group, k_codes, v_codes, k_sz, v_sz};
    int ng = d / group;
    long total = (long)B * n * Hkv;
#pragma omp parallel for schedule(dynamic, 64)
    for (long u = 0; u < total; ++u) {
        int h = (int)(u % Hkv);
        int i = (int)((u / Hkv) % n);
        int b = (int)(u / ((long)Hkv * n));
        double xin[1024], xt[1024];
        float xf[1024];
        uint8_t codes[1024];
        uint16_t sz[2 * 1024];
        for (int which = 0; which < 2; ++which) {
            const void *src = which ? v : k;
            const float *T = which ? T_v : T_k;
            int bits = which ? bits_v : bits_k;
            size_t base = (((size_t)b * n + i) * Hkv + h) * d;
            for (int j = 0; j < d; ++j)
                xin[j] = load_in(src, in_dtype, base + j);
            if (T) {
                const float *Th = T + (size_t)h * d * d;
                for (int r = 0; r < d; ++r) {
                    double acc = 0.0;
                    for (int j = 0; j < d; ++j)
                        acc += (double)Th[(size_t)r * d + j] * xin[j];
                    xt[r] = acc;
                }
            } else {
                memcpy(xt, xin, sizeof(double) * d);
            }
            for (int j = 0; j < d; ++j)
                xf[j] = (float)xt[j];
            float *dump = which ? vt_out : kt_out;
            if (dump)
                memcpy(dump + base, xf, sizeof(float) * d);
            int kappa = oracle_kappa(clip_alpha, group);
            for (int gr = 0; gr < ng; ++gr) {
                if (quantizer == 1)
                    oracle_quantize_group_quest(xf + gr * group, group, bits, codes + gr * group,
                                                &sz[2 * gr], &sz[2 * gr + 1]);
                else
                    oracle_quantize_group(xf + gr * group, group, bits, kappa, codes + gr * group,
                                          &sz[2 * gr], &sz[2 * gr + 1]);
            }
            store_token(&c, which, b, h, pos[b] + i, codes, sz);
        }
    }
    return 0;
}

/* Pack externally given codes and float16 (s, z) for tokens [t0, t0+n) of one
 * (b, kv head) into the cache planes (used to build caches from random fields). */
int oracle_pack_tokens(int B, int Hkv, int T_cap, int d, int bits_k, int bits_v, int group,
                       int b, int h, int t0, int n,
                       const uint8_t *kc, const uint8_t *vc,
                       const uint16_t *ksz, const uint16_t *vsz,
                       uint8_t *k_codes, uint16_t *k_sz, uint8_t *v_codes, uint16_t *v_sz)
{
    if (t0 < 0 || t0 + n > T_cap || b < 0 || b >= B || h < 0 || h >= Hkv || T_cap % 16)
        return -1;
    oracle_cache c = {B, Hkv, T_cap, d, bits_k, bits_v, group, k_codes, v_codes, k_sz, v_sz};
    int ng = d / group;
    for (int i = 0; i < n; ++i) {
        store_token(&c, 0, b, h, t0 + i, kc + (size_t)i * d, ksz + (size_t)i * 2 * ng);
        store_token(&c, 1, b, h, t0 + i, vc + (size_t)i * d, vsz + (size_t)i * 2 * ng);
    }
    return 0;
}

/* Read back codes and (s, z) of tokens [t0, t0+n) of one (b, kv head). */
int oracle_unpack_tokens(int B, int Hkv, int T_cap, int d, int bits_k, int bits_v, int group,
                         int b, int h, int t0, int n,
                         const uint8_t *k_codes, const uint16_t *k_sz,
                         const uint8_t *v_codes, const uint16_t *v_sz,
                         uint8_t *kc, uint8_t *vc, uint16_t *ksz, uint16_t *vsz)
{
    if (t0 < 0 || t0 + n > T_cap || b < 0 || b >= B || h < 0 || h >= Hkv || T_cap % 16)
        return -1;
    oracle_cache c = {B, Hkv, T_cap, d, bits_k, bits_v, group,
                      (uint8_t *)k_codes, (uint8_t *)v_codes, (uint16_t *)k_sz, (uint16_t *)v_sz};
    int ng = d / group;
    for (int i = 0; i < n; ++i) {
        int t = t0 + i;
        oracle_unpack_k_row(k_row_ptr(&c, b, h, t), d, bits_k, kc + (size_t)i * d);
        oracle_unpack_v_token(v_tile_ptr(&c, b, h, t), d, bits_v, t % 16, vc + (size_t)i * d);
        memcpy(ksz + (size_t)i * 2 * ng, sz_ptr(&c, c.k_sz, b, h, t), sizeof(uint16_t) * 2 * ng);
        memcpy(vsz + (size_t)i * 2 * ng, sz_ptr(&c, c.v_sz, b, h, t), sizeof(uint16_t) * 2 * ng);
    }
    return 0;
}

/* ------------------------------------------------------------------ read path */

/*
 * Attention of one query head over cached tokens [t0, t1) of its KV head, as the
 * unnormalised triple (m, l, o): m = max_t logit_t, l = sum_t exp(logit_t - m),
 * o = sum_t exp(logit_t - m) * vhat_t. logit_t = (1/sqrt(d)) * qt . khat_t with
 * qt = M q (M = T_k^{-T}, the query-side compensation; NULL = identity).
 * An empty range returns m = -inf, l = 0, o = 0.
 * Query head hq reads KV head hq / (Hq/Hkv) (contiguous GQA grouping, WUSH-KV
 * summary section 4.1).
 */
static void attend_range(const oracle_cache *c, const double *qt, int b, int h,
                         int t0, int t1, double *m_out, double *l_out, double *o)
{
    int d = c->d;
    double sm = 1.0 / sqrt((double)d);
    double *kh = (double *)malloc(sizeof(double) * d);
    double *vh = (double *)malloc(sizeof(double) * d);
    double *logit = (double *)malloc(sizeof(double) * (t1 > t0 ? (t1 - t0) : 1));
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        load_token(c, 0, b, h, t, kh);
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += qt[j] * kh[j];
        logit[t - t0] = sm * acc;
        if (logit[t - t0] > m)
            m = logit[t - t0];
    }
    double l = 0.0;
    for (int j = 0; j < d; ++j)
        o[j] = 0.0;
    for (int t = t0; t < t1; ++t) {
        double p = exp(logit[t - t0] - m);
        l += p;
        load_token(c, 1, b, h, t, vh);
        for (int j = 0; j < d; ++j)
            o[j] += p * vh[j];
    }
    *m_out = m;
    *l_out = l;
    free(kh);
    free(vh);
    free(logit);
}

static void query_transform(const void *q, int q_dtype, const float *M, int Hq, int Hkv,
                            int d, int b, int hq, double *qt)
{
    int G = Hq / Hkv, h = hq / G;
    double qin[1024];
    for (int j = 0; j < d; ++j)
        qin[j] = load_in(q, q_dtype, ((size_t)b * Hq + hq) * d + j);
    if (!M) {
        memcpy(qt, qin, sizeof(double) * d);
        return;
    }
    const float *Mh = M + (size_t)h * d * d;
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += (double)Mh[(size_t)i * d + j] * qin[j];
        qt[i] = acc;
    }
}

/*
 * Decode attention (one step): out[b][hq][:] = softmax over t < seqlens[b] of the
 * logits above, applied to the dequantized values. The result stays in the
 * value-transform domain (the inverse value transform is folded into the output
 * projection on the real model, WUSH-KV summary section 4.2). seqlen 0 gives 0.
 * q: [B][Hq][d], dtype 0 float32 / 1 bfloat16 bits. out: [B][Hq][d] float64.
 * sel (nullable): nsel (b, hq) pairs to compute; other outputs are left untouched.
 */
int oracle_decode(const void *q, int q_dtype, int B, int Hq, int Hkv, int d, const float *M,
                  int T_cap, int bits_k, int bits_v, int group,
                  const uint8_t *k_codes, const uint16_t *k_sz,
                  const uint8_t *v_codes, const uint16_t *v_sz,
                  const int32_t *seqlens, const int32_t *sel, int nsel, double *out)
{
    if (Hkv <= 0 || Hq % Hkv || d > 1024 || T_cap % 16)
        return -1;
    oracle_cache c = {B, Hkv, T_cap, d, bits_k, bits_v, group,
                      (uint8_t *)k_codes, (uint8_t *)v_codes, (uint16_t *)k_sz, (uint16_t *)v_sz};
    int npairs = sel ? nsel : B * Hq;
    for (int u = 0; u < npairs; ++u) {
        int b = sel ? sel[2 * u] : u / Hq, hq = sel ? sel[2 * u + 1] : u % Hq;
        if (b < 0 || b >= B || hq < 0 || hq >= Hq || seqlens[b] < 0 || seqlens[b] > T_cap)
            return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < npairs; ++u) {
        int b = sel ? sel[2 * u] : u / Hq, hq = sel ? sel[2 * u + 1] : u % Hq;
        int G = Hq / Hkv;
        double qt[1024], o[1024], m, l;
        query_transform(q, q_dtype, M, Hq, Hkv, d, b, hq, qt);
        attend_range(&c, qt, b, hq / G, 0, seqlens[b], &m, &l, o);
        /* accumulate privately, store once: a pair listed twice in sel is still safe */
        for (int j = 0; j < d; ++j)
            out[((size_t)b * Hq + hq) * d + j] = l > 0 ? o[j] / l : 0.0;
    }
    return 0;
}

/* Partial attention of (b, hq) over [t0, t1) as (m, l, o[d]) -- the quantities a
 * split of the sequence produces before they are merged. */
int oracle_decode_partial(const void *q, int q_dtype, int B, int Hq, int Hkv, int d,
                          const float *M, int T_cap, int bits_k, int bits_v, int group,
                          const uint8_t *k_codes, const uint16_t *k_sz,
                          const uint8_t *v_codes, const uint16_t *v_sz,
                          int b, int hq, int t0, int t1, double *m, double *l, double *o)
{
    if (t0 < 0 || t1 > T_cap || t0 > t1 || Hq % Hkv)
        return -1;
    oracle_cache c = {B, Hkv, T_cap, d, bits_k, bits_v, group,
                      (uint8_t *)k_codes, (uint8_t *)v_codes, (uint16_t *)k_sz, (uint16_t *)v_sz};
    double qt[1024];
    query_transform(q, q_dtype, M, Hq, Hkv, d, b, hq, qt);
    attend_range(&c, qt, b, hq / (Hq / Hkv), t0, t1, m, l, o);
    return 0;
}

/* Merge n partials (m_i, l_i, o_i) of one query head:
 *   M = max_i m_i,  L = sum_i exp(m_i - M) l_i,  out = sum_i exp(m_i - M) o_i / L.
 * Partials with l_i == 0 (empty ranges) contribute nothing; all empty gives 0. */
void oracle_merge(int n, const double *m, const double *l, const double *o, int d, double *out)
{
    double M = -INFINITY;
    for (int i = 0; i < n; ++i)
        if (l[i] > 0 && m[i] > M)
            M = m[i];
    double L = 0.0;
    for (int j = 0; j < d; ++j)
        out[j] = 0.0;
    for (int i = 0; i < n; ++i) {
        if (!(l[i] > 0))
            continue;
        double w = exp(m[i] - M);
        L += w * l[i];
        for (int j = 0; j < d; ++j)
            out[j] += w * o[(size_t)i * d + j];
    }
    for (int j = 0; j < d; ++j)
        out[j] = L > 0 ? out[j] / L : 0.0;
}

/*
 * Uncompressed comparator: the same decode attention directly over bfloat16 keys and
 * values [B][Hkv][T_cap][d] with bfloat16 queries [B][Hq][d] (no transform, no
 * quantization). out: [B][Hq][d] float64. sel as in oracle_decode.
 */
int oracle_bf16_decode(const uint16_t *q, int B, int Hq, int Hkv, int d,
                       const uint16_t *K, const uint16_t *V, int T_cap,
                       const int32_t *seqlens, const int32_t *sel, int nsel, double *out)
{
    if (Hkv <= 0 || Hq % Hkv || d > 1024)
        return -1;
    int npairs = sel ? nsel : B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < npairs; ++u) {
        int b = sel ? sel[2 * u] : u / Hq, hq = sel ? sel[2 * u + 1] : u % Hq;
        int h = hq / (Hq / Hkv), n = seqlens[b];
        double sm = 1.0 / sqrt((double)d);
        double qv[1024], o[1024];
        double *logit = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
        for (int j = 0; j < d; ++j)
            qv[j] = oracle_bf16_to_f64(q[((size_t)b * Hq + hq) * d + j]);
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) {
            const uint16_t *kr = K + (((size_t)b * Hkv + h) * T_cap + t) * d;
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += qv[j] * oracle_bf16_to_f64(kr[j]);
            logit[t] = sm * acc;
            if (logit[t] > m)
                m = logit[t];
        }
        double l = 0.0;
        for (int j = 0; j < d; ++j)
            o[j] = 0.0;
        for (int t = 0; t < n; ++t) {
            const uint16_t *vr = V + (((size_t)b * Hkv + h) * T_cap + t) * d;
            double p = exp(logit[t] - m);
            l += p;
            for (int j = 0; j < d; ++j)
                o[j] += p * oracle_bf16_to_f64(vr[j]);
        }
        for (int j = 0; j < d; ++j)
            out[((size_t)b * Hq + hq) * d + j] = l > 0 ? o[j] / l : 0.0;
        free(logit);
    }
    return 0;
}

/* ------------------------------------------------------------------ full-precision window */

/*
 * Full-precision window ("WUSH-KV: KV Cache Quantization with Data-Adaptive
 * Transforms", section 4.4): the first S_sink positions and the newest S_keep positions
 * of a sequence stay in full precision, and the middle positions that are neither are
 * quantized in batches of S_flush, after the new chunk has been appended and attended
 * in full precision. Reading (the page gives no formula): the flush runs after every
 * append and quantizes the oldest S_flush eligible positions while at least S_flush are
 * eligible, so a sequence of L positions has the quantized middle
 * [S_sink, S_sink + Q) with Q = S_flush * floor(max(0, L - S_sink - S_keep) / S_flush).
 * Returns Q, or -1 for invalid arguments.
 */
int oracle_window_quantized(int L, int S_sink, int S_keep, int S_flush)
{
    if (L < 0 || S_sink < 0 || S_keep < 0 || S_flush <= 0)
        return -1;
    int e = L - S_sink - S_keep;
    return e > 0 ? (e / S_flush) * S_flush : 0;
}

/*
 * Decode attention of a sequence with a full-precision window. For t < L = seqlens[b]:
 *   quantized t (S_sink <= t < S_sink + Q):  logit = (1/sqrt(d)) (M q) . khat_t,
 *                                             value = vhat_t (as oracle_decode);
 *   full-precision t:                         logit = (1/sqrt(d)) q . k_t,
 *                                             value = T_v v_t,
 * k_t, v_t as given (post-RoPE, not transformed; q . k = (M q) . (T_k k) holds exactly
 * for M = T_k^{-T}, so both kinds of logits are on the same scale), and T_v applied in
 * float64 so that every value is in the value-transform domain, as the quantized ones
 * are. out[b][hq] = sum_t p_t value_t / sum_t p_t with p_t = exp(logit_t - max); 0 if
 * L = 0.
 *   k, v: [B][T_cap][Hkv][d] in in_dtype (0 float32, 1 bfloat16 bits): the full-precision
 *         tokens (only window positions are read). Tv: [Hkv][d][d] float32 or NULL = I.
 *   cache planes: the quantized positions at their own positions.
 */
int oracle_window_decode(const void *q, int q_dtype, int B, int Hq, int Hkv, int d,
                         const float *M, const float *Tv, const void *k, const void *v,
                         int in_dtype, int T_cap, int bits_k, int bits_v, int group,
                         const uint8_t *k_codes, const uint16_t *k_sz,
                         const uint8_t *v_codes, const uint16_t *v_sz,
                         const int32_t *seqlens, int S_sink, int S_keep, int S_flush,
                         double *out)
{
    if (Hkv <= 0 || Hq % Hkv || d > 1024 || T_cap % 16 || S_sink < 0 || S_keep < 0 ||
        S_flush <= 0)
        return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > T_cap)
            return -1;
    oracle_cache c = {B, Hkv, T_cap, d, bits_k, bits_v, group,
                      (uint8_t *)k_codes, (uint8_t *)v_codes, (uint16_t *)k_sz, (uint16_t *)v_sz};
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < B * Hq; ++u) {
        int b = u / Hq, hq = u % Hq, G = Hq / Hkv, h = hq / G;
        int L = seqlens[b];
        int Q = oracle_window_quantized(L, S_sink, S_keep, S_flush);
        double sm = 1.0 / sqrt((double)d);
        double qt[1024], qin[1024], o[1024], xv[1024], val[1024];
        query_transform(q, q_dtype, M, Hq, Hkv, d, b, hq, qt);
        for (int j = 0; j < d; ++j)
            qin[j] = load_in(q, q_dtype, ((size_t)b * Hq + hq) * d + j);
        double *logit = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
        double m = -INFINITY;
        for (int t = 0; t < L; ++t) {
            int quant = t >= S_sink && t < S_sink + Q;
            double acc = 0.0;
            if (quant) {
                load_token(&c, 0, b, h, t, xv);
                for (int j = 0; j < d; ++j)
                    acc += qt[j] * xv[j];
            } else {
                for (int j = 0; j < d; ++j)
                    acc += qin[j] * load_in(k, in_dtype, (((size_t)b * T_cap + t) * Hkv + h) * d + j);
            }
            logit[t] = sm * acc;
            if (logit[t] > m)
                m = logit[t];
        }
        double l = 0.0;
        for (int j = 0; j < d; ++j)
            o[j] = 0.0;
        for (int t = 0; t < L; ++t) {
            int quant = t >= S_sink && t < S_sink + Q;
            double p = exp(logit[t] - m);
            l += p;
            if (quant) {
                load_token(&c, 1, b, h, t, val);
            } else {
                for (int j = 0; j < d; ++j)
                    xv[j] = load_in(v, in_dtype, (((size_t)b * T_cap + t) * Hkv + h) * d + j);
                if (Tv) {
                    for (int i = 0; i < d; ++i) {
                        const float *row = Tv + ((size_t)h * d + i) * d;
                        double a = 0.0;
                        for (int j = 0; j < d; ++j)
                            a += (double)row[j] * xv[j];
                        val[i] = a;
                    }
                } else {
                    memcpy(val, xv, sizeof(double) * d);
                }
            }
            for (int j = 0; j < d; ++j)
                o[j] += p * val[j];
        }
        for (int j = 0; j < d; ++j)
            out[((size_t)b * Hq + hq) * d + j] = l > 0 ? o[j] / l : 0.0;
        free(logit);
    }
    return 0;
}

/* ------------------------------------------------------------------ NOVA-KV vector quantization */

/*
 * Vector-quantized cache ("Spend Bits Where Queries Look: KV Cache Vector Quantization with
 * Attention-Preserving Transforms", NOVA-KV project page: transformed keys and values are
 * encoded once on the write path into a fixed-width cache; "the read path ... is a
 * codebook lookup plus one multiply"; equal-size codebooks keep every token the same
 * width). The page fixes neither the sub-vector size nor the codebook layout. Reading:
 *   - the d transformed coefficients of a token form d/4 groups of 4 consecutive
 *     coefficients, each coded by an 8-bit index into a codebook of 256 four-dimensional
 *     codewords (float16), one codebook per KV head for keys and one for values, shared
 *     by the groups: 2 bits per coefficient;
 *   - the "one multiply" is a per-token gain g (float16): x^_group = g * C[idx];
 *   - encoding: g = f16(f32(sqrt(sum_j x_j^2 / d))) (sum in float64), then per group the
 *     index of the codeword nearest to the coefficients after scaling by g, in float32 with
 *     a fixed operation order (this decides an integer, so both sides compute it the same
 *     way): e_m = f32(x_m - f32(g * c_m)) (the product is exact), dist = f32(e_0 * e_0),
 *     then dist = fmaf(e_m, e_m, dist) for m = 1, 2, 3; the smallest dist wins, ties to
 *     the lowest index. g == 0 codes every group as index 0.
 * Layout: idx planes [B][Hkv][T_cap][d/4] bytes, gain planes [B][Hkv][T_cap] float16,
 * codebooks [Hkv][256][4] float16.
 */
#define VQ_DIM 4
#define VQ_SIZE 256

void oracle_vq_encode(const float *x, int d, const uint16_t *cb, uint8_t *idx, uint16_t *gain)
{
    double ss = 0.0;
    for (int j = 0; j < d; ++j)
        ss += (double)x[j] * (double)x[j];
    float rms = (float)sqrt(ss / (double)d);
    uint16_t gh = oracle_f32_to_f16(rms);
    float g = (float)oracle_f16_to_f64(gh);
    *gain = gh;
    for (int grp = 0; grp < d / VQ_DIM; ++grp) {
        int best = 0;
        if (g != 0.0f) {
            float bestd = INFINITY;
            for (int i = 0; i < VQ_SIZE; ++i) {
                float dist = 0.0f;
                for (int m = 0; m < VQ_DIM; ++m) {
                    float c = (float)oracle_f16_to_f64(cb[i * VQ_DIM + m]);
                    float e = f32((double)x[grp * VQ_DIM + m] - (double)f32((double)g * c));
                    dist = m == 0 ? f32((double)e * e) : fmaf(e, e, dist);
                }
                if (dist < bestd) {
                    bestd = dist;
                    best = i;
                }
            }
        }
        idx[grp] = (uint8_t)best;
    }
}

/* Write path: x~ = f32(T x) in float64 (as oracle_quantize_append), then the encoder above;
 * token i of sequence b goes to position pos[b] + i. cb_k, cb_v: [Hkv][256][4] float16. */
int oracle_vq_append(const void *k, const void *v, int in_dtype, const float *T_k,
                     const float *T_v, const uint16_t *cb_k, const uint16_t *cb_v, int B, int n,
                     int Hkv, int d, int T_cap, const int32_t *pos, uint8_t *k_idx,
                     uint16_t *k_gain, uint8_t *v_idx, uint16_t *v_gain, float *kt_out,
                     float *vt_out)
{
    if (d <= 0 || d > 1024 || d % VQ_DIM)
        return -1;
    for (int b = 0; b < B; ++b)
        if (pos[b] < 0 || pos[b] + n > T_cap)
            return -1;
    long total = (long)B * n * Hkv;
#pragma omp parallel for schedule(dynamic, 64)
    for (long u = 0; u < total; ++u) {
        int h = (int)(u % Hkv);
        int i = (int)((u / Hkv) % n);
        int b = (int)(u / ((long)Hkv * n));
        double xin[1024];
        float xf[1024];
        for (int which = 0; which < 2; ++which) {
            const void *src = which ? v : k;
            const float *T = which ? T_v : T_k;
            size_t base = (((size_t)b * n + i) * Hkv + h) * d;
            for (int j = 0; j < d; ++j)
                xin[j] = load_in(src, in_dtype, base + j);
            for (int r = 0; r < d; ++r) {
                double acc = 0.0;
                if (T) {
                    const float *Th = T + (size_t)h * d * d;
                    for (int j = 0; j < d; ++j)
                        acc += (double)Th[(size_t)r * d + j] * xin[j];
                } else {
                    acc = xin[r];
                }
                xf[r] = (float)acc;
            }
            float *dump = which ? vt_out : kt_out;
            if (dump)
                memcpy(dump + base, xf, sizeof(float) * d);
            size_t slot = ((size_t)b * Hkv + h) * T_cap + pos[b] + i;
            const uint16_t *cb = (which ? cb_v : cb_k) + (size_t)h * VQ_SIZE * VQ_DIM;
            oracle_vq_encode(xf, d, cb, (which ? v_idx : k_idx) + slot * (d / VQ_DIM),
                             (which ? v_gain : k_gain) + slot);
        }
    }
    return 0;
}

/* Dequantized token of a VQ cache: x^_j = g * C[idx_{j/4}][j%4] (exact in float64). */
static void vq_load_token(const uint8_t *idx_plane, const uint16_t *gain_plane, const uint16_t *cb,
                          int d, size_t slot, double *xhat)
{
    double g = oracle_f16_to_f64(gain_plane[slot]);
    const uint8_t *row = idx_plane + slot * (d / VQ_DIM);
    for (int j = 0; j < d; ++j)
        xhat[j] = g * oracle_f16_to_f64(cb[(size_t)row[j / VQ_DIM] * VQ_DIM + j % VQ_DIM]);
}

/* Decode attention over a VQ cache: softmax_t((1/sqrt(d)) (M q) . k^_t) v^_t over t <
 * seqlens[b], as oracle_decode with the dequantization above. sel as in oracle_decode. */
int oracle_vq_decode(const void *q, int q_dtype, int B, int Hq, int Hkv, int d, const float *M,
                     const uint16_t *cb_k, const uint16_t *cb_v, int T_cap,
                     const uint8_t *k_idx, const uint16_t *k_gain, const uint8_t *v_idx,
                     const uint16_t *v_gain, const int32_t *seqlens, const int32_t *sel,
                     int nsel, double *out)
{
    if (Hkv <= 0 || Hq % Hkv || d > 1024 || d % VQ_DIM)
        return -1;
    int npairs = sel ? nsel : B * Hq;
    for (int u = 0; u < npairs; ++u) {
        int b = sel ? sel[2 * u] : u / Hq, hq = sel ? sel[2 * u + 1] : u % Hq;
        if (b < 0 || b >= B || hq < 0 || hq >= Hq || seqlens[b] < 0 || seqlens[b] > T_cap)
            return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < npairs; ++u) {
        int b = sel ? sel[2 * u] : u / Hq, hq = sel ? sel[2 * u + 1] : u % Hq;
        int G = Hq / Hkv, h = hq / G, L = seqlens[b];
        double qt[1024], o[1024], xh[1024];
        double sm = 1.0 / sqrt((double)d);
        query_transform(q, q_dtype, M, Hq, Hkv, d, b, hq, qt);
        const uint16_t *ck = cb_k + (size_t)h * VQ_SIZE * VQ_DIM;
        const uint16_t *cv = cb_v + (size_t)h * VQ_SIZE * VQ_DIM;
        double *logit = (double *)malloc(sizeof(double) * (L > 0 ? L : 1));
        double m = -INFINITY;
        for (int t = 0; t < L; ++t) {
            vq_load_token(k_idx, k_gain, ck, d, ((size_t)b * Hkv + h) * T_cap + t, xh);
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += qt[j] * xh[j];
            logit[t] = sm * acc;
            if (logit[t] > m)
                m = logit[t];
        }
        double l = 0.0;
        for (int j = 0; j < d; ++j)
            o[j] = 0.0;
        for (int t = 0; t < L; ++t) {
            double p = exp(logit[t] - m);
            l += p;
            vq_load_token(v_idx, v_gain, cv, d, ((size_t)b * Hkv + h) * T_cap + t, xh);
            for (int j = 0; j < d; ++j)
                o[j] += p * xh[j];
        }
        for (int j = 0; j < d; ++j)
            out[((size_t)b * Hq + hq) * d + j] = l > 0 ? o[j] / l : 0.0;
        free(logit);
    }
    return 0;
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
