/*
 * tbq4_oracle.c -- plain, slow, fp64 CPU oracle for TBQ4 long-context attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no source with the CUDA library: it has its
 * own PRNG, its own fp16 rounding, its own Hadamard transform and its own
 * bit packing.
 *
 * What it computes (sources):
 *   - The TBQ4 block: 128 values in 66 bytes, a 2-byte scale followed by 64
 *     bytes of 4-bit indices (4.125 bits per value), stored in a
 *     Hadamard-rotated domain -- trefon.com, "Kontekst 262K na jednej RTX
 *     4090: co dodalem do llama.cpp-turboq", section "Od czego zaczalem".
 *   - The codebook the page leaves open, fixed by this library: rotation
 *     R = H*D/sqrt(128) (H the 128x128 Sylvester Hadamard matrix, D a seeded
 *     +-1 diagonal), scale = fp16(max|x_rot|), 16 symmetric levels
 *     (i - 7.5)/7.5 * scale chosen by round-to-nearest-even.
 *   - Attention: plain softmax(scale * q.k) v over the dequantised cache,
 *     computed in the rotated domain and rotated back at the end (the page's
 *     "attention works in the rotated (Hadamard) domain", same section).
 *
 * Readings where the page is silent (each repeated where it is used):
 *   signs from SplitMix64 (Steele, Lea & Flood, OOPSLA 2014), bit i of output
 *   i/64 set -> s_i = -1;  D applied before H;  butterflies in ascending
 *   stride, lower = a+b, upper = a-b, each rounded to fp32, then one fp32
 *   multiply by fl32(1/sqrt(128));  index = clamp(rne(fl32(fl32(x/S)*7.5)+7.5),
 *   0, 15), index 8 when S == 0;  even element in the low nibble;  scale bytes
 *   first, little endian;  cache layout [B][Hkv][capacity][66].
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC.
 * float arithmetic on x86-64 is SSE2 single precision, so every float
 * operation below is one IEEE-754 binary32 operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OD 128           /* values per block */
#define OBLOCK 66        /* bytes per block  */

/* ---------------------------------------------------------------- threads */

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int oracle_block_bytes(void) { return OBLOCK; }

/* ------------------------------------------------------------- SplitMix64 */
/* SplitMix64 as published by Steele, Lea & Flood (2014): add the golden
 * gamma, then the variant-13 mixing function. */
void oracle_splitmix64(uint64_t seed, int n, uint64_t *out) {
    uint64_t state = seed;
    for (int k = 0; k < n; ++k) {
        state += 0x9E3779B97F4A7C15ULL;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
        out[k] = z ^ (z >> 31);
    }
}

/* The +-1 diagonal D: two SplitMix64 outputs w0, w1; s_i = 1 - 2*bit(i%64 of
 * w_{i/64}). */
void oracle_signs(uint64_t seed, int8_t *s) {
    uint64_t w[2];
    oracle_splitmix64(seed, 2, w);
    for (int i = 0; i < OD; ++i) {
        int bit = (int)((w[i / 64] >> (i % 64)) & 1u);
        s[i] = (int8_t)(1 - 2 * bit);
    }
}

/* ------------------------------------------------------------------ fp16 */
/* Right shift of an unsigned integer with round-to-nearest, ties to even. */
static uint32_t shr_rne(uint32_t m, int sh) {
    if (sh <= 0) return m;
    if (sh >= 32) return 0;      /* m < 2^24 here, so below half of 2^sh */
    uint32_t q = m >> sh;
    uint32_t r = m & ((1u << sh) - 1u);
    uint32_t half = 1u << (sh - 1);
    if (r > half || (r == half && (q & 1u))) q += 1u;
    return q;
}

/* IEEE binary32 -> binary16, round to nearest even, from the bit fields.
 * Overflow gives infinity, as IEEE rounding does. */
uint16_t oracle_f32_to_f16_bits(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7FFFFFFFu;
    if (ax >= 0x7F800000u)                      /* inf or nan */
        return (uint16_t)(sign | 0x7C00u | (ax > 0x7F800000u ? 0x200u : 0u));
    if (ax < 0x00800000u)                       /* binary32 zero/subnormal */
        return (uint16_t)sign;                  /* < 2^-126, rounds to 0 */
    int e = (int)(ax >> 23) - 127;              /* unbiased exponent */
    uint32_t mant = ax & 0x7FFFFFu;
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    if (e >= -14) {
        /* normal half: 10 mantissa bits; a carry out of the mantissa moves
         * into the exponent field, and out of e=15 into infinity. */
        uint32_t h = ((uint32_t)(e + 15) << 10) + shr_rne(mant, 13);
        return (uint16_t)(sign | h);
    }
    /* subnormal half: value / 2^-24 = (mant|2^23) * 2^(e+1) */
    uint32_t k = shr_rne(mant | 0x800000u, -(e + 1));
    return (uint16_t)(sign | k);
}

void oracle_f32_to_f16_array(const float *x, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_f16_bits(x[i]);
}

double oracle_f16_bits_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* --------------------------------------------------------------- Hadamard */
/* Sylvester Hadamard matrix, natural order: H[i][j] = (-1)^popcount(i & j). */
int oracle_hadamard_entry(int i, int j) {
    return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* R = H * D / sqrt(128) in double: R[i][j] = H[i][j] * s_j / sqrt(128). */
void oracle_rotation_matrix(const int8_t *s, double *R) {
    const double inv = 1.0 / sqrt((double)OD);
    for (int i = 0; i < OD; ++i)
        for (int j = 0; j < OD; ++j)
            R[i * OD + j] = (double)(oracle_hadamard_entry(i, j) * s[j]) * inv;
}

/* The rotation as the quantiser performs it, in binary32: sign flip, then
 * seven butterfly stages with strides 1, 2, 4, ..., 64 (lower element
 * a+b, upper element a-b, a being the lower-index element), then one
 * multiply by c = fl32(1/sqrt(128)). */
void oracle_rotate_f32(const float *x, const int8_t *s, float *out) {
    float z[OD];
    for (int i = 0; i < OD; ++i) z[i] = (s[i] < 0) ? -x[i] : x[i];
    for (int h = 1; h < OD; h <<= 1) {
        for (int i = 0; i < OD; i += 2 * h) {
            for (int j = i; j < i + h; ++j) {
                float a = z[j];
                float b = z[j + h];
                z[j] = a + b;
                z[j + h] = a - b;
            }
        }
    }
    const float c = (float)(1.0 / sqrt(128.0));   /* 0x3DB504F3 */
    for (int i = 0; i < OD; ++i) out[i] = z[i] * c;
}

/* ------------------------------------------------------------- quantiser */
/* Round half to even, written out from floor(): v - floor(v) is exact in
 * binary32 for |v| < 2^23. */
static float rne_f32(float v) {
    float f = floorf(v);
    float d = v - f;
    if (d > 0.5f) return f + 1.0f;
    if (d < 0.5f) return f;
    return (fmodf(f, 2.0f) == 0.0f) ? f : f + 1.0f;
}

/* Index of one rotated value: t = x/S, u = t*7.5, v = u+7.5 (each one
 * binary32 operation), rne, clamp to [0, 15]; S == 0 gives index 8. */
int oracle_level_index(float x_rot, float S) {
    if (S == 0.0f) return 8;
    float t = x_rot / S;
    float u = t * 7.5f;
    float v = u + 7.5f;
    float r = rne_f32(v);
    if (r < 0.0f) r = 0.0f;
    if (r > 15.0f) r = 15.0f;
    return (int)r;
}

/* Scale of one rotated block: fp16(max |x_rot|), round to nearest even,
 * saturating at 65504 (0x7BFF) instead of overflowing to infinity. */
uint16_t oracle_block_scale_bits(const float *x_rot) {
    float m = 0.0f;
    for (int i = 0; i < OD; ++i) {
        float a = fabsf(x_rot[i]);
        if (a > m) m = a;
    }
    uint16_t h = oracle_f32_to_f16_bits(m);
    if ((h & 0x7FFFu) == 0x7C00u) h = 0x7BFFu;
    return h;
}

/* One 128-value block -> 66 bytes: [scale lo][scale hi][64 index bytes],
 * byte 2+j = idx[2j] | idx[2j+1] << 4. */
void oracle_quantize_block(const float *x, const int8_t *s, uint8_t *out) {
    float xr[OD];
    oracle_rotate_f32(x, s, xr);
    uint16_t sb = oracle_block_scale_bits(xr);
    float S = (float)oracle_f16_bits_to_f64(sb);
    int idx[OD];
    for (int i = 0; i < OD; ++i) idx[i] = oracle_level_index(xr[i], S);
    out[0] = (uint8_t)(sb & 0xFFu);
    out[1] = (uint8_t)(sb >> 8);
    for (int j = 0; j < OD / 2; ++j)
        out[2 + j] = (uint8_t)(idx[2 * j] | (idx[2 * j + 1] << 4));
}

/* Dequantise one block into the rotated domain: S * (2*idx - 15) / 15. */
void oracle_dequant_block(const uint8_t *blk, double *out) {
    uint16_t sb = (uint16_t)(blk[0] | (blk[1] << 8));
    double S = oracle_f16_bits_to_f64(sb);
    for (int j = 0; j < OD / 2; ++j) {
        int lo = blk[2 + j] & 0xF;
        int hi = blk[2 + j] >> 4;
        out[2 * j] = S * (double)(2 * lo - 15) / 15.0;
        out[2 * j + 1] = S * (double)(2 * hi - 15) / 15.0;
    }
}

/* Quantise-append: src [B][n_new][Hkv][128] fp32; the block of (b, t, h) goes
 * to cache[b][h][start_pos[b] + t]; cache is [B][Hkv][capacity][66].
 * Returns the number of rows skipped because their position fell outside
 * [0, capacity). */
int64_t oracle_quantize_append(const float *src, int B, int n_new, int Hkv,
                               const int32_t *start_pos, int64_t capacity,
                               uint64_t seed, uint8_t *cache) {
    int8_t s[OD];
    oracle_signs(seed, s);
    int64_t rows = (int64_t)B * n_new * Hkv;
    int64_t skipped = 0;
#pragma omp parallel for schedule(static) reduction(+ : skipped)
    for (int64_t r = 0; r < rows; ++r) {
        int h = (int)(r % Hkv);
        int64_t t = (r / Hkv) % n_new;
        int b = (int)(r / ((int64_t)Hkv * n_new));
        int64_t pos = (int64_t)start_pos[b] + t;
        if (pos < 0 || pos >= capacity) { skipped += 1; continue; }
        uint8_t *dst = cache + (((int64_t)b * Hkv + h) * capacity + pos) * OBLOCK;
        oracle_quantize_block(src + r * OD, s, dst);
    }
    return skipped;
}

/* -------------------------------------------------------------- attention */
typedef void (*dequant_fn)(const uint8_t *blk, double *out);

/* One attention row in the rotated domain, all in double:
 *   q_rot = R q;  logit_t = scale * q_rot . Khat_t  (t < n_keys);
 *   p = softmax(logit);  o_rot = sum_t p_t Vhat_t;  o = R^T o_rot.
 * k_rows / v_rows point at the first block of the (b, kv head) stream;
 * blocks are nbytes apart and dequantised by dq. */
static void attend_row_fmt(const double *R, const double *q, const uint8_t *k_rows,
                           const uint8_t *v_rows, int64_t n_keys, double scale,
                           int nbytes, dequant_fn dq, double *o) {
    double q_rot[OD], o_rot[OD], kd[OD], vd[OD];
    for (int i = 0; i < OD; ++i) {
        double acc = 0.0;
        for (int j = 0; j < OD; ++j) acc += R[i * OD + j] * q[j];
        q_rot[i] = acc;
    }
    if (n_keys <= 0) {                      /* empty context: zero output */
        for (int i = 0; i < OD; ++i) o[i] = 0.0;
        return;
    }
    double *logit = (double *)malloc((size_t)n_keys * sizeof(double));
    double m = -INFINITY;
    for (int64_t t = 0; t < n_keys; ++t) {
        dq(k_rows + t * nbytes, kd);
        double dot = 0.0;
        for (int i = 0; i < OD; ++i) dot += q_rot[i] * kd[i];
        logit[t] = scale * dot;
        if (logit[t] > m) m = logit[t];
    }
    double l = 0.0;
    for (int i = 0; i < OD; ++i) o_rot[i] = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) {
        double p = exp(logit[t] - m);
        l += p;
        dq(v_rows + t * nbytes, vd);
        for (int i = 0; i < OD; ++i) o_rot[i] += p * vd[i];
    }
    free(logit);
    for (int i = 0; i < OD; ++i) o_rot[i] /= l;
    for (int j = 0; j < OD; ++j) {
        double acc = 0.0;
        for (int i = 0; i < OD; ++i) acc += R[i * OD + j] * o_rot[i];
        o[j] = acc;
    }
}

static void attend_row(const double *R, const double *q, const uint8_t *k_rows,
                       const uint8_t *v_rows, int64_t n_keys, double scale,
                       double *o) {
    attend_row_fmt(R, q, k_rows, v_rows, n_keys, scale, OBLOCK, oracle_dequant_block, o);
}

/* Decode attention.  q [B][Hq][128] fp32 (unrotated); caches
 * [B][Hkv][capacity][66]; seq_lens [B] = number of keys attended; q head h
 * reads kv head h / (Hq/Hkv).  out [B][Hq][128] double (unrotated).
 * rows: optional list of b*Hq + h to compute (n_rows entries, NULL = all);
 * only those rows of out are written. */
void oracle_attn_decode(const float *q, const uint8_t *k_cache,
                        const uint8_t *v_cache, const int32_t *seq_lens, int B,
                        int Hq, int Hkv, int64_t capacity, double softmax_scale,
                        uint64_t seed, const int32_t *rows, int n_rows,
                        double *out) {
    int8_t s[OD];
    oracle_signs(seed, s);
    double *R = (double *)malloc(OD * OD * sizeof(double));
    oracle_rotation_matrix(s, R);
    int G = Hq / Hkv;
    int total = rows ? n_rows : B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int k = 0; k < total; ++k) {
        int row = rows ? rows[k] : k;
        int b = row / Hq, h = row % Hq, g = h / G;
        double qd[OD];
        for (int i = 0; i < OD; ++i) qd[i] = (double)q[(int64_t)row * OD + i];
        int64_t base = ((int64_t)b * Hkv + g) * capacity * OBLOCK;
        attend_row(R, qd, k_cache + base, v_cache + base, seq_lens[b],
                   softmax_scale, out + (int64_t)row * OD);
    }
    free(R);
}

/* Chunked prefill attention for one sequence.  q [n_new][Hq][128] given as
 * float (bf16 values upcast exactly); caches [Hkv][capacity][66] already
 * hold the chunk's keys at positions n_cached .. n_cached+n_new-1.  Query i
 * sits at absolute position n_cached+i and sees keys 0 .. n_cached+i
 * (causal, aligned bottom-right).  out [n_new][Hq][128] double.
 * rows: optional list of i*Hq + h (NULL = all). */
void oracle_attn_prefill(const float *q, int n_new, int64_t n_cached,
                         const uint8_t *k_cache, const uint8_t *v_cache, int Hq,
                         int Hkv, int64_t capacity, double softmax_scale,
                         uint64_t seed, const int32_t *rows, int n_rows,
                         double *out) {
    int8_t s[OD];
    oracle_signs(seed, s);
    double *R = (double *)malloc(OD * OD * sizeof(double));
    oracle_rotation_matrix(s, R);
    int G = Hq / Hkv;
    int total = rows ? n_rows : n_new * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int k = 0; k < total; ++k) {
        int row = rows ? rows[k] : k;
        int i = row / Hq, h = row % Hq, g = h / G;
        double qd[OD];
        for (int d = 0; d < OD; ++d) qd[d] = (double)q[(int64_t)row * OD + d];
        int64_t base = (int64_t)g * capacity * OBLOCK;
        attend_row(R, qd, k_cache + base, v_cache + base, n_cached + i + 1,
                   softmax_scale, out + (int64_t)row * OD);
    }
    free(R);
}

/* ==================================================================== TBQ3 */
/* A 3-bit variant with the same rotation and the same scale.  The page
 * names TBQ3 next to TBQ4 and mentions a fix to its 3-bit packing
 * (trefon.com, "Kontekst 262K na jednej RTX 4090: co dodalem do
 * llama.cpp-turboq", section "6. Ten sam cache na Apple silicon") but gives
 * no layout, so this library fixes one:
 *   - 128 values in 50 bytes: the fp16 scale (little endian), then 48 bytes;
 *   - 8 symmetric levels (i - 3.5)/3.5 * S = S * (2i - 7)/7;
 *   - index = clamp(rne(fl32(fl32(x/S)*3.5)+3.5), 0, 7), index 4 when S == 0;
 *   - indices 8g .. 8g+7 form one 24-bit little-endian word, index 8g+k at
 *     bits 3k .. 3k+2, stored as bytes 2+3g, 3+3g, 4+3g.
 * Cache layout [B][Hkv][capacity][50]. */
#define OBLOCK3 50

int oracle_block_bytes3(void) { return OBLOCK3; }

/* Index of one rotated value against the block scale, 3-bit codebook. */
int oracle_level_index3(float x_rot, float S) {
    if (S == 0.0f) return 4;
    float t = x_rot / S;
    float u = t * 3.5f;
    float v = u + 3.5f;
    float r = rne_f32(v);
    if (r < 0.0f) r = 0.0f;
    if (r > 7.0f) r = 7.0f;
    return (int)r;
}

/* One 128-value block -> 50 bytes. */
void oracle_quantize_block3(const float *x, const int8_t *s, uint8_t *out) {
    float xr[OD];
    oracle_rotate_f32(x, s, xr);
    uint16_t sb = oracle_block_scale_bits(xr);
    float S = (float)oracle_f16_bits_to_f64(sb);
    int idx[OD];
    for (int i = 0; i < OD; ++i) idx[i] = oracle_level_index3(xr[i], S);
    out[0] = (uint8_t)(sb & 0xFFu);
    out[1] = (uint8_t)(sb >> 8);
    for (int g = 0; g < OD / 8; ++g) {
        uint32_t w = 0;
        for (int k = 0; k < 8; ++k) w |= (uint32_t)idx[8 * g + k] << (3 * k);
        out[2 + 3 * g] = (uint8_t)(w & 0xFFu);
        out[3 + 3 * g] = (uint8_t)((w >> 8) & 0xFFu);
        out[4 + 3 * g] = (uint8_t)((w >> 16) & 0xFFu);
    }
}

/* Dequantise one 3-bit block into the rotated domain: S * (2*idx - 7) / 7. */
void oracle_dequant_block3(const uint8_t *blk, double *out) {
    uint16_t sb = (uint16_t)(blk[0] | (blk[1] << 8));
    double S = oracle_f16_bits_to_f64(sb);
    for (int g = 0; g < OD / 8; ++g) {
        uint32_t w = (uint32_t)blk[2 + 3 * g] | ((uint32_t)blk[3 + 3 * g] << 8) |
                     ((uint32_t)blk[4 + 3 * g] << 16);
        for (int k = 0; k < 8; ++k) {
            int i = (int)((w >> (3 * k)) & 7u);
            out[8 * g + k] = S * (double)(2 * i - 7) / 7.0;
        }
    }
}

/* Quantise-append into a [B][Hkv][capacity][50] cache; as
 * oracle_quantize_append otherwise. */
int64_t oracle_quantize_append3(const float *src, int B, int n_new, int Hkv,
                                const int32_t *start_pos, int64_t capacity,
                                uint64_t seed, uint8_t *cache) {
    int8_t s[OD];
    oracle_signs(seed, s);
    int64_t rows = (int64_t)B * n_new * Hkv;
    int64_t skipped = 0;
#pragma omp parallel for schedule(static) reduction(+ : skipped)
    for (int64_t r = 0; r < rows; ++r) {
        int h = (int)(r % Hkv);
        int64_t t = (r / Hkv) % n_new;
        int b = (int)(r / ((int64_t)Hkv * n_new));
        int64_t pos = (int64_t)start_pos[b] + t;
        if (pos < 0 || pos >= capacity) { skipped += 1; continue; }
        uint8_t *dst = cache + (((int64_t)b * Hkv + h) * capacity + pos) * OBLOCK3;
        oracle_quantize_block3(src + r * OD, s, dst);
    }
    return skipped;
}

/* Decode attention over 3-bit caches [B][Hkv][capacity][50]; as
 * oracle_attn_decode otherwise. */
void oracle_attn_decode3(const float *q, const uint8_t *k_cache,
                         const uint8_t *v_cache, const int32_t *seq_lens, int B,
                         int Hq, int Hkv, int64_t capacity, double softmax_scale,
                         uint64_t seed, const int32_t *rows, int n_rows,
                         double *out) {
    int8_t s[OD];
    oracle_signs(seed, s);
    double *R = (double *)malloc(OD * OD * sizeof(double));
    oracle_rotation_matrix(s, R);
    int G = Hq / Hkv;
    int total = rows ? n_rows : B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int k = 0; k < total; ++k) {
        int row = rows ? rows[k] : k;
        int b = row / Hq, h = row % Hq, g = h / G;
        double qd[OD];
        for (int i = 0; i < OD; ++i) qd[i] = (double)q[(int64_t)row * OD + i];
        int64_t base = ((int64_t)b * Hkv + g) * capacity * OBLOCK3;
        attend_row_fmt(R, qd, k_cache + base, v_cache + base, seq_lens[b], softmax_scale,
                       OBLOCK3, oracle_dequant_block3, out + (int64_t)row * OD);
    }
    free(R);
}
