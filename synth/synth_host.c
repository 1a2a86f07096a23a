/*
 * Seeded synthetic expert banks for the union-of-experts quantized SwitchGLU
 * layer (host side).
 *
 * This module generates INPUTS only.  It holds none of the layer's own
 * arithmetic (no dequantisation, no matmul, no activation).  It draws the
 * weights of an expert bank and encodes them in the 4-bit affine group-64
 * format that "gather_qmm at M=1 streams 4-bit expert weights at ~half the
 * bandwidth of M=4" (mlx issue 4509, "Numbers" and the moe_bench.py script)
 * builds with mx.quantize(..., group_size=64, bits=4): per group of 64
 * consecutive input columns, w ~= scale * q + bias, q in [0, 15].
 *
 * Random numbers: the n-th output of the SplitMix64 sequence (Steele, Lea and
 * Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) seeded
 * with s is mix(s + (n + 1) * 0x9E3779B97F4A7C15).  It is counter based, so an
 * element's draws depend only on (seed, matrix, expert, row, column) and any
 * subset of a bank can be drawn on its own.  The device twin in synth_dev.cu
 * implements the same definition and produces the same bits.
 *
 * Normal draws: the sum of twelve uniforms minus six (the classical
 * Irwin-Hall approximation of N(0,1): mean 0, variance 1).  Each uniform is a
 * 16-bit field of a SplitMix64 output, so the sum is an exact integer and the
 * draw  sum * 2^-16 - 6  is exact in fp32.  No transcendental function is
 * used anywhere, so host and device agree bit for bit.
 *
 * Quantiser (the pages do not define mx.quantize; plainest min/max reading):
 *   scale = bf16_rne((max - min) / 15), bias = bf16_rne(min),
 *   q     = clamp(rint((w - bias) / scale), 0, 15)
 * with every step an IEEE-754 basic operation (correctly rounded, identical on
 * host and device).  A group whose values are all equal gets scale 1, q = 0.
 * Packing: element c of a row is nibble (c % 8), bits 4*(c%8)..4*(c%8)+3,
 * least significant first, of 32-bit word c / 8.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared -pthread.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t synth_mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* n-th output (n >= 0) of the SplitMix64 sequence seeded with `seed`. */
static inline uint64_t synth_sm64_at(uint64_t seed, uint64_t n) {
    return synth_mix64(seed + (n + 1) * SYNTH_GAMMA);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t matrix_id) {
    return synth_sm64_at(seed, matrix_id);
}

/* Approximate N(0,1) draw for element `elem` of the stream `key`. */
static inline float synth_normal(uint64_t key, uint64_t elem) {
    uint32_t acc = 0;
    for (int i = 0; i < 3; ++i) {
        uint64_t r = synth_sm64_at(key, 3 * elem + (uint64_t)i);
        acc += (uint32_t)(r & 0xFFFF) + (uint32_t)((r >> 16) & 0xFFFF) +
               (uint32_t)((r >> 32) & 0xFFFF) + (uint32_t)(r >> 48);
    }
    return (float)acc * (1.0f / 65536.0f) - 6.0f;
}

float synth_normal_at(uint64_t key, uint64_t elem) { return synth_normal(key, elem); }

static inline uint16_t synth_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf / nan */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline float synth_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Draw and quantise one group of 64 consecutive columns of one row. */
static void synth_group(uint64_t key, uint64_t elem0, uint32_t* q8, uint16_t* s, uint16_t* b) {
    float w[64];
    float mn = 0.0f, mx = 0.0f;
    for (int c = 0; c < 64; ++c) {
        w[c] = synth_normal(key, elem0 + (uint64_t)c);
        if (c == 0 || w[c] < mn) mn = w[c];
        if (c == 0 || w[c] > mx) mx = w[c];
    }
    uint16_t sb = (mx == mn) ? (uint16_t)0x3F80 : synth_bf16_rne((mx - mn) / 15.0f);
    if ((sb & 0x7FFF) == 0) sb = 0x3F80;
    uint16_t bb = synth_bf16_rne(mn);
    float sf = synth_bf16_to_f32(sb), bf = synth_bf16_to_f32(bb);
    for (int wd = 0; wd < 8; ++wd) {
        uint32_t word = 0;
        for (int j = 0; j < 8; ++j) {
            float t = nearbyintf((w[wd * 8 + j] - bf) / sf);
            int qi = (mx == mn) ? 0 : (int)t;
            if (qi < 0) qi = 0;
            if (qi > 15) qi = 15;
            word |= (uint32_t)qi << (4 * j);
        }
        q8[wd] = word;
    }
    *s = sb;
    *b = bb;
}

typedef struct {
    uint32_t* q;
    uint16_t* s;
    uint16_t* b;
    int rows, cols;
    uint64_t key;
    const int32_t* experts;
    int n_experts;
    int next;
    pthread_mutex_t mu;
} synth_job;

static void synth_one_expert(synth_job* J, int e) {
    const int rows = J->rows, cols = J->cols;
    const int gpr = cols / 64;
    uint32_t* q = J->q + (size_t)e * rows * (cols / 8);
    uint16_t* s = J->s + (size_t)e * rows * gpr;
    uint16_t* b = J->b + (size_t)e * rows * gpr;
    for (int r = 0; r < rows; ++r)
        for (int g = 0; g < gpr; ++g) {
            uint64_t elem0 = ((uint64_t)e * rows + r) * cols + (uint64_t)g * 64;
            synth_group(J->key, elem0, q + (size_t)r * (cols / 8) + g * 8,
                        s + (size_t)r * gpr + g, b + (size_t)r * gpr + g);
        }
}

static void* synth_worker(void* arg) {
    synth_job* J = (synth_job*)arg;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int i = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (i >= J->n_experts) break;
        synth_one_expert(J, J->experts[i]);
    }
    return 0;
}

/*
 * Fill experts `experts[0..n_experts)` of a bank laid out as
 *   q [E, rows, cols/8] uint32, s/b [E, rows, cols/64] bf16 bits,
 * drawn from stream (seed, matrix_id).  Other experts are left untouched.
 * cols must be a multiple of 64.  Returns 0, or -1 on bad arguments.
 */
int synth_fill_bank(uint32_t* q, uint16_t* s, uint16_t* b, int E, int rows, int cols,
                    uint64_t seed, uint64_t matrix_id, const int32_t* experts, int n_experts,
                    int n_threads) {
    if (!q || !s || !b || E <= 0 || rows <= 0 || cols <= 0 || cols % 64) return -1;
    for (int i = 0; i < n_experts; ++i)
        if (experts[i] < 0 || experts[i] >= E) return -1;
    synth_job J;
    J.q = q; J.s = s; J.b = b; J.rows = rows; J.cols = cols;
    J.key = synth_stream_key(seed, matrix_id);
    J.experts = experts; J.n_experts = n_experts; J.next = 0;
    pthread_mutex_init(&J.mu, 0);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    if (n_threads > n_experts) n_threads = n_experts > 0 ? n_experts : 1;
    pthread_t th[256];
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], 0, synth_worker, &J);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], 0);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

/*
 * mxfp4 encoding (GLM-5.2's routed banks are "mxfp4 gs32" in "Small-L fused
 * expert gather for fine-grained MoE decode", mlx discussion 3801, the post
 * that isolates one layer's routed bank; the pages define it no further, so
 * the OCP microscaling format is taken): per group of 32 consecutive input
 * columns one e8m0 scale byte X = 127 + floor(log2(max |w|)) - 2 (the largest
 * e2m1 exponent is 2), and per element the e2m1 code nearest to w * 2^-(X-127),
 * ties to the even mantissa, magnitudes above 6 saturating to 6.  An all-zero
 * group gets X = 127 and zero codes.  e2m1 code: sign bit 3, magnitude index
 * bits 2..0 for 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Codes are packed like the affine
 * ones.  Every step is exact in fp32 (power-of-two scaling, comparisons), so the
 * device twin gives the same bits.
 */
static inline uint32_t synth_e2m1_code(float v) {
    const float a = fabsf(v);
    uint32_t m;
    if (a <= 0.25f) m = 0;
    else if (a < 0.75f) m = 1;
    else if (a <= 1.25f) m = 2;
    else if (a < 1.75f) m = 3;
    else if (a <= 2.5f) m = 4;
    else if (a < 3.5f) m = 5;
    else if (a <= 5.0f) m = 6;
    else m = 7;
    return (v < 0.0f ? 8u : 0u) | m;
}

static void synth_group_mx(uint64_t key, uint64_t elem0, uint32_t* q4, uint8_t* e8) {
    float w[32];
    float amax = 0.0f;
    for (int c = 0; c < 32; ++c) {
        w[c] = synth_normal(key, elem0 + (uint64_t)c);
        if (fabsf(w[c]) > amax) amax = fabsf(w[c]);
    }
    int e = 0;
    if (amax > 0.0f) {
        uint32_t u;
        memcpy(&u, &amax, 4);
        e = (int)((u >> 23) & 0xFF) - 127 - 2;  /* floor(log2 amax) - 2; amax is normal */
    }
    /* 2^-e as an fp32 bit pattern (|e| < 30 for these draws) */
    const uint32_t inv_bits = (uint32_t)(127 - e) << 23;
    float inv;
    memcpy(&inv, &inv_bits, 4);
    for (int wd = 0; wd < 4; ++wd) {
        uint32_t word = 0;
        for (int j = 0; j < 8; ++j)
            word |= (amax > 0.0f ? synth_e2m1_code(w[wd * 8 + j] * inv) : 0u) << (4 * j);
        q4[wd] = word;
    }
    *e8 = (uint8_t)(127 + e);
}

typedef struct {
    uint32_t* q;
    uint8_t* e8;
    int rows, cols;
    uint64_t key;
    const int32_t* experts;
    int n_experts;
    int next;
    pthread_mutex_t mu;
} synth_job_mx;

static void* synth_worker_mx(void* arg) {
    synth_job_mx* J = (synth_job_mx*)arg;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int i = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (i >= J->n_experts) break;
        const int e = J->experts[i], rows = J->rows, cols = J->cols, gpr = cols / 32;
        uint32_t* q = J->q + (size_t)e * rows * (cols / 8);
        uint8_t* e8 = J->e8 + (size_t)e * rows * gpr;
        for (int r = 0; r < rows; ++r)
            for (int g = 0; g < gpr; ++g)
                synth_group_mx(J->key, ((uint64_t)e * rows + r) * cols + (uint64_t)g * 32,
                               q + (size_t)r * (cols / 8) + g * 4, e8 + (size_t)r * gpr + g);
    }
    return 0;
}

/*
 * Fill experts `experts[0..n_experts)` of an mxfp4 bank laid out as
 *   q [E, rows, cols/8] uint32 (e2m1 codes), e8 [E, rows, cols/32] uint8,
 * from the same normal draws as synth_fill_bank (stream (seed, matrix_id)).
 * cols must be a multiple of 32.  Returns 0, or -1 on bad arguments.
 */
int synth_fill_bank_mxfp4(uint32_t* q, uint8_t* e8, int E, int rows, int cols, uint64_t seed,
                          uint64_t matrix_id, const int32_t* experts, int n_experts,
                          int n_threads) {
    if (!q || !e8 || E <= 0 || rows <= 0 || cols <= 0 || cols % 32) return -1;
    for (int i = 0; i < n_experts; ++i)
        if (experts[i] < 0 || experts[i] >= E) return -1;
    synth_job_mx J;
    J.q = q; J.e8 = e8; J.rows = rows; J.cols = cols;
    J.key = synth_stream_key(seed, matrix_id);
    J.experts = experts; J.n_experts = n_experts; J.next = 0;
    pthread_mutex_init(&J.mu, 0);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    if (n_threads > n_experts) n_threads = n_experts > 0 ? n_experts : 1;
    pthread_t th[256];
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], 0, synth_worker_mx, &J);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], 0);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

/* Raw fp32 draws of one row (before quantisation); used by the quantiser's
 * round-trip test. */
int synth_draw_row(float* out, int E, int rows, int cols, uint64_t seed, uint64_t matrix_id,
                   int expert, int row) {
    if (!out || expert < 0 || expert >= E || row < 0 || row >= rows) return -1;
    uint64_t key = synth_stream_key(seed, matrix_id);
    for (int c = 0; c < cols; ++c)
        out[c] = synth_normal(key, ((uint64_t)expert * rows + row) * cols + (uint64_t)c);
    return 0;
}
