/*
 * ngram_oracle.c -- plain, slow CPU oracle for the hashed n-gram embedding lookup.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this
 * file.  It is used by tests/, by __graft_entry__.smoke() (to check one small GPU
 * invocation) and by bench.py's CPU-baseline leg.  It shares no source with the CUDA
 * library: every definition below is restated here from the pages and from the
 * published definitions of the two generators.
 *
 * What it computes (the pages):
 *   "Qwen Brought Back N-Grams. All 51 Billion Parameters of Them." (aibacon.net),
 *   section "N-grams, of all things": for every token the local bigram and trigram
 *   context is hashed into one 20M-row table, 16 rows are gathered and summed into a
 *   2560-wide vector that is added to the residual stream.  Same page, "Key
 *   Takeaways": 20,000,000 hash-addressed bigram and trigram rows, 16 rows read per
 *   token.
 *   "Qwen3.8-Flash-Next: A 51B N-gram Embedding Table with Heterogeneous Memory
 *   Prefetch" (zhichai.net), Key point 1, the gate equation
 *   h_0 = e_1gram(w_t) + W_g (elementwise) e_Ngram(w_{t-1}, w_t): the n-gram vector
 *   enters through an elementwise gate.  The same key point says a deterministic hash
 *   addresses the stored vector.
 *   "Qwen 3.8 Flash-Next Deep Dive ..." (abrarakhunji.com), Section 1 figure: the
 *   lookup consumes the stream w_{t-2}, w_{t-1}, w_t.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - hash: splitmix64 finaliser over a packed key, one seed per head, then % R;
 *   - heads: 8 bigram heads (0..7) and 8 trigram heads (8..15), one shared table;
 *   - contexts never cross a sequence row; positions before 0 come from an optional
 *     per-sequence history {w_-2, w_-1}, else from a fixed PAD id;
 *   - the gate g is a static fp32 vector of width d;
 *   - the sum is plain and unweighted; colliding heads count once per head;
 *   - table values are synthetic (no trained weights exist): a Philox4x32-10
 *     function of (seed, row, col), see oracle_table_bf16 / oracle_table_int8.
 *
 * Row formats: bf16; int8 with an fp32 row scale; FP8 E4M3 with an fp32 row scale;
 * NVFP4 (E2M1 with one E4M3 scale per 16 columns and an fp32 global scale).
 *
 * Two accumulation modes:
 *   ORACLE_ACC_F64 -- the plain definition.  The 16 products/values are summed in
 *                     double (exact for these operands), gate and add in double, and
 *                     the result is rounded once to bf16 (round to nearest even).
 *   ORACLE_ACC_F32 -- the fp32-accumulated reference: fp32 sum in head order 0..H-1
 *                     (bf16 rows: acc = acc + E; int8 rows: acc = fmaf(q, s, acc), one
 *                     correctly rounded fused multiply-add per head), then a separately
 *                     rounded fp32 multiply by g and fp32 add of the residual, then bf16
 *                     round to nearest even.  Build with -ffp-contract=off so that no
 *                     step other than the explicit fmaf is fused.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>

#define ORACLE_ACC_F64 0
#define ORACLE_ACC_F32 1

#define ORACLE_BF16 0
#define ORACLE_INT8 1
#define ORACLE_FP8 2      /* FP8 E4M3 codes, one fp32 scale per row */
#define ORACLE_NVFP4 3    /* FP4 E2M1 codes, one E4M3 scale per 16 columns, one fp32 global scale */

/* ------------------------------------------------------------------------------------
 * splitmix64 (Steele, Lea & Flood, "Fast Splittable Pseudorandom Number Generators",
 * OOPSLA 2014; the 64-bit mixer constants are those of the published SplitMix64).
 * One call advances the state by the golden gamma and returns the mixed state.
 * ---------------------------------------------------------------------------------- */
uint64_t oracle_splitmix64_next(uint64_t *state)
{
    uint64_t z;
    *state = *state + 0x9E3779B97F4A7C15ull;
    z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Head seeds: seed_h is the (h+1)-th output of splitmix64 started at base_seed. */
void oracle_head_seeds(uint64_t base_seed, uint32_t n_heads, uint64_t *seeds)
{
    uint64_t state = base_seed;
    uint32_t h;
    for (h = 0; h < n_heads; h++)
        seeds[h] = oracle_splitmix64_next(&state);
}

/* ------------------------------------------------------------------------------------
 * Philox4x32-10 (Salmon, Moraes, Dror & Shaw, "Parallel Random Numbers: As Easy as
 * 1, 2, 3", SC'11).  Counter (c0..c3), key (k0, k1); ten rounds; the key is bumped
 * by the Weyl constants between rounds.
 * ---------------------------------------------------------------------------------- */
void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    int round;
    for (round = 0; round < 10; round++) {
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;   /* multiplies word 0 */
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;   /* multiplies word 2 */
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += 0x9E3779B9u;   /* golden ratio */
        k1 += 0xBB67AE85u;   /* sqrt(3) - 1 */
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* ------------------------------------------------------------------------------------
 * bf16 round to nearest, ties to even.
 * ---------------------------------------------------------------------------------- */
static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

uint16_t oracle_bf16_from_f32(float f)
{
    uint32_t u = f32_bits(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);              /* quiet NaN */
    /* add half an ulp of bf16, plus one when the kept lsb is odd (ties to even) */
    u = u + 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

float oracle_f32_from_bf16(uint16_t b) { return bits_f32((uint32_t)b << 16); }

/* Direct round of a double to the nearest bf16 value (ties to even), no detour
 * through fp32.  bf16 keeps 8 significant bits; below 2^-126 the spacing is 2^-133. */
uint16_t oracle_bf16_from_f64(double y)
{
    int e;
    double q, fl, rem, r;
    if (y != y) return 0x7FC0u;
    if (y == 0.0) return (uint16_t)(signbit(y) ? 0x8000u : 0x0000u);
    (void)frexp(fabs(y), &e);               /* |y| = m * 2^e, m in [0.5, 1) */
    {
        int ulp_exp = e - 8;                /* spacing of 8 significant bits */
        if (ulp_exp < -133) ulp_exp = -133;
        q = ldexp(fabs(y), -ulp_exp);       /* exact: power-of-two scaling */
        fl = floor(q);
        rem = q - fl;                       /* exact */
        if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
        r = ldexp(fl, ulp_exp);
    }
    if (r >= 0x1p128) return (uint16_t)(y < 0 ? 0xFF80u : 0x7F80u);   /* overflow */
    {
        float rf = (float)r;                /* exact: r is a bf16 value */
        uint16_t b = (uint16_t)(f32_bits(rf) >> 16);
        return (uint16_t)(y < 0 ? (b | 0x8000u) : b);
    }
}

/* ------------------------------------------------------------------------------------
 * Synthetic table values (no trained weights exist; the pages call the table
 * learned).  The value of element (row, col) is a pure function of (seed, row, col).
 *
 * bf16: Philox counter (col/2, row, 1, 0), key (seed low 32, seed high 32).  Even
 *       columns take words (x0, x1), odd columns (x2, x3).  S is the sum of the four
 *       16-bit halves of those two words, C = 2S - 262140 is an even integer in
 *       [-262140, 262140] (Irwin-Hall of order 4, centred), v = C * K in fp32 with
 *       K = 0x1.1bc77ap-22 so that std(v) = 0.02, and the stored value is bf16(v).
 * int8: Philox counter (col/4, row, 2, 0); word x[col % 4]; q = (sum of its four
 *       bytes - 510) >> 2 (arithmetic), in [-128, 127].  Row scale: counter
 *       (0, row, 3, 0), s = K8 * (0.75 + (x0 >> 8) * 2^-25) in fp32 with separate
 *       roundings and K8 = 0x1.1bc5f4p-11, so that std(q * s) is about 0.02.
 * ---------------------------------------------------------------------------------- */
static void seed_key(uint64_t seed, uint32_t key[2])
{
    key[0] = (uint32_t)(seed & 0xFFFFFFFFu);
    key[1] = (uint32_t)(seed >> 32);
}

uint16_t oracle_table_bf16(uint64_t seed, uint64_t row, uint32_t col)
{
    uint32_t key[2], ctr[4], x[4], a, b;
    int32_t S, C;
    float v;
    seed_key(seed, key);
    ctr[0] = col >> 1; ctr[1] = (uint32_t)row; ctr[2] = 1u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    if ((col & 1u) == 0) { a = x[0]; b = x[1]; } else { a = x[2]; b = x[3]; }
    S = (int32_t)(a & 0xFFFFu) + (int32_t)(a >> 16) + (int32_t)(b & 0xFFFFu) + (int32_t)(b >> 16);
    C = 2 * S - 262140;
    v = (float)C * 0x1.1bc77ap-22f;
    return oracle_bf16_from_f32(v);
}

int8_t oracle_table_int8(uint64_t seed, uint64_t row, uint32_t col)
{
    uint32_t key[2], ctr[4], x[4], w;
    int32_t sum;
    seed_key(seed, key);
    ctr[0] = col >> 2; ctr[1] = (uint32_t)row; ctr[2] = 2u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    w = x[col & 3u];
    sum = (int32_t)(w & 0xFFu) + (int32_t)((w >> 8) & 0xFFu)
        + (int32_t)((w >> 16) & 0xFFu) + (int32_t)(w >> 24);
    /* arithmetic shift right by 2 == floor division by 4 */
    return (int8_t)((sum - 510) >= 0 ? (sum - 510) / 4 : -((510 - sum + 3) / 4));
}

float oracle_row_scale(uint64_t seed, uint64_t row)
{
    uint32_t key[2], ctr[4], x[4];
    float t, s;
    seed_key(seed, key);
    ctr[0] = 0u; ctr[1] = (uint32_t)row; ctr[2] = 3u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    t = (float)(x[0] >> 8) * 0x1p-25f;
    s = 0.75f + t;
    return 0x1.1bc5f4p-11f * s;
}

/* ------------------------------------------------------------------------------------
 * Low-precision element formats (OCP 8-bit floating point and Microscaling formats).
 *   E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is subnormal
 *         (m/8 * 2^-6); S.1111.111 is NaN; no infinities.  Largest finite 448.
 *   E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal
 *         (m * 0.5).  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 * ---------------------------------------------------------------------------------- */
double oracle_e4m3_value(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                  /* m/8 * 2^(1-7) */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

double oracle_e2m1_value(uint8_t nib)
{
    int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + m / 2.0, e - 1);
    return s ? -v : v;
}

/* Synthetic FP8 rows.  Element (row, col): Philox counter (col/4, row, 4, 0), word
 * w = x[col % 4]; sign = bit 31, exponent field 4 + bits[3:4] + bits[5:6] (4..10, never
 * NaN), mantissa bits[0:2].  Row scale: counter (0, row, 5, 0),
 * s = K * (0.75 + (x0 >> 8) * 2^-25) with K = 0x1.4dp-8 (std of the values ~0.02). */
uint8_t oracle_table_fp8(uint64_t seed, uint64_t row, uint32_t col)
{
    uint32_t key[2], ctr[4], x[4], w, e;
    seed_key(seed, key);
    ctr[0] = col >> 2; ctr[1] = (uint32_t)row; ctr[2] = 4u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    w = x[col & 3u];
    e = 4u + ((w >> 3) & 3u) + ((w >> 5) & 3u);
    return (uint8_t)(((w >> 31) << 7) | (e << 3) | (w & 7u));
}

float oracle_row_scale_fp8(uint64_t seed, uint64_t row)
{
    uint32_t key[2], ctr[4], x[4];
    float t, s;
    seed_key(seed, key);
    ctr[0] = 0u; ctr[1] = (uint32_t)row; ctr[2] = 5u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    t = (float)(x[0] >> 8) * 0x1p-25f;
    s = 0.75f + t;
    return 0x1.4dp-8f * s;
}

/* Synthetic NVFP4 rows.  Column c's 4-bit code: Philox counter (c/32, row, 6, 0), word
 * x[(c/8) % 4], nibble c % 8 (bits 4*(c%8)..).  Block b's E4M3 scale (columns 16b ..
 * 16b+15): counter (b/4, row, 7, 0), word w = x[b % 4]; positive, exponent field
 * 5 + bits[0:1] + bit[2] (5..9), mantissa bits[3:5].  Global scale 0x1.4fp-9 (std of
 * the values ~0.02). */
uint8_t oracle_table_fp4(uint64_t seed, uint64_t row, uint32_t col)
{
    uint32_t key[2], ctr[4], x[4];
    seed_key(seed, key);
    ctr[0] = col >> 5; ctr[1] = (uint32_t)row; ctr[2] = 6u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    return (uint8_t)((x[(col >> 3) & 3u] >> (4u * (col & 7u))) & 15u);
}

uint8_t oracle_block_scale_fp4(uint64_t seed, uint64_t row, uint32_t block)
{
    uint32_t key[2], ctr[4], x[4], w, e;
    seed_key(seed, key);
    ctr[0] = block >> 2; ctr[1] = (uint32_t)row; ctr[2] = 7u; ctr[3] = 0u;
    oracle_philox4x32_10(ctr, key, x);
    w = x[block & 3u];
    e = 5u + (w & 3u) + ((w >> 2) & 1u);
    return (uint8_t)((e << 3) | ((w >> 3) & 7u));
}

#define ORACLE_FP4_GLOBAL_SCALE 0x1.4fp-9f

/* Bytes of one NVFP4 row: d/2 code bytes, then d/16 scale bytes padded to 16. */
uint32_t oracle_fp4_row_bytes(uint32_t d) { return d / 2 + ((d / 16 + 15) / 16) * 16; }

void oracle_fill_fp8(uint64_t seed, uint64_t row0, uint64_t n_rows, uint32_t d,
                     uint8_t *q_out, float *scale_out)
{
    uint64_t r; uint32_t c;
    for (r = 0; r < n_rows; r++) {
        for (c = 0; c < d; c++)
            q_out[r * d + c] = oracle_table_fp8(seed, row0 + r, c);
        scale_out[r] = oracle_row_scale_fp8(seed, row0 + r);
    }
}

void oracle_fill_fp4(uint64_t seed, uint64_t row0, uint64_t n_rows, uint32_t d, uint8_t *out)
{
    const uint32_t rb = oracle_fp4_row_bytes(d);
    uint64_t r; uint32_t c, b;
    for (r = 0; r < n_rows; r++) {
        uint8_t *row = out + r * rb;
        memset(row, 0, rb);
        for (c = 0; c < d; c++)
            row[c / 2] |= (uint8_t)(oracle_table_fp4(seed, row0 + r, c) << (4 * (c & 1u)));
        for (b = 0; b < d / 16; b++)
            row[d / 2 + b] = oracle_block_scale_fp4(seed, row0 + r, b);
    }
}

/* Materialise rows [row0, row0 + n_rows) x d of the synthetic table on the host. */
void oracle_fill_bf16(uint64_t seed, uint64_t row0, uint64_t n_rows, uint32_t d, uint16_t *out)
{
    uint64_t r; uint32_t c;
    for (r = 0; r < n_rows; r++)
        for (c = 0; c < d; c++)
            out[r * d + c] = oracle_table_bf16(seed, row0 + r, c);
}

void oracle_fill_int8(uint64_t seed, uint64_t row0, uint64_t n_rows, uint32_t d,
                      int8_t *q_out, float *scale_out)
{
    uint64_t r; uint32_t c;
    for (r = 0; r < n_rows; r++) {
        for (c = 0; c < d; c++)
            q_out[r * d + c] = oracle_table_int8(seed, row0 + r, c);
        scale_out[r] = oracle_row_scale(seed, row0 + r);
    }
}

/* ------------------------------------------------------------------------------------
 * Context formation and hashing.
 * ---------------------------------------------------------------------------------- */
typedef struct {
    uint64_t base_seed;
    uint32_t n_bigram_heads;
    uint32_t n_trigram_heads;
    uint32_t pad_id;
    uint32_t vocab_size;
} oracle_hash_params;

/* Token (s, t) of a [n_seq][T] batch: w0 = w_t, w1 = w_{t-1}, w2 = w_{t-2}.  Earlier
 * positions come from history[s] = {w_-2, w_-1} (oldest first) when given, else PAD.
 * A token id outside [0, vocab_size) is replaced by PAD (the GPU library flags it). */
static uint32_t checked_id(int32_t w, const oracle_hash_params *hp)
{
    if (w < 0 || (uint32_t)w >= hp->vocab_size) return hp->pad_id;
    return (uint32_t)w;
}

static void context_of(const int32_t *tokens, const int32_t *history, uint32_t T,
                       uint32_t s, uint32_t t, const oracle_hash_params *hp,
                       uint32_t *w0, uint32_t *w1, uint32_t *w2)
{
    const int32_t *row = tokens + (size_t)s * T;
    uint32_t hist_old = hp->pad_id, hist_new = hp->pad_id;   /* w_-2, w_-1 */
    if (history != NULL) {
        hist_old = checked_id(history[2 * (size_t)s + 0], hp);
        hist_new = checked_id(history[2 * (size_t)s + 1], hp);
    }
    *w0 = checked_id(row[t], hp);
    if (t >= 1) *w1 = checked_id(row[t - 1], hp); else *w1 = hist_new;
    if (t >= 2) *w2 = checked_id(row[t - 2], hp);
    else if (t == 1) *w2 = hist_new;
    else *w2 = hist_old;
}

/* Indices of one token: head h < n_bigram uses the bigram key (w1 << 21) | w0, the
 * others the trigram key (w2 << 42) | (w1 << 21) | w0; row = mix(key ^ seed_h) % R. */
static void token_indices(uint32_t w0, uint32_t w1, uint32_t w2, const uint64_t *seeds,
                          const oracle_hash_params *hp, uint64_t R, uint32_t *idx)
{
    uint64_t k2 = ((uint64_t)w1 << 21) | (uint64_t)w0;
    uint64_t k3 = ((uint64_t)w2 << 42) | ((uint64_t)w1 << 21) | (uint64_t)w0;
    uint32_t H = hp->n_bigram_heads + hp->n_trigram_heads, h;
    for (h = 0; h < H; h++) {
        uint64_t key = (h < hp->n_bigram_heads) ? k2 : k3;
        uint64_t state = key ^ seeds[h];
        uint64_t mixed = oracle_splitmix64_next(&state);
        idx[h] = (uint32_t)(mixed % R);
    }
}

/* idx_out: [N][H] uint32, N = n_seq * T, H = heads.  Returns 0, or -1 on bad args. */
int oracle_indices(const int32_t *tokens, const int32_t *history, uint32_t n_seq, uint32_t T,
                   uint64_t R, const oracle_hash_params *hp, uint32_t *idx_out)
{
    uint64_t seeds[64];
    uint32_t H = hp->n_bigram_heads + hp->n_trigram_heads, s, t;
    if (H == 0 || H > 64 || R == 0) return -1;
    oracle_head_seeds(hp->base_seed, H, seeds);
    for (s = 0; s < n_seq; s++)
        for (t = 0; t < T; t++) {
            uint32_t w0, w1, w2;
            context_of(tokens, history, T, s, t, hp, &w0, &w1, &w2);
            token_indices(w0, w1, w2, seeds, hp, R, idx_out + ((size_t)s * T + t) * H);
        }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Forward: gather the H rows of each selected token, sum, gate, add, round to bf16.
 *
 *   tokens [n_seq][T] int32, history [n_seq][2] int32 or NULL,
 *   residual [N][d] bf16 bits, gate [d] fp32,
 *   sel: flat token ids (s * T + t) to compute, or NULL for all N (n_sel = N),
 *   out [n_sel][d] bf16 bits,
 *   y_out [n_sel][d] double or NULL: the pre-rounding value of the chosen mode,
 *   mag_out [n_sel][d] double or NULL: |r| + |g| * sum_h |E_h| (error-bound scale),
 *   idx_out [n_sel][H] uint32 or NULL.
 *   Rows: table_bf16 / (table_i8, scale) when non-NULL, else regenerated from
 *   table_seed through the synthetic-table definition above.
 *   n_threads > 1 splits the token loop across OpenMP threads (per-token work and
 *   arithmetic are unchanged).
 * ---------------------------------------------------------------------------------- */
/* Element (row, col) of the table: bf16 value v (s = 1, unused), or the pair (q, s)
 * with value q * s (int8: q the integer, s the row scale; fp8: q the E4M3 value, s the
 * row scale; nvfp4: q the E2M1 value, s the E4M3 block scale -- the global scale gs is
 * applied to the head sum, see head_sum).  Returns the exact value q * s (* gs for nvfp4)
 * in double.  For fp8 / nvfp4 a materialised table is passed as table_i8 (bytes) and the
 * scales as `scale` (fp8: per row; nvfp4: the global scale at scale[0], block scales
 * inside the row bytes). */
static double row_value(int dtype, const uint16_t *table_bf16, const int8_t *table_i8,
                        const float *scale, uint64_t seed, uint64_t row, uint32_t col,
                        uint32_t d, float *v_or_q, float *s_out)
{
    if (dtype == ORACLE_FP8) {
        const uint8_t code = table_i8 ? (uint8_t)table_i8[row * d + col] : oracle_table_fp8(seed, row, col);
        const float sc = scale ? scale[row] : oracle_row_scale_fp8(seed, row);
        *v_or_q = (float)oracle_e4m3_value(code);          /* exact */
        *s_out = sc;
        return (double)*v_or_q * (double)sc;
    }
    if (dtype == ORACLE_NVFP4) {
        const uint32_t rb = oracle_fp4_row_bytes(d);
        uint8_t code, bs;
        float gs, cs;
        if (table_i8) {
            const uint8_t *r = (const uint8_t *)table_i8 + row * rb;
            code = (uint8_t)((r[col / 2] >> (4 * (col & 1u))) & 15u);
            bs = r[d / 2 + col / 16];
        } else {
            code = oracle_table_fp4(seed, row, col);
            bs = oracle_block_scale_fp4(seed, row, col / 16);
        }
        gs = scale ? scale[0] : ORACLE_FP4_GLOBAL_SCALE;
        cs = (float)oracle_e4m3_value(bs);                  /* exact */
        *v_or_q = (float)oracle_e2m1_value(code);           /* exact */
        *s_out = cs;
        return (double)*v_or_q * (double)cs * (double)gs;  /* exact in double */
    }
    if (dtype == ORACLE_BF16) {
        uint16_t b = table_bf16 ? table_bf16[row * d + col] : oracle_table_bf16(seed, row, col);
        float f = oracle_f32_from_bf16(b);
        *v_or_q = f;
        *s_out = 1.0f;
        return (double)f;
    } else {
        int8_t q = table_i8 ? table_i8[row * d + col] : oracle_table_int8(seed, row, col);
        float sc = scale ? scale[row] : oracle_row_scale(seed, row);
        *v_or_q = (float)q;                        /* exact */
        *s_out = sc;
        return (double)q * (double)sc;             /* exact in double */
    }
}

/* The head sum of one column of one token (rows idx[0..H-1]):
 *   acc64 the exact sum (fp64; exact for these operands),
 *   acc32 the fp32 sum in head order: bf16 rows acc = acc + v; scaled rows
 *         acc = fmaf(q, s, acc), one rounding per head (int8, fp8, nvfp4 alike; q exact
 *         in fp32 in every case); for nvfp4 s is the E4M3 block scale (q * s exact) and
 *         the table's fp32 global scale multiplies the sum once at the end,
 *         acc32 = fp32(gs * acc32),
 *   mag   sum_h |E_h| (error-bound scale). */
static void head_sum(int dtype, const uint16_t *table_bf16, const int8_t *table_i8,
                     const float *row_scale, uint64_t table_seed, const uint32_t *idx,
                     uint32_t H, uint32_t c, uint32_t d, float *acc32, double *acc64, double *mag)
{
    uint32_t h;
    float a32 = 0.0f;
    double a64 = 0.0, m = 0.0;
    for (h = 0; h < H; h++) {
        float v, sc;
        double e64 = row_value(dtype, table_bf16, table_i8, row_scale, table_seed, idx[h], c, d,
                               &v, &sc);
        a64 += e64;
        if (dtype == ORACLE_BF16)
            a32 = a32 + v;
        else
            a32 = fmaf(v, sc, a32);
        m += fabs(e64);
    }
    if (dtype == ORACLE_NVFP4) {
        const float gs = row_scale ? row_scale[0] : ORACLE_FP4_GLOBAL_SCALE;
        a32 = gs * a32;                                     /* rounded once */
    }
    *acc32 = a32;
    *acc64 = a64;
    *mag = m;
}

/* gate_tok: NULL for the shared gate [d] fp32; else the per-token gate [N][d] bf16 bits
 * (gate is then unused): g = fp32(gate_tok[flat][c]), the same arithmetic otherwise. */
int oracle_forward(int dtype, const uint16_t *table_bf16, const int8_t *table_i8,
                   const float *row_scale, uint64_t table_seed, uint64_t R, uint32_t d,
                   const oracle_hash_params *hp,
                   const int32_t *tokens, const int32_t *history, uint32_t n_seq, uint32_t T,
                   const uint16_t *residual, const float *gate, const uint16_t *gate_tok,
                   const int64_t *sel, uint64_t n_sel, int acc_mode, int n_threads,
                   uint16_t *out, double *y_out, double *mag_out, uint32_t *idx_out)
{
    uint64_t seeds[64];
    uint32_t H = hp->n_bigram_heads + hp->n_trigram_heads;
    uint64_t N = (uint64_t)n_seq * T;
    int64_t i;
    if (H == 0 || H > 64 || R == 0 || d == 0) return -1;
    if (sel == NULL) n_sel = N;
    oracle_head_seeds(hp->base_seed, H, seeds);

#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (i = 0; i < (int64_t)n_sel; i++) {
        uint64_t flat = sel ? (uint64_t)sel[i] : (uint64_t)i;
        uint32_t s = (uint32_t)(flat / T), t = (uint32_t)(flat % T);
        uint32_t w0, w1, w2, idx[64], h, c;
        if (flat >= N) continue;
        context_of(tokens, history, T, s, t, hp, &w0, &w1, &w2);
        token_indices(w0, w1, w2, seeds, hp, R, idx);
        if (idx_out)
            for (h = 0; h < H; h++) idx_out[(size_t)i * H + h] = idx[h];
        for (c = 0; c < d; c++) {
            double acc64, mag, y64;
            float acc32;
            float r32 = oracle_f32_from_bf16(residual[flat * d + c]);
            float g32 = gate_tok ? oracle_f32_from_bf16(gate_tok[flat * d + c]) : gate[c];
            head_sum(dtype, table_bf16, table_i8, row_scale, table_seed, idx, H, c, d,
                     &acc32, &acc64, &mag);
            if (acc_mode == ORACLE_ACC_F64) {
                y64 = (double)r32 + (double)g32 * acc64;
                out[(size_t)i * d + c] = oracle_bf16_from_f64(y64);
            } else {
                float prod = g32 * acc32;          /* rounded separately (no FMA) */
                float y32 = r32 + prod;
                y64 = (double)y32;
                out[(size_t)i * d + c] = oracle_bf16_from_f32(y32);
            }
            if (y_out) y_out[(size_t)i * d + c] = y64;
            if (mag_out) mag_out[(size_t)i * d + c] = fabs((double)r32) + fabs((double)g32) * mag;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * Backward of out = residual + g (elementwise) sum_h E[idx_h], with dy = dL/dout given
 * as bf16 [N][d] (the gradient with respect to the residual is dy itself).
 * ---------------------------------------------------------------------------------- */

/* Gradient with respect to the table: only the rows the batch read have one.  The
 * occurrences are i = flat * H + h in ascending order; row idx[i] receives the
 * contribution of token flat = i / H once per occurrence (a row read by two heads of
 * one token receives it twice).  The distinct rows are listed in order of first
 * occurrence (uniq_out, U entries; the same list as the dedup step).  For the rows
 * u in sel_u (ascending positions in that list; NULL = all U rows):
 *   shared gate [d]:        grad[u] = g (elementwise) sum_i dy[flat(i)]
 *   per-token gate [N][d]:  grad[u] = sum_i g[flat(i)] (elementwise) dy[flat(i)]
 *   ACC_F64: fp64 (products of bf16 and fp32 values are exact in fp64; sums in
 *            ascending i);
 *   ACC_F32: shared: S = fp32 sum in ascending i (acc = acc + dy, from 0), then
 *            grad = fp32(g * S); per-token: acc = fmaf(g_t, dy_t, acc) in ascending i.
 * grad_out [n_sel][d] double; mag_out [n_sel][d] (sum_i |g dy|) or NULL.
 * Returns U, or -1 on bad arguments. */
int64_t oracle_backward_rows(uint64_t R, uint32_t d, const oracle_hash_params *hp,
                             const int32_t *tokens, const int32_t *history, uint32_t n_seq,
                             uint32_t T, const uint16_t *dy, const float *gate,
                             const uint16_t *gate_tok, const int64_t *sel_u, uint64_t n_sel,
                             int acc_mode, int n_threads, uint32_t *uniq_out, double *grad_out,
                             double *mag_out)
{
    const uint32_t H = hp->n_bigram_heads + hp->n_trigram_heads;
    const uint64_t N = (uint64_t)n_seq * T, M = N * H;
    uint32_t *idx, *u_of, *keys, *vals, *start, *occ;
    uint64_t P = 16, i, U = 0;
    int64_t k;
    if (H == 0 || H > 64 || R == 0 || d == 0) return -1;
    if (M == 0) return 0;
    idx = malloc(M * sizeof(uint32_t));
    u_of = malloc(M * sizeof(uint32_t));
    while (P < 2 * M) P <<= 1;
    keys = malloc(P * sizeof(uint32_t));
    vals = malloc(P * sizeof(uint32_t));
    start = calloc(M + 1, sizeof(uint32_t));
    occ = malloc(M * sizeof(uint32_t));
    if (!idx || !u_of || !keys || !vals || !start || !occ) {
        free(idx); free(u_of); free(keys); free(vals); free(start); free(occ);
        return -1;
    }
    oracle_indices(tokens, history, n_seq, T, R, hp, idx);
    /* first-occurrence numbering through a plain open-addressing map row -> u */
    for (i = 0; i < P; i++) keys[i] = 0xFFFFFFFFu;
    for (i = 0; i < M; i++) {
        uint64_t slot = ((uint64_t)idx[i] * 0x9E3779B97F4A7C15ull) & (P - 1);
        while (keys[slot] != 0xFFFFFFFFu && keys[slot] != idx[i]) slot = (slot + 1) & (P - 1);
        if (keys[slot] == 0xFFFFFFFFu) {
            keys[slot] = idx[i];
            vals[slot] = (uint32_t)U;
            uniq_out[U++] = idx[i];
        }
        u_of[i] = vals[slot];
    }
    /* the occurrences of each u in ascending i (counting sort, stable by construction) */
    for (i = 0; i < M; i++) start[u_of[i] + 1]++;
    for (i = 0; i < U; i++) start[i + 1] += start[i];
    {
        uint32_t *fill = malloc(U * sizeof(uint32_t));
        if (!fill) { free(idx); free(u_of); free(keys); free(vals); free(start); free(occ); return -1; }
        memcpy(fill, start, U * sizeof(uint32_t));
        for (i = 0; i < M; i++) occ[fill[u_of[i]]++] = (uint32_t)i;
        free(fill);
    }
    if (sel_u == NULL) n_sel = U;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (k = 0; k < (int64_t)n_sel; k++) {
        const uint64_t u = sel_u ? (uint64_t)sel_u[k] : (uint64_t)k;
        uint32_t c, j;
        if (u >= U) continue;
        for (c = 0; c < d; c++) {
            float acc32 = 0.0f;
            double acc64 = 0.0, mag = 0.0;
            for (j = start[u]; j < start[u + 1]; j++) {
                const uint64_t flat = occ[j] / H;
                const float dy32 = oracle_f32_from_bf16(dy[flat * d + c]);
                const float g32 = gate_tok ? oracle_f32_from_bf16(gate_tok[flat * d + c]) : gate[c];
                if (gate_tok) {
                    acc32 = fmaf(g32, dy32, acc32);
                    acc64 += (double)g32 * (double)dy32;
                } else {
                    acc32 = acc32 + dy32;
                    acc64 += (double)dy32;
                }
                mag += fabs((double)g32 * (double)dy32);
            }
            if (!gate_tok) {
                acc32 = gate[c] * acc32;
                acc64 = (double)gate[c] * acc64;
            }
            grad_out[(size_t)k * d + c] = (acc_mode == ORACLE_ACC_F64) ? acc64 : (double)acc32;
            if (mag_out) mag_out[(size_t)k * d + c] = mag;
        }
    }
    free(idx); free(u_of); free(keys); free(vals); free(start); free(occ);
    return (int64_t)U;
}

/* Gradient with respect to the gate; e[t] = the head sum of token t (head_sum).
 *   shared gate:    dg[c] = sum over all N tokens of dy[t][c] * e[t][c]     (out [d])
 *   per-token gate: dg[t][c] = dy[t][c] * e[t][c] for the tokens in sel      (out [n_sel][d])
 *   ACC_F64: e exact; products and the sum in fp64.
 *   ACC_F32: e = the fp32 head-order sum (as in forward); p = dy * e is exact in fp64;
 *            shared: the fp64 sum in ascending t, rounded once to fp32; per-token: p
 *            rounded to fp32.
 * mag_out (same shape, or NULL): |dy| * sum_h |E_h| (summed over t for the shared gate).
 * The shared gate sums every token (sel is ignored). */
int oracle_backward_gate(int dtype, const uint16_t *table_bf16, const int8_t *table_i8,
                         const float *row_scale, uint64_t table_seed, uint64_t R, uint32_t d,
                         const oracle_hash_params *hp, const int32_t *tokens,
                         const int32_t *history, uint32_t n_seq, uint32_t T, const uint16_t *dy,
                         int per_token, const int64_t *sel, uint64_t n_sel, int acc_mode,
                         int n_threads, double *dg_out, double *mag_out)
{
    uint64_t seeds[64];
    const uint32_t H = hp->n_bigram_heads + hp->n_trigram_heads;
    const uint64_t N = (uint64_t)n_seq * T;
    double *terms = NULL, *mags = NULL;
    int64_t i;
    if (H == 0 || H > 64 || R == 0 || d == 0) return -1;
    if (!per_token || sel == NULL) n_sel = N;
    if (!per_token) {
        /* every token's terms first (in parallel), then one sum per column in ascending t */
        terms = malloc(N * d * sizeof(double));
        mags = malloc(N * d * sizeof(double));
        if (N > 0 && (!terms || !mags)) { free(terms); free(mags); return -1; }
    }
    oracle_head_seeds(hp->base_seed, H, seeds);
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (i = 0; i < (int64_t)n_sel; i++) {
        const uint64_t flat = (per_token && sel) ? (uint64_t)sel[i] : (uint64_t)i;
        const uint32_t s = (uint32_t)(flat / T), t = (uint32_t)(flat % T);
        uint32_t w0, w1, w2, idx[64], c;
        if (flat >= N) continue;
        context_of(tokens, history, T, s, t, hp, &w0, &w1, &w2);
        token_indices(w0, w1, w2, seeds, hp, R, idx);
        for (c = 0; c < d; c++) {
            float acc32;
            double acc64, mag, p;
            const double dy64 = (double)oracle_f32_from_bf16(dy[flat * d + c]);
            head_sum(dtype, table_bf16, table_i8, row_scale, table_seed, idx, H, c, d,
                     &acc32, &acc64, &mag);
            p = dy64 * ((acc_mode == ORACLE_ACC_F64) ? acc64 : (double)acc32);
            if (per_token) {
                dg_out[(size_t)i * d + c] = (acc_mode == ORACLE_ACC_F64) ? p : (double)(float)p;
                if (mag_out) mag_out[(size_t)i * d + c] = fabs(dy64) * mag;
            } else {
                terms[flat * d + c] = p;
                mags[flat * d + c] = fabs(dy64) * mag;
            }
        }
    }
    if (!per_token) {
        uint32_t c;
        uint64_t t;
        for (c = 0; c < d; c++) {
            double sum = 0.0, m = 0.0;
            for (t = 0; t < N; t++) {
                sum += terms[t * d + c];
                m += mags[t * d + c];
            }
            dg_out[c] = (acc_mode == ORACLE_ACC_F64) ? sum : (double)(float)sum;
            if (mag_out) mag_out[c] = m;
        }
        free(terms);
        free(mags);
    }
    return 0;
}
