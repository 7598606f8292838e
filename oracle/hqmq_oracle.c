/*
 * hqmq_oracle.c -- plain, slow, obviously-correct CPU oracle for HQMQ
 * (Hurwitz Quaternion Multiplicative Quantization) KV-cache encode/decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, __graft_entry__.smoke() and the cpu_baseline
 * leg of bench.py use it.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (cited below by the short tag in brackets):
 *   [ABS]   arXiv 2605.27646 abstract, as printed on paperdance.org/p/2605.27646
 *           and thelatestinai.com/papers/2605.27646
 *   [NL M]  gist.science/nl/paper/2605.27646, "Technische Samenvatting",
 *           section "Methodologie"
 *   [NL 1]  same page, "1. Multiplicatieve Samenstelling van Codeboeken"
 *   [NL 2]  same page, "2. Theoretische Rechtvaardiging voor Willekeurige Initialisatie"
 *   [NL 3]  same page, "3. Mediane-Multiplier Uitbijterextractie (Med3x)"
 *   [NL ML] same page, "Memory en Latentie"
 *   [PT 1], [PT 3] gist.science/pt/paper/2605.27646, "Resumo Tecnico",
 *           sections 1 and 3 (same content as NL 1 / NL 3)
 *   [FR]    signal-ia-rouge.vercel.app article, section "La mecanique"
 *
 * Readings where the pages are silent:
 *   quaternion order (w,i,j,k) = 4 consecutive elements; Hamilton product with
 *   ij = k; the 2T enumeration p in [0,24); global index s*24+p with ties to
 *   the lowest index; codebook RNG = Philox4x32-10 + Box-Muller in fp64;
 *   fp32 chunk norm in a fixed fma order; fp16 radius; lower median; strict
 *   r > C*r_med; LSB-first bit packing in groups of 32 chunks; the optional
 *   quantized radius uniform on [0, thr] in 24 S levels.
 *
 * Precision: the argmax and the outlier test are integer-valued decisions, so
 * they are taken in fp32, the precision of the GPU kernels.  The codebook is
 * drawn in fp64 and rounded once to fp32.  Every fp32 step below is a single
 * IEEE operation (compiled with -ffp-contract=off), so its rounding is fixed.
 *
 * Parity pins for every function are in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_BF16 0
#define OR_F32 1
#define OR_GRAN_CHUNK 0
#define OR_GRAN_ELEMENT 1

#define OR_FLAG_OVERFLOW 1u
#define OR_FLAG_SATURATED 2u
#define OR_FLAG_NONFINITE 4u
#define OR_FLAG_BAD_INDEX 8u

typedef struct {
    uint32_t flags;
    uint32_t reserved;
    uint64_t n_outliers;
    uint64_t n_saturated;
    uint64_t n_nonfinite;
} oracle_status;

/* ------------------------------------------------------------------------ */
/* Scalar formats                                                            */
/* ------------------------------------------------------------------------ */

static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* bf16 -> fp32 is exact: the bf16 bits are the upper half of the fp32 bits. */
float oracle_bf16_to_f32(uint16_t h) { return u2f((uint32_t)h << 16); }

/* fp32 -> bf16, IEEE round-to-nearest-even on the upper 16 bits; any NaN
 * becomes the quiet NaN 0x7FC0 (sign kept). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u = f2u(f);
    if (isnan(f)) return (uint16_t)(((u >> 16) & 0x8000u) | 0x7FC0u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* fp16 -> fp32 (exact), written from the binary16 layout:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
float oracle_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 31) {
        if (m) return sign ? -NAN : NAN;
        return sign ? -INFINITY : INFINITY;
    }
    if (e == 0) v = ldexp((double)m, -24);                 /* subnormal */
    else v = ldexp(1.0 + (double)m / 1024.0, e - 15);       /* normal    */
    return (float)(sign ? -v : v);
}

/* fp32 -> fp16, round-to-nearest-even.  The value is exact in fp64, so the
 * rounding is done on the scaled fp64 value with rint() (ties to even in the
 * default rounding mode).  Finite values whose rounding would be +-inf are
 * saturated to +-65504 and *saturated is set; inf stays inf, NaN -> 0x7E00. */
uint16_t oracle_f32_to_f16_sat(float f, int *saturated)
{
    uint16_t sign = (f2u(f) >> 16) & 0x8000u;
    if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
    if (isinf(f)) return (uint16_t)(sign | 0x7C00u);
    double a = fabs((double)f);
    if (a >= 65520.0) {                  /* rounds to inf under RN-even */
        if (saturated) *saturated = 1;
        return (uint16_t)(sign | 0x7BFFu);
    }
    if (a < ldexp(1.0, -14)) {           /* subnormal range: step 2^-24  */
        double q = rint(a * ldexp(1.0, 24));  /* 0..1024; 1024 == min normal */
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e;
    double m = frexp(a, &e);             /* a = m * 2^e, m in [0.5, 1)   */
    m *= 2.0; e -= 1;                    /* a = m * 2^e, m in [1, 2)     */
    double q = rint((m - 1.0) * 1024.0);
    if (q == 1024.0) { q = 0.0; e += 1; }
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)q);
}

/* ------------------------------------------------------------------------ */
/* Quaternion algebra [NL M]: x in H, stored (w, i, j, k).                   */
/* ------------------------------------------------------------------------ */

/* Hamilton product a*b in fp64, from i^2 = j^2 = k^2 = ijk = -1. */
void oracle_qmul_f64(const double *a, const double *b, double *out)
{
    double w = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
    double x = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
    double y = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
    double z = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
    out[0] = w; out[1] = x; out[2] = y; out[3] = z;
}

/* The 24 elements of the binary tetrahedral group 2T [NL 1], [ABS]:
 *   p = 2a + sg (a in 0..3 = axis w,i,j,k; sg = 0 for +, 1 for -):
 *       the 8 units +-1, +-i, +-j, +-k;
 *   p = 8 + m (m in 0..15): 1/2 ((-1)^m0, (-1)^m1, (-1)^m2, (-1)^m3),
 *       m_c = bit c of m.                                                    */
void oracle_2t_element(int p, double *q)
{
    q[0] = q[1] = q[2] = q[3] = 0.0;
    if (p < 8) {
        q[p >> 1] = (p & 1) ? -1.0 : 1.0;
    } else {
        int m = p - 8;
        for (int c = 0; c < 4; ++c) q[c] = ((m >> c) & 1) ? -0.5 : 0.5;
    }
}

/* Effective codeword q_p * q_s [NL 1] in fp32: each component is the sum, left
 * to right, of the four Hamilton terms in the order written in
 * oracle_qmul_f64, each term an fp32 product (exact, since q_p entries are
 * 0, +-1 or +-1/2) and each partial sum rounded to fp32. */
void oracle_codeword_f32(int p, const float *qs, float *c)
{
    double qp[4];
    oracle_2t_element(p, qp);
    float a0 = (float)qp[0], a1 = (float)qp[1], a2 = (float)qp[2], a3 = (float)qp[3];
    float b0 = qs[0], b1 = qs[1], b2 = qs[2], b3 = qs[3];
    float t;
    t = a0 * b0; t = t - a1 * b1; t = t - a2 * b2; t = t - a3 * b3; c[0] = t;
    t = a0 * b1; t = t + a1 * b0; t = t + a2 * b3; t = t - a3 * b2; c[1] = t;
    t = a0 * b2; t = t - a1 * b3; t = t + a2 * b0; t = t + a3 * b1; c[2] = t;
    t = a0 * b3; t = t + a1 * b2; t = t - a2 * b1; t = t + a3 * b0; c[3] = t;
}

/* ------------------------------------------------------------------------ */
/* Secondary codebook [NL 1], [PT 1]: S random unit quaternions for each     */
/* (layer, head, role), drawn with no calibration data; [ABS]: seeded.       */
/* ------------------------------------------------------------------------ */

/* Philox4x32-10 counter-based generator, from its published definition
 * (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
 * SC'11): ten rounds of a multiply-xor S-box with multipliers 0xD2511F53 and
 * 0xCD9E8D57, the two-word key bumped by the Weyl constants 0x9E3779B9 and
 * 0xBB67AE85 between rounds. */
void oracle_philox4x32_10(const uint32_t *ctr_in, const uint32_t *key_in, uint32_t *out)
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint64_t prod_a = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t prod_b = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi_a = (uint32_t)(prod_a >> 32), lo_a = (uint32_t)prod_a;
        uint32_t hi_b = (uint32_t)(prod_b >> 32), lo_b = (uint32_t)prod_b;
        uint32_t n0 = hi_b ^ c1 ^ k0;
        uint32_t n1 = lo_b;
        uint32_t n2 = hi_a ^ c3 ^ k1;
        uint32_t n3 = lo_a;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* One secondary codeword q_{g,s}: four uniforms u = (v + 1/2) 2^-32 from
 * Philox4x32-10(counter = (s, g, 0, 0), key = (seed lo, seed hi)); two
 * Box-Muller pairs (Box & Muller 1958) give four N(0,1) deviates z; the unit
 * quaternion is z / |z| in fp64, rounded once to fp32.  A normalised Gaussian
 * 4-vector is Haar-uniform on S^3. */
void oracle_codeword_secondary(uint64_t seed, uint32_t g, uint32_t s, float *q)
{
    const double two_pi = 6.283185307179586; /* fp64 nearest to 2*pi */
    uint32_t ctr[4] = {s, g, 0u, 0u};
    uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
    uint32_t v[4];
    oracle_philox4x32_10(ctr, key, v);
    double u[4];
    for (int i = 0; i < 4; ++i) u[i] = ((double)v[i] + 0.5) * 2.3283064365386963e-10; /* 2^-32 */
    double rad0 = sqrt(-2.0 * log(u[0]));
    double rad1 = sqrt(-2.0 * log(u[2]));
    double th0 = two_pi * u[1];
    double th1 = two_pi * u[3];
    double z[4];
    z[0] = rad0 * cos(th0);
    z[1] = rad0 * sin(th0);
    z[2] = rad1 * cos(th1);
    z[3] = rad1 * sin(th1);
    double n2 = z[0] * z[0] + z[1] * z[1] + z[2] * z[2] + z[3] * z[3];
    double n = sqrt(n2);
    if (!(n > 1e-300)) { q[0] = 1.0f; q[1] = q[2] = q[3] = 0.0f; return; }
    for (int i = 0; i < 4; ++i) q[i] = (float)(z[i] / n);
}

/* Codebook rows for groups group0 .. group0+n_groups-1, layout [g][s][4]. */
void oracle_make_codebook(uint64_t seed, uint32_t S, uint32_t n_groups, uint32_t group0, float *out)
{
    for (uint32_t gl = 0; gl < n_groups; ++gl)
        for (uint32_t s = 0; s < S; ++s)
            oracle_codeword_secondary(seed, group0 + gl, s, out + ((size_t)gl * S + s) * 4);
}

/* ------------------------------------------------------------------------ */
/* Polar split [NL M]: r = |x|, u = x / r.                                    */
/* ------------------------------------------------------------------------ */

/* r = sqrt(x0^2 + x1^2 + x2^2 + x3^2) in fp32 with the order fixed:
 * r2 = fma(x3,x3, fma(x2,x2, fma(x1,x1, x0*x0))), r = sqrt(r2). */
float oracle_chunk_norm(const float *x)
{
    float r2 = x[0] * x[0];
    r2 = fmaf(x[1], x[1], r2);
    r2 = fmaf(x[2], x[2], r2);
    r2 = fmaf(x[3], x[3], r2);
    return sqrtf(r2);
}

/* Order key of a non-negative fp32 magnitude: its bit pattern (monotone for
 * +0 .. +inf); every NaN maps to 0x7FFFFFFF, above +inf. */
static uint32_t mag_key(float v) { return isnan(v) ? 0x7FFFFFFFu : f2u(v); }

static float load_elem(const void *x, int dtype, size_t e)
{
    if (dtype == OR_BF16) return oracle_bf16_to_f32(((const uint16_t *)x)[e]);
    return ((const float *)x)[e];
}

/* ------------------------------------------------------------------------ */
/* Search [NL 1]: u -> argmax_{c in C} <u, c>, C = {q_p q_s}, 24S words.      */
/* ------------------------------------------------------------------------ */

/* fp32 score <u, c>, products and sums left to right, each rounded. */
static float dot4_f32(const float *u, const float *c)
{
    float t = u[0] * c[0];
    t = t + u[1] * c[1];
    t = t + u[2] * c[2];
    t = t + u[3] * c[3];
    return t;
}

/* Build the explicit 24*S codeword table of one head: row s*24+p. */
static void build_table(const float *qs_head, uint32_t S, float *table)
{
    for (uint32_t s = 0; s < S; ++s)
        for (int p = 0; p < 24; ++p)
            oracle_codeword_f32(p, qs_head + (size_t)s * 4, table + ((size_t)s * 24 + p) * 4);
}

/* Brute-force nearest codeword of one chunk x (already zeroed where Med3x
 * says so).  Returns the index (ties -> lowest index), writes the fp32 norm,
 * the best and the second-best score (over all other codewords).
 * r == 0 -> index 0; r not finite -> index 0. */
static uint32_t search_chunk(const float *x, const float *table, uint32_t S,
                             float *r_out, float *best_out, float *second_out)
{
    float r = oracle_chunk_norm(x);
    *r_out = r;
    *best_out = 0.0f; *second_out = 0.0f;
    if (!(r > 0.0f) || isinf(r)) return 0u;       /* zero, NaN or inf */
    float u[4] = {x[0] / r, x[1] / r, x[2] / r, x[3] / r};
    float best = -INFINITY, second = -INFINITY;
    uint32_t bi = 0;
    uint32_t n = 24u * S;
    for (uint32_t i = 0; i < n; ++i) {
        float sc = dot4_f32(u, table + (size_t)i * 4);
        if (sc > best) { second = best; best = sc; bi = i; }
        else if (sc > second) second = sc;
    }
    *best_out = best; *second_out = second;
    return bi;
}

/* fp32 score of codeword `idx` for chunk x, same arithmetic as search_chunk. */
float oracle_score(const float *x, const float *qs_head, uint32_t S, uint32_t idx)
{
    float r = oracle_chunk_norm(x);
    if (!(r > 0.0f) || isinf(r) || idx >= 24u * S) return 0.0f;
    float u[4] = {x[0] / r, x[1] / r, x[2] / r, x[3] / r};
    float c[4];
    oracle_codeword_f32((int)(idx % 24u), qs_head + (size_t)(idx / 24u) * 4, c);
    return dot4_f32(u, c);
}

uint32_t oracle_index_bits(uint32_t S)
{
    uint64_t n = 24ull * S;
    uint32_t b = 0;
    while ((1ull << b) < n) ++b;
    return b;
}

/* LSB-first packing: in a group of 32 consecutive chunks, bit i of chunk k's
 * index is bit k*b+i of the group's b-word stream (word (k*b+i)/32, bit
 * (k*b+i)%32). */
static void put_index(uint32_t *words, uint32_t b, size_t chunk, uint32_t idx)
{
    size_t grp = chunk / 32, k = chunk % 32;
    uint32_t *w = words + grp * b;
    for (uint32_t i = 0; i < b; ++i) {
        size_t bit = k * b + i;
        if ((idx >> i) & 1u) w[bit / 32] |= 1u << (bit % 32);
    }
}

uint32_t oracle_get_index(const uint32_t *words, uint32_t b, size_t chunk)
{
    size_t grp = chunk / 32, k = chunk % 32;
    const uint32_t *w = words + grp * b;
    uint32_t idx = 0;
    for (uint32_t i = 0; i < b; ++i) {
        size_t bit = k * b + i;
        idx |= ((w[bit / 32] >> (bit % 32)) & 1u) << i;
    }
    return idx;
}

/* Chunk j of a [B,H,T,D] tensor: element base 4j, head (j / (T*D/4)) % H. */
static int head_of_chunk(size_t j, int H, int T, int D)
{
    size_t per_slab = (size_t)T * (size_t)D / 4;
    return (int)((j / per_slab) % (size_t)H);
}

/* Load chunk j in fp32 and apply the Med3x zeroing [NL 3]:
 * chunk mode: a chunk with r > thr becomes 0; element mode: an element with
 * |x| > thr becomes 0.  Returns 1 if the chunk was an outlier (chunk mode). */
static int load_chunk(const void *x, int dtype, size_t j, const float *thr_h,
                      int gran, float *c)
{
    for (int i = 0; i < 4; ++i) c[i] = load_elem(x, dtype, 4 * j + i);
    if (!thr_h) return 0;
    if (gran == OR_GRAN_CHUNK) {
        float r = oracle_chunk_norm(c);
        if (r > *thr_h) { c[0] = c[1] = c[2] = c[3] = 0.0f; return 1; }
        return 0;
    }
    for (int i = 0; i < 4; ++i)
        if (fabsf(c[i]) > *thr_h) c[i] = 0.0f;
    return 0;
}

static void status_add(oracle_status *st, uint32_t flag, uint64_t *ctr, uint64_t n)
{
    if (!st || n == 0) return;
    st->flags |= flag;
    *ctr += n;
}

/* Encode a [B,H,T,D] tensor [NL M], [NL 1]: per chunk the fp16 radius and
 * the packed codeword index.  codebook: [H][S][4] fp32 of this call's heads.
 * thr: [H] Med3x thresholds or NULL.  words: zero-initialised by this call.
 * A chunk whose radius is not finite gets index 0 and radius 0x7E00 and is
 * counted as non-finite.  best/second (optional, per chunk) receive the two
 * top fp32 scores (0 for zero / non-finite chunks). */
void oracle_encode(const void *x, int dtype, int B, int H, int T, int D,
                   const float *codebook, uint32_t S, const float *thr, int gran,
                   uint32_t *words, uint16_t *radius, float *best, float *second,
                   oracle_status *st)
{
    size_t n_chunks = (size_t)B * H * T * D / 4;
    uint32_t b = oracle_index_bits(S);
    memset(words, 0, (n_chunks / 32) * b * sizeof(uint32_t));
    float *tables = (float *)malloc((size_t)H * 24 * S * 4 * sizeof(float));
    for (int h = 0; h < H; ++h)
        build_table(codebook + (size_t)h * S * 4, S, tables + (size_t)h * 24 * S * 4);
    uint64_t n_sat = 0, n_nf = 0;
    for (size_t j = 0; j < n_chunks; ++j) {
        int h = head_of_chunk(j, H, T, D);
        float c[4];
        load_chunk(x, dtype, j, thr ? thr + h : NULL, gran, c);
        float r, bs, sc;
        uint32_t idx = search_chunk(c, tables + (size_t)h * 24 * S * 4, S, &r, &bs, &sc);
        uint16_t rh;
        if (isnan(r) || isinf(r)) { rh = 0x7E00u; ++n_nf; idx = 0; }
        else {
            int sat = 0;
            rh = oracle_f32_to_f16_sat(r, &sat);
            n_sat += (uint64_t)sat;
        }
        radius[j] = rh;
        put_index(words, b, j, idx);
        if (best) best[j] = bs;
        if (second) second[j] = sc;
    }
    status_add(st, OR_FLAG_SATURATED, st ? &st->n_saturated : NULL, n_sat);
    status_add(st, OR_FLAG_NONFINITE, st ? &st->n_nonfinite : NULL, n_nf);
    free(tables);
}

/* Encode only the listed chunks (for sampled parity at full size): writes the
 * index, radius, best and second score of each listed chunk. */
void oracle_encode_chunks(const void *x, int dtype, int B, int H, int T, int D,
                          const float *codebook, uint32_t S, const float *thr, int gran,
                          const int64_t *chunks, int64_t n, uint32_t *idx_out,
                          uint16_t *radius_out, float *best, float *second)
{
    (void)B;
    float *table = (float *)malloc((size_t)24 * S * 4 * sizeof(float));
    int cur_h = -1;
    for (int64_t q = 0; q < n; ++q) {
        size_t j = (size_t)chunks[q];
        int h = head_of_chunk(j, H, T, D);
        if (h != cur_h) { build_table(codebook + (size_t)h * S * 4, S, table); cur_h = h; }
        float c[4];
        load_chunk(x, dtype, j, thr ? thr + h : NULL, gran, c);
        float r, bs, sc;
        uint32_t idx = search_chunk(c, table, S, &r, &bs, &sc);
        uint16_t rh;
        if (isnan(r) || isinf(r)) { rh = 0x7E00u; idx = 0; }
        else rh = oracle_f32_to_f16_sat(r, NULL);
        idx_out[q] = idx;
        radius_out[q] = rh;
        if (best) best[q] = bs;
        if (second) second[q] = sc;
    }
    free(table);
}

/* ------------------------------------------------------------------------ */
/* Med3x [NL 3], [PT 3]: median chunk norm r_med over the current batch;     */
/* chunks with r > C * r_med are outliers, kept in fp16 with a flag.          */
/* ------------------------------------------------------------------------ */

static int cmp_u32(const void *a, const void *b)
{
    uint32_t x = *(const uint32_t *)a, y = *(const uint32_t *)b;
    return (x > y) - (x < y);
}

/* Per head h: r_med = the lower median (rank N/2 - 1 of N ascending) of the
 * chunk norms (chunk mode) or of the element magnitudes |x| (element mode)
 * over all batches and tokens of this call; thr = fl32(C * r_med).
 * rmed/thr: [H]. */
void oracle_med3_threshold(const void *x, int dtype, int B, int H, int T, int D,
                           float C, int gran, float *rmed, float *thr)
{
    size_t per_slab_chunks = (size_t)T * D / 4;
    size_t n_per_head = (gran == OR_GRAN_CHUNK) ? (size_t)B * per_slab_chunks
                                                : (size_t)B * T * D;
    uint32_t *keys = (uint32_t *)malloc(n_per_head * sizeof(uint32_t));
    for (int h = 0; h < H; ++h) {
        size_t n = 0;
        for (int b = 0; b < B; ++b) {
            size_t slab = (size_t)b * H + h;
            for (size_t c = 0; c < per_slab_chunks; ++c) {
                size_t j = slab * per_slab_chunks + c;
                float v[4];
                for (int i = 0; i < 4; ++i) v[i] = load_elem(x, dtype, 4 * j + i);
                if (gran == OR_GRAN_CHUNK) keys[n++] = mag_key(oracle_chunk_norm(v));
                else for (int i = 0; i < 4; ++i) keys[n++] = mag_key(fabsf(v[i]));
            }
        }
        qsort(keys, n, sizeof(uint32_t), cmp_u32);
        uint32_t k = keys[n / 2 - 1];
        float m = (k == 0x7FFFFFFFu) ? NAN : u2f(k);
        rmed[h] = m;
        thr[h] = C * m;
    }
    free(keys);
}

/* Outlier list [NL 3]: ascending flat index; chunk mode stores (chunk index,
 * the 4 original values in fp16), element mode (element index, fp16 value).
 * slab_off[B*H+1]: entries of slab (b,h) are [slab_off[bh], slab_off[bh+1]).
 * Entries past cap are not written; returns the required count. */
int64_t oracle_extract(const void *x, int dtype, int B, int H, int T, int D,
                       const float *thr, int gran, uint32_t *out_idx, uint16_t *out_val,
                       uint32_t *slab_off, uint64_t cap, oracle_status *st)
{
    size_t per_slab_chunks = (size_t)T * D / 4;
    size_t n_slabs = (size_t)B * H;
    uint64_t cnt = 0, n_sat = 0;
    for (size_t slab = 0; slab < n_slabs; ++slab) {
        int h = (int)(slab % (size_t)H);
        if (slab_off) slab_off[slab] = (uint32_t)cnt;
        for (size_t c = 0; c < per_slab_chunks; ++c) {
            size_t j = slab * per_slab_chunks + c;
            float v[4];
            for (int i = 0; i < 4; ++i) v[i] = load_elem(x, dtype, 4 * j + i);
            if (gran == OR_GRAN_CHUNK) {
                if (oracle_chunk_norm(v) > thr[h]) {
                    if (cnt < cap) {
                        out_idx[cnt] = (uint32_t)j;
                        for (int i = 0; i < 4; ++i) {
                            int sat = 0;
                            out_val[cnt * 4 + i] = oracle_f32_to_f16_sat(v[i], &sat);
                            n_sat += (uint64_t)sat;
                        }
                    }
                    ++cnt;
                }
            } else {
                for (int i = 0; i < 4; ++i) {
                    if (fabsf(v[i]) > thr[h]) {
                        if (cnt < cap) {
                            int sat = 0;
                            out_idx[cnt] = (uint32_t)(4 * j + i);
                            out_val[cnt] = oracle_f32_to_f16_sat(v[i], &sat);
                            n_sat += (uint64_t)sat;
                        }
                        ++cnt;
                    }
                }
            }
        }
    }
    if (slab_off) slab_off[n_slabs] = (uint32_t)cnt;
    if (st) {
        st->n_outliers += cnt;
        if (cnt > cap) st->flags |= OR_FLAG_OVERFLOW;
    }
    status_add(st, OR_FLAG_SATURATED, st ? &st->n_saturated : NULL, n_sat);
    return (int64_t)cnt;
}

/* ------------------------------------------------------------------------ */
/* Decode: x_hat = r * (q_p q_s) [NL M], outliers restored [NL 3].            */
/* ------------------------------------------------------------------------ */

static void store_elem(void *y, int out_dtype, size_t e, float v)
{
    if (out_dtype == OR_BF16) ((uint16_t *)y)[e] = oracle_f32_to_bf16(v);
    else ((float *)y)[e] = v;
}

/* Decode a whole call.  y[e] = round(fl32(r * c_i)) with r the fp16 radius
 * widened exactly and c the fp32 codeword of oracle_codeword_f32.  Outliers
 * (n_out entries of out_idx/out_val, or none if out_idx == NULL):
 * chunk mode: the chunk becomes round(fp16 value); element mode:
 * y[e] = round(fl32(fl32(r * c_i) + v)).  An index >= 24*S is flagged and
 * decodes to 0. */
void oracle_decode(const uint32_t *words, const uint16_t *radius, const float *codebook,
                   uint32_t S, const uint32_t *out_idx, const uint16_t *out_val,
                   int64_t n_out, int gran, int B, int H, int T, int D, void *y,
                   int out_dtype, oracle_status *st)
{
    size_t n_chunks = (size_t)B * H * T * D / 4;
    uint32_t b = oracle_index_bits(S);
    float *acc = (float *)malloc(n_chunks * 4 * sizeof(float));
    uint64_t n_bad = 0;
    for (size_t j = 0; j < n_chunks; ++j) {
        int h = head_of_chunk(j, H, T, D);
        uint32_t idx = oracle_get_index(words, b, j);
        float r = oracle_f16_to_f32(radius[j]);
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (idx >= 24u * S) { ++n_bad; r = 0.0f; }
        else oracle_codeword_f32((int)(idx % 24u), codebook + ((size_t)h * S + idx / 24u) * 4, c);
        for (int i = 0; i < 4; ++i) acc[4 * j + i] = r * c[i];
    }
    if (out_idx && n_out > 0) {
        if (gran == OR_GRAN_CHUNK) {
            for (int64_t q = 0; q < n_out; ++q) {
                size_t j = out_idx[q];
                for (int i = 0; i < 4; ++i) acc[4 * j + i] = oracle_f16_to_f32(out_val[4 * q + i]);
            }
        } else {
            for (int64_t q = 0; q < n_out; ++q) {
                size_t e = out_idx[q];
                acc[e] = acc[e] + oracle_f16_to_f32(out_val[q]);
            }
        }
    }
    for (size_t e = 0; e < n_chunks * 4; ++e) store_elem(y, out_dtype, e, acc[e]);
    if (st && n_bad) { st->flags |= OR_FLAG_BAD_INDEX; }
    free(acc);
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar conversions and helpers (for the Python side). */
/* ------------------------------------------------------------------------ */

void oracle_f32_to_bf16_array(const float *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(in[i]);
}

void oracle_bf16_to_f32_array(const uint16_t *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_f32(in[i]);
}

int64_t oracle_f32_to_f16_sat_array(const float *in, uint16_t *out, int64_t n)
{
    int64_t n_sat = 0;
    for (int64_t i = 0; i < n; ++i) {
        int sat = 0;
        out[i] = oracle_f32_to_f16_sat(in[i], &sat);
        n_sat += sat;
    }
    return n_sat;
}

void oracle_f16_to_f32_array(const uint16_t *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f32(in[i]);
}

void oracle_chunk_norm_array(const float *x, float *r, int64_t n_chunks)
{
    for (int64_t j = 0; j < n_chunks; ++j) r[j] = oracle_chunk_norm(x + 4 * j);
}

void oracle_get_index_array(const uint32_t *words, uint32_t b, const int64_t *chunks,
                            int64_t n, uint32_t *out)
{
    for (int64_t q = 0; q < n; ++q) out[q] = oracle_get_index(words, b, (size_t)chunks[q]);
}

/* fp32 score of codeword idx[q] for the listed chunks (after Med3x zeroing). */
void oracle_score_chunks(const void *x, int dtype, int B, int H, int T, int D,
                         const float *codebook, uint32_t S, const float *thr, int gran,
                         const int64_t *chunks, const uint32_t *idx, int64_t n, float *out)
{
    (void)B;
    for (int64_t q = 0; q < n; ++q) {
        size_t j = (size_t)chunks[q];
        int h = head_of_chunk(j, H, T, D);
        float c[4];
        load_chunk(x, dtype, j, thr ? thr + h : NULL, gran, c);
        out[q] = oracle_score(c, codebook + (size_t)h * S * 4, S, idx[q]);
    }
}

/* ------------------------------------------------------------------------ */
/* Quantized radius (our reading of the pages' bit budget [ABS], [NL 3]:     */
/* about 2 log2(24 S) bits per chunk, i.e. a radius code of as many levels  */
/* as there are codewords).  With Med3x every bulk chunk has r <= thr, so   */
/* the fp16 radius is quantized uniformly on [0, thr_h] into L = 24 S       */
/* levels, code k stored in b = ceil(log2(24 S)) bits, packed like the      */
/* indices.  Outliers are in the list; their codes are zero, so k = 0.      */
/* ------------------------------------------------------------------------ */

/* Step and inverse step of head h: delta = fl32(thr / (L-1)),
 * inv = fl32((L-1) / thr); both 0 when thr is not a positive finite value. */
static void qr_steps(float thr, uint32_t L, float *delta, float *inv)
{
    float lm1 = (float)(L - 1u);
    if (!(thr > 0.0f) || isinf(thr) || L < 2u) { *delta = 0.0f; *inv = 0.0f; return; }
    *delta = thr / lm1;
    *inv = lm1 / thr;
}

/* Level of one radius: k = min(L-1, floor(fl32(fl32(r * inv) + 0.5))),
 * every step one fp32 operation; a NaN radius gives 0. */
uint32_t oracle_radius_level(uint16_t radius_f16, float thr, uint32_t L)
{
    float delta, inv;
    qr_steps(thr, L, &delta, &inv);
    float r = oracle_f16_to_f32(radius_f16);
    float q = r * inv;
    if (isnan(q)) return 0u;
    float t = q + 0.5f;
    float k = floorf(t);
    if (k >= (float)(L - 1u)) return L - 1u;
    if (k < 0.0f) return 0u;
    return (uint32_t)k;
}

/* Radius codes of a whole call: rcode_words laid out like the index words. */
void oracle_quantize_radius(const uint16_t *radius, const float *thr, int B, int H, int T, int D,
                            uint32_t S, uint32_t *rcode_words)
{
    size_t n_chunks = (size_t)B * H * T * D / 4;
    uint32_t b = oracle_index_bits(S), L = 24u * S;
    memset(rcode_words, 0, (n_chunks / 32) * b * sizeof(uint32_t));
    for (size_t j = 0; j < n_chunks; ++j) {
        int h = head_of_chunk(j, H, T, D);
        put_index(rcode_words, b, j, oracle_radius_level(radius[j], thr[h], L));
    }
}

/* Decoded radius of level k: fl32(k * delta). */
float oracle_radius_of_level(uint32_t k, float thr, uint32_t L)
{
    float delta, inv;
    qr_steps(thr, L, &delta, &inv);
    return (float)k * delta;
}

/* oracle_decode with the radius of chunk j taken from its code:
 * r = fl32(k * delta_h).  Everything else (codeword, outliers, rounding,
 * bad-index rule) as in oracle_decode. */
void oracle_decode_qradius(const uint32_t *words, const uint32_t *rcode_words, const float *thr,
                           const float *codebook, uint32_t S, const uint32_t *out_idx,
                           const uint16_t *out_val, int64_t n_out, int gran, int B, int H, int T,
                           int D, void *y, int out_dtype, oracle_status *st)
{
    size_t n_chunks = (size_t)B * H * T * D / 4;
    uint32_t b = oracle_index_bits(S), L = 24u * S;
    float *acc = (float *)malloc(n_chunks * 4 * sizeof(float));
    uint64_t n_bad = 0;
    for (size_t j = 0; j < n_chunks; ++j) {
        int h = head_of_chunk(j, H, T, D);
        uint32_t idx = oracle_get_index(words, b, j);
        uint32_t k = oracle_get_index(rcode_words, b, j);
        float r = oracle_radius_of_level(k < L ? k : L - 1u, thr[h], L);
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (idx >= 24u * S) { ++n_bad; r = 0.0f; }
        else oracle_codeword_f32((int)(idx % 24u), codebook + ((size_t)h * S + idx / 24u) * 4, c);
        for (int e = 0; e < 4; ++e) acc[4 * j + e] = r * c[e];
    }
    if (out_idx && n_out > 0) {
        if (gran == OR_GRAN_CHUNK) {
            for (int64_t q = 0; q < n_out; ++q) {
                size_t j = out_idx[q];
                for (int i = 0; i < 4; ++i) acc[4 * j + i] = oracle_f16_to_f32(out_val[4 * q + i]);
            }
        } else {
            for (int64_t q = 0; q < n_out; ++q) {
                size_t e = out_idx[q];
                acc[e] = acc[e] + oracle_f16_to_f32(out_val[q]);
            }
        }
    }
    for (size_t e = 0; e < n_chunks * 4; ++e) store_elem(y, out_dtype, e, acc[e]);
    if (st && n_bad) { st->flags |= OR_FLAG_BAD_INDEX; }
    free(acc);
}

/* ------------------------------------------------------------------------ */
/* Joint (index, radius level) code: the pages' bit budget [ABS], [FR]      */
/* "La mecanique" (3.79 bits per element at S = 8: log2(192^2) bits per    */
/* chunk of 4 elements) reached by coding each chunk's pair as one digit   */
/* D = idx * L + k in base L^2 (L = 24 S) and n consecutive chunks of a     */
/* slab as one number V = sum_c D_c (L^2)^c (least significant chunk       */
/* first), n the largest count with L^(2n) < 2^64; V takes w = bit length  */
/* of L^(2n) - 1 bits.  Each slab's blocks (its last one padded with zero   */
/* digits) are packed LSB-first into its own run of 32-bit words.           */
/* ------------------------------------------------------------------------ */

uint32_t oracle_joint_block_chunks(uint32_t S)
{
    uint64_t m = (uint64_t)(24u * S) * (uint64_t)(24u * S);   /* L^2 */
    uint64_t p = 1;
    uint32_t n = 0;
    while (p <= UINT64_MAX / m) { p *= m; ++n; }                /* p = L^(2n) fits */
    return n;
}

uint32_t oracle_joint_block_bits(uint32_t S)
{
    uint64_t m = (uint64_t)(24u * S) * (uint64_t)(24u * S);
    uint32_t n = oracle_joint_block_chunks(S);
    uint64_t top = 1;
    for (uint32_t i = 0; i < n; ++i) top *= m;                  /* L^(2n) */
    top -= 1u;                                                  /* largest V */
    uint32_t w = 0;
    while (w < 64 && (top >> w) != 0) ++w;
    return w;
}

/* words of one slab's run */
uint64_t oracle_joint_slab_words(int T, int D, uint32_t S)
{
    uint64_t cps = (uint64_t)T * D / 4;
    uint32_t n = oracle_joint_block_chunks(S), w = oracle_joint_block_bits(S);
    uint64_t nb = (cps + n - 1) / n;
    return (nb * w + 31) / 32;
}

/* bit i of a word run */
static void put_bits(uint32_t *run, uint64_t bit0, uint32_t w, uint64_t v)
{
    for (uint32_t i = 0; i < w; ++i)
        if ((v >> i) & 1u) run[(bit0 + i) / 32] |= 1u << ((bit0 + i) % 32);
}

static uint64_t get_bits(const uint32_t *run, uint64_t bit0, uint32_t w)
{
    uint64_t v = 0;
    for (uint32_t i = 0; i < w; ++i)
        v |= (uint64_t)((run[(bit0 + i) / 32] >> ((bit0 + i) % 32)) & 1u) << i;
    return v;
}

/* Joint code of a call from its index words and radius-code words (both
 * laid out as b-bit fields in groups of 32 chunks).  joint: B*H runs of
 * oracle_joint_slab_words(T, D, S) words, zeroed here.  Returns the number
 * of chunks whose index or level is not below L (stored as digit 0). */
uint64_t oracle_pack_joint(const uint32_t *words, const uint32_t *rcode_words, int B, int H, int T,
                           int D, uint32_t S, uint32_t *joint)
{
    uint32_t b = oracle_index_bits(S), L = 24u * S;
    uint64_t m = (uint64_t)L * L;
    uint32_t n = oracle_joint_block_chunks(S), w = oracle_joint_block_bits(S);
    uint64_t cps = (uint64_t)T * D / 4, wps = oracle_joint_slab_words(T, D, S);
    uint64_t nb = (cps + n - 1) / n, bad = 0;
    memset(joint, 0, (size_t)B * H * wps * sizeof(uint32_t));
    for (uint64_t s = 0; s < (uint64_t)B * H; ++s) {
        for (uint64_t q = 0; q < nb; ++q) {
            uint64_t v = 0, p = 1;
            for (uint32_t c = 0; c < n; ++c) {
                uint64_t j = q * n + c;
                uint64_t d = 0;
                if (j < cps) {
                    uint32_t idx = oracle_get_index(words, b, s * cps + j);
                    uint32_t k = oracle_get_index(rcode_words, b, s * cps + j);
                    if (idx < L && k < L) d = (uint64_t)idx * L + k;
                    else ++bad;
                }
                v += d * p;
                p *= m;                        /* (the last product may wrap: unused) */
            }
            put_bits(joint + s * wps, q * w, w, v);
        }
    }
    return bad;
}

/* The (index, level) pair of every chunk of a call from its joint code. */
void oracle_unpack_joint(const uint32_t *joint, int B, int H, int T, int D, uint32_t S,
                         uint32_t *idx, uint32_t *k)
{
    uint32_t L = 24u * S;
    uint64_t m = (uint64_t)L * L;
    uint32_t n = oracle_joint_block_chunks(S), w = oracle_joint_block_bits(S);
    uint64_t cps = (uint64_t)T * D / 4, wps = oracle_joint_slab_words(T, D, S);
    uint64_t nb = (cps + n - 1) / n;
    for (uint64_t s = 0; s < (uint64_t)B * H; ++s) {
        for (uint64_t q = 0; q < nb; ++q) {
            uint64_t v = get_bits(joint + s * wps, q * w, w);
            for (uint32_t c = 0; c < n; ++c) {
                uint64_t j = q * n + c;
                uint64_t d = v % m;
                v /= m;
                if (j < cps) {
                    idx[s * cps + j] = (uint32_t)(d / L);
                    k[s * cps + j] = (uint32_t)(d % L);
                }
            }
        }
    }
}

/* The pages' outlier flag [NL 3] ("met een 1-bit vlag"): bit c of word g is
 * set when chunk 32 g + c is in the (chunk-mode) outlier list.  flags:
 * n_chunks / 32 words, zeroed here. */
void oracle_list_flags(const uint32_t *out_idx, int64_t n_out, uint64_t n_chunks, uint32_t *flags)
{
    memset(flags, 0, (size_t)(n_chunks / 32) * sizeof(uint32_t));
    for (int64_t q = 0; q < n_out; ++q) {
        uint64_t j = out_idx[q];
        if (j < n_chunks) flags[j / 32] |= 1u << (j % 32);
    }
}

/* The chunk-mode outlier list (chunk indices, in order) read back from the
 * flags: the values stay in the list's order, so entry q of the list is the
 * q-th set flag.  Returns the number of set flags (written up to cap). */
int64_t oracle_list_from_flags(const uint32_t *flags, uint64_t n_chunks, uint32_t *out_idx,
                               int64_t cap)
{
    int64_t n = 0;
    for (uint64_t j = 0; j < n_chunks; ++j)
        if ((flags[j / 32] >> (j % 32)) & 1u) {
            if (n < cap) out_idx[n] = (uint32_t)j;
            ++n;
        }
    return n;
}
