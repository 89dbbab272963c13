/*
 * sz_oracle.c -- plain single-threaded CPU reference of the SplitZip BF16
 * exponent codec.  TEST INFRASTRUCTURE ONLY (see sz_oracle.h): only the
 * tests, the smoke check and the bench's CPU-baseline leg may use it.
 *
 * Every step is written the slow, obvious way, in the order the SplitZip
 * explainer gives it ("SplitZip: Ultra Fast Lossless KV Compression for
 * Disaggregated LLM Serving", gist.science):
 *   1. split each BF16 number into sign, exponent and mantissa (section 1,
 *      "La structure de la Note");
 *   2. the exponents repeat, the mantissas do not (section 2);
 *   3. give the 16 most common exponents a fixed 4-bit code, pack two codes
 *      per byte, and write every other exponent as an escape record
 *      (position, raw exponent) (section 3, "La strategie SplitZip");
 *   4. decode looks each code up, recombines it with sign and mantissa, and
 *      overwrites the escaped places (section 4, "Pourquoi est-ce rapide ?").
 * Losslessness is the claim of "Les Resultats": decode(encode(x)) == x bit
 * for bit.
 */
#include "sz_oracle.h"

#include <stdlib.h>
#include <string.h>

/* ---- step 1: the three fields of a BF16 bit pattern --------------------- */
/* BF16 = 1 sign bit | 8 exponent bits | 7 mantissa bits (most to least
 * significant). */
static unsigned field_sign(uint16_t x) { return (unsigned)(x >> 15) & 1u; }
static unsigned field_exponent(uint16_t x) { return (unsigned)(x >> 7) & 0xFFu; }
static unsigned field_mantissa(uint16_t x) { return (unsigned)x & 0x7Fu; }

static uint16_t join_fields(unsigned sign, unsigned exponent, unsigned mantissa) {
    return (uint16_t)((sign << 15) | (exponent << 7) | mantissa);
}

/* The sign+mantissa byte: sign in bit 7, mantissa in bits 6..0. */
static uint8_t sm_byte(uint16_t x) {
    return (uint8_t)((field_sign(x) << 7) | field_mantissa(x));
}

/* ---- little-endian helpers ---------------------------------------------- */
static void put_u16(uint8_t *p, uint16_t v) {
    p[0] = (uint8_t)(v & 0xFF);
    p[1] = (uint8_t)(v >> 8);
}
static void put_u32(uint8_t *p, uint32_t v) {
    for (int b = 0; b < 4; ++b) p[b] = (uint8_t)((v >> (8 * b)) & 0xFF);
}
static void put_u64(uint8_t *p, uint64_t v) {
    for (int b = 0; b < 8; ++b) p[b] = (uint8_t)((v >> (8 * b)) & 0xFF);
}
static uint16_t get_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get_u32(const uint8_t *p) {
    uint32_t v = 0;
    for (int b = 3; b >= 0; --b) v = (v << 8) | p[b];
    return v;
}
static uint64_t get_u64(const uint8_t *p) {
    uint64_t v = 0;
    for (int b = 7; b >= 0; --b) v = (v << 8) | p[b];
    return v;
}

/* ---- step 2: how often each exponent occurs ----------------------------- */
void szo_histogram(const uint16_t *x, uint64_t n, uint64_t hist[256]) {
    for (int e = 0; e < 256; ++e) hist[e] = 0;
    for (uint64_t i = 0; i < n; ++i) hist[field_exponent(x[i])] += 1;
}

/* ---- step 3a: the "Top 16" list ---------------------------------------- */
typedef struct {
    uint64_t count;
    unsigned exponent;
} exp_key;

/* Most common first; among equal counts, the lower exponent first. */
static int more_common_first(const void *pa, const void *pb) {
    const exp_key *a = (const exp_key *)pa;
    const exp_key *b = (const exp_key *)pb;
    if (a->count != b->count) return a->count > b->count ? -1 : 1;
    if (a->exponent != b->exponent) return a->exponent < b->exponent ? -1 : 1;
    return 0;
}

void szo_select_top16(const uint64_t hist[256], uint8_t codebook[16]) {
    exp_key keys[256];
    for (unsigned e = 0; e < 256; ++e) {
        keys[e].count = hist[e];
        keys[e].exponent = e;
    }
    qsort(keys, 256, sizeof(exp_key), more_common_first);
    for (int k = 0; k < 16; ++k) codebook[k] = (uint8_t)keys[k].exponent;
}

uint64_t szo_container_size(uint64_t n, uint64_t e) {
    return (uint64_t)SZO_HEADER_BYTES + n + (n + 1) / 2 + 5 * e;
}

/* ---- step 3b: one pass writing the streams ------------------------------ */
#define NO_CODE 0xFFFFu

static int codebook_is_valid(const uint8_t codebook[16]) {
    for (int a = 0; a < 16; ++a)
        for (int b = a + 1; b < 16; ++b)
            if (codebook[a] == codebook[b]) return 0;
    return 1;
}

int szo_encode_with_codebook(const uint16_t *x, uint64_t n,
                             const uint8_t codebook[16], uint8_t *out,
                             uint64_t cap, uint64_t *out_size,
                             uint64_t *n_escapes) {
    if ((x == NULL && n > 0) || codebook == NULL || out == NULL ||
        out_size == NULL || n_escapes == NULL)
        return SZO_ERR_NULL;
    if (n > 0xFFFFFFFFull) return SZO_ERR_TOO_LARGE; /* positions are u32 */
    if (!codebook_is_valid(codebook)) return SZO_ERR_CORRUPT;

    /* code of each exponent, or NO_CODE for an escape */
    unsigned code_of[256];
    for (int e = 0; e < 256; ++e) code_of[e] = NO_CODE;
    for (unsigned k = 0; k < 16; ++k) code_of[codebook[k]] = k;

    /* count the escapes first: the raw-exponent stream starts after all the
     * positions, so its offset needs the count */
    uint64_t e_count = 0;
    for (uint64_t i = 0; i < n; ++i)
        if (code_of[field_exponent(x[i])] == NO_CODE) e_count += 1;

    const uint64_t size = szo_container_size(n, e_count);
    if (cap < size) return SZO_ERR_CAPACITY;

    const uint64_t off_sm = SZO_HEADER_BYTES;
    const uint64_t off_codes = off_sm + n;
    const uint64_t off_pos = off_codes + (n + 1) / 2;
    const uint64_t off_raw = off_pos + 4 * e_count;

    /* header */
    memset(out, 0, SZO_HEADER_BYTES);
    out[0] = 'S';
    out[1] = 'Z';
    out[2] = 'K';
    out[3] = 'V';
    out[4] = 1; /* version */
    out[5] = 1; /* dtype: BF16 */
    put_u16(out + 6, 0);
    put_u64(out + 8, n);
    put_u64(out + 16, e_count);
    for (int k = 0; k < 16; ++k) out[24 + k] = codebook[k];
    /* bytes 40..47 stay zero */

    /* code bytes start at zero so that a missing odd tail nibble is 0 */
    memset(out + off_codes, 0, (size_t)((n + 1) / 2));

    uint64_t k_esc = 0;
    for (uint64_t i = 0; i < n; ++i) {
        const uint16_t v = x[i];
        out[off_sm + i] = sm_byte(v);
        const unsigned ex = field_exponent(v);
        unsigned nibble;
        if (code_of[ex] == NO_CODE) {
            nibble = 0; /* placeholder; the escape record carries the value */
            put_u32(out + off_pos + 4 * k_esc, (uint32_t)i);
            out[off_raw + k_esc] = (uint8_t)ex;
            k_esc += 1;
        } else {
            nibble = code_of[ex];
        }
        if (i % 2 == 0)
            out[off_codes + i / 2] |= (uint8_t)nibble;
        else
            out[off_codes + i / 2] |= (uint8_t)(nibble << 4);
    }

    *out_size = size;
    *n_escapes = e_count;
    return SZO_OK;
}

int szo_encode(const uint16_t *x, uint64_t n, uint8_t *out, uint64_t cap,
               uint64_t *out_size, uint64_t *n_escapes) {
    if (x == NULL && n > 0) return SZO_ERR_NULL;
    uint64_t hist[256];
    uint8_t codebook[16];
    szo_histogram(x, n, hist);
    szo_select_top16(hist, codebook);
    return szo_encode_with_codebook(x, n, codebook, out, cap, out_size, n_escapes);
}

/* ---- step 4: decode ----------------------------------------------------- */
int szo_decode(const uint8_t *in, uint64_t in_bytes, uint16_t *x, uint64_t n) {
    if (in == NULL || (x == NULL && n > 0)) return SZO_ERR_NULL;
    if (in_bytes < SZO_HEADER_BYTES) return SZO_ERR_CORRUPT;
    if (in[0] != 'S' || in[1] != 'Z' || in[2] != 'K' || in[3] != 'V') return SZO_ERR_CORRUPT;
    if (in[4] != 1 || in[5] != 1 || get_u16(in + 6) != 0) return SZO_ERR_CORRUPT;
    for (int b = 40; b < 48; ++b)
        if (in[b] != 0) return SZO_ERR_CORRUPT;
    if (get_u64(in + 8) != n) return SZO_ERR_CORRUPT;
    if (n > 0xFFFFFFFFull) return SZO_ERR_CORRUPT;
    const uint64_t e_count = get_u64(in + 16);
    if (e_count > n) return SZO_ERR_CORRUPT;
    if (szo_container_size(n, e_count) > in_bytes) return SZO_ERR_CORRUPT;

    uint8_t codebook[16];
    for (int k = 0; k < 16; ++k) codebook[k] = in[24 + k];
    if (!codebook_is_valid(codebook)) return SZO_ERR_CORRUPT;
    int in_codebook[256];
    for (int e = 0; e < 256; ++e) in_codebook[e] = 0;
    for (int k = 0; k < 16; ++k) in_codebook[codebook[k]] = 1;

    const uint64_t off_sm = SZO_HEADER_BYTES;
    const uint64_t off_codes = off_sm + n;
    const uint64_t off_pos = off_codes + (n + 1) / 2;
    const uint64_t off_raw = off_pos + 4 * e_count;

    /* an odd count leaves the high nibble of the last code byte unused: 0 */
    if (n % 2 == 1 && (in[off_codes + n / 2] >> 4) != 0) return SZO_ERR_CORRUPT;

    /* look each code up and recombine with the sign and the mantissa */
    for (uint64_t i = 0; i < n; ++i) {
        const uint8_t s = in[off_sm + i];
        const uint8_t byte = in[off_codes + i / 2];
        const unsigned nibble = (i % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
        x[i] = join_fields((s >> 7) & 1u, codebook[nibble], s & 0x7Fu);
    }

    /* overwrite the escaped places with their raw exponents */
    uint64_t prev = 0;
    for (uint64_t k = 0; k < e_count; ++k) {
        const uint64_t p = get_u32(in + off_pos + 4 * k);
        const unsigned ex = in[off_raw + k];
        if (p >= n) return SZO_ERR_CORRUPT;
        if (k > 0 && p <= prev) return SZO_ERR_CORRUPT; /* strictly ascending */
        if (in_codebook[ex]) return SZO_ERR_CORRUPT;    /* would have had a code */
        const uint8_t byte = in[off_codes + p / 2];
        const unsigned nibble = (p % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
        if (nibble != 0) return SZO_ERR_CORRUPT;        /* placeholder is 0 */
        const uint8_t s = in[off_sm + p];
        x[p] = join_fields((s >> 7) & 1u, ex, s & 0x7Fu);
        prev = p;
    }
    return SZO_OK;
}
