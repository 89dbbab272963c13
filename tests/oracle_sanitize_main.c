/* Memory-safety drive of the CPU oracle (test infrastructure).
 *
 * Built with -fsanitize=address,undefined next to oracle/sz_oracle.c by
 * tests/test_oracle_sanitized.py.  Every buffer is a heap block of exactly
 * the size the call is allowed to touch, so any read or write outside it is
 * reported by the sanitizer and fails the run.  Covered: round trips over
 * small and multi-tile sizes, an encode whose capacity is one byte short,
 * a codebook with a repeated entry, every truncation of small containers,
 * and many containers with bytes flipped or header fields rewritten (the
 * decoder must reject them or decode without touching memory it does not
 * own).  Prints "ok" and exits 0 when nothing failed. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "sz_oracle.h"

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;

static uint64_t next_u64(void) { /* xorshift64* */
    rng_state ^= rng_state >> 12;
    rng_state ^= rng_state << 25;
    rng_state ^= rng_state >> 27;
    return rng_state * 0x2545F4914F6CDD1Dull;
}

static int failures = 0;

#define CHECK(cond, ...)                                \
    do {                                                \
        if (!(cond)) {                                  \
            fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__); \
            fprintf(stderr, __VA_ARGS__);               \
            fputc('\n', stderr);                        \
            ++failures;                                 \
        }                                               \
    } while (0)

/* KV-like values: a few common exponents, some rare ones, arbitrary
 * sign and mantissa. */
static void fill(uint16_t *x, uint64_t n, int kind) {
    for (uint64_t i = 0; i < n; ++i) {
        uint64_t r = next_u64();
        uint32_t e;
        if (kind == 0) e = 120u + (uint32_t)(r % 12u);                         /* compressible */
        else if (kind == 1) e = (r % 100u) < 97u ? 118u + (uint32_t)(r % 14u) : (uint32_t)(r >> 40) & 0xFFu;
        else e = (uint32_t)(r >> 40) & 0xFFu;                                  /* incompressible */
        x[i] = (uint16_t)(((r >> 8) & 0x8000u) | (e << 7) | ((r >> 16) & 0x7Fu));
    }
}

static uint64_t bound(uint64_t n) {
    return 48u + n + (n + 1) / 2 + 5u * (n - (n + 15) / 16);
}

/* Encode into an exactly-sized copy; returns the container (malloc'd, size
 * *sz) or NULL. */
static uint8_t *encode_exact(const uint16_t *x, uint64_t n, uint64_t *sz) {
    uint64_t cap = bound(n);
    uint8_t *tmp = (uint8_t *)malloc(cap ? cap : 1);
    uint64_t size = 0, e = 0;
    int st = szo_encode(x, n, tmp, cap, &size, &e);
    CHECK(st == SZO_OK, "encode n=%llu status %d", (unsigned long long)n, st);
    if (st != SZO_OK) { free(tmp); return NULL; }
    CHECK(size == szo_container_size(n, e), "size formula n=%llu", (unsigned long long)n);
    uint8_t *c = (uint8_t *)malloc(size);
    memcpy(c, tmp, size);
    free(tmp);
    /* the same bytes with a capacity of exactly the size */
    uint8_t *again = (uint8_t *)malloc(size);
    uint64_t size2 = 0, e2 = 0;
    CHECK(szo_encode(x, n, again, size, &size2, &e2) == SZO_OK && size2 == size && memcmp(again, c, size) == 0,
          "exact-capacity encode n=%llu", (unsigned long long)n);
    free(again);
    /* one byte short: refused, and nothing written past the block */
    if (size > 0) {
        uint8_t *shortbuf = (uint8_t *)malloc(size - 1 ? size - 1 : 1);
        CHECK(szo_encode(x, n, shortbuf, size - 1, &size2, &e2) == SZO_ERR_CAPACITY,
              "short capacity n=%llu", (unsigned long long)n);
        free(shortbuf);
    }
    *sz = size;
    return c;
}

/* Decode from an exactly-sized copy of in[0..len) into an exactly-sized
 * output; returns the status. */
static int decode_exact(const uint8_t *in, uint64_t len, uint64_t n, uint16_t *out_copy) {
    uint8_t *c = (uint8_t *)malloc(len ? len : 1);
    if (len) memcpy(c, in, len);
    uint16_t *y = (uint16_t *)malloc(n ? n * 2 : 2);
    int st = szo_decode(c, len, y, n);
    if (out_copy && st == SZO_OK) memcpy(out_copy, y, n * 2);
    free(y);
    free(c);
    return st;
}

static void round_trips(void) {
    static const uint64_t sizes[] = {0, 1, 2, 3, 15, 16, 17, 255, 4096, 16385, 65537, 3 * 65536 + 101};
    for (size_t s = 0; s < sizeof(sizes) / sizeof(sizes[0]); ++s) {
        for (int kind = 0; kind < 3; ++kind) {
            uint64_t n = sizes[s];
            uint16_t *x = (uint16_t *)malloc(n ? n * 2 : 2);
            fill(x, n, kind);
            uint64_t size = 0;
            uint8_t *c = encode_exact(x, n, &size);
            if (c) {
                uint16_t *y = (uint16_t *)malloc(n ? n * 2 : 2);
                int st = decode_exact(c, size, n, y);
                CHECK(st == SZO_OK, "decode n=%llu kind %d status %d", (unsigned long long)n, kind, st);
                CHECK(st != SZO_OK || n == 0 || memcmp(x, y, n * 2) == 0, "round trip n=%llu", (unsigned long long)n);
                /* the wrong element count is rejected */
                CHECK(decode_exact(c, size, n + 1, NULL) != SZO_OK, "n+1 accepted");
                if (n) CHECK(decode_exact(c, size, n - 1, NULL) != SZO_OK, "n-1 accepted");
                free(y);
                free(c);
            }
            free(x);
        }
    }
}

static void bad_codebook(void) {
    uint16_t x[64];
    fill(x, 64, 0);
    uint8_t cb[16];
    for (int i = 0; i < 16; ++i) cb[i] = (uint8_t)(120 + i);
    cb[9] = cb[3];
    uint64_t cap = bound(64), size = 0, e = 0;
    uint8_t *out = (uint8_t *)malloc(cap);
    CHECK(szo_encode_with_codebook(x, 64, cb, out, cap, &size, &e) != SZO_OK, "repeated codebook accepted");
    free(out);
}

static void truncations_and_flips(void) {
    for (int kind = 0; kind < 3; ++kind) {
        const uint64_t n = kind == 2 ? 40 : 300;
        uint16_t *x = (uint16_t *)malloc(n * 2);
        fill(x, n, kind == 2 ? 2 : 1);
        uint64_t size = 0;
        uint8_t *c = encode_exact(x, n, &size);
        if (!c) { free(x); continue; }
        for (uint64_t len = 0; len < size; ++len)
            CHECK(decode_exact(c, len, n, NULL) != SZO_OK, "truncated to %llu accepted", (unsigned long long)len);
        uint8_t *m = (uint8_t *)malloc(size);
        uint16_t *y = (uint16_t *)malloc(n * 2);
        for (int t = 0; t < 4000; ++t) {
            memcpy(m, c, size);
            int flips = 1 + (int)(next_u64() % 3);
            for (int f = 0; f < flips; ++f) m[next_u64() % size] ^= (uint8_t)(1u << (next_u64() % 8));
            int st = decode_exact(m, size, n, y);
            /* a flip inside sm bytes decodes (to other values); anything
             * else must be rejected or decode without a memory error */
            CHECK(st == SZO_OK || st == SZO_ERR_CORRUPT, "flip status %d", st);
        }
        /* header fields rewritten with small and extreme values */
        static const int offs[] = {8, 16};  /* n, e */
        static const uint64_t vals[] = {0, 1, 0xFFFFFFFFull, 0x100000000ull, 0xFFFFFFFFFFFFFFFFull};
        for (size_t o = 0; o < 2; ++o) {
            for (size_t v = 0; v < sizeof(vals) / sizeof(vals[0]); ++v) {
                memcpy(m, c, size);
                memcpy(m + offs[o], &vals[v], 8);
                int st = decode_exact(m, size, n, y);
                /* another element count never matches the caller's; a
                 * smaller escape count can leave a well-formed container
                 * inside the larger buffer, which decodes */
                if (offs[o] == 8)
                    CHECK(st == SZO_ERR_CORRUPT, "header n = %llx status %d", (unsigned long long)vals[v], st);
                else
                    CHECK(st == SZO_OK || st == SZO_ERR_CORRUPT, "header e = %llx status %d",
                          (unsigned long long)vals[v], st);
            }
        }
        free(y);
        free(m);
        free(c);
        free(x);
    }
}

int main(void) {
    round_trips();
    bad_codebook();
    truncations_and_flips();
    if (failures) {
        fprintf(stderr, "%d failure(s)\n", failures);
        return 1;
    }
    puts("ok");
    return 0;
}
