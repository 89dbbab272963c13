/*
 * sz_oracle.h -- plain single-threaded CPU reference of the SplitZip BF16
 * exponent codec.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the bench's CPU-baseline leg use it to check the CUDA library; the CUDA
 * library never includes, links or calls it, and it shares no code with it.
 *
 * Source of the method: "SplitZip: Ultra Fast Lossless KV Compression for
 * Disaggregated LLM Serving" (gist.science explainer, French and Japanese
 * pages), sections 1-4.  Byte layout: the container format below, which the
 * pages leave open; it is restated independently in include/splitzip.h for
 * the CUDA side.
 *
 * Container (all integers little-endian):
 *   off  0  magic "SZKV"               4 B
 *   off  4  version = 1                u8
 *   off  5  dtype   = 1 (BF16)         u8
 *   off  6  flags   = 0                u16
 *   off  8  n_elems                    u64
 *   off 16  n_escapes                  u64
 *   off 24  codebook[16]               u8 x 16 (exponent of code k)
 *   off 40  reserved = 0               u8 x 8
 *   off 48  sm[n]       sign<<7 | mantissa
 *           codes[ceil(n/2)]  element 2j low nibble, 2j+1 high nibble
 *           pos[e]      u32, strictly ascending element indices
 *           rawexp[e]   u8, the exponent at pos[k]
 *   size = 48 + n + ceil(n/2) + 5e
 */
#ifndef SZ_ORACLE_H
#define SZ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SZO_OK 0
#define SZO_ERR_NULL (-1)
#define SZO_ERR_TOO_LARGE (-2)
#define SZO_ERR_CAPACITY (-3)
#define SZO_ERR_CORRUPT (-5)

#define SZO_HEADER_BYTES 48u

/* Exponent histogram: hist[E] = number of elements whose 8-bit exponent
 * field is E. */
void szo_histogram(const uint16_t *x, uint64_t n, uint64_t hist[256]);

/* Top-16 codebook: all 256 exponents ordered by (count descending, exponent
 * ascending); codebook[k] = k-th exponent of that order. */
void szo_select_top16(const uint64_t hist[256], uint8_t codebook[16]);

/* Container size for n elements and e escapes. */
uint64_t szo_container_size(uint64_t n, uint64_t e);

/* Encode x[0..n) into out (capacity cap bytes).  On success writes the
 * container size to *out_size and the escape count to *n_escapes. */
int szo_encode(const uint16_t *x, uint64_t n, uint8_t *out, uint64_t cap,
               uint64_t *out_size, uint64_t *n_escapes);

/* Encode with a caller-chosen codebook (16 distinct exponents). */
int szo_encode_with_codebook(const uint16_t *x, uint64_t n,
                             const uint8_t codebook[16], uint8_t *out,
                             uint64_t cap, uint64_t *out_size,
                             uint64_t *n_escapes);

/* Decode a container of in_bytes bytes into x[0..n).  Rejects anything that
 * is not a well-formed container for exactly n elements. */
int szo_decode(const uint8_t *in, uint64_t in_bytes, uint16_t *x, uint64_t n);

#ifdef __cplusplus
}
#endif
#endif
