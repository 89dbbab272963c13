/*
 * splitzip.h -- C ABI of the SplitZip lossless BF16 KV-cache codec for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "SplitZip: Ultra Fast Lossless KV Compression for Disaggregated LLM
 * Serving" (gist.science explainer, French and Japanese pages).
 *   - section 1 "La structure de la Note": a BF16 number is a sign, an 8-bit
 *     exponent and a 7-bit mantissa;
 *   - section 2 "La decouverte secrete": mantissas look random, exponents
 *     repeat;
 *   - section 3 "La strategie SplitZip": the 16 most common exponents get a
 *     fixed 4-bit code, two codes share a byte, and every other exponent is
 *     written as an escape note (position, raw exponent);
 *   - section 4 "Pourquoi est-ce rapide ?": fixed-length codes make encode a
 *     straight pass; decode looks each code up, recombines it with sign and
 *     mantissa and overwrites the escaped places;
 *   - "Les Resultats": the round trip is lossless, bit for bit.
 *
 * ------------------------------------------------------------------------
 * Container format (the pages fix no bytes; this library defines them).
 * All integers little-endian.  H = 48 header bytes.
 *
 *   off  0  magic "SZKV"              4 bytes  'S','Z','K','V'
 *   off  4  version = 1               u8
 *   off  5  dtype   = 1 (BF16)        u8
 *   off  6  flags   = 0               u16
 *   off  8  n_elems                   u64
 *   off 16  n_escapes  (e)            u64
 *   off 24  codebook[16]              u8: exponent of code k, k = 0..15
 *   off 40  reserved = 0              8 bytes
 *   off 48  sm[n]         sign in bit 7, mantissa in bits 6..0
 *           codes[ceil(n/2)]  element 2j in the low nibble of byte j,
 *                         element 2j+1 in the high nibble; an odd count
 *                         leaves the last high nibble 0
 *           pos[e]        u32 element indices, strictly ascending
 *           rawexp[e]     u8 exponent of element pos[k]
 *   size = 48 + n + ceil(n/2) + 5e
 *
 * Codebook: the 256 exponents ordered by (count descending, exponent
 * ascending); code k is the k-th.  An element whose exponent is not in the
 * codebook is an escape: its nibble is the placeholder 0 and it gets one
 * (pos, rawexp) record.  Hence e = n - (sum of the 16 codebook counts).
 * The top 16 of 256 bins hold at least ceil(n/16) elements, so the worst
 * case is size <= 48 + n + ceil(n/2) + 5(n - ceil(n/16)) (SZ_MAX_BYTES).
 * ------------------------------------------------------------------------
 *
 * Conventions for every entry point:
 *   - "d_" pointers are CUDA device pointers on the current device; "h_"
 *     pointers are host pointers.  The caller owns every buffer, including
 *     the workspace; the library never allocates device memory and never
 *     synchronises the stream.  Work is enqueued on `stream` (a
 *     cudaStream_t; NULL = legacy default stream) and runs asynchronously.
 *   - Errors the host can see (null pointer, size, alignment, workspace or
 *     capacity too small, launch failure) are returned at once and nothing
 *     is enqueued.  Errors only the device can see (corrupt container,
 *     workspace histogram that does not describe the input, a device-side
 *     wait that ran out) are written as an sz_status to the caller's d_status
 *     word(s), which the call first sets to SZ_OK.  A container whose status
 *     is not SZ_OK must not be used.
 *   - Vector path: device buffers must be 16-byte aligned (SZ_ERR_ALIGN
 *     otherwise); there is no scalar fallback for misaligned buffers.
 *   - Element counts are limited to n < 2^32 (escape positions are u32).
 *   - A device error leaves the affected container's size word(s) at 0: a
 *     size is written only after every CTA that worked on that container
 *     finished its share without an error.  A status of SZ_OK with a
 *     nonzero size is a complete container.
 *   - The calling thread's current device must have an ordinal below 64
 *     (per-device facts are kept in a 64-entry table); a larger ordinal
 *     returns SZ_ERR_INVALID before anything is enqueued.
 */
#ifndef SPLITZIP_H
#define SPLITZIP_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t sz_status;

#define SZ_OK 0
#define SZ_ERR_NULL (-1)           /* a required pointer is NULL */
#define SZ_ERR_TOO_LARGE (-2)      /* n >= 2^32, or a size overflows */
#define SZ_ERR_CAPACITY (-3)       /* output buffer smaller than needed */
#define SZ_ERR_ALIGN (-4)          /* buffer not 16-byte aligned, page size not a multiple of 64 */
#define SZ_ERR_CORRUPT (-5)        /* container malformed, or input != workspace histogram */
#define SZ_ERR_CUDA (-6)           /* a CUDA runtime call failed */
#define SZ_ERR_DEVICE_TIMEOUT (-7) /* a bounded device-side wait ran out */
#define SZ_ERR_INVALID (-8)        /* bad argument (codebook with repeats, counts) */
#define SZ_ERR_WORKSPACE (-9)      /* workspace smaller than planned */

#define SZ_HEADER_BYTES 48u

/* Worst-case container size for n elements (see the format above). */
#define SZ_MAX_BYTES(n) \
    (48ull + (uint64_t)(n) + ((uint64_t)(n) + 1) / 2 + 5ull * ((uint64_t)(n) - ((uint64_t)(n) + 15) / 16))

/* ------------------------------------------------------------------ plan */
/*
 * sz_plan -- sizes for one tensor of n_elems BF16 values.
 *   *max_compressed_bytes  worst-case container size (SZ_MAX_BYTES)
 *   *workspace_bytes       device workspace needed by every single-tensor
 *                          call below for this n (one workspace serves the
 *                          histogram, encode and decode of one tensor)
 * Host only; never touches the device.  SZ_ERR_TOO_LARGE if n >= 2^32.
 */
sz_status sz_plan(uint64_t n_elems, uint64_t *max_compressed_bytes, uint64_t *workspace_bytes);

/* ------------------------------------------------------------- histogram */
/*
 * sz_histogram_codebook -- exponent histogram and top-16 codebook
 * (explainer section 3, the "Top 16" list).
 *   d_in            n BF16 values (uint16 bit patterns), 16-byte aligned
 *   d_codebook16    out: 16 bytes, codebook[k] = exponent of code k
 *   d_hist256_or_null  optional out: uint32[256] exponent counts
 *   d_ws, ws_bytes  workspace of at least sz_plan's size, 16-byte aligned.
 *                   The histogram stays in the workspace: sz_encode of the
 *                   same input reads it from there to size the escape
 *                   stream, so the same workspace must be passed to it.
 * n may be 0 (codebook = exponents 0..15).
 */
sz_status sz_histogram_codebook(const uint16_t *d_in, uint64_t n, uint8_t *d_codebook16,
                                uint32_t *d_hist256_or_null, void *d_ws, uint64_t ws_bytes,
                                void *stream);

/* ---------------------------------------------------------------- encode */
/*
 * sz_encode -- write the container of d_in[0..n) (explainer section 3:
 * sign+mantissa bytes, 4-bit codes two per byte, escape records).
 *   d_codebook16    16 distinct exponents (normally from
 *                   sz_histogram_codebook; any 16 distinct exponents are
 *                   accepted, repeats give SZ_ERR_INVALID in *d_status)
 *   d_out, out_cap  container buffer, 16-byte aligned.  out_cap must be at
 *                   least 48 + n + ceil(n/2) (host check); the device checks
 *                   the exact size against out_cap (SZ_ERR_CAPACITY).
 *                   sz_plan's max_compressed_bytes always suffices for a
 *                   codebook from sz_histogram_codebook.
 *   d_out_bytes     out: uint64 container size (0 on a device error: the
 *                   size is written by the CTA that completes the stream's
 *                   tile count, and only when no CTA reported an error)
 *   d_status        out (required): int32 device status (SZ_OK,
 *                   SZ_ERR_CORRUPT when the workspace histogram does not
 *                   describe d_in, SZ_ERR_CAPACITY, SZ_ERR_INVALID,
 *                   SZ_ERR_DEVICE_TIMEOUT); set to SZ_OK first
 *   d_ws, ws_bytes  the workspace passed to sz_histogram_codebook for this
 *                   same input (its histogram gives the escape count).
 * The escape stream is compacted in element order across tiles without
 * any block waiting for another: the histogram call kept the exponent
 * counts of the first and last segment piece of every CTA's range of tiles,
 * and from those each CTA's first escape index follows (placed by the
 * histogram call for its own codebook, again here for another one).  A
 * pipeline wait that runs out gives SZ_ERR_DEVICE_TIMEOUT.  The same
 * workspace may serve several sz_encode calls after one histogram call
 * (with other codebooks, or after an error).
 */
sz_status sz_encode(const uint16_t *d_in, uint64_t n, const uint8_t *d_codebook16, uint8_t *d_out,
                    uint64_t out_cap, uint64_t *d_out_bytes, int32_t *d_status, void *d_ws,
                    uint64_t ws_bytes, void *stream);

/*
 * sz_compress -- histogram, codebook and container of d_in[0..n) in one call
 * (sz_histogram_codebook + sz_encode with the codebook chosen there).  A
 * stream of at most 2^20 elements is compressed by blocks of 4,096
 * elements in two launches after one memset; a longer one by the
 * histogram kernel and the encode kernel.
 *   d_out, out_cap  container buffer, 16-byte aligned; out_cap at least
 *                   48 + n + ceil(n/2) (host check), sz_plan's
 *                   max_compressed_bytes always suffices
 *   d_out_bytes     out: uint64 container size (0 on a device error)
 *   d_codebook16_or_null  optional out: the 16-entry codebook
 *   d_status        out (required): int32 device status, set to SZ_OK first
 *   d_ws, ws_bytes  workspace of sz_plan's size, 16-byte aligned
 * The container is byte for byte the two-call path's.
 */
sz_status sz_compress(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap, uint64_t *d_out_bytes,
                      uint8_t *d_codebook16_or_null, int32_t *d_status, void *d_ws, uint64_t ws_bytes,
                      void *stream);

/* ---------------------------------------------------------------- decode */
/*
 * sz_decode -- rebuild d_out[0..n) from a container (explainer section 4:
 * look the code up, recombine with sign and mantissa, overwrite escapes).
 *   d_in, in_bytes  container bytes, 16-byte aligned; in_bytes may exceed
 *                   the container size (the rest is ignored)
 *   d_out           n uint16 outputs, 16-byte aligned
 *   d_status        out (required): int32 device status; SZ_ERR_CORRUPT for
 *                   a bad magic/version/dtype/flags/reserved field, a
 *                   header n other than n, a size above in_bytes, repeated
 *                   codebook entries, escape positions out of range or not
 *                   strictly ascending, an escaped exponent that is in the
 *                   codebook, or a nonzero placeholder / odd-tail nibble.
 *                   d_out holds no meaningful data unless it reads SZ_OK.
 *   d_ws, ws_bytes  workspace of sz_plan's size (the first escape index of
 *                   every 16,384-element sub-tile, found by binary search).
 * A stream of at most 2^17 elements is decoded by blocks of 4,096 elements
 * in one launch after the status memset (no index kernel), with the same
 * checks; a longer one by the index kernel and the pipelined decode.
 */
sz_status sz_decode(const uint8_t *d_in, uint64_t in_bytes, uint16_t *d_out, uint64_t n,
                    int32_t *d_status, void *d_ws, uint64_t ws_bytes, void *stream);

/* --------------------------------------------------------- batched/paged */
/*
 * A batch is a list of segments; each segment is one logical stream (one
 * (layer, K/V) tensor, or one request's paged KV) with its own codebook and
 * its own container.  A segment's stream is a run of pages of page_elems
 * elements taken in page-list order (the last page may be partial); a
 * contiguous tensor is one page of n elements, or several pages pointing
 * into it.
 */
typedef struct sz_segment {
    uint64_t n_elems;    /* elements in the segment's stream (< 2^32) */
    uint64_t page_begin; /* index of the segment's first page in the page-pointer array */
    uint64_t out_offset; /* byte offset of its container in the container buffer */
    uint64_t tile_begin; /* first global tile index of the segment */
} sz_segment;

/*
 * sz_plan_batched -- fill h_segs[0..n_segs) from the segment lengths.
 *   h_seg_elems     n_segs element counts
 *   page_elems      elements per page; a multiple of 64 when any segment
 *                   spans more than one page (SZ_ERR_ALIGN otherwise)
 *   h_segs          out: the segment table (pages numbered consecutively,
 *                   containers at 256-byte aligned offsets, each slot
 *                   SZ_MAX_BYTES(n_elems) long); copy it to the device for
 *                   the batched calls.  The container offsets depend only
 *                   on the segment lengths: a plan of the same lengths with
 *                   another page_elems finds the same containers, so a
 *                   batch can be decoded into pages of another size.
 *   *total_pages    out: page pointers the page array must hold
 *   *n_tiles        out: tiles of the whole batch (pass to the calls below)
 *   *out_bytes      out: container buffer size
 *   *workspace_bytes out: device workspace for the batched calls
 * Host only.
 */
sz_status sz_plan_batched(uint32_t n_segs, const uint64_t *h_seg_elems, uint64_t page_elems,
                          sz_segment *h_segs, uint64_t *total_pages, uint64_t *n_tiles,
                          uint64_t *out_bytes, uint64_t *workspace_bytes);

/*
 * sz_histogram_codebook_batched -- exponent histogram and top-16 codebook
 * of every segment (a memset and one kernel launch for the whole batch).  The
 * codebooks and escape counts stay in the workspace for sz_encode_batched.
 *   d_segs          the table from sz_plan_batched, in device memory
 *   n_tiles         from sz_plan_batched
 *   d_pages         device array of page pointers (16-byte aligned pages)
 *   d_codebooks_or_null  optional out: uint8[n_segs][16]
 *   d_status        out: int32[n_segs] device status per segment (set to
 *                   SZ_OK first; SZ_ERR_ALIGN for a misaligned page)
 */
sz_status sz_histogram_codebook_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                                        const uint16_t *const *d_pages, uint64_t page_elems,
                                        uint8_t *d_codebooks_or_null, int32_t *d_status, void *d_ws,
                                        uint64_t ws_bytes, void *stream);

/*
 * sz_encode_batched -- write every segment's container (one kernel launch
 * for the whole batch), with the codebooks that sz_histogram_codebook_batched
 * left in the same workspace for the same pages.
 *   d_out, out_cap  container buffer (16-byte aligned); segment k's
 *                   container starts at d_out + d_segs[k].out_offset
 *   d_out_bytes     out: uint64[n_segs] container sizes (0 on error)
 *   d_status        in/out: int32[n_segs]; keeps the histogram call's
 *                   errors and adds the encode's (first error wins)
 */
sz_status sz_encode_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                            const uint16_t *const *d_pages, uint64_t page_elems, uint8_t *d_out,
                            uint64_t out_cap, uint64_t *d_out_bytes, int32_t *d_status, void *d_ws,
                            uint64_t ws_bytes, void *stream);

/*
 * sz_decode_batched -- decode every segment's container into its pages.
 *   d_in, in_cap    container buffer; segment k's container starts at
 *                   d_in + d_segs[k].out_offset and may use the rest of
 *                   the buffer
 *   d_pages         device array of destination page pointers (16-byte
 *                   aligned), laid out like the encode's source pages
 *   d_status        out: int32[n_segs] device status per segment
 */
sz_status sz_decode_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                            const uint8_t *d_in, uint64_t in_cap, uint16_t *const *d_pages,
                            uint64_t page_elems, int32_t *d_status, void *d_ws, uint64_t ws_bytes,
                            void *stream);

/* ------------------------------------------- one pass, caller's codebook(s) */
/*
 * Encoding with a codebook chosen beforehand -- one kept from an earlier
 * request or chunk, or shared across layers -- needs no histogram pass: the
 * input is read once.  The explainer's method picks each tensor's own top
 * 16 (section 3); a codebook that is not the tensor's own stays lossless but
 * may leave more escapes.  The container is byte for byte the one the
 * two-call path (sz_histogram_codebook + sz_encode) writes with the same
 * codebook.
 *
 * Three kernels: the encode writes the sign+mantissa and code streams in
 * place and parks each tile's escape records (up to 1/16 of the tile,
 * 4,096 per 65,536-element tile) in the workspace; a placement kernel then
 * counts each segment's escapes, writes the header and moves the records
 * into place; a third kernel reads again the input of every tile with more
 * escapes than its slot holds (spread over the GPU), and its last block
 * writes every segment's size (0 for a segment with an error).
 *
 * sz_plan_one_pass -- worst-case container (every element an escape:
 * 48 + n + ceil(n/2) + 5n) and workspace bytes (16,420 bytes per 65,536
 * elements, about 1/8 of the input's bytes, plus 16 bytes per range and 4
 * per segment).  Host only.
 */
sz_status sz_plan_one_pass(uint64_t n_elems, uint64_t *max_compressed_bytes, uint64_t *workspace_bytes);

/*
 * sz_encode_one_pass -- the container of d_in[0..n) with d_codebook16.
 *   d_codebook16    16 distinct exponents (device memory); repeats give
 *                   SZ_ERR_INVALID in *d_status
 *   d_out, out_cap  container buffer, 16-byte aligned; out_cap must be at
 *                   least 48 + n + ceil(n/2) (host check); the device checks
 *                   the exact size (SZ_ERR_CAPACITY, *d_out_bytes = 0)
 *   d_out_bytes, d_status  out, as for sz_encode (both set first)
 *   d_ws, ws_bytes  workspace of sz_plan_one_pass's size, 16-byte aligned
 */
sz_status sz_encode_one_pass(const uint16_t *d_in, uint64_t n, const uint8_t *d_codebook16, uint8_t *d_out,
                             uint64_t out_cap, uint64_t *d_out_bytes, int32_t *d_status, void *d_ws,
                             uint64_t ws_bytes, void *stream);

/*
 * sz_workspace_one_pass_batched -- workspace bytes of
 * sz_encode_one_pass_batched for a batch of n_tiles tiles (from
 * sz_plan_batched).  Host only.
 */
sz_status sz_workspace_one_pass_batched(uint32_t n_segs, uint64_t n_tiles, uint64_t *workspace_bytes);

/*
 * sz_encode_one_pass_batched -- every segment's container with its own
 * caller codebook, in one read of the input.
 *   d_codebooks     uint8[n_segs][16] device array (row k: segment k)
 *   d_segs, n_tiles, d_pages, page_elems, d_out, out_cap  as for
 *                   sz_encode_batched; a plan's container slots hold any
 *                   codebook's container up to 48 + n + ceil(n/2) + 5(n -
 *                   ceil(n/16)) bytes, more escapes than that give
 *                   SZ_ERR_CAPACITY
 *   d_out_bytes, d_status  out: uint64[n_segs], int32[n_segs] (set first)
 */
sz_status sz_encode_one_pass_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                                     const uint16_t *const *d_pages, uint64_t page_elems,
                                     const uint8_t *d_codebooks, uint8_t *d_out, uint64_t out_cap,
                                     uint64_t *d_out_bytes, int32_t *d_status, void *d_ws, uint64_t ws_bytes,
                                     void *stream);

/* ------------------------- histogram kept while the cache is written */
/*
 * The codebook is each tensor's own top 16 (explainer section 3), so the
 * two-call path reads the input twice: once to count exponents, once to
 * encode.  A serving engine can instead count each chunk of KV as it is
 * written during prefill, into a running histogram per tensor or request;
 * at transfer time sz_select_codebook(_batched) turns the histograms into
 * the exact codebooks and sz_encode_one_pass(_batched) reads the cache
 * once.  The containers are byte for byte those of the two-call path
 * (explainer, "Le probleme des methodes d'envoi actuelles": the compressor
 * must keep pace with the prefill team producing the notes).
 *
 * sz_histogram_accumulate -- add the exponent counts of d_in[0..n) to the
 * caller's uint32[256] histogram (zero it before the first chunk, e.g.
 * with cudaMemsetAsync).  No workspace; n = 0 enqueues nothing.  The caller
 * keeps each histogram's total below 2^32 (the container's element limit).
 *   d_in            n BF16 values, 16-byte aligned
 *   d_hist256       in/out uint32[256], 4-byte aligned
 */
sz_status sz_histogram_accumulate(const uint16_t *d_in, uint64_t n, uint32_t *d_hist256, void *stream);

/*
 * sz_histogram_accumulate_batched -- add the exponent counts of every
 * segment of a batch (newly written pages or chunks, laid out as for
 * sz_plan_batched: d_segs from a plan of the new data's lengths) to the
 * caller's histograms, one launch.
 *   d_hist_index_or_null  uint32[n_segs]: segment k adds to histogram
 *                   d_hist_index[k] (several segments may share one, e.g.
 *                   the eight heads' slices of one tensor's new tokens);
 *                   NULL: segment k adds to histogram k
 *   d_hists         in/out uint32[rows][256], 4-byte aligned
 *   d_status        out int32[n_segs]: SZ_ERR_ALIGN for a misaligned page
 *                   (that segment's counts are then incomplete); set to
 *                   SZ_OK first
 */
sz_status sz_histogram_accumulate_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                                          const uint16_t *const *d_pages, uint64_t page_elems,
                                          const uint32_t *d_hist_index_or_null, uint32_t *d_hists,
                                          int32_t *d_status, void *stream);

/*
 * sz_select_codebook -- the codebook of a histogram: the 16 exponents
 * first in (count descending, exponent ascending) order, code k = the k-th
 * (explainer section 3), the same choice sz_histogram_codebook makes.
 *   d_hist256          uint32[256]
 *   d_codebook16       out: 16 bytes
 *   d_escapes_or_null  optional out: uint64 escape count (total - the 16
 *                      codebook counts), 8-byte aligned
 * sz_select_codebook_batched does the same for n_hists histograms
 * (uint32[n_hists][256] -> uint8[n_hists][16], uint64[n_hists]), one
 * block per histogram.
 */
sz_status sz_select_codebook(const uint32_t *d_hist256, uint8_t *d_codebook16, uint64_t *d_escapes_or_null,
                             void *stream);
sz_status sz_select_codebook_batched(uint32_t n_hists, const uint32_t *d_hists, uint8_t *d_codebooks,
                                     uint64_t *d_escapes_or_null, void *stream);

/* ------------------------------------------------------- no-allocation path */
/*
 * sz_encode_static -- the whole compression of one tensor (histogram,
 * codebook, container) without any workspace from the caller and without
 * allocating: for callers that cannot allocate device memory at the moment
 * they compress -- code running inside an allocator or memory-pool callback,
 * or an engine that reserved all device memory up front.  The explainer has
 * no counterpart; it is an interface of this library only.
 *
 * Its scratch is one file-scope device array of SZ_STATIC_SCRATCH_BYTES,
 * present on every GPU that loads the library until the process exits.
 *   d_in, n         n <= SZ_STATIC_MAX_ELEMS (2^28 elements, 512 MiB of
 *                   BF16); larger n returns SZ_ERR_TOO_LARGE
 *   d_out, out_cap, d_out_bytes, d_status  as for sz_encode
 *   d_codebook16_or_null  optional out: the 16-entry codebook
 * The container is byte for byte the one sz_histogram_codebook + sz_encode
 * write (the same kernels run; their waits follow sz_set_wait_limit_ns).
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls on a device share the one array: calls that overlap on the GPU
 * (other streams, other host threads) race and must be serialised by the
 * caller.
 */
#define SZ_STATIC_MAX_ELEMS (1ull << 28)
#define SZ_STATIC_SCRATCH_BYTES (1536ull + 2064ull * 1024ull)
sz_status sz_encode_static(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap,
                           uint64_t *d_out_bytes, uint8_t *d_codebook16_or_null, int32_t *d_status,
                           void *stream);

/* ------------------------------------------------------------ diagnostics */
/*
 * sz_set_wait_limit_ns -- upper bound, in nanoseconds of device time, of
 * every device-side wait of every entry point (a pipeline stage of the
 * encode or decode kernel waiting for its bulk copy).
 * Default 1e9 (one second).  A wait that runs out sets
 * SZ_ERR_DEVICE_TIMEOUT in the segment's status and the kernel returns.
 * Applies to calls made after it, process-wide.
 */
sz_status sz_set_wait_limit_ns(uint64_t limit_ns);

/*
 * sz_debug_set_flags -- test hook.  Bit 0: the encode and decode kernels'
 * copy threads issue no bulk copy, so every stage wait of their consumer
 * threads runs out (exercises the timeout path without faulting
 * anything).  Bit 1: the decode kernel's copy thread publishes the values
 * part of its stages but never their escape part, so the consumers' wait
 * for escape records runs out after the values are stored.  0 restores
 * normal operation.
 */
sz_status sz_debug_set_flags(uint32_t flags);

/* Tile size in elements of the batched calls and of single streams of 2^27
 * elements or more: 65536 (a tile never crosses a page, so the last tile of
 * a page may be shorter).  Single-stream calls on shorter streams cut them
 * into tiles of 16384 elements, so that a mid-size stream still spreads over
 * every CTA; the containers do not depend on the tile size. */
uint64_t sz_tile_elems(void);

/* Library version string, e.g. "splitzip-b200 1.0 sm_100a". */
const char *sz_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SPLITZIP_H */
