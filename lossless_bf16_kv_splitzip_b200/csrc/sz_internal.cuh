// sz_internal.cuh -- shared device-side definitions of the SplitZip B200
// kernels: tile geometry, the tile -> (segment, page, offset) mapping, the
// per-segment record, TMA / mbarrier helpers and small PTX helpers.
//
// Method: "SplitZip: Ultra Fast Lossless KV Compression for Disaggregated LLM
// Serving" (gist.science explainer), sections 1-4; container layout as
// documented in include/splitzip.h.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "splitzip.h"

namespace sz {

// ---------------------------------------------------------------- geometry
// Sub-tile: one pass of the 256 consumer threads, 4 chunks x 16 elements
// each.  Chunk c of thread t covers sub-tile elements [(c*256 + t)*16, +16),
// so a warp-wide 16-byte access is 512 contiguous bytes.
// Tile: 4 sub-tiles (65,536 elements) inside one page; the unit of work
// scheduling.  Single-stream calls on streams shorter than
// kSmallTileBelow elements use tiles of one sub-tile (16,384 elements)
// instead, so that a mid-size stream still spreads over every CTA slot.
// Range: a run of consecutive tiles of the batch, one CTA's share in both
// the histogram and the encode kernel (the two use the same partition).  A
// range cut by segment boundaries holds several pieces; the histogram kernel
// keeps the exponent counts of its first and last piece, which is all the
// encode needs to place each CTA's escape records.
constexpr int kThreads = 256;                 // consumer threads
constexpr int kWarps = kThreads / 32;
constexpr int kPipeThreads = kThreads + 32;   // + one producer warp
constexpr int kChunk = 16;
constexpr int kChunks = 4;
constexpr uint32_t kSub = kThreads * kChunk * kChunks;  // 16,384 elements
constexpr uint32_t kSubsPerTile = 4;                    // the most sub-tiles in a tile
constexpr uint32_t kTile = kSub * kSubsPerTile;         // 65,536 elements: batched calls, long streams
constexpr uint64_t kSmallTileBelow = 1ull << 27;        // single streams shorter than this: kSub tiles
constexpr uint64_t kHeader = 48;
constexpr uint32_t kMaxSmemSegs = 256;  // segment starts cached in shared memory
constexpr uint64_t kMaxRanges = 1024;   // ranges of one call (workspace bound)
constexpr uint64_t kRangesPerSM = 3;    // encode CTAs resident per SM
constexpr uint32_t kSlotDiv = 16;       // one-pass encode: escape records staged per tile = tile / 16 (6.25 %)

// Per-segment record kept in the workspace between kernels (32 bytes).
struct SegMeta {
    uint8_t codebook[16];
    uint64_t n_escapes;  // e = n - sum of the codebook's counts
    uint32_t valid;      // 1 when the 16 entries are distinct and the counts fit n
    uint32_t pad;
};
static_assert(sizeof(SegMeta) == 32, "SegMeta layout");

constexpr uint32_t kDebugNoSignal = 1u;  // producer never signals its stages

__host__ __device__ inline uint64_t container_size(uint64_t n, uint64_t e) {
    return kHeader + n + (n + 1) / 2 + 5 * e;
}
__host__ __device__ inline uint64_t div_up(uint64_t a, uint64_t b) { return (a + b - 1) / b; }

// The range partition of n_tiles tiles: `tiles` tiles per range, `count`
// ranges (the last may be shorter); at most kMaxRanges ranges.
struct RangePlan {
    uint64_t tiles;
    uint64_t count;
};
__host__ __device__ inline RangePlan plan_ranges(uint64_t n_tiles, uint64_t sms) {
    RangePlan p;
    uint64_t want = sms * kRangesPerSM;
    if (want > kMaxRanges) want = kMaxRanges;
    if (want == 0) want = 1;
    p.tiles = n_tiles ? div_up(n_tiles, want) : 1;
    p.count = div_up(n_tiles, p.tiles);
    return p;
}

// Escape bookkeeping of one range, written by the select of the segments
// that own its first and last pieces (u32: escapes < n < 2^32).
//   first_off  escapes of the first piece's segment before the range
//   first_cnt  escapes in the first piece
//   last_cnt   escapes in the last piece, when it is another piece whose
//              segment continues past the range
struct RangeRec {
    uint32_t first_off;
    uint32_t first_cnt;
    uint32_t last_cnt;
    uint32_t pad;
};
__host__ __device__ inline uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }
__host__ __device__ inline uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }
__host__ __device__ inline uint32_t umin32(uint32_t a, uint32_t b) { return a < b ? a : b; }

// Tiles of a segment of n elements in pages of page_elems: every page is cut
// into tiles of 2^tile_shift elements (its last tile may be short).
__host__ __device__ inline uint64_t tiles_per_page(uint64_t page_elems, uint32_t tile_shift) {
    return (page_elems + (1ull << tile_shift) - 1) >> tile_shift;
}
__host__ __device__ inline uint64_t segment_tiles(uint64_t n, uint64_t page_elems, uint32_t tile_shift) {
    if (n == 0) return 0;
    const uint64_t full = n / page_elems, rem = n - full * page_elems;
    return full * tiles_per_page(page_elems, tile_shift) + ((rem + (1ull << tile_shift) - 1) >> tile_shift);
}

// ------------------------------------------------------------ tile lookup
// Where the tiles come from.  Single-tensor calls use one implicit segment
// (one page = the whole tensor); batched calls read the segment table.
struct Batch {
    const sz_segment *segs;  // nullptr for a single tensor
    uint32_t n_segs;
    uint64_t page_elems;
    uint32_t tiles_per_page;  // ceil(page_elems / tile_elems), precomputed on the host
    uint32_t tile_subs;       // sub-tiles per tile: kSubsPerTile, or 1 for short single streams
    uint32_t tile_elems;      // kSub * tile_subs
    uint32_t tile_shift;      // log2(tile_elems)
    uint32_t group_tiles;     // the decode deals tiles round robin in groups of this many
    uint64_t n_tiles;
    sz_segment single;        // the implicit segment of a single-tensor call
};

__host__ __device__ inline uint64_t seg_tiles(const Batch &b, uint64_t n) {
    return segment_tiles(n, b.page_elems, b.tile_shift);
}

// Tile size of a batch: tile_subs sub-tiles of kSub elements.  The decode
// deals tiles round robin in groups of about kTile elements -- one tile, or
// several pages shorter than a tile -- so that a CTA meets a new segment at
// most once per group.
__host__ __device__ inline void set_tiles(Batch &b, uint32_t tile_subs) {
    b.tile_subs = tile_subs;
    b.tile_elems = kSub * tile_subs;
    b.tile_shift = tile_subs == 1 ? 14u : 16u;
    b.tiles_per_page = (uint32_t)tiles_per_page(b.page_elems, b.tile_shift);
    const uint64_t te = b.page_elems < (uint64_t)kTile ? b.page_elems : (uint64_t)kTile;
    const uint64_t g = (uint64_t)kTile / (te > 0 ? te : 1);
    b.group_tiles = g > 0 ? (uint32_t)g : 1u;
}
// one-pass encode: escape records a tile's workspace slot holds
__host__ __device__ inline uint32_t slot_cap(const Batch &b) { return b.tile_elems / kSlotDiv; }

struct TileRef {
    uint32_t seg;
    uint32_t local;    // tile index within the segment
    uint64_t n;        // elements of the segment
    uint32_t page;     // page index within the segment
    uint64_t elem0;    // first element of the tile in the segment's stream
    uint32_t in_page;  // offset of the tile within its page (elements)
    uint32_t len;      // elements in the tile
    uint32_t n_subs;   // sub-tiles in the tile
    uint32_t tiles;    // tiles of the segment
};

// Segment-start cache: tile_begin of every segment in shared memory when
// the batch is small enough, else binary search in global memory.
struct SegCache {
    uint64_t tile_begin[kMaxSmemSegs + 1];
};

// Must be reached by every thread of the block.
__device__ inline void seg_cache_fill(SegCache &c, const Batch &b) {
    if (b.segs != nullptr && b.n_segs <= kMaxSmemSegs) {
        for (uint32_t i = threadIdx.x; i < b.n_segs; i += blockDim.x) c.tile_begin[i] = b.segs[i].tile_begin;
        if (threadIdx.x == 0) c.tile_begin[b.n_segs] = b.n_tiles;
    }
    __syncthreads();
}

__device__ inline uint32_t find_segment(const SegCache &c, const Batch &b, uint64_t tile) {
    if (b.segs == nullptr) return 0;
    uint32_t lo = 0, hi = b.n_segs;  // largest k with tile_begin[k] <= tile
    if (b.n_segs <= kMaxSmemSegs) {
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            if (c.tile_begin[mid] <= tile) lo = mid; else hi = mid;
        }
    } else {
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            if (b.segs[mid].tile_begin <= tile) lo = mid; else hi = mid;
        }
    }
    return lo;
}

__device__ inline sz_segment load_segment(const Batch &b, uint32_t k) {
    sz_segment s;
    if (b.segs == nullptr) {
        s.n_elems = b.single.n_elems;
        s.page_begin = b.single.page_begin;
        s.out_offset = b.single.out_offset;
        s.tile_begin = b.single.tile_begin;
    } else {
        const sz_segment *g = b.segs + k;
        s.n_elems = g->n_elems;
        s.page_begin = g->page_begin;
        s.out_offset = g->out_offset;
        s.tile_begin = g->tile_begin;
    }
    return s;
}

// Geometry of global tile `tile` of segment k.  Tile and page counts fit in
// 32 bits (n < 2^32), so the divisions here are 32-bit.
__device__ inline TileRef resolve_tile(const Batch &b, const sz_segment &s, uint32_t k, uint64_t tile) {
    TileRef r;
    r.seg = k;
    r.local = (uint32_t)(tile - s.tile_begin);
    r.n = s.n_elems;
    const uint32_t tpp = b.tiles_per_page;
    const uint32_t te = b.tile_elems;
    r.page = tpp == 1 ? r.local : r.local / tpp;
    r.in_page = (r.local - r.page * tpp) << b.tile_shift;
    r.elem0 = (uint64_t)r.page * b.page_elems + r.in_page;
    const uint64_t page_len = umin64(b.page_elems, r.n - (uint64_t)r.page * b.page_elems);
    r.len = (uint32_t)umin64(te, page_len - r.in_page);
    r.n_subs = (r.len + kSub - 1) / kSub;
    const uint64_t full = r.n / b.page_elems;
    const uint64_t rem = r.n - full * b.page_elems;
    r.tiles = (uint32_t)(full * tpp + ((rem + te - 1) >> b.tile_shift));
    return r;
}

// 16 codebook entries, all different (one thread, byte loads: any alignment).
__device__ inline bool codebook16_distinct(const uint8_t *cb) {
    uint64_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        lo |= (uint64_t)cb[i] << (8 * i);
        hi |= (uint64_t)cb[8 + i] << (8 * i);
    }
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int k = i + 1; k < 16; ++k)
            ok &= ((((i < 8) ? lo : hi) >> (8 * (i & 7))) & 0xFFu) != ((((k < 8) ? lo : hi) >> (8 * (k & 7))) & 0xFFu);
    return ok;
}

// 256-bit codebook membership in 8 registers, selected without local memory.
__device__ __forceinline__ bool in_set8(const uint32_t (&set)[8], uint32_t x) {
    const uint32_t w = x >> 5;
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v = (w == (uint32_t)i) ? set[i] : v;
    return (v >> (x & 31)) & 1u;
}

// Little-endian u32 at p, 4-byte aligned or not.
__device__ __forceinline__ void store_u32_le(uint8_t *p, uint32_t v, bool aligned) {
    if (aligned) {
        *reinterpret_cast<uint32_t *>(p) = v;
    } else {
        p[0] = (uint8_t)v;
        p[1] = (uint8_t)(v >> 8);
        p[2] = (uint8_t)(v >> 16);
        p[3] = (uint8_t)(v >> 24);
    }
}

// ------------------------------------------------------------ status words
__device__ inline void set_status(int32_t *status, int32_t code) {
    if (status != nullptr) atomicCAS(reinterpret_cast<int *>(status), 0, code);
}

// --------------------------------------------------------------- PTX bits
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Streaming loads/stores: each byte is touched once by the kernel.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    return __ldcs(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void st_stream_v4(void *p, uint4 v) {
    __stcs(reinterpret_cast<uint4 *>(p), v);
}
__device__ __forceinline__ void st_stream_u64(void *p, uint64_t v) {
    __stcs(reinterpret_cast<unsigned long long *>(p), (unsigned long long)v);
}

// Read a little-endian u32 at any byte address.
__device__ __forceinline__ uint32_t load_u32_any(const uint8_t *p) {
    if ((reinterpret_cast<uintptr_t>(p) & 3) == 0) return *reinterpret_cast<const uint32_t *>(p);
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}

// Consumer-only barrier (named barrier 1): the 256 consumer threads, never
// the producer warp.
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}

// ------------------------------------------- programmatic dependent launch
// A kernel launched with launch_after() may start while the kernel before
// it in the stream is still running; it calls grid_dependency_wait() before
// it reads anything that kernel wrote (the wait returns once that kernel has
// finished and its memory operations are visible; without a prerequisite
// kernel it returns at once).  A kernel calls allow_dependents() to let the
// next launch_after() kernel start early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Ask, once per device, for the largest shared-memory carveout for
// `Kernel`: an SM then keeps room for blocks of a big-shared-memory kernel
// next to this one's (the decode kernel starting while the index kernel
// still runs), and a kernel whose blocks each take a slice of the shared
// memory gets as many of them on an SM as its other limits allow.  Best
// effort: a refusal leaves the driver's choice.
template <auto Kernel>
void prefer_max_shared() {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
    const uint64_t bit = 1ull << dev;
    if (done.load(std::memory_order_relaxed) & bit) return;
    if (cudaFuncSetAttribute(Kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess)
        done.fetch_or(bit, std::memory_order_relaxed);
    else
        (void)cudaGetLastError();
}

template <typename... Params, typename... Args>
cudaError_t launch_after(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                         Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// Rank of exponent `tid` (count c) in the order (count descending, exponent
// ascending): the number of exponents before it; ranks 0..15 are the
// codebook.  Every one of the 256 threads of the block calls it (thread t =
// exponent t).
// Only the exponents that occur are compared: they are compacted, in
// ascending order, as keys count << 8 | (255 - exponent) -- one key is
// greater than another exactly when it comes first -- and an exponent that
// does not occur ranks after all that do, in ascending order (its rank is
// the number of occurring exponents plus the absent ones below it).
struct RankShared {
    unsigned long long key[256];
    uint32_t warp[kWarps];
};
__device__ inline uint32_t exponent_rank(uint32_t c, uint32_t tid, RankShared &rs) {
    const uint32_t lane = tid & 31, wid = tid >> 5;
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, c != 0);
    if (lane == 0) rs.warp[wid] = __popc(m);
    __syncthreads();
    uint32_t before = 0, nnz = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const uint32_t x = rs.warp[w];
        before += (uint32_t)w < wid ? x : 0u;
        nnz += x;
    }
    const uint32_t pos = before + __popc(m & ((1u << lane) - 1u));  // occurring exponents below tid
    const unsigned long long mine = ((unsigned long long)c << 8) | (255u - tid);
    if (c) rs.key[pos] = mine;
    __syncthreads();
    uint32_t rank = 0;
    if (c == 0) {
        rank = nnz + (tid - pos);
    } else {
#pragma unroll 4
        for (uint32_t u = 0; u < nnz; ++u) rank += rs.key[u] > mine;
    }
    __syncthreads();  // the scratch may be reused
    return rank;
}

// ------------------------------------------------- mbarrier + 1-D TMA copy
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Raise the transaction count of the current phase by `bytes` without
// arriving (the phase still waits for its arrivals).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for phase `parity` of `bar` to complete, for at most limit_ns of
// device time.  Returns false when the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}
// One bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing `bytes` of transaction count on `bar`.
__device__ __forceinline__ void tma_load_1d(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------- launch arguments
// What the select of a segment reads and writes.
struct SelectCtx {
    Batch batch;
    const uint32_t *seg_hist;  // [n_segs][256]
    const uint32_t *rhist;     // [2][256][ranges]: first, last piece of each range (rhist_at)
    SegMeta *meta;             // [n_segs]
    RangeRec *rrec;            // [ranges]
    uint64_t range_tiles;      // tiles per range
    uint8_t *codebooks_out;    // optional [n_segs][16]
    uint32_t *hist_out;        // optional [256] (single only)
};

// Ranges of a call, and the index of the count of exponent x in the first
// (which = 0) or last (1) piece of range b: range-minor, so that the select
// reads one exponent's counts of consecutive ranges as consecutive words.
__host__ __device__ inline uint64_t range_count(uint64_t n_tiles, uint64_t range_tiles) {
    return n_tiles ? (n_tiles + range_tiles - 1) / range_tiles : 1;
}
__host__ __device__ inline uint64_t rhist_at(uint64_t ranges, uint32_t which, uint32_t x, uint64_t b) {
    return ((uint64_t)which * 256 + x) * ranges + b;
}

struct HistArgs {
    SelectCtx sel;
    const uint16_t *const *pages;  // batched: page pointers
    const uint16_t *base;          // single-tensor input
    uint32_t *seg_hist;            // [n_segs][256], zero on entry
    uint32_t *seg_done;            // [n_segs] tiles counted so far, zero on entry
    uint32_t *rhist;               // [2][256][ranges] (rhist_at)
    int32_t *status;               // [n_segs] or nullptr
    uint32_t *accum;               // accumulate mode: caller histograms [rows][256] (else nullptr)
    const uint32_t *accum_index;   // accumulate mode: row of segment k (nullptr: row k)
    int32_t *reset_status;         // optional: set to SZ_OK by block 0 (the encode's status, single stream)
    uint64_t *reset_size;          // optional: set to 0 by block 0 (the encode's size word)
};

// Select with a caller codebook (single tensor), ahead of the encode.
struct ReselectArgs {
    SelectCtx sel;
    const uint8_t *codebook_in;
    int32_t *status;      // set to SZ_OK here
    uint64_t *out_bytes;  // set to 0 here
    uint32_t *enc_done;   // set to 0 here
};

struct EncodeArgs {
    Batch batch;
    const uint16_t *const *pages;
    const uint16_t *base;
    uint8_t *out;
    uint64_t out_cap;
    uint64_t *out_bytes;      // [n_segs]
    int32_t *status;          // [n_segs]
    const SegMeta *meta;      // [n_segs]
    const RangeRec *rrec;     // [ranges]
    uint64_t range_tiles;     // tiles per range = per CTA
    uint64_t wait_limit_ns;
    uint32_t debug_flags;
    uint32_t *enc_done;       // [n_segs] tiles whose pieces are complete, zero on entry (two-pass)
    // one-pass mode (caller codebooks, no histogram pass)
    const uint8_t *codebooks_in;  // [n_segs][16]
    uint32_t *tile_cnt;           // [n_tiles] escapes of each tile
    uint32_t *slots;              // [n_tiles][slot_cap] records: raw << 16 | offset in the tile
    RangeRec *rcnt;               // [ranges] first_cnt / last_cnt: escapes of the first / last piece
};

// A tile whose escapes overflowed its record slot, left for the rescan.
struct OvfItem {
    uint64_t tile;  // global tile index
    uint64_t base;  // index of the tile's first escape record in its segment
    uint64_t e;     // escapes of the segment
    uint32_t cnt;   // escapes of the tile
    uint32_t seg;
};

// Scratch of the short-stream path of one-call compression (sz_compress).
struct SmallWs {
    uint32_t *seg_hist;    // [256] stream counts          } zero on entry
    uint32_t *done;        // slices counted               }
    uint32_t *done2;       // slices encoded               }
    SegMeta *meta;
    uint32_t *block_off;   // [slices] first escape index of each slice
    uint32_t *block_hist;  // [slices][256]
};

// The escape placement that follows a one-pass encode.
struct PlaceArgs {
    Batch batch;
    const uint16_t *const *pages;
    const uint16_t *base;
    const uint8_t *codebooks_in;  // [n_segs][16]
    uint8_t *out;
    uint64_t out_cap;
    uint64_t *out_bytes;          // [n_segs]
    int32_t *status;              // [n_segs]
    const uint32_t *tile_cnt;     // [n_tiles]
    const uint32_t *slots;        // [n_tiles][slot_cap]
    const RangeRec *rcnt;         // [ranges]
    uint64_t range_tiles;
    uint32_t *ovf_count;          // overflowed tiles listed so far (zero on entry)
    OvfItem *ovf;                 // [n_tiles]
    uint32_t *seg_e;              // [n_segs] escape count of each segment (placement -> rescan)
    uint32_t *blocks_done;        // rescan blocks finished (zero on entry)
};

struct DecodeArgs {
    Batch batch;
    uint16_t *const *pages;  // batched destination pages
    uint16_t *base;          // single-tensor output
    const uint8_t *in;
    uint64_t in_cap;         // bytes available from d_in (single: in_bytes)
    int32_t *status;         // [n_segs]
    uint32_t *sub_start;     // per segment: 4*tiles+1 escape start indices
    uint64_t tiles_per_cta;
    uint64_t wait_limit_ns;
    uint32_t debug_flags;
};

// ------------------------------------------------------------- host side
// Process-wide settings of sz_set_wait_limit_ns and sz_debug_set_flags.
uint64_t wait_limit_ns();
uint32_t debug_flags();

// The implicit batch of a single-tensor call: one segment, one page.
Batch single_batch(uint64_t n);

// Device facts the launchers need, looked up once per device ordinal
// (ordinals 0..kMaxDevices-1; a larger ordinal gives SZ_ERR_INVALID).
constexpr int kMaxDevices = 64;
struct DeviceInfo {
    bool ready = false;
    int sms = 0, dec_occ = 1;
};
sz_status device_info(DeviceInfo &out);

// Scratch of the pipelined compression of one stream.  `zero` .. `zero` +
// zero_bytes must cover seg_hist, seg_done and enc_done (cleared by the call).
struct CompressScratch {
    uint8_t *zero;
    uint64_t zero_bytes;
    uint32_t *seg_hist;  // [256]
    uint32_t *seg_done;  // [1]
    uint32_t *enc_done;  // [1]
    SegMeta *meta;       // [1]
    uint32_t *rhist;     // [2][256][ranges] (rhist_at)
    RangeRec *rrec;      // [ranges]
};
// Histogram kernel (with the select) and encode kernel of d_in[0..n): the
// container of sz_histogram_codebook + sz_encode, in one call.
sz_status compress_pipelined(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap,
                             uint64_t *d_out_bytes, uint8_t *d_codebook16_or_null, int32_t *d_status,
                             const CompressScratch &w, const DeviceInfo &dev, cudaStream_t s);

}  // namespace sz
