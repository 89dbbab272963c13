// sz_decode.cu -- container reader.
//
// SplitZip explainer (gist.science), section 4 "Pourquoi est-ce rapide ?":
// decoding looks each 4-bit code up, joins the exponent it names to the
// sign and mantissa, and, where an escape note exists, overwrites that
// place with the raw exponent -- linear work with no detours.
//
// Two launches.  (1) esc_index_kernel: for every 16,384-element sub-tile,
// the index of its first escape in the ascending position stream (one
// binary search per sub-tile, all in parallel); it also checks each
// segment's header.  (2) decode_kernel, warp-specialised like the encode,
// 3 CTAs per SM, groups of tiles (about 65,536 elements each) dealt round
// robin, so that the CTAs' stores land close together in memory:
//   producer thread  TMA bulk copies of the sub-tile's sm bytes (16 KiB),
//                    codes (8 KiB) and a 16-byte aligned superset of its
//                    escape positions and exponents into a 2-stage ring;
//   8 consumer warps turn codes + sm bytes into BF16 with register-only
//                    PRMT lookups and write 16-byte stores (the escaped
//                    places get codebook[0]); then, after one barrier per
//                    sub-tile -- into which the wait for the next stage's
//                    data is folded -- one thread per escape checks its
//                    record (inside the sub-tile, strictly ascending, raw
//                    exponent outside the codebook, placeholder code 0) and
//                    overwrites the value.
// Monotone sub-tile starts plus in-sub-tile checks prove the whole escape
// stream well formed.  Every mbarrier wait is bounded.
//
// Streams of up to 2^21 elements take one launch instead: small_decode_kernel,
// one block per 4,096-element slice, each finding its slice's escape records
// by binary search.
#include "sz_internal.cuh"

namespace sz {

// ------------------------------------------------------------ the header
struct Header {
    uint64_t n, e;
    uint64_t cb_lo, cb_hi;  // codebook bytes 0-7 and 8-15, little-endian
    bool ok;
    bool misaligned;        // container not on a 16-byte boundary: not read at all
};

__device__ __forceinline__ uint32_t cb_entry(uint64_t lo, uint64_t hi, int k) {  // k compile-time after unrolling
    return (uint32_t)(((k < 8) ? lo : hi) >> (8 * (k & 7))) & 0xFFu;
}

// Parse and check the fixed fields of the container at c (cap bytes
// available) for a stream of `n` elements.
__device__ inline Header read_header(const uint8_t *c, uint64_t cap, uint64_t n) {
    Header h{};
    h.ok = false;
    h.misaligned = (reinterpret_cast<uintptr_t>(c) & 15) != 0;
    if (h.misaligned || cap < kHeader) return h;
    const uint64_t w0 = *reinterpret_cast<const uint64_t *>(c);
    h.n = *reinterpret_cast<const uint64_t *>(c + 8);
    h.e = *reinterpret_cast<const uint64_t *>(c + 16);
    h.cb_lo = *reinterpret_cast<const uint64_t *>(c + 24);
    h.cb_hi = *reinterpret_cast<const uint64_t *>(c + 32);
    const uint64_t rsv = *reinterpret_cast<const uint64_t *>(c + 40);
    bool distinct = true;
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int k = i + 1; k < 16; ++k) distinct &= cb_entry(h.cb_lo, h.cb_hi, i) != cb_entry(h.cb_lo, h.cb_hi, k);
    h.ok = w0 == 0x00000101564B5A53ull && rsv == 0 && h.n == n && n < (1ull << 32) && h.e <= n &&
           container_size(n, h.e) <= cap && distinct;
    return h;
}

// ------------------------------------------------- per-sub-tile escape index
// Entry j of segment k (j = S*tile + sub, S = sub-tiles per tile, j =
// 0..S*tiles_k) = index of the first escape whose position is >= the first
// element of that sub-tile (sub-tiles past a short tile's end start at the
// tile's end); entry S*tiles_k = e.  Entries of segment k start at
// S*tile_begin_k + k.  kWarp (few entries, where latency rules): one warp per
// entry, a 32-way search over the ascending position stream (each round
// probes 32 evenly spaced records and keeps the interval where the positions
// reach the target, so about log32 e dependent loads); else one thread per
// entry and a binary search (log2 e dependent loads, 32x fewer threads).
// On a corrupt stream either search still ends, on some index; the decode's
// per-sub-tile checks reject the records.  The entry of the segment's
// sentinel also writes the segment's status (SZ_OK, or the header's error):
// the decode kernel after it only ever sets errors.
__device__ inline uint64_t warp_first_at_least(const uint8_t *pos, uint64_t e, uint64_t target, uint32_t lane) {
    uint64_t lo = 0, hi = e;  // the answer is in [lo, hi]
    while (lo < hi) {
        const uint64_t step = (hi - lo + 31) / 32;
        const uint64_t p = lo + (uint64_t)(lane + 1) * step - 1;
        bool ge = true;  // probes past the interval count as reaching the target
        if (p < hi) ge = load_u32_any(pos + 4 * p) >= target;
        const uint32_t b = __ballot_sync(0xFFFFFFFFu, ge);
        if (b == 0) return hi;  // every probe is below: the answer is hi
        const uint64_t f = (uint64_t)(__ffs(b) - 1);
        const uint64_t nhi = umin64(hi, lo + (f + 1) * step - 1);
        lo = f == 0 ? lo : lo + f * step;
        hi = nhi;
    }
    return lo;
}

template <bool kBatched, bool kWarp>
__global__ void __launch_bounds__(256) esc_index_kernel(const DecodeArgs a, uint64_t n_entries) {
    __shared__ uint64_t s_entry_begin[kMaxSmemSegs + 1];
    grid_dependency_wait();  // the kernel that wrote the containers has finished
    // The decode kernel may start now: every container is complete, so it
    // may read headers, sm bytes and codes before its own wait (only the
    // index entries and status words written here need that wait).
    allow_dependents();
    const uint32_t S = a.batch.tile_subs;
    const uint32_t ns = kBatched ? a.batch.n_segs : 1u;
    const bool cached = kBatched && ns <= kMaxSmemSegs;
    if (cached) {
        for (uint32_t i = threadIdx.x; i < ns; i += blockDim.x)
            s_entry_begin[i] = S * a.batch.segs[i].tile_begin + i;
    }
    __syncthreads();
    const uint32_t lane = kWarp ? threadIdx.x & 31 : 0u;
    const uint64_t j_glob = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> (kWarp ? 5 : 0);
    if (j_glob >= n_entries) return;
    uint32_t k = 0;
    if (kBatched) {  // largest k with S*tile_begin_k + k <= j_glob
        uint32_t lo = 0, hi = ns;
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            const uint64_t b = cached ? s_entry_begin[mid] : S * a.batch.segs[mid].tile_begin + mid;
            if (b <= j_glob) lo = mid; else hi = mid;
        }
        k = lo;
    }
    const sz_segment seg = load_segment(a.batch, k);
    const uint64_t j = j_glob - (S * seg.tile_begin + k);
    const uint64_t tiles = seg_tiles(a.batch, seg.n_elems);
    uint32_t *ts = a.sub_start + S * seg.tile_begin + k;
    if (j > S * tiles) return;
    const uint64_t cap = seg.out_offset <= a.in_cap ? a.in_cap - seg.out_offset : 0;
    const uint8_t *c = a.in + seg.out_offset;
    const Header h = read_header(c, cap, seg.n_elems);
    if (j == S * tiles) {  // the sentinel entry: the segment's status and its escape count
        if (lane == 0) {
            a.status[k] = h.ok ? SZ_OK : (h.misaligned ? SZ_ERR_ALIGN : SZ_ERR_CORRUPT);
            ts[j] = h.ok ? (uint32_t)h.e : 0u;
        }
        return;
    }
    uint64_t idx = 0;
    if (h.ok) {
        const TileRef r = resolve_tile(a.batch, seg, k, seg.tile_begin + j / S);
        const uint64_t first = r.elem0 + umin32((uint32_t)(j % S) * kSub, r.len);
        const uint64_t n = h.n;
        const uint8_t *pos = c + kHeader + n + (n + 1) / 2;
        if (kWarp) {
            idx = warp_first_at_least(pos, h.e, first, lane);
        } else {  // first index with pos >= first
            uint64_t lo = 0, hi = h.e;
            while (lo < hi) {
                const uint64_t mid = (lo + hi) >> 1;
                if (load_u32_any(pos + 4 * mid) < first) lo = mid + 1; else hi = mid;
            }
            idx = lo;
        }
    }
    if (lane == 0) ts[j] = (uint32_t)idx;
}

// -------------------------------------------------------------- decode
// Code lookup tables built from the codebook, for PRMT byte selection:
//   hA..hD  byte k = codebook[k] >> 1            (codes 0-3, 4-7, 8-11, 12-15)
//   lA, lB  byte j = (codebook[j] & 1) << 6 | (codebook[j+8] & 1) << 7
// A code nibble with bit 3 clear selects its byte directly; with bit 3 set
// PRMT replicates the selected byte's bit 7, which is the low exponent bit of
// code j+8 -- so bit 6 of the result is always the low exponent bit.
struct DecTables {
    uint32_t hA, hB, hC, hD, lA, lB;
};

__device__ inline DecTables make_tables(uint64_t cb_lo, uint64_t cb_hi) {
    DecTables t;
    uint32_t h[4] = {0, 0, 0, 0}, l[2] = {0, 0};
#pragma unroll
    for (int k = 0; k < 16; ++k) h[k >> 2] |= (cb_entry(cb_lo, cb_hi, k) >> 1) << (8 * (k & 3));
#pragma unroll
    for (int j = 0; j < 8; ++j)
        l[j >> 2] |= (((cb_entry(cb_lo, cb_hi, j) & 1u) << 6) | ((cb_entry(cb_lo, cb_hi, j + 8) & 1u) << 7))
                     << (8 * (j & 3));
    t.hA = h[0]; t.hB = h[1]; t.hC = h[2]; t.hD = h[3];
    t.lA = l[0]; t.lB = l[1];
    return t;
}

// Four elements: `sel` holds their four code nibbles (low 16 bits), `smw`
// their four sm bytes.  Out: two words of two BF16 each.
__device__ __forceinline__ void decode_quad(uint32_t sel, uint32_t smw, const DecTables &T, uint32_t &o0,
                                            uint32_t &o1) {
    const uint32_t s7 = sel & 0x7777u;
    const uint32_t r0 = prmt(T.hA, T.hB, s7);          // exponent >> 1 for codes 0-7
    const uint32_t r1 = prmt(T.hC, T.hD, s7);          // ... for codes 8-15
    const uint32_t m = prmt(0x7F7F7F7Fu, 0x7F7F7F7Fu, sel);  // 0x7F: code < 8, 0x00: code >= 8
    const uint32_t hiE = (r0 & m) | (r1 & ~m);
    const uint32_t t = prmt(T.lA, T.lB, sel);          // bit 6 = low exponent bit
    const uint32_t out_hi = (smw & 0x80808080u) | hiE;                       // sign | exp >> 1
    const uint32_t out_lo = (smw & 0x7F7F7F7Fu) | ((t << 1) & 0x80808080u);  // exp & 1 | mantissa
    o0 = prmt(out_lo, out_hi, 0x5140u);
    o1 = prmt(out_lo, out_hi, 0x7362u);
}

__device__ __forceinline__ void decode_chunk(uint4 sm, uint64_t codes, const DecTables &T, uint4 &out0,
                                             uint4 &out1) {
    const uint32_t c0 = (uint32_t)codes, c1 = (uint32_t)(codes >> 32);
    decode_quad(c0, sm.x, T, out0.x, out0.y);
    decode_quad(c0 >> 16, sm.y, T, out0.z, out0.w);
    decode_quad(c1, sm.z, T, out1.x, out1.y);
    decode_quad(c1 >> 16, sm.w, T, out1.z, out1.w);
}

// Replace the exponent of element j (0..15, runtime) of a decoded chunk:
// every word is rewritten through a select, so the chunk stays in registers.
__device__ __forceinline__ void patch_elem(uint4 &o0, uint4 &o1, int j, uint32_t raw) {
    const int q = j >> 1;
    const uint32_t sh = (j & 1) ? 16u : 0u;
    const uint32_t mask = ~(0x7F80u << sh);
    const uint32_t val = (raw & 0xFFu) << (7 + sh);
#define SZ_PATCH(word, idx) word = (q == (idx)) ? ((word & mask) | val) : word
    SZ_PATCH(o0.x, 0); SZ_PATCH(o0.y, 1); SZ_PATCH(o0.z, 2); SZ_PATCH(o0.w, 3);
    SZ_PATCH(o1.x, 4); SZ_PATCH(o1.y, 5); SZ_PATCH(o1.z, 6); SZ_PATCH(o1.w, 7);
#undef SZ_PATCH
}

constexpr int kDecStages = 2;  // 3 CTAs per SM
constexpr uint32_t kEscCap = 1024;  // escape records bulk-copied per sub-tile; more: read directly

constexpr uint32_t kDFlagEnd = 1u;
constexpr uint32_t kDFlagInSmem = 2u;   // sm + codes came by TMA into the stage
constexpr uint32_t kDFlagTileEnd = 4u;  // last sub-tile of its tile
constexpr uint32_t kDFlagEscSmem = 8u;  // the escape records came by TMA into the stage (DecEscMeta)
constexpr uint32_t kDFlagEarly = 16u;   // described and copied before the grid dependency wait
constexpr uint32_t kDebugNoEscapeSignal = 2u;  // test hook: the producer publishes values parts only

// What the producer read and copied before the grid dependency wait.
struct DecEarly {
    uint32_t n;  // leading sub-tiles whose sm + code copies were issued
    uint32_t k;  // segment whose header was read (0xFFFFFFFF: none)
    sz_segment seg;
    Header h;
};

// A stage's description in two parts, each published by its own arrival:
// the values part (full[s]) needs only the container, the escape part
// (escs[s]) needs the index kernel's sub-tile starts, so the consumers
// decode and store a stage's values while the index may still be running.
struct DecMeta {
    uint16_t *dst;      // global destination of the sub-tile's first element
    const uint8_t *c;   // the segment's container
    uint64_t elem0;     // first element of the sub-tile in the segment stream
    uint64_t n, e;
    uint64_t cb_lo, cb_hi;
    uint64_t tile;      // global tile of the sub-tile
    uint32_t seg, len, flags, pad;
};
struct DecEscMeta {
    uint32_t lo, cnt;   // the sub-tile's escape records [lo, lo + cnt)
    uint32_t pos_skew;  // byte offset of record lo's position inside the staged copy
    uint32_t raw_skew;  // byte offset of record lo's exponent inside the staged copy
    uint32_t flags;     // kDFlagEscSmem
};

struct __align__(128) DecShared {
    uint8_t sm[kDecStages][kSub];
    uint8_t codes[kDecStages][kSub / 2];
    uint8_t pos[kDecStages][4 * kEscCap + 32];  // 16-byte aligned superset of the positions
    uint8_t raw[kDecStages][kEscCap + 32];      // 16-byte aligned superset of the exponents
    DecMeta meta[kDecStages];
    DecEscMeta emeta[kDecStages];
    uint64_t full[kDecStages];   // values part: sm + codes arrived, meta written
    uint64_t escs[kDecStages];   // escape part: records arrived, emeta written
    uint64_t empty[kDecStages];
    SegCache segc;
    DecEarly early;  // producer only: what it read and copied before the grid dependency wait
    int go[2];  // stage j's data arrived (slot j & 1)
    int eok;    // the current stage's escape part arrived
};

// Tiles are dealt round robin in groups of about kTile elements: one tile
// of a contiguous tensor, several when pages are smaller than a tile, so
// that a CTA meets a new segment (header, codebook tables) at most once per
// group.  Group g holds tiles [g * group, (g + 1) * group).
__host__ __device__ inline uint64_t tiles_per_group(const Batch &b) { return b.group_tiles; }

// The tile a CTA of `grid` decodes after tile t.
__device__ __forceinline__ uint64_t next_dealt_tile(uint64_t t, uint64_t group, uint32_t grid) {
    if (group == 1) return t + grid;
    return (t + 1) % group == 0 ? t + 1 + (uint64_t)(grid - 1) * group : t + 1;
}

// A stage wait of this CTA ran out.  Its tiles before `from` (in the order
// it decodes them) are complete; every segment with a tile at or after
// `from` gets SZ_ERR_DEVICE_TIMEOUT.
__device__ void decode_timeout_from(const DecodeArgs &a, const SegCache &c, uint64_t from) {
    const uint64_t group = tiles_per_group(a.batch);
    uint32_t last = 0xFFFFFFFFu;
    for (uint64_t t = from; t < a.batch.n_tiles; t = next_dealt_tile(t, group, gridDim.x)) {
        const uint32_t k = find_segment(c, a.batch, t);
        if (k != last) set_status(a.status + k, SZ_ERR_DEVICE_TIMEOUT);
        last = k;
    }
}

// ------------------------------------------------------------ producer
// Before the grid dependency wait (the index kernel's end): the header of
// the CTA's first segment and the values part of its first kDecStages
// sub-tiles (description, sm + code copies, arrival) -- what the containers
// alone give, not the index entries or status words the index kernel
// writes; the consumers start on those values at once.  The containers are
// complete here: the index kernel lets this kernel start only after its own
// wait for the kernel that wrote them.  Stops at the first sub-tile that is
// short, in another segment, or whose header or alignment rules out bulk
// copies.  Sets no status (the index kernel writes it).
template <bool kBatched>
__device__ void decode_prefetch(const DecodeArgs &a, DecShared &sh) {
    DecEarly &p = sh.early;  // the producer thread's own (shared memory: no registers held over the wait)
    p.n = 0;
    p.k = 0xFFFFFFFFu;
    if ((a.debug_flags & kDebugNoSignal) != 0) return;
    const uint64_t group = tiles_per_group(a.batch);
    for (uint64_t t = (uint64_t)blockIdx.x * group; t < a.batch.n_tiles && p.n < (uint32_t)kDecStages;
         t = next_dealt_tile(t, group, gridDim.x)) {
        const uint32_t k = find_segment(sh.segc, a.batch, t);
        if (k != p.k) {
            if (p.k != 0xFFFFFFFFu) return;
            p.k = k;
            p.seg = load_segment(a.batch, k);
            const uint64_t cap = p.seg.out_offset <= a.in_cap ? a.in_cap - p.seg.out_offset : 0;
            p.h = read_header(a.in + p.seg.out_offset, cap, p.seg.n_elems);
        }
        if (!p.h.ok || (p.seg.n_elems % 16) != 0) return;
        const TileRef r = resolve_tile(a.batch, p.seg, k, t);
        const uint8_t *c = a.in + p.seg.out_offset;
        uint16_t *dst = kBatched ? a.pages[p.seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        if ((reinterpret_cast<uintptr_t>(dst) & 15) != 0) return;
        for (uint32_t sub = 0; sub < r.n_subs && p.n < (uint32_t)kDecStages; ++sub) {
            if (r.len - sub * kSub < kSub) return;
            const uint64_t elem0 = r.elem0 + (uint64_t)sub * kSub;
            DecMeta &m = sh.meta[p.n];
            m.dst = dst + sub * kSub;
            m.c = c;
            m.elem0 = elem0;
            m.n = p.h.n;
            m.e = p.h.e;
            m.cb_lo = p.h.cb_lo;
            m.cb_hi = p.h.cb_hi;
            m.tile = t;
            m.seg = k;
            m.len = kSub;
            m.flags = kDFlagInSmem | kDFlagEarly | (sub + 1 == r.n_subs ? kDFlagTileEnd : 0u);
            mbar_arrive_expect_tx(&sh.full[p.n], kSub + kSub / 2);
            tma_load_1d(sh.sm[p.n], c + kHeader + elem0, kSub, &sh.full[p.n]);
            tma_load_1d(sh.codes[p.n], c + kHeader + p.h.n + elem0 / 2, kSub / 2, &sh.full[p.n]);
            ++p.n;
        }
    }
}

// One thread: per sub-tile, wait for the stage to be free, then publish
// its values part (description; sm bytes and codes by bulk copy) on
// full[s] and its escape part (record range; when they fit and stay inside
// the buffer, a 16-byte aligned superset of its escape positions and
// exponents by bulk copy) on escs[s] -- for the first sh.early.n sub-tiles
// only the escape part, the values part went out before the wait.
template <bool kBatched>
__device__ void decode_producer(const DecodeArgs &a, DecShared &sh) {
    if ((a.debug_flags & kDebugNoSignal) != 0) return;  // test hook: nothing is ever signalled
    const DecEarly &pf = sh.early;
    uint32_t j = 0;
    uint32_t cur = 0xFFFFFFFFu;
    sz_segment seg{};
    Header h{};
    const uint8_t *c = nullptr;
    uint64_t cap = 0;
    bool tma_ok = false;
    const uint64_t group = tiles_per_group(a.batch);
    for (uint64_t t = (uint64_t)blockIdx.x * group; t < a.batch.n_tiles; t = next_dealt_tile(t, group, gridDim.x)) {
        const uint32_t k = find_segment(sh.segc, a.batch, t);
        if (k != cur) {
            cur = k;
            seg = k == pf.k ? pf.seg : load_segment(a.batch, k);
            cap = seg.out_offset <= a.in_cap ? a.in_cap - seg.out_offset : 0;
            c = a.in + seg.out_offset;
            h = k == pf.k ? pf.h : read_header(c, cap, seg.n_elems);
            tma_ok = (seg.n_elems % 16) == 0;  // code and position streams 16-byte aligned
            if (!h.ok) set_status(a.status + k, h.misaligned ? SZ_ERR_ALIGN : SZ_ERR_CORRUPT);
        }
        if (!h.ok) continue;
        const TileRef r = resolve_tile(a.batch, seg, k, t);
        uint16_t *dst = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        const bool dst_aligned = (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
        if (!dst_aligned) set_status(a.status + k, SZ_ERR_ALIGN);
        // the tile's five sub-tile starts; the last sub-tile of a tile ends
        // where the next tile starts (the segment's last: at e), so the
        // ranges cover every escape record
        const uint32_t S = a.batch.tile_subs;
        const uint32_t *ts = a.sub_start + S * (seg.tile_begin + r.local) + k;
        uint32_t tsv[kSubsPerTile + 1];
#pragma unroll
        for (uint32_t q = 0; q <= kSubsPerTile; ++q) tsv[q] = q <= S ? ts[q] : 0u;
        const uint64_t pos_off = kHeader + h.n + (h.n + 1) / 2;
        const uint64_t raw_off = pos_off + 4 * h.e;
        for (uint32_t sub = 0; sub < r.n_subs; ++sub, ++j) {
            const int s = (int)(j % kDecStages);
            if (j >= (uint32_t)kDecStages && !mbar_wait(&sh.empty[s], ((j / kDecStages) - 1) & 1u, a.wait_limit_ns)) {
                set_status(a.status + k, SZ_ERR_DEVICE_TIMEOUT);
                return;
            }
            const uint64_t elem0 = r.elem0 + (uint64_t)sub * kSub;
            const uint32_t len = umin32(kSub, r.len - sub * kSub);
            uint32_t lo = tsv[0], hi = tsv[0];
#pragma unroll
            for (uint32_t q = 0; q <= kSubsPerTile; ++q)
                if (q == S) hi = tsv[q];
#pragma unroll
            for (uint32_t q = 0; q < kSubsPerTile; ++q) {
                if (q == sub) {
                    lo = tsv[q];
                    if (sub + 1 < r.n_subs) hi = tsv[q + 1];
                }
            }
            if (hi < lo || hi > h.e || hi - lo > len) {  // sub-tile starts not monotone
                set_status(a.status + k, SZ_ERR_CORRUPT);
                hi = lo = 0;
            }
            const uint32_t cnt = hi - lo;
            const bool tma = tma_ok && len == kSub;
            if (j >= pf.n) {  // the values part (the first pf.n went out before the wait)
                DecMeta &m = sh.meta[s];
                m.dst = dst_aligned ? dst + sub * kSub : nullptr;
                m.c = c;
                m.elem0 = elem0;
                m.n = h.n;
                m.e = h.e;
                m.cb_lo = h.cb_lo;
                m.cb_hi = h.cb_hi;
                m.tile = t;
                m.seg = k;
                m.len = len;
                m.flags = (sub + 1 == r.n_subs ? kDFlagTileEnd : 0u) | (tma ? kDFlagInSmem : 0u);
                if (tma) {
                    mbar_arrive_expect_tx(&sh.full[s], kSub + kSub / 2);
                    tma_load_1d(sh.sm[s], c + kHeader + elem0, kSub, &sh.full[s]);
                    tma_load_1d(sh.codes[s], c + kHeader + h.n + elem0 / 2, kSub / 2, &sh.full[s]);
                } else {
                    mbar_arrive(&sh.full[s]);
                }
            }
            // test hook: the escape parts are never published
            if ((a.debug_flags & kDebugNoEscapeSignal) != 0) return;
            // the escape part: aligned supersets [ps & ~15, ceil16(pe)) of
            // the records, which must lie inside the caller's buffer
            DecEscMeta &em = sh.emeta[s];
            em.lo = lo;
            em.cnt = cnt;
            em.flags = 0;
            uint32_t bytes = 0;
            if (tma && cnt > 0 && cnt <= kEscCap) {
                const uint64_t p0 = (pos_off + 4 * (uint64_t)lo) & ~15ull;
                const uint64_t p1 = (pos_off + 4 * (uint64_t)hi + 15) & ~15ull;
                const uint64_t r0 = (raw_off + lo) & ~15ull;
                const uint64_t r1 = (raw_off + hi + 15) & ~15ull;
                if (p1 <= cap && r1 <= cap) {
                    em.flags = kDFlagEscSmem;
                    em.pos_skew = (uint32_t)(pos_off + 4 * (uint64_t)lo - p0);
                    em.raw_skew = (uint32_t)(raw_off + lo - r0);
                    bytes = (uint32_t)(p1 - p0) + (uint32_t)(r1 - r0);
                    mbar_arrive_expect_tx(&sh.escs[s], bytes);
                    tma_load_1d(sh.pos[s], c + p0, (uint32_t)(p1 - p0), &sh.escs[s]);
                    tma_load_1d(sh.raw[s], c + r0, (uint32_t)(r1 - r0), &sh.escs[s]);
                }
            }
            if (!bytes) mbar_arrive(&sh.escs[s]);
        }
    }
    const int s = (int)(j % kDecStages);
    if (j >= (uint32_t)kDecStages && !mbar_wait(&sh.empty[s], ((j / kDecStages) - 1) & 1u, a.wait_limit_ns)) return;
    sh.meta[s].flags = kDFlagEnd;
    mbar_arrive(&sh.full[s]);
}

// ------------------------------------------------------------ consumers
// One chunk: 16 sm bytes + 8 code bytes -> 16 BF16 values, stored.  The
// escaped places get codebook[0] here and are overwritten afterwards.
__device__ __forceinline__ void decode_store_chunk(const DecMeta &m, DecShared &sh, int s, const DecTables &T, int q,
                                                   int tid, int32_t *status) {
    const uint32_t off = (q * kThreads + tid) * kChunk;
    if (off >= m.len) return;
    const uint32_t cnt = umin32(kChunk, m.len - off);
    uint4 smv = make_uint4(0, 0, 0, 0);
    uint64_t codes = 0;
    if (m.flags & kDFlagInSmem) {
        smv = *reinterpret_cast<const uint4 *>(sh.sm[s] + off);
        codes = *reinterpret_cast<const unsigned long long *>(sh.codes[s] + off / 2);
    } else {
        const uint8_t *in_sm = m.c + kHeader + m.elem0;
        const uint8_t *codes_base = m.c + kHeader + m.n;
        if (cnt == (uint32_t)kChunk && (m.n % 8) == 0) {
            smv = ld_stream_v4(in_sm + off);
            codes = *reinterpret_cast<const unsigned long long *>(codes_base + (m.elem0 + off) / 2);
        } else {
            uint32_t sw[4] = {0, 0, 0, 0};
#pragma unroll
            for (int jj = 0; jj < kChunk; ++jj)
                if (jj < (int)cnt) sw[jj >> 2] |= (uint32_t)in_sm[off + jj] << (8 * (jj & 3));
            smv = make_uint4(sw[0], sw[1], sw[2], sw[3]);
            const uint8_t *cb = codes_base + (m.elem0 + off) / 2;
#pragma unroll
            for (int b = 0; b < kChunk / 2; ++b)
                if (2 * b < (int)cnt) codes |= (uint64_t)cb[b] << (8 * b);
            // odd element count: the unused high nibble must be 0
            if ((cnt & 1) && ((codes >> (4 * cnt)) & 0xFu) != 0) set_status(status, SZ_ERR_CORRUPT);
            if (cnt < (uint32_t)kChunk) codes &= (1ull << (4 * cnt)) - 1ull;
        }
    }
    uint4 o0, o1;
    decode_chunk(smv, codes, T, o0, o1);
    if (m.dst == nullptr) return;
    if (cnt == (uint32_t)kChunk) {
        *reinterpret_cast<uint4 *>(m.dst + off) = o0;
        *reinterpret_cast<uint4 *>(m.dst + off + 8) = o1;
    } else {
        const uint32_t w[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
        for (int jj = 0; jj < kChunk; ++jj)
            if (jj < (int)cnt) m.dst[off + jj] = (uint16_t)(w[jj >> 1] >> (16 * (jj & 1)));
    }
}

template <bool kBatched>
__device__ void decode_consumers(const DecodeArgs &a, DecShared &sh) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t cur = 0xFFFFFFFFu;
    DecTables T{};
    uint32_t cbset[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    // thread 0: this CTA's first tile not yet decoded completely (every
    // consumer has passed the barrier below when it is read)
    uint64_t next_tile = (uint64_t)blockIdx.x * tiles_per_group(a.batch);
    // One consumer barrier per sub-tile: after its values are stored, thread
    // 0 waits for the stage's escape part and the next stage's values part,
    // then the barrier orders every store before the escape patches and
    // hands both arrivals to all.  The consumers do not wait for the index
    // kernel before a stage described before the grid dependency wait (its
    // values need only the container, and that path sets no status); every
    // other status write comes after their own grid dependency wait.
    if (tid == 0) sh.go[0] = mbar_wait(&sh.full[0], 0u, a.wait_limit_ns) ? 1 : 0;
    consumer_sync();
    for (uint32_t j = 0;; ++j) {
        const int s = (int)(j % kDecStages);
        if (!sh.go[j & 1]) {  // the same decision in every consumer thread
            grid_dependency_wait();
            if (tid == 0) decode_timeout_from(a, sh.segc, next_tile);
            return;
        }
        const DecMeta m = sh.meta[s];
        if (m.flags & kDFlagEnd) return;
        if (!(m.flags & kDFlagEarly)) grid_dependency_wait();
        if (m.seg != cur) {
            T = make_tables(m.cb_lo, m.cb_hi);
#pragma unroll
            for (int i = 0; i < 8; ++i) cbset[i] = 0;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const uint32_t x = cb_entry(m.cb_lo, m.cb_hi, q);
#pragma unroll
                for (int i = 0; i < 8; ++i) cbset[i] |= ((x >> 5) == (uint32_t)i) ? (1u << (x & 31)) : 0u;
            }
            cur = m.seg;
        }
        int32_t *status = a.status + m.seg;

        // ---- every chunk: codes -> exponents, joined with sign and mantissa
#pragma unroll
        for (int q = 0; q < kChunks; ++q) decode_store_chunk(m, sh, s, T, q, tid, status);

        const int s_next = (int)((j + 1) % kDecStages);
        if (tid == 0) {
            const bool e_ok = mbar_wait(&sh.escs[s], (j / kDecStages) & 1u, a.wait_limit_ns);
            sh.eok = e_ok ? 1 : 0;
            sh.go[(j + 1) & 1] =
                e_ok && mbar_wait(&sh.full[s_next], ((j + 1) / kDecStages) & 1u, a.wait_limit_ns) ? 1 : 0;
        }
        consumer_sync();
        grid_dependency_wait();  // returns at once: the escape part was published after it
        if (!sh.eok) {  // the same decision in every consumer thread
            if (tid == 0) decode_timeout_from(a, sh.segc, next_tile);
            return;
        }

        // ---- escapes, one per thread, after every chunk store of the
        // sub-tile: check the record and overwrite its value's exponent
        const DecEscMeta em = sh.emeta[s];
        if (em.cnt) {
            const bool es = (em.flags & kDFlagEscSmem) != 0;
            const bool ss = (m.flags & kDFlagInSmem) != 0;
            const uint8_t *gpos = m.c + kHeader + m.n + (m.n + 1) / 2;
            const uint8_t *graw = gpos + 4 * m.e;
            const uint8_t *spos = sh.pos[s] + em.pos_skew;
            const uint8_t *sraw = sh.raw[s] + em.raw_skew;
            const uint8_t *gsm = m.c + kHeader + m.elem0;
            const uint8_t *gcodes = m.c + kHeader + m.n;
            for (uint32_t i = tid; i < em.cnt; i += kThreads) {
                const uint64_t g = (uint64_t)em.lo + i;
                const uint64_t p = es ? *reinterpret_cast<const uint32_t *>(spos + 4 * i) : load_u32_any(gpos + 4 * g);
                const uint32_t x = es ? sraw[i] : graw[g];
                bool bad = p < m.elem0 || p - m.elem0 >= m.len || in_set8(cbset, x);
                if (i > 0) {
                    const uint64_t pp = es ? *reinterpret_cast<const uint32_t *>(spos + 4 * (i - 1))
                                           : load_u32_any(gpos + 4 * (g - 1));
                    bad |= pp >= p;
                }
                if (!bad) {
                    const uint32_t l = (uint32_t)(p - m.elem0);
                    const uint32_t cbyte = ss ? sh.codes[s][l >> 1] : gcodes[(p >> 1)];
                    if (((cbyte >> (4 * (l & 1))) & 0xFu) != 0) bad = true;  // placeholder must be 0
                    const uint32_t smb = ss ? sh.sm[s][l] : gsm[l];
                    if (!bad && m.dst != nullptr)
                        m.dst[l] = (uint16_t)(((smb & 0x80u) << 8) | (x << 7) | (smb & 0x7Fu));
                }
                if (bad) set_status(status, SZ_ERR_CORRUPT);
            }
        }
        if (tid == 0 && (m.flags & kDFlagTileEnd))
            next_tile = next_dealt_tile(m.tile, tiles_per_group(a.batch), gridDim.x);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
    }
}

template <bool kBatched>
__global__ void __launch_bounds__(kPipeThreads, 3) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    DecShared &sh = *reinterpret_cast<DecShared *>(smem_raw);
    const int tid = threadIdx.x;
    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.escs[s], 1);
            mbar_init(&sh.empty[s], kWarps);
        }
        fence_mbar_init();
    }
    seg_cache_fill(sh.segc, a.batch);  // all threads (the caller's table); ends with __syncthreads
    if (tid >= kThreads) {
        if (tid == kThreads) {
            decode_prefetch<kBatched>(a, sh);
            grid_dependency_wait();  // the index kernel before it has finished
            decode_producer<kBatched>(a, sh);
        }
    } else {
        decode_consumers<kBatched>(a, sh);  // waits for the index kernel itself, where it must
    }
}

// ----------------------------------------------------------- small streams
// A short stream decoded by a grid of blocks in one launch, without the
// sub-tile index kernel: block b decodes elements [b*S, (b+1)*S) (S a
// multiple of 16), thread t chunks t, t + 256, ... straight from the
// container, and after one barrier (every placeholder value stored) checks
// and patches the escape records of its slice.  Its records [lo, hi) come
// from two binary searches, the block's end search being the next block's
// start search, so the slices tile [0, e): the last block checks hi = e, a
// block with hi < lo reports it, and every record is checked against its
// predecessor -- the large path's checks, on the same containers.  The
// status word is set to SZ_OK by the caller's memset.
constexpr uint32_t kSmallSlice = 4096;  // elements per block

__device__ __forceinline__ uint64_t lower_pos(const uint8_t *pos, uint64_t e, uint64_t key) {
    uint64_t lo = 0, hi = e;  // first record with position >= key
    while (lo < hi) {
        const uint64_t mid = (lo + hi) >> 1;
        if (load_u32_any(pos + 4 * mid) < key) lo = mid + 1; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kThreads) small_decode_kernel(const uint8_t *c, uint64_t cap, uint16_t *out,
                                                                uint64_t n, uint32_t slice, int32_t *status) {
    __shared__ uint64_t s_range[2];
    const uint32_t tid = threadIdx.x;
    const Header h = read_header(c, cap, n);
    if (!h.ok) {
        if (tid == 0 && blockIdx.x == 0) set_status(status, h.misaligned ? SZ_ERR_ALIGN : SZ_ERR_CORRUPT);
        return;
    }
    const uint64_t first = (uint64_t)blockIdx.x * slice;
    const uint64_t last = umin64(first + slice, n);
    const uint8_t *sm = c + kHeader;
    const uint8_t *codes = c + kHeader + n;
    const uint8_t *pos = c + kHeader + n + (n + 1) / 2;
    const uint8_t *raw = pos + 4 * h.e;
    if (tid < 2) s_range[tid] = (tid == 0) ? lower_pos(pos, h.e, first) : lower_pos(pos, h.e, last);
    const DecTables T = make_tables(h.cb_lo, h.cb_hi);
    for (uint64_t off = first + tid * kChunk; off < last; off += kThreads * kChunk) {
        const uint32_t cnt = (uint32_t)umin64(kChunk, n - off);
        uint4 smv;
        uint64_t cw = 0;
        if (cnt == (uint32_t)kChunk && (n % 8) == 0) {
            smv = *reinterpret_cast<const uint4 *>(sm + off);
            cw = *reinterpret_cast<const unsigned long long *>(codes + off / 2);
        } else {
            uint32_t sw[4] = {0, 0, 0, 0};
#pragma unroll
            for (int j = 0; j < kChunk; ++j)
                if (j < (int)cnt) sw[j >> 2] |= (uint32_t)sm[off + j] << (8 * (j & 3));
            smv = make_uint4(sw[0], sw[1], sw[2], sw[3]);
#pragma unroll
            for (int b = 0; b < kChunk / 2; ++b)
                if (2 * b < (int)cnt) cw |= (uint64_t)codes[off / 2 + b] << (8 * b);
            if ((cnt & 1) && ((cw >> (4 * cnt)) & 0xFu) != 0) set_status(status, SZ_ERR_CORRUPT);  // odd tail
            if (cnt < (uint32_t)kChunk) cw &= (1ull << (4 * cnt)) - 1ull;
        }
        uint4 o0, o1;
        decode_chunk(smv, cw, T, o0, o1);
        if (cnt == (uint32_t)kChunk) {
            st_stream_v4(out + off, o0);
            st_stream_v4(out + off + 8, o1);
        } else {
            const uint32_t w[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
            for (int j = 0; j < kChunk; ++j)
                if (j < (int)cnt) out[off + j] = (uint16_t)(w[j >> 1] >> (16 * (j & 1)));
        }
    }
    __syncthreads();  // the block's values stored; the searches done
    const uint64_t lo = s_range[0], hi = s_range[1];
    if (tid == 0 && (hi < lo || (last == n && hi != h.e))) set_status(status, SZ_ERR_CORRUPT);
    if (hi < lo) return;
    uint32_t cbset[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const uint32_t x = cb_entry(h.cb_lo, h.cb_hi, q);
#pragma unroll
        for (int i = 0; i < 8; ++i) cbset[i] |= ((x >> 5) == (uint32_t)i) ? (1u << (x & 31)) : 0u;
    }
    for (uint64_t i = lo + tid; i < hi; i += kThreads) {
        const uint64_t p = load_u32_any(pos + 4 * i);
        const uint32_t x = raw[i];
        bool bad = p < first || p >= last || in_set8(cbset, x) || (i > 0 && load_u32_any(pos + 4 * (i - 1)) >= p);
        if (!bad && ((codes[p >> 1] >> (4 * (p & 1))) & 0xFu) != 0) bad = true;  // placeholder must be 0
        if (!bad) {
            const uint32_t smb = sm[p];
            out[p] = (uint16_t)(((smb & 0x80u) << 8) | (x << 7) | (smb & 0x7Fu));
        }
        if (bad) set_status(status, SZ_ERR_CORRUPT);
    }
}

cudaError_t launch_small_decode(const uint8_t *c, uint64_t cap, uint16_t *out, uint64_t n, int32_t *status,
                                cudaStream_t s) {
    const uint64_t blocks = umax64(1, div_up(n, kSmallSlice));
    small_decode_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(c, cap, out, n, kSmallSlice, status);
    return cudaGetLastError();
}

// Also writes every segment's status word (no memset before it).  A warp
// per entry while the warps fit about one wave of the GPU, a thread per
// entry beyond.
constexpr uint64_t kWarpIndexMax = 8192;
cudaError_t launch_esc_index(const DecodeArgs &a, bool batched, cudaStream_t s) {
    const uint64_t entries = (uint64_t)a.batch.tile_subs * a.batch.n_tiles + (batched ? a.batch.n_segs : 1u);
    const bool warp = entries <= kWarpIndexMax;
    const dim3 grid((unsigned)div_up(entries, warp ? 256 / 32 : 256)), block(256);
    // The warp build runs where latency rules (a few thousand entries): with
    // the largest shared-memory carveout on its SMs, decode blocks start
    // next to its blocks and copy their first stages while it searches
    // (a 64 MiB stream decodes in 36.9 instead of 38.9 us).  The thread build
    // (long streams) keeps the driver's carveout: there the early decode
    // blocks only compete with the searches.
    cudaError_t e;
    if (batched) {
        if (warp) prefer_max_shared<esc_index_kernel<true, true>>();
        e = warp ? launch_after(esc_index_kernel<true, true>, grid, block, 0, s, a, entries)
                 : launch_after(esc_index_kernel<true, false>, grid, block, 0, s, a, entries);
    } else {
        if (warp) prefer_max_shared<esc_index_kernel<false, true>>();
        e = warp ? launch_after(esc_index_kernel<false, true>, grid, block, 0, s, a, entries)
                 : launch_after(esc_index_kernel<false, false>, grid, block, 0, s, a, entries);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a0, bool batched, int grid, int sms, cudaStream_t s) {
    DecodeArgs a = a0;
    if (a.batch.n_tiles == 0) return cudaSuccess;
    const size_t smem = sizeof(DecShared);
    const uint64_t groups = div_up(a.batch.n_tiles, tiles_per_group(a.batch));
    // A short index kernel (its warp build) holds one SM slot of this kernel
    // per block while it runs.  When the CTAs left beside it take at most
    // 1.5 groups each on average, leaving those slots out lets every CTA
    // start at once and copy its first stages while the index runs (16 MiB
    // stream: 20.5 -> 18.4 us, no CTA starting after the index's end instead
    // of 64; at 20 MiB, 1.76 groups each, it was no better).
    const uint64_t entries = (uint64_t)a.batch.tile_subs * a.batch.n_tiles + (batched ? a.batch.n_segs : 1u);
    if (entries <= kWarpIndexMax) {
        const uint64_t index_blocks = div_up(entries, 256 / 32);
        const uint64_t beside = umax64((uint64_t)sms, (uint64_t)grid > index_blocks ? (uint64_t)grid - index_blocks : 0);
        if (2 * groups <= 3 * beside) grid = (int)umin64((uint64_t)grid, beside);
    }
    // groups of tiles are dealt round robin: CTA b decodes groups b, b + grid, ...
    grid = (int)umax64(1, umin64((uint64_t)grid, groups));
    cudaError_t e;
    if (batched) {
        e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_after(decode_kernel<true>, dim3(grid), dim3(kPipeThreads), smem, s, a);
    } else {
        e = cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_after(decode_kernel<false>, dim3(grid), dim3(kPipeThreads), smem, s, a);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

int decode_blocks_per_sm() {
    const size_t smem = sizeof(DecShared);
    cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<true>, kPipeThreads, smem);
    return occ > 0 ? occ : 1;
}

}  // namespace sz
