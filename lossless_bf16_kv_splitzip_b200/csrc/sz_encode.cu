// sz_encode.cu -- container writer.
//
// SplitZip explainer (gist.science), section 3 "La strategie SplitZip":
// each BF16 value leaves its sign+mantissa byte, its exponent becomes the
// 4-bit code of its codebook slot (two codes per byte), and an exponent
// outside the codebook becomes an escape note (position, raw exponent).
// Section 4: fixed-length codes make this one straight pass -- every output
// byte's address follows from the element index, and the first escape
// index of each CTA's share of tiles is already known from the histogram
// pass's range records, so CTAs are independent.
//
// One persistent CTA per slot, warp-specialised:
//   producer warp   walks the CTA's tiles, 1-D TMA bulk copy of each
//                   16,384-element sub-tile (32 KiB) into a 2-stage
//                   shared-memory ring (3 CTAs per SM), signalled by
//                   mbarriers;
//   8 consumer warps read the stage, write the sm stream (16-byte stores)
//                   and code stream (8-byte stores), scan the escape counts
//                   across the CTA and write the escape records in element
//                   order, then release the stage.
// Every mbarrier wait is bounded (SZ_ERR_DEVICE_TIMEOUT).
#include "sz_internal.cuh"

namespace sz {

constexpr int kEncStages = 2;  // x 32 KiB; 3 CTAs per SM
constexpr uint32_t kEscStage = 512;  // staged escape records per sub-tile; more: written directly

constexpr uint32_t kFlagEnd = 1u;        // no more sub-tiles
constexpr uint32_t kFlagInSmem = 2u;     // data came by TMA into the stage
constexpr uint32_t kFlagLastSub = 4u;    // last sub-tile of its piece (the range's tiles of one segment)
constexpr uint32_t kFlagHeader = 8u;     // first sub-tile of the segment: write the header
// one-pass mode (kFlagLastSub then marks the last sub-tile of a tile)
constexpr uint32_t kFlagPieceEnd = 32u;     // last sub-tile of the piece
constexpr uint32_t kFlagPieceOpens = 64u;   // the piece opens the range
constexpr uint32_t kFlagPieceCloses = 128u; // the piece closes the range

struct EncMeta {
    const uint16_t *src;  // global address of the sub-tile's first element
    uint64_t elem0;       // first element of the sub-tile in the segment stream
    uint64_t piece_end;   // global tile after the piece's last tile
    uint32_t seg;
    uint32_t len;         // elements of the sub-tile
    uint32_t flags;
    uint32_t esc_base;    // first escape index of the piece (one-pass: the global tile)
    uint32_t esc_count;   // escapes the piece must produce (one-pass: unused)
    uint32_t sub_in_tile; // sub-tile index within its tile
    uint32_t piece_tiles; // tiles of the piece
    uint32_t seg_tiles;   // tiles of the segment
};

struct __align__(128) EncShared {
    uint8_t stage[kEncStages][kSub * 2];
    EncMeta meta[kEncStages];
    uint64_t full[kEncStages];
    uint64_t empty[kEncStages];
    SegCache segc;
    uint64_t warp_tot[2][kWarps];  // double-buffered by sub-tile parity
    int go[2];                     // stage j's data arrived (slot j & 1)
    // escape records of a sub-tile, (raw exponent << 16 | offset in the
    // sub-tile), written in element order and copied out coalesced one
    // sub-tile later; double-buffered by sub-tile parity
    uint32_t esc[2][kEscStage];
};

// Four lookup tables, one per position k of an element in its quad of 4:
// entry e = code(e) << 4k for a codebook exponent, 1 << (16 + k) for an
// escape (placeholder code 0).  OR-ing a quad's four entries gives its four
// code nibbles in bits 0..15 and its escape flags in bits 16..19.  Static, so
// that a lookup addresses it as [byte offset + constant].
__shared__ __align__(16) uint32_t s_lut[4][256];

__device__ __forceinline__ uint32_t lut_at(int k, uint32_t byte_off) {
    return *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(s_lut[k]) + byte_off);
}

// ---------------------------------------------------------- chunk encode
// 16 consecutive BF16 values (two uint4) -> 16 sm bytes, 8 code bytes and an
// escape mask.  Escape mask layout: element j = 4q + k of the chunk is bit
// k + 16 (q & 1) + 4 (q >> 1).
__device__ __forceinline__ void encode_chunk(const uint4 v0, const uint4 v1, uint4 &sm, uint64_t &codes,
                                             uint32_t &esc) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t smw[4], B[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t a = w[2 * q], b = w[2 * q + 1];
        const uint32_t hi = prmt(a, b, 0x7531u);  // high bytes of the 4 values: sign | exp >> 1
        const uint32_t lo = prmt(a, b, 0x6420u);  // low bytes: exp & 1 | mantissa
        smw[q] = (hi & 0x80808080u) | (lo & 0x7F7F7F7Fu);
        // byte offset 4 * exponent of each value (exponent in bits 7..14 of its half)
        B[q] = lut_at(0, (a >> 5) & 0x3FCu) | lut_at(1, (a >> 21) & 0x3FCu) | lut_at(2, (b >> 5) & 0x3FCu) |
               lut_at(3, (b >> 21) & 0x3FCu);
    }
    sm = make_uint4(smw[0], smw[1], smw[2], smw[3]);
    codes = (uint64_t)prmt(B[0], B[1], 0x5410u) | ((uint64_t)prmt(B[2], B[3], 0x5410u) << 32);
    esc = prmt(B[0], B[1], 0x7632u) | (prmt(B[2], B[3], 0x7632u) << 4);
}

__device__ __forceinline__ uint32_t byte_of(uint4 v, int b) {  // b is a compile-time constant
    const uint32_t w = (b < 4) ? v.x : (b < 8) ? v.y : (b < 12) ? v.z : v.w;
    return (w >> (8 * (b & 3))) & 0xFFu;
}

// Escape mask in element order (bit j = element j), from the layout above.
__device__ __forceinline__ uint32_t esc_in_element_order(uint32_t m) {
    return (m & 0xFu) | ((m >> 12) & 0xF0u) | ((m << 4) & 0xF00u) | ((m >> 8) & 0xF000u);
}

__device__ __forceinline__ uint32_t esc_bit_of_elem(int j) {
    return 1u << ((j & 3) | (((j >> 2) & 1) << 4) | ((j >> 3) << 2));
}

// Element of the chunk whose escape flag is bit b of the mask.
__device__ __forceinline__ int elem_of_esc_bit(int b) { return (b & 3) | (((b >> 4) & 1) << 2) | (((b >> 2) & 1) << 3); }


__device__ __forceinline__ uint32_t field16(uint64_t v, int c) { return (uint32_t)(v >> (16 * c)) & 0xFFFFu; }

// Read chunk (c, tid) of a stage: 32 bytes at (c*256 + tid)*32 (two 16-byte
// reads; a quarter-warp's reads meet each bank twice, cheaper here than the
// selects that would avoid it).
__device__ __forceinline__ void read_chunk_smem(const uint8_t *stage, int c, int tid, uint4 &v0, uint4 &v1) {
    const uint4 *p = reinterpret_cast<const uint4 *>(stage + (uint32_t)(c * kThreads + tid) * 32u);
    v0 = p[0];
    v1 = p[1];
}

// Chunk from global memory, `cnt` (<= 16) valid elements, the rest zero.
__device__ __forceinline__ void read_chunk_global(const uint16_t *p, uint32_t cnt, uint4 &v0, uint4 &v1) {
    uint32_t wv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t lo = (2 * q < (int)cnt) ? (uint32_t)p[2 * q] : 0u;
        const uint32_t hi = (2 * q + 1 < (int)cnt) ? (uint32_t)p[2 * q + 1] : 0u;
        wv[q] = lo | (hi << 16);
    }
    v0 = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    v1 = make_uint4(wv[4], wv[5], wv[6], wv[7]);
}

// ------------------------------------------------------------ producer
// Before the grid dependency wait: the bulk copies of the CTA's first
// kEncStages sub-tiles, which need only the caller's input and the batch
// geometry, not what the kernel before this one writes (codebooks, escape
// counts) -- the copies then overlap that kernel's end.  Stops at the first
// sub-tile that is short or misaligned.  Returns how many leading sub-tiles
// were issued: their stages have the transaction count set, and the
// producer arrives on them once their descriptions are written.  The input
// is complete here: the kernel before this one in the stream started only
// after the input's writers finished (it is a plain launch or a memset).
template <bool kBatched>
__device__ uint32_t encode_prefetch(const EncodeArgs &a, EncShared &sh) {
    if ((a.debug_flags & kDebugNoSignal) != 0) return 0;
    const uint64_t t_begin = (uint64_t)blockIdx.x * a.range_tiles;
    const uint64_t t_end = umin64(t_begin + a.range_tiles, a.batch.n_tiles);
    uint32_t j = 0;
    for (uint64_t t = t_begin; t < t_end && j < (uint32_t)kEncStages; ++t) {
        const uint32_t k = find_segment(sh.segc, a.batch, t);
        const sz_segment seg = load_segment(a.batch, k);
        const TileRef r = resolve_tile(a.batch, seg, k, t);
        const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        if ((reinterpret_cast<uintptr_t>(src) & 15) != 0) return j;
        for (uint32_t sub = 0; sub < r.n_subs && j < (uint32_t)kEncStages; ++sub, ++j) {
            if (r.len - sub * kSub < kSub) return j;
            mbar_expect_tx(&sh.full[j], kSub * 2);
            tma_load_1d(sh.stage[j], src + sub * kSub, kSub * 2, &sh.full[j]);
        }
    }
    return j;
}

template <bool kBatched, bool kOnePass>
__device__ void encode_producer(const EncodeArgs &a, EncShared &sh, uint32_t n_early) {
    if ((a.debug_flags & kDebugNoSignal) != 0) return;  // test hook: nothing is ever signalled
    const uint64_t t_begin = (uint64_t)blockIdx.x * a.range_tiles;
    const uint64_t t_end = umin64(t_begin + a.range_tiles, a.batch.n_tiles);
    RangeRec rr{};
    if (t_begin < t_end) rr = a.rrec[blockIdx.x];
    uint32_t j = 0;
    uint32_t cur = 0xFFFFFFFFu;
    sz_segment seg{};
    bool seg_ok = false;
    uint64_t e_total = 0;
    uint32_t p_base = 0, p_count = 0;  // the piece's first escape index and escape count
    uint64_t p_first = 0, p_last = 0;  // the piece's first and last tile
    uint64_t seg_end = 0;              // tile after the segment's last tile
    for (uint64_t t = t_begin; t < t_end; ++t) {
        const uint32_t k = find_segment(sh.segc, a.batch, t);
        if (k != cur) {  // a new piece: the range's tiles of segment k
            cur = k;
            seg = load_segment(a.batch, k);
            bool valid;
            if (kOnePass) {  // the caller's codebook; the container size is known only later
                valid = codebook16_distinct(a.codebooks_in + 16 * (size_t)k);
                e_total = 0;
            } else {
                valid = a.meta[k].valid != 0;
                e_total = a.meta[k].n_escapes;
            }
            const bool fits = seg.out_offset <= a.out_cap &&
                              container_size(seg.n_elems, e_total) <= a.out_cap - seg.out_offset;
            const bool aligned = (reinterpret_cast<uintptr_t>(a.out + seg.out_offset) & 15) == 0;
            seg_ok = valid && fits && aligned;
            if (!valid) set_status(a.status + k, SZ_ERR_INVALID);
            else if (!fits) set_status(a.status + k, SZ_ERR_CAPACITY);
            else if (!aligned) set_status(a.status + k, SZ_ERR_ALIGN);
            seg_end = seg.tile_begin + seg_tiles(a.batch, seg.n_elems);
            p_first = t;
            p_last = umin64(seg_end, t_end) - 1;
            if (t == t_begin) {  // opens the range
                p_base = rr.first_off;
                p_count = rr.first_cnt;
            } else if (seg_end > t_end) {  // closes the range, the segment goes on
                p_base = 0;
                p_count = rr.last_cnt;
            } else {  // the whole segment
                p_base = 0;
                p_count = (uint32_t)e_total;
            }
        }
        const TileRef r = resolve_tile(a.batch, seg, k, t);
        if (!seg_ok) {  // every tile of the segment is skipped
            // sub-tiles of it copied before the wait go out as empty ones
            for (uint32_t sub = 0; sub < r.n_subs && j < n_early; ++sub, ++j) {
                EncMeta &m = sh.meta[j % kEncStages];
                m = EncMeta{};
                m.seg = k;
                mbar_arrive(&sh.full[j % kEncStages]);
            }
            continue;
        }
        const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        const bool aligned = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
        if (!aligned) set_status(a.status + k, SZ_ERR_ALIGN);
        for (uint32_t sub = 0; sub < r.n_subs; ++sub, ++j) {
            const int s = (int)(j % kEncStages);
            if (j >= (uint32_t)kEncStages && !mbar_wait(&sh.empty[s], ((j / kEncStages) - 1) & 1u, a.wait_limit_ns)) {
                set_status(a.status + k, SZ_ERR_DEVICE_TIMEOUT);
                return;
            }
            EncMeta &m = sh.meta[s];
            m.src = src + sub * kSub;
            m.elem0 = r.elem0 + (uint64_t)sub * kSub;
            m.seg = k;
            m.len = aligned ? umin32(kSub, r.len - sub * kSub) : 0u;  // nothing is read from a misaligned page
            m.sub_in_tile = sub;
            m.piece_end = p_last + 1;
            m.piece_tiles = (uint32_t)(p_last + 1 - p_first);
            m.seg_tiles = (uint32_t)(seg_end - seg.tile_begin);
            uint32_t f = 0;
            if (kOnePass) {
                m.esc_base = (uint32_t)t;
                m.esc_count = 0;
                if (sub + 1 == r.n_subs) f |= kFlagLastSub;
                if (t == p_last && sub + 1 == r.n_subs) {
                    f |= kFlagPieceEnd;
                    if (p_first == t_begin) f |= kFlagPieceOpens;
                    if (p_last + 1 == t_end) f |= kFlagPieceCloses;
                }
            } else {
                m.esc_base = p_base;
                m.esc_count = p_count;
                if (t == p_last && sub + 1 == r.n_subs) f |= kFlagLastSub;
                if (r.local == 0 && sub == 0) f |= kFlagHeader;
            }
            const bool tma = m.len == kSub;
            if (tma) f |= kFlagInSmem;
            m.flags = f;
            if (j < n_early) {  // copied before the wait (same source, a full sub-tile)
                mbar_arrive(&sh.full[s]);
            } else if (tma) {
                mbar_arrive_expect_tx(&sh.full[s], kSub * 2);
                tma_load_1d(sh.stage[s], m.src, kSub * 2, &sh.full[s]);
            } else {
                mbar_arrive(&sh.full[s]);
            }
        }
    }
    const int s = (int)(j % kEncStages);
    if (j >= (uint32_t)kEncStages && !mbar_wait(&sh.empty[s], ((j / kEncStages) - 1) & 1u, a.wait_limit_ns)) return;
    sh.meta[s].flags = kFlagEnd;
    mbar_arrive(&sh.full[s]);
}

// ------------------------------------------------------------ consumers
// A sub-tile's staged escape records waiting to be copied out.
struct PendingEsc {
    uint32_t cnt;           // records staged (0: none)
    uint64_t first;         // segment index of the first record
    uint64_t lim;           // records may not reach this index
    uint64_t elem0;         // first element of the sub-tile
    uint8_t *pos_base;
    uint8_t *raw_base;
    bool pos_aligned;
    int32_t *status;
    uint32_t *slot;         // one-pass: the tile's record slot
    uint32_t tile_off;      // one-pass: offset of the sub-tile in its tile
};

// Every consumer thread takes records tid, tid + 256, ...: consecutive
// threads write consecutive positions and exponents (one-pass: consecutive
// slot entries, the first slot_cap records of the tile; lim = slot_cap).
template <bool kOnePass>
__device__ __forceinline__ void copy_out_escapes(const uint32_t *stg, const PendingEsc &p, int tid) {
    if constexpr (kOnePass) {
        for (uint32_t i = tid; i < p.cnt; i += kThreads) {
            const uint64_t g = p.first + i;
            if (g >= p.lim) break;
            const uint32_t rec = stg[i];
            p.slot[g] = (rec & 0xFF0000u) | (p.tile_off + (rec & 0xFFFFu));
        }
    } else {
        for (uint32_t i = tid; i < p.cnt; i += kThreads) {
            const uint64_t g = p.first + i;
            if (g >= p.lim) {  // more escapes than the histograms said
                set_status(p.status, SZ_ERR_CORRUPT);
                break;
            }
            const uint32_t rec = stg[i];
            store_u32_le(p.pos_base + 4 * g, (uint32_t)(p.elem0 + (rec & 0xFFFFu)), p.pos_aligned);
            p.raw_base[g] = (uint8_t)(rec >> 16);
        }
    }
}

// Escape counts of the thread's 4 chunks -> (exclusive prefix within the
// warp, warp total), both packed as four 16-bit fields.  When no chunk holds
// more than one escape -- the usual case -- ballots do it; otherwise a
// shuffle scan of the packed counts.
__device__ __forceinline__ bool warp_escape_scan(const uint32_t (&esc)[kChunks], int lane, uint64_t &excl,
                                                 uint64_t &total) {
    uint32_t cnt[kChunks];
    uint32_t any_multi = 0;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
        cnt[c] = __popc(esc[c]);
        any_multi |= cnt[c] > 1u;
    }
    excl = 0;
    total = 0;
    if (!__any_sync(0xFFFFFFFFu, any_multi)) {
        const uint32_t below = (1u << lane) - 1u;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            const uint32_t b = __ballot_sync(0xFFFFFFFFu, cnt[c] != 0);
            excl |= (uint64_t)__popc(b & below) << (16 * c);
            total |= (uint64_t)__popc(b) << (16 * c);
        }
        return false;
    }
    uint64_t v = 0;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) v |= (uint64_t)cnt[c] << (16 * c);
    uint64_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint64_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    excl = incl - v;
    total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    return true;  // some chunk of the warp has several escapes
}

// A stage wait ran out.  The pieces of this CTA's range before tile `from`
// are complete: their records are written and they were counted.  Every
// segment with a piece at or after `from` gets SZ_ERR_DEVICE_TIMEOUT, and
// none of them is counted here, so their sizes are never written.
__device__ void timeout_from(const EncodeArgs &a, const SegCache &c, uint64_t from, uint64_t t_end) {
    for (uint64_t t = from; t < t_end;) {
        const uint32_t k = find_segment(c, a.batch, t);  // the segment that holds tile t
        set_status(a.status + k, SZ_ERR_DEVICE_TIMEOUT);
        const sz_segment sk = load_segment(a.batch, k);
        t = sk.tile_begin + seg_tiles(a.batch, sk.n_elems);
    }
}

template <bool kBatched, bool kOnePass>
__device__ void encode_consumers(const EncodeArgs &a, EncShared &sh) {
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    uint32_t cur = 0xFFFFFFFFu;
    uint8_t *out = nullptr;
    uint64_t n = 0, e_total = 0;
    bool codes_aligned = false, pos_aligned = false;
    uint32_t running = 0;  // escapes of the current piece so far (one-pass: of the tile)
    uint32_t piece_acc = 0;  // one-pass: escapes of the current piece so far
    PendingEsc pend{};
    const uint64_t t_begin = umin64((uint64_t)blockIdx.x * a.range_tiles, a.batch.n_tiles);
    const uint64_t t_end = umin64(t_begin + a.range_tiles, a.batch.n_tiles);
    uint64_t counted_end = t_begin;  // thread 0: the pieces before this tile are complete

    // The wait for stage j+1 is folded into sub-tile j's scan barrier: one
    // consumer barrier per sub-tile.
    if (tid == 0) sh.go[0] = mbar_wait(&sh.full[0], 0u, a.wait_limit_ns) ? 1 : 0;
    consumer_sync();
    for (uint32_t j = 0;; ++j) {
        const int s = (int)(j % kEncStages);
        if (!sh.go[j & 1]) {  // the same decision in every consumer thread
            if (tid == 0) timeout_from(a, sh.segc, counted_end, t_end);
            return;
        }
        const EncMeta m = sh.meta[s];
        if (m.flags & kFlagEnd) {
            consumer_sync();  // the last sub-tile's staged records are complete
            copy_out_escapes<kOnePass>(sh.esc[(j + 1) & 1], pend, tid);
            return;
        }
        if (m.seg != cur) {  // every consumer is past the previous sub-tile's compute
#pragma unroll
            for (int k = 0; k < 4; ++k) s_lut[k][tid] = 1u << (16 + k);
            consumer_sync();
            const uint8_t *cbk = kOnePass ? a.codebooks_in + 16 * (size_t)m.seg : a.meta[m.seg].codebook;
            if (tid < 16) {
                const uint32_t x = cbk[tid];
#pragma unroll
                for (int k = 0; k < 4; ++k) s_lut[k][x] = (uint32_t)tid << (4 * k);
            }
            const sz_segment seg = load_segment(a.batch, m.seg);
            out = a.out + seg.out_offset;
            n = seg.n_elems;
            e_total = kOnePass ? 0 : a.meta[m.seg].n_escapes;
            codes_aligned = (n % 8) == 0;
            pos_aligned = ((kHeader + n + (n + 1) / 2) & 3) == 0;
            cur = m.seg;
            consumer_sync();
        }
        int32_t *status = a.status + m.seg;
        if ((m.flags & kFlagHeader) && tid < 6) {
            uint64_t v = 0;
            if (tid == 0) v = 0x00000101564B5A53ull;  // "SZKV", version 1, dtype 1, flags 0
            if (tid == 1) v = n;
            if (tid == 2) v = e_total;
            if (tid == 3 || tid == 4) {
                const uint8_t *cb = a.meta[m.seg].codebook + 8 * (tid - 3);
                for (int i = 7; i >= 0; --i) v = (v << 8) | cb[i];
            }
            reinterpret_cast<uint64_t *>(out)[tid] = v;
        }
        uint8_t *out_sm = out + kHeader + m.elem0;
        uint8_t *codes_base = out + kHeader + n;  // element i's nibble is in byte i/2
        const uint8_t *stage = sh.stage[s];
        const bool in_smem = (m.flags & kFlagInSmem) != 0;

        uint32_t esc[kChunks];
        if (in_smem && codes_aligned) {  // a full sub-tile in shared memory
            uint8_t *psm = out_sm + tid * kChunk;
            uint8_t *pcw = codes_base + (m.elem0 + tid * kChunk) / 2;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint4 v0, v1, smv;
                uint64_t cw;
                read_chunk_smem(stage, c, tid, v0, v1);
                encode_chunk(v0, v1, smv, cw, esc[c]);
                st_stream_v4(psm + c * kThreads * kChunk, smv);
                st_stream_u64(pcw + c * kThreads * kChunk / 2, cw);
            }
        } else {
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            const uint32_t off = (c * kThreads + tid) * kChunk;
            esc[c] = 0;
            if (off >= m.len) continue;
            uint4 v0, v1, smv;
            uint64_t cw;
            // ragged or unaligned chunk: guarded element loads, encoded as a
            // full chunk, cnt of it kept
            const uint32_t cnt = umin32(kChunk, m.len - off);
            read_chunk_global(m.src + off, cnt, v0, v1);
            uint32_t e;
            encode_chunk(v0, v1, smv, cw, e);
            uint32_t keep = 0;
#pragma unroll
            for (int q = 0; q < kChunk; ++q)
                if (q < (int)cnt) keep |= esc_bit_of_elem(q);
            esc[c] = e & keep;
            if (cnt < (uint32_t)kChunk) cw &= (1ull << (4 * cnt)) - 1ull;  // odd tail nibble = 0
            if (cnt == (uint32_t)kChunk && codes_aligned) {
                st_stream_v4(out_sm + off, smv);
                st_stream_u64(codes_base + (m.elem0 + off) / 2, cw);
            } else {
#pragma unroll
                for (int q = 0; q < kChunk; ++q)
                    if (q < (int)cnt) out_sm[off + q] = (uint8_t)byte_of(smv, q);
                uint8_t *cb = codes_base + (m.elem0 + off) / 2;
#pragma unroll
                for (int b = 0; b < kChunk / 2; ++b)
                    if (2 * b < (int)cnt) cb[b] = (uint8_t)(cw >> (8 * b));
            }
        }
        }

        // ---- escapes: position of every escape in the sub-tile's order
        uint64_t wexcl, wtot;
        const bool multi = warp_escape_scan(esc, lane, wexcl, wtot);
        uint64_t *wt = sh.warp_tot[j & 1];
        if (lane == 0) wt[wid] = wtot;
        const int s_next = (int)((j + 1) % kEncStages);
        if (tid == 0) sh.go[(j + 1) & 1] = mbar_wait(&sh.full[s_next], ((j + 1) / kEncStages) & 1u, a.wait_limit_ns) ? 1 : 0;
        consumer_sync();
        // warp totals -> this warp's exclusive prefix and the sub-tile total
        // (packed fields): an 8-lane shuffle scan instead of 8 sums per thread
        uint64_t wv = lane < kWarps ? wt[lane] : 0ull;
        uint64_t wi = wv;
#pragma unroll
        for (int d = 1; d < kWarps; d <<= 1) {
            const uint64_t y = __shfl_up_sync(0xFFFFFFFFu, wi, d);
            if (lane >= d) wi += y;
        }
        const uint64_t tot = __shfl_sync(0xFFFFFFFFu, wi, kWarps - 1);
        const uint64_t warp_excl = __shfl_sync(0xFFFFFFFFu, wi - wv, wid);
        const uint64_t thr_excl = warp_excl + wexcl;
        const uint32_t sub_total = field16(tot, 0) + field16(tot, 1) + field16(tot, 2) + field16(tot, 3);

        // ---- the previous sub-tile's staged records, coalesced
        copy_out_escapes<kOnePass>(sh.esc[(j + 1) & 1], pend, tid);
        pend.cnt = 0;

        // ---- this sub-tile's records, in element order
        if (sub_total) {
            const uint64_t pos_off = kHeader + n + (n + 1) / 2;
            uint8_t *pos_base = out + pos_off;
            uint8_t *raw_base = pos_base + 4 * e_total;
            // the records this sub-tile may write: [first, last) of the segment
            // (one-pass: of the tile's slot)
            const uint64_t first = kOnePass ? (uint64_t)running : (uint64_t)m.esc_base + running;
            const uint32_t cap = slot_cap(a.batch);
            const uint64_t lim = kOnePass ? (uint64_t)cap : umin64(e_total, (uint64_t)m.esc_base + m.esc_count);
            uint32_t *slot = kOnePass ? a.slots + (size_t)m.esc_base * cap : nullptr;
            const uint32_t tile_off = m.sub_in_tile * kSub;
            const bool staged = sub_total <= kEscStage;
            uint32_t *stg = sh.esc[j & 1];
            uint32_t chunk_base = 0;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint32_t idx = chunk_base + field16(thr_excl, c);  // index within the sub-tile
                chunk_base += field16(tot, c);
                if (!esc[c]) continue;
                const uint32_t off = (c * kThreads + tid) * kChunk;
                // the usual case, one escape in the chunk: no ordering loop
                uint32_t msk = multi ? esc_in_element_order(esc[c]) : 0u;
                int q = 0;
                if (!multi) {
                    q = elem_of_esc_bit(__ffs(esc[c]) - 1);
                } else {
                    q = __ffs(msk) - 1;
                    msk &= msk - 1;
                }
                for (;;) {  // ascending element order
                    const uint32_t x = in_smem ? (uint32_t)reinterpret_cast<const uint16_t *>(stage)[off + q]
                                               : (uint32_t)m.src[off + q];
                    const uint32_t raw = (x >> 7) & 0xFFu;
                    if (staged) {
                        stg[idx] = (raw << 16) | (off + q);
                    } else if (kOnePass) {
                        const uint64_t g = first + idx;
                        if (g < lim) slot[g] = (raw << 16) | (tile_off + off + q);
                    } else {
                        const uint64_t g = first + idx;
                        if (g >= lim) {  // more escapes than the histograms said
                            set_status(status, SZ_ERR_CORRUPT);
                            break;
                        }
                        store_u32_le(pos_base + 4 * g, (uint32_t)(m.elem0 + off + q), pos_aligned);
                        raw_base[g] = (uint8_t)raw;
                    }
                    ++idx;
                    if (!msk) break;
                    q = __ffs(msk) - 1;
                    msk &= msk - 1;
                }
            }
            if (staged) {
                pend.cnt = sub_total;
                pend.first = first;
                pend.lim = lim;
                pend.elem0 = m.elem0;
                pend.pos_base = pos_base;
                pend.raw_base = raw_base;
                pend.pos_aligned = pos_aligned;
                pend.status = status;
                pend.slot = slot;
                pend.tile_off = tile_off;
            }
        }
        running += sub_total;
        if (kOnePass && (m.flags & kFlagLastSub)) {  // end of a tile: its count, and the piece's
            piece_acc += running;
            if (tid == 0) {
                a.tile_cnt[m.esc_base] = running;
                if (m.flags & kFlagPieceEnd) {
                    if (m.flags & kFlagPieceOpens) a.rcnt[blockIdx.x].first_cnt = piece_acc;
                    else if (m.flags & kFlagPieceCloses) a.rcnt[blockIdx.x].last_cnt = piece_acc;
                }
            }
            if (m.flags & kFlagPieceEnd) piece_acc = 0;
            running = 0;
        }
        if (m.flags & (kOnePass ? kFlagPieceEnd : kFlagLastSub)) {
            // End of a piece.  Its last records go out now instead of one
            // sub-tile later, so that once the barrier below is passed every
            // record of the piece is written.  Two-pass: the piece's escape
            // count is checked, then its tiles are added to the segment's
            // completion count; the piece that completes it writes the size,
            // if no piece of the segment reported an error -- a segment with
            // an error keeps size 0.
            consumer_sync();
            copy_out_escapes<kOnePass>(sh.esc[j & 1], pend, tid);
            pend.cnt = 0;
            consumer_sync();
            if (tid == 0) {
                if (!kOnePass) {
                    if (running != m.esc_count) set_status(status, SZ_ERR_CORRUPT);
                    __threadfence();
                    if (atomicAdd(a.enc_done + m.seg, m.piece_tiles) + m.piece_tiles == m.seg_tiles) {
                        __threadfence();  // every piece's status is visible
                        if (*reinterpret_cast<volatile const int32_t *>(status) == SZ_OK)
                            a.out_bytes[m.seg] = container_size(n, e_total);
                    }
                }
                counted_end = m.piece_end;
            }
            if (!kOnePass) running = 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[s]);
    }
}

template <bool kBatched, bool kOnePass>
__global__ void __launch_bounds__(kPipeThreads, 3) encode_kernel(const EncodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    EncShared &sh = *reinterpret_cast<EncShared *>(smem_raw);
    const int tid = threadIdx.x;
    allow_dependents();  // the escape placement (one-pass) may start its prologue
    if (tid == 0) {
        for (int s = 0; s < kEncStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kWarps);
        }
        fence_mbar_init();
    }
    seg_cache_fill(sh.segc, a.batch);  // all threads (the caller's table); ends with __syncthreads
    uint32_t n_early = 0;
    if (tid == kThreads) n_early = encode_prefetch<kBatched>(a, sh);
    grid_dependency_wait();  // the kernel before it (histogram, select) has finished

    // Segments with no elements have no tiles: CTA 0 writes their header
    // (one-pass: the escape placement does).
    if (!kOnePass && blockIdx.x == 0 && tid < kThreads) {
        const uint32_t ns = kBatched ? a.batch.n_segs : 1;
        for (uint32_t k = tid; k < ns; k += kThreads) {
            const sz_segment s = load_segment(a.batch, k);
            if (s.n_elems != 0) continue;
            if (a.meta[k].valid == 0) { set_status(a.status + k, SZ_ERR_INVALID); continue; }
            if (s.out_offset + kHeader > a.out_cap) { set_status(a.status + k, SZ_ERR_CAPACITY); continue; }
            if ((reinterpret_cast<uintptr_t>(a.out + s.out_offset) & 15) != 0) {
                set_status(a.status + k, SZ_ERR_ALIGN);
                continue;
            }
            uint64_t *h = reinterpret_cast<uint64_t *>(a.out + s.out_offset);
            const uint8_t *cb = a.meta[k].codebook;
            uint64_t c0 = 0, c1 = 0;
            for (int i = 7; i >= 0; --i) { c0 = (c0 << 8) | cb[i]; c1 = (c1 << 8) | cb[8 + i]; }
            h[0] = 0x00000101564B5A53ull;  // "SZKV", version 1, dtype 1, flags 0
            h[1] = 0;
            h[2] = 0;
            h[3] = c0;
            h[4] = c1;
            h[5] = 0;
            a.out_bytes[k] = kHeader;
        }
    }

    if (tid >= kThreads) {
        if (tid == kThreads) encode_producer<kBatched, kOnePass>(a, sh, n_early);
    } else {
        encode_consumers<kBatched, kOnePass>(a, sh);
    }
}

// ----------------------------------------------------------- small streams
constexpr uint32_t kTinyColWords = 256 * 32;  // exponent counts: 256 bins x 32 lane columns

// A short stream over a grid of blocks, each one 4,096-element slice (one
// chunk per thread), in two launches after one memset: the counting kernel
// keeps every slice's 256 exponent counts and adds them to the stream's;
// the block that completes the count (one atomic completion count, no
// wait) selects the top 16 and turns the slices' counts into each slice's
// first escape index.  The encode kernel then writes every slice's bytes
// and records in place; its last block to finish writes the size if no
// block reported an error.  status and size are reset by the first kernel.
constexpr uint32_t kSlice = kThreads * kChunk;  // 4,096 elements per block

__global__ void __launch_bounds__(kThreads) small_hist_kernel(const uint16_t *in, uint64_t n, SmallWs w,
                                                              uint8_t *codebook_out, int32_t *status,
                                                              uint64_t *out_bytes) {
    extern __shared__ __align__(16) uint32_t s_col[];  // kTinyColWords
    __shared__ RankShared s_rank;
    __shared__ uint32_t s_warp[kWarps];
    __shared__ uint32_t s_carry;
    __shared__ uint8_t s_cb[16];
    __shared__ unsigned long long s_top;
    __shared__ int s_last;
    const uint32_t tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const uint32_t nb = (uint32_t)umax64(1, div_up(n, kSlice));  // an empty stream: one block
    for (uint32_t i = tid; i < kTinyColWords; i += kThreads) s_col[i] = 0;
    if (tid == 0) {
        if (blockIdx.x == 0) {
            *status = SZ_OK;
            *out_bytes = 0;
        }
        s_top = 0;
        s_carry = 0;
    }
    __syncthreads();
    const uint64_t off = (uint64_t)blockIdx.x * kSlice + tid * kChunk;
    const uint32_t col = smem_u32(s_col) + lane * 4;
    if (off < n) {
        const uint32_t cnt = (uint32_t)umin64(kChunk, n - off);
        if (cnt == (uint32_t)kChunk) {
            const uint4 v0 = ld_stream_v4(in + off), v1 = ld_stream_v4(in + off + 8);
            const uint32_t x[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {  // (half & 0x7F80) = exponent * 128 = the byte offset of its row
                asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(col + (x[q] & 0x7F80u)) : "memory");
                asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(col + ((x[q] >> 16) & 0x7F80u)) : "memory");
            }
        } else {
            for (uint32_t j = 0; j < cnt; ++j)
                asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(col + ((uint32_t)in[off + j] & 0x7F80u)) : "memory");
        }
    }
    __syncthreads();
    uint32_t c = 0;
#pragma unroll 8
    for (uint32_t i = 0; i < 32; ++i) c += s_col[tid * 32 + ((i + tid) & 31)];
    w.block_hist[(size_t)blockIdx.x * 256 + tid] = c;
    if (c) atomicAdd(&w.seg_hist[tid], c);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(w.done, 1u) + 1 == nb;
    __syncthreads();
    if (!s_last) return;
    // ---- the last block: select, escape count, first escape index per slice
    __threadfence();
    c = __ldcg(w.seg_hist + tid);
    const uint32_t rank = exponent_rank(c, tid, s_rank);
    if (rank < 16) {
        s_cb[rank] = (uint8_t)tid;
        atomicAdd(&s_top, (unsigned long long)c);
    }
    __syncthreads();
    if (tid < 16) {
        w.meta->codebook[tid] = s_cb[tid];
        if (codebook_out) codebook_out[tid] = s_cb[tid];
    }
    if (tid == 0) {
        w.meta->n_escapes = n - s_top;
        w.meta->valid = 1;
        w.meta->pad = 0;
    }
    uint32_t cbq[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) cbq[q] = s_cb[q];
    for (uint32_t base = 0; base < nb; base += kThreads) {
        const uint32_t b = base + tid;
        uint32_t esc = 0;
        if (b < nb) {
            uint32_t in_cb = 0;
#pragma unroll
            for (int q = 0; q < 16; ++q) in_cb += __ldcg(w.block_hist + (size_t)b * 256 + cbq[q]);
            esc = (uint32_t)umin64(kSlice, n - (uint64_t)b * kSlice) - in_cb;
        }
        uint32_t incl = esc;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= (uint32_t)d) incl += y;
        }
        if (lane == 31) s_warp[wid] = incl;
        __syncthreads();
        uint32_t before = 0, total = 0;
#pragma unroll
        for (int q = 0; q < kWarps; ++q) {
            const uint32_t x = s_warp[q];
            before += ((uint32_t)q < wid) ? x : 0u;
            total += x;
        }
        const uint32_t carry = s_carry;
        if (b < nb) w.block_off[b] = carry + before + incl - esc;
        __syncthreads();
        if (tid == 0) s_carry = carry + total;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads) small_encode_kernel(const uint16_t *in, uint64_t n, SmallWs w,
                                                                uint8_t *out, uint64_t out_cap,
                                                                uint64_t *out_bytes, int32_t *status) {
    __shared__ uint32_t s_warp[kWarps];
    __shared__ int s_last;
    const uint32_t tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const uint32_t nb = (uint32_t)umax64(1, div_up(n, kSlice));  // an empty stream: one block
#pragma unroll
    for (int k = 0; k < 4; ++k) s_lut[k][tid] = 1u << (16 + k);
    __syncthreads();
    if (tid < 16) {
        const uint32_t x = w.meta->codebook[tid];
#pragma unroll
        for (int k = 0; k < 4; ++k) s_lut[k][x] = (uint32_t)tid << (4 * k);
    }
    const uint64_t e_total = w.meta->n_escapes;
    if (container_size(n, e_total) > out_cap) {  // the same decision in every block
        if (tid == 0 && blockIdx.x == 0) set_status(status, SZ_ERR_CAPACITY);
        return;
    }
    if (blockIdx.x == 0 && tid < 6) {
        uint64_t v = 0;
        if (tid == 0) v = 0x00000101564B5A53ull;  // "SZKV", version 1, dtype 1, flags 0
        if (tid == 1) v = n;
        if (tid == 2) v = e_total;
        if (tid == 3 || tid == 4)
            for (int i = 7; i >= 0; --i) v = (v << 8) | w.meta->codebook[8 * (tid - 3) + i];
        reinterpret_cast<uint64_t *>(out)[tid] = v;
    }
    __syncthreads();  // the LUT is complete
    const uint64_t pos_off = kHeader + n + (n + 1) / 2;
    const bool pos_aligned = (pos_off & 3) == 0;
    uint8_t *codes = out + kHeader + n;
    uint8_t *pos = out + pos_off;
    uint8_t *raw = pos + 4 * e_total;
    const uint64_t off = (uint64_t)blockIdx.x * kSlice + tid * kChunk;
    uint32_t esc = 0;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (off < n) {
        const uint32_t cnt = (uint32_t)umin64(kChunk, n - off);
        if (cnt == (uint32_t)kChunk) {
            v0 = ld_stream_v4(in + off);
            v1 = ld_stream_v4(in + off + 8);
        } else {
            read_chunk_global(in + off, cnt, v0, v1);
        }
        uint4 smv;
        uint64_t cw;
        uint32_t m;
        encode_chunk(v0, v1, smv, cw, m);
        uint32_t keep = 0;
#pragma unroll
        for (int q = 0; q < kChunk; ++q)
            if (q < (int)cnt) keep |= esc_bit_of_elem(q);
        esc = esc_in_element_order(m & keep);
        if (cnt < (uint32_t)kChunk) cw &= (1ull << (4 * cnt)) - 1ull;  // odd tail nibble = 0
        if (cnt == (uint32_t)kChunk) {
            st_stream_v4(out + kHeader + off, smv);
        } else {
#pragma unroll
            for (int q = 0; q < kChunk; ++q)
                if (q < (int)cnt) out[kHeader + off + q] = (uint8_t)byte_of(smv, q);
        }
        if (cnt == (uint32_t)kChunk && (n % 8) == 0) {
            st_stream_u64(codes + off / 2, cw);
        } else {
#pragma unroll
            for (int b = 0; b < kChunk / 2; ++b)
                if (2 * b < (int)cnt) codes[off / 2 + b] = (uint8_t)(cw >> (8 * b));
        }
    }
    const uint32_t k = __popc(esc);
    uint32_t incl = k;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= (uint32_t)d) incl += y;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
        const uint32_t x = s_warp[q];
        before += ((uint32_t)q < wid) ? x : 0u;
        total += x;
    }
    const uint64_t b0 = w.block_off[blockIdx.x];
    const uint64_t b1 = blockIdx.x + 1 < nb ? (uint64_t)w.block_off[blockIdx.x + 1] : e_total;
    uint64_t g = b0 + before + incl - k;
    while (esc) {
        const int q = __ffs(esc) - 1;
        esc &= esc - 1;
        const uint32_t x = (q < 8) ? ((q < 4) ? (q < 2 ? v0.x : v0.y) : (q < 6 ? v0.z : v0.w))
                                   : ((q < 12) ? (q < 10 ? v1.x : v1.y) : (q < 14 ? v1.z : v1.w));
        if (g < b1) {  // never past the slice's share
            store_u32_le(pos + 4 * g, (uint32_t)(off + q), pos_aligned);
            raw[g] = (uint8_t)((x >> (16 * (q & 1) + 7)) & 0xFFu);
        }
        ++g;
    }
    if (tid == 0 && b0 + total != b1) set_status(status, SZ_ERR_CORRUPT);  // the input changed
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(w.done2, 1u) + 1 == nb;
    __syncthreads();
    if (s_last && tid == 0) {
        __threadfence();
        if (*reinterpret_cast<volatile int32_t *>(status) == SZ_OK) *out_bytes = container_size(n, e_total);
    }
}

cudaError_t launch_small_encode(const uint16_t *in, uint64_t n, const SmallWs &w, uint8_t *out, uint64_t out_cap,
                                uint64_t *out_bytes, uint8_t *codebook_out, int32_t *status, cudaStream_t s) {
    const uint32_t nb = (uint32_t)umax64(1, div_up(n, kSlice));
    small_hist_kernel<<<nb, kThreads, kTinyColWords * sizeof(uint32_t), s>>>(in, n, w, codebook_out, status,
                                                                            out_bytes);
    small_encode_kernel<<<nb, kThreads, 0, s>>>(in, n, w, out, out_cap, out_bytes, status);
    return cudaGetLastError();
}


// One CTA per range of the partition the histogram kernel used (one-pass:
// of the partition the escape placement will use).
template <bool kBatched, bool kOnePass>
cudaError_t launch_encode_t(const EncodeArgs &a, cudaStream_t s) {
    const size_t smem = sizeof(EncShared);
    const int grid = (int)umax64(1, div_up(a.batch.n_tiles, a.range_tiles));
    cudaError_t e =
        cudaFuncSetAttribute(encode_kernel<kBatched, kOnePass>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_after(encode_kernel<kBatched, kOnePass>, dim3(grid), dim3(kPipeThreads), smem, s, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_encode(const EncodeArgs &a, bool batched, cudaStream_t s) {
    return batched ? launch_encode_t<true, false>(a, s) : launch_encode_t<false, false>(a, s);
}

cudaError_t launch_encode_one_pass(const EncodeArgs &a, bool batched, cudaStream_t s) {
    return batched ? launch_encode_t<true, true>(a, s) : launch_encode_t<false, true>(a, s);
}

}  // namespace sz
