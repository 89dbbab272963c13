// sz_encode.cu -- container writer.
//
// SplitZip explainer (gist.science), section 3 "La strategie SplitZip":
// each BF16 value leaves its sign+mantissa byte, its exponent becomes the
// 4-bit code of its codebook slot (two codes per byte), and an exponent
// outside the codebook becomes an escape note (position, raw exponent).
// Section 4: fixed-length codes make this one straight pass -- every output
// byte's address is known from the element index, except the escape
// records, whose place is the number of escapes before them.
//
// One persistent kernel: CTAs draw tiles from an atomic ticket (so a tile's
// predecessors are always running or done), write the sm and code streams
// with coalesced 16-byte / 8-byte stores, count escapes per thread-chunk,
// scan the counts across the CTA, and find the tile's starting escape index
// with a decoupled lookback over the tiles before it in the same segment.
#include "sz_internal.cuh"

namespace sz {

// ---------------------------------------------------------- chunk encode
// 16 consecutive BF16 values (two uint4) -> 16 sm bytes, 8 code bytes and an
// escape mask.  The LUT maps exponent -> code (0..15) or 0x80 (escape; its
// low nibble 0 is the placeholder code).  Escape mask layout: element j of
// the chunk is bit 8*(j%4) + j/4.
__device__ __forceinline__ void encode_chunk(const uint4 v0, const uint4 v1, const uint8_t *lut,
                                             uint4 &sm, uint64_t &codes, uint32_t &esc) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t smw[4], B[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t a = w[2 * q], b = w[2 * q + 1];
        const uint32_t hi = prmt(a, b, 0x7531u);  // high bytes of the 4 values
        const uint32_t lo = prmt(a, b, 0x6420u);  // low bytes
        smw[q] = (hi & 0x80808080u) | (lo & 0x7F7F7F7Fu);
        const uint32_t c0 = lut[(a >> 7) & 0xFFu];
        const uint32_t c1 = lut[(a >> 23) & 0xFFu];
        const uint32_t c2 = lut[(b >> 7) & 0xFFu];
        const uint32_t c3 = lut[(b >> 23) & 0xFFu];
        B[q] = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
    }
    sm = make_uint4(smw[0], smw[1], smw[2], smw[3]);
    esc = ((B[0] & 0x80808080u) >> 7) | ((B[1] & 0x80808080u) >> 6) | ((B[2] & 0x80808080u) >> 5) |
          ((B[3] & 0x80808080u) >> 4);
    uint32_t P[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t nib = B[q] & 0x0F0F0F0Fu;
        P[q] = nib | (nib >> 4);  // byte 0 = n0 | n1<<4, byte 2 = n2 | n3<<4
    }
    const uint32_t lo32 = prmt(P[0], P[1], 0x6420u);
    const uint32_t hi32 = prmt(P[2], P[3], 0x6420u);
    codes = (uint64_t)lo32 | ((uint64_t)hi32 << 32);
}

// Exponent of chunk element j (runtime j; selects, no local-memory array).
__device__ __forceinline__ uint32_t exponent_of_chunk_elem(const uint4 v0, const uint4 v1, int j) {
    const int q = j >> 1;
    const uint4 v = (q & 4) ? v1 : v0;
    const uint32_t word = (q & 2) ? ((q & 1) ? v.w : v.z) : ((q & 1) ? v.y : v.x);
    return (j & 1) ? (word >> 23) & 0xFFu : (word >> 7) & 0xFFu;
}

__device__ __forceinline__ uint32_t byte_of(uint4 v, int b) {  // b is a compile-time constant
    const uint32_t w = (b < 4) ? v.x : (b < 8) ? v.y : (b < 12) ? v.z : v.w;
    return (w >> (8 * (b & 3))) & 0xFFu;
}

// Escape mask in element order (bit j = element j), from the interleaved
// layout above: for each quad q, bits 8b + q (b = 0..3) are gathered by one
// multiply -- the four products of 1 + 2^7 + 2^14 + 2^21 do not overlap, and
// bits 21..24 receive b = 0..3 in order.
__device__ __forceinline__ uint32_t esc_in_element_order(uint32_t m) {
    uint32_t r = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) r |= ((((m >> q) & 0x01010101u) * 0x00204081u) >> 21 & 0xFu) << (4 * q);
    return r;
}

__device__ __forceinline__ uint32_t esc_bit_of_elem(int j) { return 1u << (8 * (j & 3) + (j >> 2)); }

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

// Warp-wide inclusive scan of a packed u64 (four 16-bit counters).
__device__ __forceinline__ uint64_t warp_incl_scan(uint64_t v, int lane) {
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint64_t y = __shfl_up_sync(0xFFFFFFFFu, v, d);
        if (lane >= d) v += y;
    }
    return v;
}

__device__ __forceinline__ uint32_t field16(uint64_t v, int c) { return (uint32_t)(v >> (16 * c)) & 0xFFFFu; }

template <bool kBatched>
__global__ void __launch_bounds__(kThreads, 2) encode_kernel(const EncodeArgs a) {
    __shared__ SegCache s_segc;
    __shared__ __align__(16) uint8_t s_lut[256];
    __shared__ uint64_t s_warp[kWarps];
    __shared__ unsigned long long s_tile;
    __shared__ uint32_t s_excl;
    __shared__ int s_timeout;

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (kBatched) seg_cache_fill(s_segc, a.batch);

    // Segments with no elements have no tiles: CTA 0 writes their header.
    if (blockIdx.x == 0) {
        const uint32_t ns = kBatched ? a.batch.n_segs : 1;
        for (uint32_t k = tid; k < ns; k += kThreads) {
            const sz_segment s = load_segment(a.batch, k);
            if (s.n_elems != 0) continue;
            if (a.meta[k].valid == 0) { set_status(a.status ? a.status + k : nullptr, SZ_ERR_INVALID); continue; }
            if (s.out_offset + kHeader > a.out_cap) { set_status(a.status ? a.status + k : nullptr, SZ_ERR_CAPACITY); continue; }
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

    uint32_t cur = 0xFFFFFFFFu;
    sz_segment seg{};
    uint64_t e_total = 0;
    bool seg_ok = false;

    while (true) {
        __syncthreads();  // every thread is done with the previous tile's shared state
        if (tid == 0) s_tile = atomicAdd(a.ticket, 1ull);
        __syncthreads();
        const uint64_t tile = s_tile;
        if (tile >= a.batch.n_tiles) break;
        const uint32_t k = find_segment(s_segc, a.batch, tile);
        int32_t *status = a.status ? a.status + k : nullptr;
        if (k != cur) {
            seg = load_segment(a.batch, k);
            s_lut[tid] = 0x80;
            __syncthreads();
            const SegMeta *m = a.meta + k;
            if (tid < 16) s_lut[m->codebook[tid]] = (uint8_t)tid;
            e_total = m->n_escapes;
            const bool valid = m->valid != 0;
            const bool fits = seg.out_offset <= a.out_cap &&
                              container_size(seg.n_elems, e_total) <= a.out_cap - seg.out_offset;
            seg_ok = valid && fits;
            if (tid == 0 && !valid) set_status(status, SZ_ERR_INVALID);
            if (tid == 0 && valid && !fits) set_status(status, SZ_ERR_CAPACITY);
            __syncthreads();
            cur = k;
        }
        // An invalid segment is skipped by every one of its tiles, so no
        // tile ever waits on it.
        if (!seg_ok) continue;

        const TileRef r = resolve_tile(a.batch, seg, k, tile);
        const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        uint8_t *out = a.out + seg.out_offset;
        uint8_t *out_sm = out + kHeader + r.elem0;
        uint8_t *codes_base = out + kHeader + r.n;  // element i's nibble is in byte i/2
        const bool codes_aligned = (r.n % 8) == 0;
        const bool src_aligned = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
        if (!src_aligned) {  // only batched pages can be misaligned here
            if (tid == 0) set_status(status, SZ_ERR_ALIGN);
        }

        // Header of the segment: written once, by its first tile.
        if (r.local == 0 && tid < 6) {
            uint64_t v = 0;
            if (tid == 0) v = 0x00000101564B5A53ull;
            if (tid == 1) v = r.n;
            if (tid == 2) v = e_total;
            if (tid == 3 || tid == 4) {
                for (int i = 7; i >= 0; --i) v = (v << 8) | a.meta[k].codebook[8 * (tid - 3) + i];
            }
            reinterpret_cast<uint64_t *>(out)[tid] = v;
        }

        uint4 in[2 * kChunks];
        uint32_t esc[kChunks];
        if (r.len == kTile && codes_aligned && src_aligned) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint16_t *p = src + (c * kThreads + tid) * kChunk;
                in[2 * c] = ld_stream_v4(p);
                in[2 * c + 1] = ld_stream_v4(p + 8);
            }
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint32_t off = (c * kThreads + tid) * kChunk;
                uint4 smv;
                uint64_t cw;
                encode_chunk(in[2 * c], in[2 * c + 1], s_lut, smv, cw, esc[c]);
                st_stream_v4(out_sm + off, smv);
                st_stream_u64(codes_base + (r.elem0 + off) / 2, cw);
            }
        } else {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint32_t off = (c * kThreads + tid) * kChunk;
                esc[c] = 0;
                in[2 * c] = make_uint4(0, 0, 0, 0);
                in[2 * c + 1] = make_uint4(0, 0, 0, 0);
                if (!src_aligned || off >= r.len) continue;
                if (off + kChunk <= r.len && codes_aligned) {
                    in[2 * c] = ld_stream_v4(src + off);
                    in[2 * c + 1] = ld_stream_v4(src + off + 8);
                    uint4 smv;
                    uint64_t cw;
                    encode_chunk(in[2 * c], in[2 * c + 1], s_lut, smv, cw, esc[c]);
                    st_stream_v4(out_sm + off, smv);
                    st_stream_u64(codes_base + (r.elem0 + off) / 2, cw);
                } else {
                    // ragged or unaligned chunk: assemble the cnt values with
                    // guarded loads, encode as a full chunk, keep cnt of it
                    const uint32_t cnt = umin32(kChunk, r.len - off);
                    uint32_t wv[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint32_t lo = (2 * q < (int)cnt) ? (uint32_t)src[off + 2 * q] : 0u;
                        const uint32_t hi = (2 * q + 1 < (int)cnt) ? (uint32_t)src[off + 2 * q + 1] : 0u;
                        wv[q] = lo | (hi << 16);
                    }
                    in[2 * c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    in[2 * c + 1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
                    uint4 smv;
                    uint64_t cw;
                    uint32_t e;
                    encode_chunk(in[2 * c], in[2 * c + 1], s_lut, smv, cw, e);
                    uint32_t keep = 0;
#pragma unroll
                    for (int j = 0; j < kChunk; ++j)
                        if (j < (int)cnt) keep |= esc_bit_of_elem(j);
                    esc[c] = e & keep;
                    if (cnt < (uint32_t)kChunk) cw &= (1ull << (4 * cnt)) - 1ull;  // odd tail nibble = 0
#pragma unroll
                    for (int j = 0; j < kChunk; ++j)
                        if (j < (int)cnt) out_sm[off + j] = (uint8_t)byte_of(smv, j);
                    uint8_t *cb = codes_base + (r.elem0 + off) / 2;
#pragma unroll
                    for (int b = 0; b < kChunk / 2; ++b)
                        if (2 * b < (int)cnt) cb[b] = (uint8_t)(cw >> (8 * b));
                }
            }
        }

        // ---- escapes: CTA scan of the per-chunk counts, packed 4 x 16 bit
        uint64_t cnt = 0;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) cnt |= (uint64_t)__popc(esc[c]) << (16 * c);
        const uint64_t incl = warp_incl_scan(cnt, lane);
        if (lane == 31) s_warp[wid] = incl;
        __syncthreads();
        uint64_t warp_excl = 0, tile_tot = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const uint64_t v = s_warp[w];
            if (w < wid) warp_excl += v;
            tile_tot += v;
        }
        const uint64_t thr_excl = warp_excl + incl - cnt;
        const uint32_t total = field16(tile_tot, 0) + field16(tile_tot, 1) + field16(tile_tot, 2) +
                               field16(tile_tot, 3);

        // ---- decoupled lookback (warp 0)
        if (wid == 0) {
            const bool publish = (a.debug_flags & kDebugNoPublish) == 0;
            uint64_t *st = a.tile_status;
            uint32_t excl = 0;
            bool timeout = false;
            if (tile == seg.tile_begin) {
                if (lane == 0 && publish) st_relaxed_u64(st + tile, kFlagPrefix | total);
            } else {
                if (lane == 0 && publish) st_relaxed_u64(st + tile, kFlagAggregate | total);
                const int64_t first = (int64_t)seg.tile_begin;
                int64_t pred = (int64_t)tile - 1;
                const uint64_t t0 = globaltimer_ns();
                while (true) {
                    const int64_t idx = pred - lane;
                    const uint64_t s = idx >= first ? ld_relaxed_u64(st + idx) : kFlagPrefix;
                    const uint32_t not_ready = __ballot_sync(0xFFFFFFFFu, (s & kFlagMask) == 0);
                    const uint32_t prefix = __ballot_sync(0xFFFFFFFFu, (s & kFlagMask) == kFlagPrefix);
                    const int p_lane = prefix ? __ffs(prefix) - 1 : 32;
                    const uint32_t upto = p_lane >= 31 ? 0xFFFFFFFFu : ((2u << p_lane) - 1u);
                    if (not_ready & upto) {
                        const bool expired = globaltimer_ns() - t0 > a.wait_limit_ns;
                        if (__any_sync(0xFFFFFFFFu, expired)) {
                            timeout = true;
                            break;
                        }
                        __nanosleep(100);
                        continue;
                    }
                    const uint32_t v = (lane <= p_lane) ? (uint32_t)s : 0u;
                    excl += __reduce_add_sync(0xFFFFFFFFu, v);
                    if (p_lane < 32) break;
                    pred -= 32;
                }
                // Publish even after a timeout so later tiles are not stuck.
                if (lane == 0 && publish) st_relaxed_u64(st + tile, kFlagPrefix | (uint64_t)(excl + total));
            }
            if (lane == 0) {
                s_excl = excl;
                s_timeout = timeout ? 1 : 0;
            }
        }
        __syncthreads();
        const uint32_t tile_excl = s_excl;
        if (s_timeout) {
            if (tid == 0) set_status(status, SZ_ERR_DEVICE_TIMEOUT);
            continue;
        }

        // ---- escape records, in element order
        const uint64_t pos_off = kHeader + r.n + (r.n + 1) / 2;
        uint8_t *pos_base = out + pos_off;
        uint8_t *raw_base = pos_base + 4 * e_total;
        const bool pos_aligned = (pos_off & 3) == 0;
        uint32_t chunk_base = 0;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            uint32_t m = esc[c] ? esc_in_element_order(esc[c]) : 0u;
            uint64_t idx = (uint64_t)tile_excl + chunk_base + field16(thr_excl, c);
            chunk_base += field16(tile_tot, c);
            while (m) {  // ascending element order
                const int j = __ffs(m) - 1;
                m &= m - 1;
                const uint64_t p = r.elem0 + (uint64_t)(c * kThreads + tid) * kChunk + j;
                if (idx >= e_total) {  // more escapes than the histogram said
                    set_status(status, SZ_ERR_CORRUPT);
                    break;
                }
                store_u32_le(pos_base + 4 * idx, (uint32_t)p, pos_aligned);
                raw_base[idx] = (uint8_t)exponent_of_chunk_elem(in[2 * c], in[2 * c + 1], j);
                ++idx;
            }
        }

        // The segment's last tile knows the final escape count.
        if (tid == 0 && r.local + 1 == segment_tiles(r.n, a.batch.page_elems)) {
            if ((uint64_t)tile_excl + total == e_total) {
                a.out_bytes[k] = container_size(r.n, e_total);
            } else {
                set_status(status, SZ_ERR_CORRUPT);
            }
        }
    }
}

cudaError_t launch_encode(const EncodeArgs &a, bool batched, int grid, cudaStream_t s) {
    if (a.batch.n_tiles == 0 && !batched && a.batch.single.n_elems != 0) return cudaSuccess;
    grid = (int)umax64(1, umin64((uint64_t)grid, umax64(a.batch.n_tiles, 1)));
    if (batched)
        encode_kernel<true><<<grid, kThreads, 0, s>>>(a);
    else
        encode_kernel<false><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

int encode_blocks_per_sm() {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, encode_kernel<true>, kThreads, 0);
    return occ > 0 ? occ : 1;
}

}  // namespace sz
