// sz_decode.cu -- container reader.
//
// SplitZip explainer (gist.science), section 4 "Pourquoi est-ce rapide ?":
// decoding looks each 4-bit code up, joins the exponent it names to the
// sign and mantissa, and, where an escape note exists, overwrites that
// place with the raw exponent -- linear work with no detours.
//
// Two launches: (1) every tile finds where its escapes start in the
// ascending position stream (one binary search per tile, all tiles in
// parallel); (2) every tile decodes its elements in registers, patches its
// escapes there, and writes the BF16 values with 16-byte stores.  The
// escape list of each tile is checked as it is used: ascending, inside the
// tile, raw exponent outside the codebook, placeholder code 0 -- together
// with monotone tile starts this proves the whole stream well formed.
#include "sz_internal.cuh"

namespace sz {

// ------------------------------------------------------------ the header
struct Header {
    uint64_t n, e;
    uint64_t cb_lo, cb_hi;  // codebook bytes 0-7 and 8-15, little-endian
    bool ok;
};

__device__ __forceinline__ uint32_t cb_entry(const Header &h, int k) {  // k compile-time after unrolling
    return (uint32_t)(((k < 8) ? h.cb_lo : h.cb_hi) >> (8 * (k & 7))) & 0xFFu;
}

// Parse and check the fixed fields of the container at c (cap bytes
// available) for a stream of `n` elements.
__device__ inline Header read_header(const uint8_t *c, uint64_t cap, uint64_t n) {
    Header h{};
    h.ok = false;
    if (cap < kHeader) return h;
    const uint64_t w0 = *reinterpret_cast<const uint64_t *>(c);
    h.n = *reinterpret_cast<const uint64_t *>(c + 8);
    h.e = *reinterpret_cast<const uint64_t *>(c + 16);
    h.cb_lo = *reinterpret_cast<const uint64_t *>(c + 24);
    h.cb_hi = *reinterpret_cast<const uint64_t *>(c + 32);
    const uint64_t rsv = *reinterpret_cast<const uint64_t *>(c + 40);
    h.ok = w0 == 0x00000101564B5A53ull && rsv == 0 && h.n == n && n < (1ull << 32) && h.e <= n &&
           container_size(n, h.e) <= cap;
    return h;
}

__device__ inline bool codebook_distinct(const Header &h) {
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int k = i + 1; k < 16; ++k) ok &= cb_entry(h, i) != cb_entry(h, k);
    return ok;
}

// ----------------------------------------------------- per-tile escape index
// Entry j of segment k (j = 0..tiles_k) = index of the first escape whose
// position is >= the first element of tile j (entry tiles_k = e).  Entries
// of segment k start at tile_begin_k + k.  One thread per entry.
template <bool kBatched>
__global__ void __launch_bounds__(256) esc_index_kernel(const DecodeArgs a, uint64_t n_entries) {
    __shared__ uint64_t s_entry_begin[kMaxSmemSegs + 1];
    const uint32_t ns = kBatched ? a.batch.n_segs : 1u;
    const bool cached = kBatched && ns <= kMaxSmemSegs;
    if (cached) {
        for (uint32_t i = threadIdx.x; i < ns; i += blockDim.x) s_entry_begin[i] = a.batch.segs[i].tile_begin + i;
        __syncthreads();
    }
    const uint64_t j_glob = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j_glob >= n_entries) return;
    uint32_t k = 0;
    if (kBatched) {  // largest k with tile_begin_k + k <= j_glob
        uint32_t lo = 0, hi = ns;
        while (hi - lo > 1) {
            const uint32_t mid = (lo + hi) >> 1;
            const uint64_t b = cached ? s_entry_begin[mid] : a.batch.segs[mid].tile_begin + mid;
            if (b <= j_glob) lo = mid; else hi = mid;
        }
        k = lo;
    }
    const sz_segment seg = load_segment(a.batch, k);
    const uint64_t j = j_glob - (seg.tile_begin + k);
    const uint64_t tiles = segment_tiles(seg.n_elems, a.batch.page_elems);
    int32_t *status = a.status + k;
    uint32_t *ts = a.tile_start + seg.tile_begin + k;
    if (j > tiles) return;
    const uint64_t cap = seg.out_offset <= a.in_cap ? a.in_cap - seg.out_offset : 0;
    const uint8_t *c = a.in + seg.out_offset;
    const Header h = read_header(c, cap, seg.n_elems);
    if (j == tiles) {  // the sentinel thread reports the header of its segment
        if (!h.ok || !codebook_distinct(h)) set_status(status, SZ_ERR_CORRUPT);
        ts[j] = h.ok ? (uint32_t)h.e : 0u;
        return;
    }
    if (!h.ok) {
        ts[j] = 0;
        return;
    }
    const uint64_t n = h.n, e = h.e;
    const uint64_t tpp = tiles_per_page(a.batch.page_elems);
    const uint64_t first = (j / tpp) * a.batch.page_elems + (j % tpp) * kTile;
    const uint8_t *pos = c + kHeader + n + (n + 1) / 2;
    uint64_t lo = 0, hi = e;  // first index with pos >= first
    while (lo < hi) {
        const uint64_t mid = (lo + hi) >> 1;
        if (load_u32_any(pos + 4 * mid) < first) lo = mid + 1; else hi = mid;
    }
    ts[j] = (uint32_t)lo;
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

__device__ inline DecTables make_tables(const Header &hd) {
    DecTables t;
    uint32_t h[4] = {0, 0, 0, 0}, l[2] = {0, 0};
#pragma unroll
    for (int k = 0; k < 16; ++k) h[k >> 2] |= (cb_entry(hd, k) >> 1) << (8 * (k & 3));
#pragma unroll
    for (int j = 0; j < 8; ++j)
        l[j >> 2] |= (((cb_entry(hd, j) & 1u) << 6) | ((cb_entry(hd, j + 8) & 1u) << 7)) << (8 * (j & 3));
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

constexpr int kEscBatch = 2048;  // escapes staged in shared memory per round

template <bool kBatched>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeArgs a) {
    __shared__ SegCache s_segc;
    __shared__ uint16_t s_epos[kEscBatch];  // tile-local offsets
    __shared__ uint8_t s_eraw[kEscBatch];
    __shared__ uint32_t s_inset[8];         // codebook membership bitmap

    const int tid = threadIdx.x;
    if (kBatched) seg_cache_fill(s_segc, a.batch);

    uint32_t cur = 0xFFFFFFFFu;
    sz_segment seg{};
    Header h{};
    bool seg_ok = false;
    DecTables T{};
    const uint8_t *c = nullptr;

    for (uint64_t tile = blockIdx.x; tile < a.batch.n_tiles; tile += gridDim.x) {
        const uint32_t k = find_segment(s_segc, a.batch, tile);
        int32_t *status = a.status + k;
        if (k != cur) {
            __syncthreads();  // done with the previous segment's shared bitmap
            seg = load_segment(a.batch, k);
            const uint64_t cap = seg.out_offset <= a.in_cap ? a.in_cap - seg.out_offset : 0;
            c = a.in + seg.out_offset;
            h = read_header(c, cap, seg.n_elems);
            seg_ok = h.ok && codebook_distinct(h);
            if (tid < 8) {
                uint32_t w = 0;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t e = cb_entry(h, i);
                    if ((e >> 5) == (uint32_t)tid) w |= 1u << (e & 31);
                }
                s_inset[tid] = w;
            }
            T = make_tables(h);
            cur = k;
            if (tid == 0 && !seg_ok) set_status(status, SZ_ERR_CORRUPT);
            __syncthreads();
        }
        if (!seg_ok) continue;

        const TileRef r = resolve_tile(a.batch, seg, k, tile);
        uint16_t *dst = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        const bool dst_aligned = (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
        const uint8_t *in_sm = c + kHeader + r.elem0;
        const uint8_t *codes_base = c + kHeader + r.n;
        const bool codes_aligned = (r.n % 8) == 0;
        const uint8_t *pos = c + kHeader + r.n + (r.n + 1) / 2;
        const uint8_t *raw = pos + 4 * h.e;
        const uint32_t *ts = a.tile_start + seg.tile_begin + k;
        uint32_t lo = ts[r.local], hi = ts[r.local + 1];
        if (!dst_aligned && tid == 0) set_status(status, SZ_ERR_ALIGN);
        if (hi < lo || hi > h.e || hi - lo > r.len) {  // tile starts not monotone
            if (tid == 0) set_status(status, SZ_ERR_CORRUPT);
            hi = lo = 0;
        }

        // ---- decode all chunks into registers
        uint4 o[2 * kChunks];
        uint64_t cw[kChunks];
        const bool fast = r.len == kTile && codes_aligned && dst_aligned;
        if (fast) {
            uint4 smv[kChunks];
#pragma unroll
            for (int q = 0; q < kChunks; ++q) {
                const uint32_t off = (q * kThreads + tid) * kChunk;
                smv[q] = ld_stream_v4(in_sm + off);
                cw[q] = __ldcs(reinterpret_cast<const unsigned long long *>(codes_base + (r.elem0 + off) / 2));
            }
#pragma unroll
            for (int q = 0; q < kChunks; ++q) decode_chunk(smv[q], cw[q], T, o[2 * q], o[2 * q + 1]);
        } else {
#pragma unroll
            for (int q = 0; q < kChunks; ++q) {
                const uint32_t off = (q * kThreads + tid) * kChunk;
                const uint32_t cnt = off < r.len ? umin32(kChunk, r.len - off) : 0u;
                uint4 smv = make_uint4(0, 0, 0, 0);
                uint64_t codes = 0;
                if (cnt == (uint32_t)kChunk && codes_aligned) {
                    smv = ld_stream_v4(in_sm + off);
                    codes = *reinterpret_cast<const unsigned long long *>(codes_base + (r.elem0 + off) / 2);
                } else if (cnt) {
                    uint32_t sw[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int j = 0; j < kChunk; ++j)
                        if (j < (int)cnt) sw[j >> 2] |= (uint32_t)in_sm[off + j] << (8 * (j & 3));
                    smv = make_uint4(sw[0], sw[1], sw[2], sw[3]);
                    const uint8_t *cb = codes_base + (r.elem0 + off) / 2;
#pragma unroll
                    for (int b = 0; b < kChunk / 2; ++b)
                        if (2 * b < (int)cnt) codes |= (uint64_t)cb[b] << (8 * b);
                    // odd element count: the unused high nibble must be 0
                    if ((cnt & 1) && ((codes >> (4 * cnt)) & 0xFu) != 0) set_status(status, SZ_ERR_CORRUPT);
                    if (cnt < (uint32_t)kChunk) codes &= (1ull << (4 * cnt)) - 1ull;
                }
                cw[q] = codes;
                decode_chunk(smv, codes, T, o[2 * q], o[2 * q + 1]);
            }
        }

        // ---- escapes of this tile, staged through shared memory
        for (uint32_t b0 = lo; b0 < hi; b0 += kEscBatch) {
            const uint32_t nb = umin32(kEscBatch, hi - b0);
            __syncthreads();
            for (uint32_t i = tid; i < nb; i += kThreads) {
                const uint64_t p = load_u32_any(pos + 4 * (uint64_t)(b0 + i));
                const uint32_t x = raw[b0 + i];
                bool bad = p < r.elem0 || p >= r.elem0 + r.len;
                if (b0 + i > lo) bad |= load_u32_any(pos + 4 * (uint64_t)(b0 + i - 1)) >= p;
                bad |= (s_inset[x >> 5] >> (x & 31)) & 1u;
                if (bad) set_status(status, SZ_ERR_CORRUPT);
                s_epos[i] = bad ? 0xFFFFu : (uint16_t)(p - r.elem0);
                s_eraw[i] = (uint8_t)x;
            }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < kChunks; ++q) {
                const uint32_t off = (q * kThreads + tid) * kChunk;
                uint32_t a0 = 0, a1 = nb;  // first staged escape at or after off
                while (a0 < a1) {
                    const uint32_t mid = (a0 + a1) >> 1;
                    if (s_epos[mid] < off) a0 = mid + 1; else a1 = mid;
                }
                for (uint32_t i = a0; i < nb && s_epos[i] < off + kChunk; ++i) {
                    const int j = (int)(s_epos[i] - off);
                    if (((cw[q] >> (4 * j)) & 0xFu) != 0) set_status(status, SZ_ERR_CORRUPT);
                    patch_elem(o[2 * q], o[2 * q + 1], j, s_eraw[i]);
                }
            }
        }

        // ---- store
        if (fast) {
#pragma unroll
            for (int q = 0; q < kChunks; ++q) {
                const uint32_t off = (q * kThreads + tid) * kChunk;
                st_stream_v4(dst + off, o[2 * q]);
                st_stream_v4(dst + off + 8, o[2 * q + 1]);
            }
        } else {
#pragma unroll
            for (int q = 0; q < kChunks; ++q) {
                const uint32_t off = (q * kThreads + tid) * kChunk;
                const uint32_t cnt = off < r.len ? umin32(kChunk, r.len - off) : 0u;
                if (cnt == (uint32_t)kChunk && dst_aligned) {
                    st_stream_v4(dst + off, o[2 * q]);
                    st_stream_v4(dst + off + 8, o[2 * q + 1]);
                } else if (cnt && dst_aligned) {
                    const uint32_t w[8] = {o[2 * q].x, o[2 * q].y, o[2 * q].z, o[2 * q].w,
                                           o[2 * q + 1].x, o[2 * q + 1].y, o[2 * q + 1].z, o[2 * q + 1].w};
#pragma unroll
                    for (int j = 0; j < kChunk; ++j)
                        if (j < (int)cnt) dst[off + j] = (uint16_t)(w[j >> 1] >> (16 * (j & 1)));
                }
            }
        }
    }
}

cudaError_t launch_esc_index(const DecodeArgs &a, bool batched, cudaStream_t s) {
    const uint64_t entries = a.batch.n_tiles + (batched ? a.batch.n_segs : 1u);
    const uint64_t grid = div_up(entries, 256);
    if (batched)
        esc_index_kernel<true><<<(unsigned)grid, 256, 0, s>>>(a, entries);
    else
        esc_index_kernel<false><<<(unsigned)grid, 256, 0, s>>>(a, entries);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, bool batched, int grid, cudaStream_t s) {
    if (a.batch.n_tiles == 0) return cudaSuccess;
    grid = (int)umax64(1, umin64((uint64_t)grid, a.batch.n_tiles));
    if (batched)
        decode_kernel<true><<<grid, kThreads, 0, s>>>(a);
    else
        decode_kernel<false><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

int decode_blocks_per_sm() {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<true>, kThreads, 0);
    return occ > 0 ? occ : 1;
}

}  // namespace sz
