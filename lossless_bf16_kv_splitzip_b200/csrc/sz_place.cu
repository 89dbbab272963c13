// sz_place.cu -- escape placement after a one-pass encode.
//
// SplitZip explainer (gist.science), section 3: the escape notes follow the
// codes, all positions first, then all raw exponents -- so the exponent
// stream starts at 4e bytes past the positions, and e is known only when the
// whole segment is encoded.  A one-pass encode with the caller's codebook
// (no histogram pass) therefore writes the sign+mantissa and code streams in
// place and parks each tile's escape records in a workspace slot; this
// kernel then counts every segment's escapes from the per-tile and per-range
// counts, writes the header and the size, and moves the records into place;
// tiles whose records overflowed their slot are listed and rescanned by a
// second kernel spread over the GPU.
//
// One block per range, the partition the encode used.  No block waits for
// another: every count it reads was written by the launch before it.
#include "sz_internal.cuh"

namespace sz {

struct PlaceShared {
    SegCache segc;
    unsigned long long red[kWarps];
    uint32_t warp[kWarps];
    uint32_t base[kThreads];  // per tile of the current chunk: index of its first record in the segment
    uint32_t cnt[kThreads];   // per tile of the current chunk: its records
    uint64_t elem0[kThreads];     // per tile: its first element in the segment's stream
    int32_t status;           // the segment's status as thread 0 read it
};

// Sum over the block's 256 threads (every thread must call it).
__device__ uint64_t block_sum(uint64_t v, PlaceShared &sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, d);
    if (lane == 0) sh.red[wid] = v;
    __syncthreads();
    uint64_t tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += sh.red[w];
    __syncthreads();
    return tot;
}

// Exclusive scan over the block's 256 threads; *total = the sum.
__device__ uint32_t block_excl_scan(uint32_t v, uint32_t *total, PlaceShared &sh) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) sh.warp[wid] = incl;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const uint32_t x = sh.warp[w];
        before += (w < wid) ? x : 0u;
        tot += x;
    }
    __syncthreads();
    *total = tot;
    return before + incl - v;
}

__device__ inline void write_header(uint8_t *out, uint64_t n, uint64_t e, const uint8_t *cb) {
    uint64_t c0 = 0, c1 = 0;
    for (int i = 7; i >= 0; --i) {
        c0 = (c0 << 8) | cb[i];
        c1 = (c1 << 8) | cb[8 + i];
    }
    uint64_t *h = reinterpret_cast<uint64_t *>(out);
    h[0] = 0x00000101564B5A53ull;  // "SZKV", version 1, dtype 1, flags 0
    h[1] = n;
    h[2] = e;
    h[3] = c0;
    h[4] = c1;
    h[5] = 0;
}

// Word i (0..7, runtime) of eight registers, selected without local memory.
__device__ __forceinline__ uint32_t word_of(const uint32_t (&w)[8], uint32_t i) {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) v = (i == (uint32_t)j) ? w[j] : v;
    return v;
}

// A tile whose slot overflowed: its escapes found again in its input, in
// element order, by the whole block.  A round covers 16,384 elements, four
// chunks of 16 per thread loaded up front; an exclusive scan of the
// per-thread counts places each thread's records.  s_esc: 256-entry table,
// nonzero for exponents outside the codebook.
template <bool kBatched>
__device__ void rescan_tile(const PlaceArgs &a, const OvfItem &it, const uint8_t *s_esc, PlaceShared &sh) {
    const uint32_t k = it.seg;
    const sz_segment seg = load_segment(a.batch, k);
    const TileRef r = resolve_tile(a.batch, seg, k, it.tile);
    const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
    const uint64_t n = seg.n_elems;
    const uint64_t pos_off = kHeader + n + (n + 1) / 2;
    uint8_t *pos_base = a.out + seg.out_offset + pos_off;
    uint8_t *raw_base = pos_base + 4 * it.e;
    const bool pos_aligned = (pos_off & 3) == 0;
    uint32_t done = 0;
    for (uint32_t o = 0; o < r.len; o += kSub) {
        uint32_t w[kChunks][8];
        uint32_t mask[kChunks];
#pragma unroll
        for (int q = 0; q < kChunks; ++q) {
            const uint32_t first = o + (q * kThreads + threadIdx.x) * kChunk;
#pragma unroll
            for (int x = 0; x < 8; ++x) w[q][x] = 0;
            if (first + kChunk <= r.len) {
                const uint4 v0 = ld_stream_v4(src + first), v1 = ld_stream_v4(src + first + 8);
                w[q][0] = v0.x; w[q][1] = v0.y; w[q][2] = v0.z; w[q][3] = v0.w;
                w[q][4] = v1.x; w[q][5] = v1.y; w[q][6] = v1.z; w[q][7] = v1.w;
            } else if (first < r.len) {
#pragma unroll
                for (int e = 0; e < kChunk; ++e)
                    if (first + e < r.len) w[q][e >> 1] |= (uint32_t)src[first + e] << (16 * (e & 1));
            }
        }
#pragma unroll
        for (int q = 0; q < kChunks; ++q) {
            const uint32_t first = o + (q * kThreads + threadIdx.x) * kChunk;
            mask[q] = 0;
#pragma unroll
            for (int e = 0; e < kChunk; ++e) {
                const uint32_t raw = (w[q][e >> 1] >> (16 * (e & 1) + 7)) & 0xFFu;
                if (first + e < r.len && s_esc[raw]) mask[q] |= 1u << e;
            }
        }
        // records of one thread are not contiguous across its four chunks:
        // scan per chunk row, rows in order
#pragma unroll
        for (int q = 0; q < kChunks; ++q) {
            const uint32_t first = o + (q * kThreads + threadIdx.x) * kChunk;
            uint32_t total = 0;
            uint32_t idx = done + block_excl_scan(__popc(mask[q]), &total, sh);
            uint32_t m = mask[q];
            while (m) {
                const int e = __ffs(m) - 1;
                m &= m - 1;
                if (idx < it.cnt) {  // never more than the encode counted
                    const uint64_t g = it.base + idx;
                    store_u32_le(pos_base + 4 * g, (uint32_t)(r.elem0 + first + e), pos_aligned);
                    raw_base[g] = (uint8_t)((word_of(w[q], e >> 1) >> (16 * (e & 1) + 7)) & 0xFFu);
                }
                ++idx;
            }
            done += total;
        }
    }
    if (threadIdx.x == 0 && done != it.cnt) set_status(a.status + k, SZ_ERR_CORRUPT);  // the input changed
}

// Zero-length segments have no tiles: block 0 writes their header (their
// size, like every segment's, is written after the rescan).
__device__ void place_empty_segments(const PlaceArgs &a) {
    const uint32_t ns = a.batch.segs ? a.batch.n_segs : 1u;
    for (uint32_t k = threadIdx.x; k < ns; k += blockDim.x) {
        const sz_segment s = load_segment(a.batch, k);
        if (s.n_elems != 0) continue;
        const uint8_t *cb = a.codebooks_in + 16 * (size_t)k;
        if (!codebook16_distinct(cb)) { set_status(a.status + k, SZ_ERR_INVALID); continue; }
        if (s.out_offset > a.out_cap || a.out_cap - s.out_offset < kHeader) {
            set_status(a.status + k, SZ_ERR_CAPACITY);
            continue;
        }
        if ((reinterpret_cast<uintptr_t>(a.out + s.out_offset) & 15) != 0) {
            set_status(a.status + k, SZ_ERR_ALIGN);
            continue;
        }
        write_header(a.out + s.out_offset, 0, 0, cb);
        a.seg_e[k] = 0;
    }
}

template <bool kBatched>
__global__ void __launch_bounds__(kThreads) place_kernel(const PlaceArgs a) {
    __shared__ PlaceShared sh;
    allow_dependents();      // the rescan kernel may start its prologue
    grid_dependency_wait();  // the one-pass encode before it has finished
    seg_cache_fill(sh.segc, a.batch);  // ends with __syncthreads
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (blockIdx.x == 0) place_empty_segments(a);

    const uint64_t R = a.range_tiles;
    const uint64_t b = blockIdx.x;
    const uint64_t t_begin = b * R;
    const uint64_t t_end = umin64(t_begin + R, a.batch.n_tiles);
    uint64_t t = t_begin;
    while (t < t_end) {
        const uint32_t k = find_segment(sh.segc, a.batch, t);
        const sz_segment seg = load_segment(a.batch, k);
        const uint64_t seg_end = seg.tile_begin + seg_tiles(a.batch, seg.n_elems);
        const uint64_t ps = t, pe = umin64(seg_end, t_end);  // this range's piece of segment k
        t = pe;
        // the encode refused the segment: skip it.  Thread 0 reads the word
        // (another block may set it meanwhile) and the block takes its decision.
        if (tid == 0) sh.status = *reinterpret_cast<volatile const int32_t *>(a.status + k);
        __syncthreads();
        const bool refused = sh.status != 0;
        __syncthreads();
        if (refused) continue;

        // the segment's escapes: its pieces in earlier ranges, in this one,
        // and in later ones
        const uint64_t b_first = seg.tile_begin / R, b_last = (seg_end - 1) / R;
        uint64_t acc = 0;
        if (ps == t_begin && seg.tile_begin < t_begin)
            for (uint64_t bb = b_first + tid; bb < b; bb += kThreads)
                acc += (bb == b_first && seg.tile_begin != b_first * R) ? a.rcnt[bb].last_cnt : a.rcnt[bb].first_cnt;
        const uint64_t pre = block_sum(acc, sh);
        acc = 0;
        if (pe == t_end && seg_end > t_end)
            for (uint64_t bb = b + 1 + tid; bb <= b_last; bb += kThreads) acc += a.rcnt[bb].first_cnt;
        for (uint64_t tt = ps + tid; tt < pe; tt += kThreads) acc += a.tile_cnt[tt];
        const uint64_t e = pre + block_sum(acc, sh);

        const uint64_t n = seg.n_elems;
        uint8_t *out = a.out + seg.out_offset;
        if (container_size(n, e) > a.out_cap - seg.out_offset) {  // the same decision in every block of k
            if (tid == 0) set_status(a.status + k, SZ_ERR_CAPACITY);
            continue;
        }
        const uint8_t *cb = a.codebooks_in + 16 * (size_t)k;
        if (ps == seg.tile_begin && tid == 0) {
            write_header(out, n, e, cb);
            a.seg_e[k] = (uint32_t)e;  // the size is written after the rescan
        }
        const uint64_t pos_off = kHeader + n + (n + 1) / 2;
        uint8_t *pos_base = out + pos_off;
        uint8_t *raw_base = pos_base + 4 * e;
        const bool pos_aligned = (pos_off & 3) == 0;

        // the piece's tiles, kThreads at a time: the first record index of
        // each; then one warp per tile moves its slot records (coalesced,
        // four loads in flight per lane); tiles whose slot overflowed are
        // listed for the rescan kernel
        uint64_t carry = pre;
        for (uint64_t c0 = ps; c0 < pe; c0 += kThreads) {
            const uint64_t tt = c0 + tid;
            const uint32_t cnt = tt < pe ? a.tile_cnt[tt] : 0u;
            uint32_t total = 0;
            const uint32_t excl = block_excl_scan(cnt, &total, sh);
            sh.cnt[tid] = cnt;
            sh.base[tid] = (uint32_t)(carry + excl);
            sh.elem0[tid] = tt < pe ? resolve_tile(a.batch, seg, k, tt).elem0 : 0;
            __syncthreads();
            const uint32_t nt = (uint32_t)umin64(kThreads, pe - c0);
            const uint32_t cap = slot_cap(a.batch);
            for (uint32_t i = wid; i < nt; i += kWarps) {
                const uint32_t ci = sh.cnt[i];
                if (ci > cap) continue;
                const uint32_t *slot = a.slots + (c0 + i) * cap;
                const uint64_t bi = sh.base[i], e0 = sh.elem0[i];
                for (uint32_t j0 = lane; j0 < ci; j0 += 128) {
                    uint32_t rec[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) rec[u] = (j0 + 32 * u < ci) ? slot[j0 + 32 * u] : 0u;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t jj = j0 + 32 * u;
                        if (jj >= ci) break;
                        const uint64_t g = bi + jj;
                        store_u32_le(pos_base + 4 * g, (uint32_t)(e0 + (rec[u] & 0xFFFFu)), pos_aligned);
                        raw_base[g] = (uint8_t)(rec[u] >> 16);
                    }
                }
            }
            if (tid < nt && cnt > cap) {  // left for the rescan kernel
                OvfItem it;
                it.tile = tt;
                it.base = sh.base[tid];
                it.e = e;
                it.cnt = cnt;
                it.seg = k;
                a.ovf[atomicAdd(a.ovf_count, 1u)] = it;
            }
            carry += total;
            __syncthreads();  // before the next chunk's counts land
        }
    }
}

// The tiles the placement listed, spread over the whole GPU, one block per
// tile at a time (nothing listed: every block goes straight to the end).
// The last block to finish writes every segment's size: the container size
// for a segment whose status is still SZ_OK after the encode, the placement
// and the rescans, else 0.
template <bool kBatched>
__global__ void __launch_bounds__(kThreads) rescan_kernel(const PlaceArgs a) {
    __shared__ PlaceShared sh;
    __shared__ uint8_t s_esc[256];
    __shared__ int s_last;
    grid_dependency_wait();  // the placement before it has finished
    const uint32_t count = *a.ovf_count;
    uint32_t cur = 0xFFFFFFFFu;
    for (uint32_t i = blockIdx.x; i < count; i += gridDim.x) {
        const OvfItem it = a.ovf[i];
        if (it.seg != cur) {  // block-uniform
            __syncthreads();
            s_esc[threadIdx.x] = 1;
            __syncthreads();
            if (threadIdx.x < 16) s_esc[a.codebooks_in[16 * (size_t)it.seg + threadIdx.x]] = 0;
            __syncthreads();
            cur = it.seg;
        }
        rescan_tile<kBatched>(a, it, s_esc, sh);
    }
    __syncthreads();  // every status this block sets is set
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(a.blocks_done, 1u) + 1 == gridDim.x;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const uint32_t ns = a.batch.segs ? a.batch.n_segs : 1u;
    for (uint32_t k = threadIdx.x; k < ns; k += blockDim.x) {
        const int32_t st = *reinterpret_cast<volatile const int32_t *>(a.status + k);
        a.out_bytes[k] = st == SZ_OK ? container_size(load_segment(a.batch, k).n_elems, a.seg_e[k]) : 0;
    }
}

cudaError_t launch_place(const PlaceArgs &a, bool batched, int sms, cudaStream_t s) {
    const int grid = (int)umax64(1, div_up(a.batch.n_tiles, a.range_tiles));
    const int rgrid = (int)umax64(1, umin64(a.batch.n_tiles, 2ull * (uint64_t)sms));
    cudaError_t e;
    if (batched) {
        e = launch_after(place_kernel<true>, dim3(grid), dim3(kThreads), 0, s, a);
        if (e == cudaSuccess) e = launch_after(rescan_kernel<true>, dim3(rgrid), dim3(kThreads), 0, s, a);
    } else {
        e = launch_after(place_kernel<false>, dim3(grid), dim3(kThreads), 0, s, a);
        if (e == cudaSuccess) e = launch_after(rescan_kernel<false>, dim3(rgrid), dim3(kThreads), 0, s, a);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sz
