// sz_hist.cu -- exponent histograms and top-16 codebook selection.
//
// SplitZip explainer (gist.science), section 2 "La decouverte secrete": the
// exponents repeat; section 3 "La strategie SplitZip": the 16 most common
// exponents get the 4-bit codes.  The histogram pass reads the input once
// and keeps, besides each segment's 256 counts, the 256 counts of every
// 65,536-element tile.  The select step orders the 256 exponents by (count
// descending, exponent ascending), keeps the first 16, and turns the tile
// histograms into the number of escapes of every tile -- an exclusive scan
// of those gives each tile the index of its first escape record, so the
// encode needs no cross-tile communication.
#include "sz_internal.cuh"

namespace sz {

// ------------------------------------------------------------- histogram
// Shared-memory layout: 256 bins x 32 lane columns of u32, bin-major, so the
// counter of (bin e, lane l) is word e*32 + l and lives in bank l: the 32
// lanes of a warp never collide, whatever exponents they hold.  All warps of
// the CTA share the 32 columns (lane l of every warp adds into column l).
// The columns are never cleared: a tile's counts are the difference of the
// column sums before and after it (modulo 2^32).
constexpr uint32_t kHistWords = 256 * 32;

__device__ __forceinline__ void red_add1(uint32_t saddr) {
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(saddr) : "memory");
}

// Count the two BF16 exponents of one 32-bit word.  The exponent field sits
// in bits 7..14 of each half, so (half & 0x7F80) is already exponent*128 =
// the byte offset of row `exponent`; adding lane*4 selects the column.
__device__ __forceinline__ void count_word(uint32_t w, uint32_t col) {
    red_add1(col + (w & 0x7F80u));
    red_add1(col + ((w >> 16) & 0x7F80u));
}

__device__ __forceinline__ void count_v4(uint4 v, uint32_t col) {
    count_word(v.x, col);
    count_word(v.y, col);
    count_word(v.z, col);
    count_word(v.w, col);
}

template <bool kBatched>
__global__ void __launch_bounds__(kThreads) hist_kernel(const HistArgs a) {
    extern __shared__ __align__(128) uint32_t s_hist[];  // kHistWords
    __shared__ SegCache s_segc;
    static_assert(kThreads == 256, "one thread per bin");

    for (uint32_t i = threadIdx.x; i < kHistWords; i += kThreads) s_hist[i] = 0;
    seg_cache_fill(s_segc, a.batch);  // ends with __syncthreads

    const uint32_t tid = threadIdx.x;
    const uint32_t col = smem_u32(s_hist) + (tid & 31) * 4;
    const uint64_t t_begin = (uint64_t)blockIdx.x * a.tiles_per_cta;
    const uint64_t t_end = umin64(t_begin + a.tiles_per_cta, a.batch.n_tiles);

    uint32_t prev = 0;     // column sum of bin `tid` at the last tile boundary
    uint32_t seg_acc = 0;  // bin `tid` count of the current segment in this CTA
    uint32_t cur = 0xFFFFFFFFu;
    sz_segment seg{};
    for (uint64_t t = t_begin; t < t_end; ++t) {
        const uint32_t k = find_segment(s_segc, a.batch, t);
        if (k != cur) {
            if (cur != 0xFFFFFFFFu && seg_acc) atomicAdd(&a.seg_hist[(size_t)cur * 256 + tid], seg_acc);
            seg_acc = 0;
            cur = k;
            seg = load_segment(a.batch, k);
        }
        const TileRef r = resolve_tile(a.batch, seg, k, t);
        const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        const bool ok = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
        if (!ok && tid == 0) set_status(a.status ? a.status + k : nullptr, SZ_ERR_ALIGN);
        for (uint32_t sub = 0; ok && sub < r.n_subs; ++sub) {
            const uint16_t *p = src + sub * kSub;
            const uint32_t len = umin32(kSub, r.len - sub * kSub);
            // bulk prefetch of the next sub-tile into L2 while this one is counted
            if (tid == 0 && sub + 1 < r.n_subs) {
                const uint32_t next = (umin32(kSub, r.len - (sub + 1) * kSub) * 2u) & ~15u;
                if (next) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p + kSub), "r"(next) : "memory");
            }
            if (len == kSub) {
                uint4 v[2 * kChunks];
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    const uint16_t *q = p + (c * kThreads + tid) * kChunk;
                    v[2 * c] = ld_stream_v4(q);
                    v[2 * c + 1] = ld_stream_v4(q + 8);
                }
#pragma unroll
                for (int i = 0; i < 2 * kChunks; ++i) count_v4(v[i], col);
            } else {
                for (int c = 0; c < kChunks; ++c) {
                    const uint32_t off = (c * kThreads + tid) * kChunk;
                    if (off + kChunk <= len) {
                        count_v4(ld_stream_v4(p + off), col);
                        count_v4(ld_stream_v4(p + off + 8), col);
                    } else {
                        for (uint32_t j = off; j < len; ++j) red_add1(col + (p[j] & 0x7F80u));
                    }
                }
            }
        }
        __syncthreads();
        // fold the 32 columns of bin `tid`, starting at its own lane so a
        // warp's 32 reads fall in 32 different banks
        uint32_t sum = 0;
#pragma unroll 8
        for (uint32_t i = 0; i < 32; ++i) sum += s_hist[tid * 32 + ((i + tid) & 31)];
        const uint32_t cnt = sum - prev;
        prev = sum;
        a.tile_hist[t * 256 + tid] = cnt;
        seg_acc += cnt;
        __syncthreads();  // folds done before the next tile's counts land
    }
    if (cur != 0xFFFFFFFFu && seg_acc) atomicAdd(&a.seg_hist[(size_t)cur * 256 + tid], seg_acc);
}

// ---------------------------------------------------------- top-16 select
// One block per segment.  Threads 0..255: the rank of exponent t is the
// number of exponents before it in (count desc, exponent asc); ranks 0..15
// form the codebook and e = n - (sum of their counts).  With a caller's
// codebook, that codebook is used instead (repeated entries: invalid).
// Then all threads: escapes of tile j = its length - (its counts of the 16
// codebook exponents), and an exclusive scan over the segment's tiles gives
// every tile the index of its first escape record.
constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectArgs a) {
    __shared__ uint32_t s_cnt[256];
    __shared__ uint8_t s_cb[16];
    __shared__ unsigned long long s_sum;
    __shared__ int s_valid;
    __shared__ uint32_t s_warp[kSelThreads / 32];
    __shared__ uint32_t s_carry;
    const uint32_t k = blockIdx.x;
    const uint32_t t = threadIdx.x;
    const sz_segment seg = load_segment(a.batch, k);
    const uint64_t n = seg.n_elems;
    if (t < 256) s_cnt[t] = a.seg_hist[(size_t)k * 256 + t];
    if (t == 0) {
        s_sum = 0;
        s_valid = 1;
        s_carry = 0;
    }
    __syncthreads();
    if (a.codebook_in == nullptr) {
        if (t < 256) {
            const uint32_t c = s_cnt[t];
            uint32_t rank = 0;
#pragma unroll 8
            for (uint32_t u = 0; u < 256; ++u) {
                const uint32_t cu = s_cnt[u];
                rank += (cu > c) || (cu == c && u < t);
            }
            if (rank < 16) {
                s_cb[rank] = (uint8_t)t;
                atomicAdd(&s_sum, (unsigned long long)c);
            }
        }
    } else {
        if (t < 16) s_cb[t] = a.codebook_in[t];
        __syncthreads();
        if (t < 16) {
            for (int j = 0; j < 16; ++j)
                if (j != (int)t && s_cb[j] == s_cb[t]) s_valid = 0;
            atomicAdd(&s_sum, (unsigned long long)s_cnt[s_cb[t]]);
        }
    }
    __syncthreads();
    const uint64_t top = s_sum;
    const bool valid = s_valid != 0 && top <= n;
    const uint64_t e = valid ? n - top : 0;
    if (t < 16) {
        a.meta[k].codebook[t] = s_cb[t];
        if (a.codebooks_out) a.codebooks_out[(size_t)k * 16 + t] = s_cb[t];
    }
    if (a.hist_out && t < 256) a.hist_out[t] = s_cnt[t];
    if (t == 0) {
        a.meta[k].n_escapes = e;
        a.meta[k].valid = valid ? 1u : 0u;
        a.meta[k].pad = 0;
    }

    // per-tile first escape index
    uint32_t cb[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) cb[q] = s_cb[q];
    const uint32_t tiles = (uint32_t)segment_tiles(n, a.batch.page_elems);
    const int lane = t & 31, wid = t >> 5;
    for (uint32_t base = 0; base < tiles; base += kSelThreads) {
        const uint32_t j = base + t;
        uint32_t cnt = 0;
        if (j < tiles) {
            const uint32_t *h = a.tile_hist + (size_t)(seg.tile_begin + j) * 256;
            uint32_t in_cb = 0;
#pragma unroll
            for (int q = 0; q < 16; ++q) in_cb += h[cb[q]];
            const TileRef r = resolve_tile(a.batch, seg, k, seg.tile_begin + j);
            cnt = r.len - in_cb;
        }
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) s_warp[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            uint32_t w = s_warp[lane];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, d);
                if (lane >= d) w += y;
            }
            s_warp[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const uint32_t carry = s_carry;
        const uint32_t excl = carry + (wid ? s_warp[wid - 1] : 0u) + incl - cnt;
        if (j < tiles) a.tile_off[seg.tile_begin + j] = excl;
        __syncthreads();
        if (t == kSelThreads - 1) s_carry = carry + s_warp[kSelThreads / 32 - 1];
        __syncthreads();
    }
}

// ------------------------------------------------------------ launchers
cudaError_t launch_hist(const HistArgs &a0, bool batched, int grid, cudaStream_t s) {
    HistArgs a = a0;
    if (a.batch.n_tiles == 0) return cudaSuccess;
    grid = (int)umin64((uint64_t)grid, a.batch.n_tiles);
    a.tiles_per_cta = div_up(a.batch.n_tiles, (uint64_t)grid);
    grid = (int)div_up(a.batch.n_tiles, a.tiles_per_cta);
    const size_t smem = kHistWords * sizeof(uint32_t);
    if (batched)
        hist_kernel<true><<<grid, kThreads, smem, s>>>(a);
    else
        hist_kernel<false><<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s) {
    const uint32_t segs = a.batch.segs ? a.batch.n_segs : 1u;
    if (segs == 0) return cudaSuccess;
    select_kernel<<<segs, kSelThreads, 0, s>>>(a);
    return cudaGetLastError();
}

int hist_blocks_per_sm() {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, hist_kernel<true>, kThreads,
                                                  kHistWords * sizeof(uint32_t));
    return occ > 0 ? occ : 1;
}

}  // namespace sz
