// sz_hist.cu -- exponent histogram and top-16 codebook selection.
//
// SplitZip explainer (gist.science), section 2 "La decouverte secrete": the
// exponents repeat; section 3 "La strategie SplitZip": the 16 most common
// exponents get the 4-bit codes.  The histogram is the full read of the
// input that finds them; the select step orders all 256 exponents by
// (count descending, exponent ascending) and keeps the first 16.
#include "sz_internal.cuh"

namespace sz {

// ------------------------------------------------------------- histogram
// Shared-memory layout: 256 bins x 32 lane columns of u32, bin-major, so the
// counter of (bin e, lane l) is word e*32 + l and lives in bank l: the 32
// lanes of a warp never collide, whatever exponents they hold.  All warps of
// the CTA share the 32 columns (lane l of every warp adds into column l).
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

// Fold the 32 columns of each bin and add them to the global histogram.
// Thread b owns bin b; it walks the columns starting at its own lane so a
// warp's 32 reads fall in 32 different banks.
__device__ void flush_hist(uint32_t *s_hist, uint32_t *g_hist) {
    __syncthreads();
    const uint32_t b = threadIdx.x;
    uint32_t sum = 0;
#pragma unroll 8
    for (uint32_t i = 0; i < 32; ++i) {
        const uint32_t idx = b * 32 + ((i + b) & 31);
        sum += s_hist[idx];
        s_hist[idx] = 0;
    }
    if (sum) atomicAdd(&g_hist[b], sum);
    __syncthreads();
}

template <bool kBatched>
__global__ void __launch_bounds__(kThreads) hist_kernel(const HistArgs a) {
    extern __shared__ __align__(128) uint32_t s_hist[];  // kHistWords
    __shared__ SegCache s_segc;
    static_assert(kThreads == 256, "one thread per bin in flush_hist");

    for (uint32_t i = threadIdx.x; i < kHistWords; i += kThreads) s_hist[i] = 0;
    if (kBatched) seg_cache_fill(s_segc, a.batch);
    __syncthreads();

    const uint32_t tid = threadIdx.x;
    const uint32_t col = (uint32_t)__cvta_generic_to_shared(s_hist) + (tid & 31) * 4;
    const uint64_t t_begin = (uint64_t)blockIdx.x * a.tiles_per_cta;
    const uint64_t t_end = umin64(t_begin + a.tiles_per_cta, a.batch.n_tiles);

    uint32_t cur = 0xFFFFFFFFu;
    sz_segment seg{};
    for (uint64_t t = t_begin; t < t_end; ++t) {
        const uint32_t k = find_segment(s_segc, a.batch, t);
        if (k != cur) {
            if (cur != 0xFFFFFFFFu) flush_hist(s_hist, a.hist + (size_t)cur * 256);
            cur = k;
            seg = load_segment(a.batch, k);
        }
        const TileRef r = resolve_tile(a.batch, seg, k, t);
        const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
        if (kBatched && (reinterpret_cast<uintptr_t>(src) & 15) != 0) {
            if (tid == 0) set_status(a.status ? a.status + k : nullptr, SZ_ERR_ALIGN);
            continue;
        }
        if (r.len == kTile) {
            uint4 v[2 * kChunks];
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                const uint16_t *p = src + (c * kThreads + tid) * kChunk;
                v[2 * c] = ld_stream_v4(p);
                v[2 * c + 1] = ld_stream_v4(p + 8);
            }
#pragma unroll
            for (int i = 0; i < 2 * kChunks; ++i) count_v4(v[i], col);
        } else {
            for (int c = 0; c < kChunks; ++c) {
                const uint32_t off = (c * kThreads + tid) * kChunk;
                if (off + kChunk <= r.len) {
                    count_v4(ld_stream_v4(src + off), col);
                    count_v4(ld_stream_v4(src + off + 8), col);
                } else {
                    for (uint32_t j = off; j < r.len; ++j) red_add1(col + (src[j] & 0x7F80u));
                }
            }
        }
    }
    if (cur != 0xFFFFFFFFu) flush_hist(s_hist, a.hist + (size_t)cur * 256);
}

// ---------------------------------------------------------- top-16 select
// One block per segment, one thread per exponent.  The rank of exponent t is
// the number of exponents that come before it in (count desc, exponent asc);
// ranks 0..15 form the codebook.  e = n - (sum of the 16 counts).
__global__ void __launch_bounds__(256) select_kernel(const SelectArgs a) {
    __shared__ uint32_t s_cnt[256];
    __shared__ uint8_t s_cb[16];
    __shared__ unsigned long long s_sum;
    const uint32_t k = blockIdx.x;
    const uint32_t t = threadIdx.x;
    const uint32_t c = a.hist[(size_t)k * 256 + t];
    s_cnt[t] = c;
    if (t == 0) s_sum = 0;
    __syncthreads();
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
    __syncthreads();
    const uint64_t n = a.segs ? a.segs[k].n_elems : a.single_n;
    if (t < 16) {
        a.meta[k].codebook[t] = s_cb[t];
        if (a.codebooks_out) a.codebooks_out[(size_t)k * 16 + t] = s_cb[t];
    }
    if (a.hist_out) a.hist_out[t] = c;
    if (t == 0) {
        const uint64_t top = s_sum;
        a.meta[k].n_escapes = top <= n ? n - top : 0;
        a.meta[k].valid = top <= n ? 1u : 0u;  // a histogram larger than n is not this input's
        a.meta[k].pad = 0;
    }
}

// Escape count for a caller-chosen codebook (single-tensor sz_encode): the
// histogram left in the workspace by sz_histogram_codebook gives
// e = n - sum(hist[codebook[k]]); repeated entries make the codebook invalid.
__global__ void prepare_kernel(const uint8_t *codebook, const uint32_t *hist, uint64_t n, SegMeta *meta) {
    __shared__ uint8_t s_cb[16];
    const uint32_t t = threadIdx.x;
    if (t < 16) s_cb[t] = codebook[t];
    __syncthreads();
    if (t == 0) {
        uint32_t valid = 1;
        uint64_t top = 0;
        for (int i = 0; i < 16; ++i) {
            for (int j = i + 1; j < 16; ++j) valid &= (s_cb[i] != s_cb[j]) ? 1u : 0u;
            top += hist[s_cb[i]];
            meta->codebook[i] = s_cb[i];
        }
        if (top > n) valid = 0;
        meta->n_escapes = valid ? n - top : 0;
        meta->valid = valid;
        meta->pad = 0;
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
    if (batched) {
        cudaFuncSetAttribute(hist_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        hist_kernel<true><<<grid, kThreads, smem, s>>>(a);
    } else {
        cudaFuncSetAttribute(hist_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        hist_kernel<false><<<grid, kThreads, smem, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s) {
    if (a.n_segs == 0) return cudaSuccess;
    select_kernel<<<a.n_segs, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prepare(const uint8_t *codebook, const uint32_t *hist, uint64_t n, SegMeta *meta,
                           cudaStream_t s) {
    prepare_kernel<<<1, 32, 0, s>>>(codebook, hist, n, meta);
    return cudaGetLastError();
}

int hist_blocks_per_sm() {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, hist_kernel<true>, kThreads,
                                                  kHistWords * sizeof(uint32_t));
    return occ > 0 ? occ : 1;
}

}  // namespace sz
