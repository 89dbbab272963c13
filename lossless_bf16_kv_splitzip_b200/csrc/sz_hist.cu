// sz_hist.cu -- exponent histograms and top-16 codebook selection.
//
// SplitZip explainer (gist.science), section 2 "La decouverte secrete": the
// exponents repeat; section 3 "La strategie SplitZip": the 16 most common
// exponents get the 4-bit codes.  The histogram pass reads the input once
// and keeps, besides each segment's 256 counts, the 256 counts of the first
// and last segment piece of every range (the encode's per-CTA share of
// tiles).  The block that completes a segment orders its 256 exponents by
// (count descending, exponent ascending), keeps the first 16, and turns the
// piece counts into the escape count of each of the segment's pieces -- an
// exclusive scan of those gives every encode CTA the index of its first
// escape record, so the encode needs no cross-CTA communication.  There is
// no wait anywhere: the last block of a segment is found with one atomic
// completion count per segment.
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

// ---------------------------------------------------------- top-16 select
// Shared state of one segment's select (256 threads).
struct SelShared {
    RankShared rank;
    uint32_t cnt[256];
    uint32_t warp[kWarps];
    unsigned long long top;
    uint32_t carry;
    int valid;
    int flag;
    uint8_t cb[16];
};

// Codebook, escape count and range records of segment k, by the kThreads
// threads of one block (every one of them must call it).  Thread t holds
// exponent t: its rank is the number of exponents before it in (count
// descending, exponent ascending); ranks 0..15 form the codebook and
// e = n - (sum of their counts).  With a caller's codebook, that codebook is
// used instead (repeated entries: invalid).  Then, for every range the
// segment reaches, the escapes of the segment's piece in it = the piece's
// length - its counts of the 16 codebook exponents; an exclusive scan over
// the ranges places each piece.  Counts written by other blocks are read
// from L2 (__ldcg): they were published before the completion count that
// made this block the segment's last.
__device__ void select_segment(const SelectCtx &a, uint32_t k, const uint8_t *codebook_in, SelShared &ss) {
    const uint32_t tid = threadIdx.x;
    const int lane = tid & 31, wid = tid >> 5;
    const sz_segment seg = load_segment(a.batch, k);
    const uint64_t n = seg.n_elems;
    const uint32_t c = __ldcg(a.seg_hist + (size_t)k * 256 + tid);
    ss.cnt[tid] = c;
    __syncthreads();
    if (codebook_in == nullptr) {
        const uint32_t rank = exponent_rank(c, tid, ss.rank);
        if (rank < 16) ss.cb[rank] = (uint8_t)tid;
    } else if (tid < 16) {
        ss.cb[tid] = codebook_in[tid];
    }
    __syncthreads();
    if (wid == 0) {
        unsigned long long v = 0;
        bool dup = false;
        if (lane < 16) {
            const uint32_t x = ss.cb[lane];
            v = ss.cnt[x];
            for (int j = 0; j < 16; ++j) dup |= (j != lane) && ss.cb[j] == x;
        }
#pragma unroll
        for (int d = 8; d >= 1; d >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, d);
        const bool any_dup = __any_sync(0xFFFFFFFFu, dup) != 0;
        if (lane == 0) {
            ss.top = v;
            ss.valid = (!any_dup && v <= n) ? 1 : 0;
            ss.carry = 0;
        }
    }
    __syncthreads();
    const bool valid = ss.valid != 0;
    const uint64_t e = valid ? n - ss.top : 0;
    if (tid < 16) {
        a.meta[k].codebook[tid] = ss.cb[tid];
        if (a.codebooks_out) a.codebooks_out[(size_t)k * 16 + tid] = ss.cb[tid];
    }
    if (a.hist_out) a.hist_out[tid] = c;
    if (tid == 0) {
        a.meta[k].n_escapes = e;
        a.meta[k].valid = valid ? 1u : 0u;
        a.meta[k].pad = 0;
    }
    if (n == 0) return;

    // ---- the segment's pieces: one per range it reaches
    const uint64_t R = a.range_tiles;
    const uint64_t G = range_count(a.batch.n_tiles, R);
    const uint64_t t_first = seg.tile_begin;
    const uint64_t t_last = t_first + seg_tiles(a.batch, n) - 1;
    const uint64_t b_first = t_first / R, b_last = t_last / R;
    if (b_first == b_last) {  // inside one range: only a range-opening segment has a record
        if (tid == 0 && t_first == b_first * R) {
            a.rrec[b_first].first_off = 0;
            a.rrec[b_first].first_cnt = (uint32_t)e;
        }
        return;
    }
    uint32_t cbq[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) cbq[q] = ss.cb[q];
    for (uint64_t base = b_first; base <= b_last; base += kThreads) {
        const uint64_t b = base + tid;
        uint32_t cnt = 0;
        bool opens = false;  // the piece opens its range (else it closes it)
        if (b <= b_last) {
            const uint64_t ps = umax64(t_first, b * R), pe = umin64(t_last + 1, (b + 1) * R);
            opens = ps == b * R;
            uint64_t in = 0;
#pragma unroll
            for (int q = 0; q < 16; ++q) in += __ldcg(a.rhist + rhist_at(G, opens ? 0u : 1u, cbq[q], b));
            const TileRef r0 = resolve_tile(a.batch, seg, k, ps);
            const TileRef r1 = resolve_tile(a.batch, seg, k, pe - 1);
            const uint64_t len = r1.elem0 + r1.len - r0.elem0;
            cnt = in <= len ? (uint32_t)(len - in) : 0u;
        }
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += y;
        }
        if (lane == 31) ss.warp[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            uint32_t w = lane < kWarps ? ss.warp[lane] : 0u;
#pragma unroll
            for (int d = 1; d < kWarps; d <<= 1) {
                const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, d);
                if (lane >= d) w += y;
            }
            if (lane < kWarps) ss.warp[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const uint32_t carry = ss.carry;
        const uint32_t excl = carry + (wid ? ss.warp[wid - 1] : 0u) + incl - cnt;
        if (b <= b_last) {
            RangeRec &rr = a.rrec[b];
            if (opens) {
                rr.first_off = excl;
                rr.first_cnt = cnt;
            } else {
                rr.last_cnt = cnt;
            }
        }
        __syncthreads();
        if (tid == 0) ss.carry = carry + ss.warp[kWarps - 1];
        __syncthreads();
    }
}

// Segments with no elements have no tiles, so no range completes them:
// their codebook is exponents 0..15 (all counts zero) and e = 0.
__device__ inline void empty_segments(const HistArgs &h) {
    const SelectCtx &a = h.sel;
    const uint32_t ns = a.batch.segs ? a.batch.n_segs : 1u;
    for (uint32_t k = threadIdx.x; k < ns; k += kThreads) {
        if (load_segment(a.batch, k).n_elems != 0) continue;
        SegMeta &m = a.meta[k];
        for (int q = 0; q < 16; ++q) {
            m.codebook[q] = (uint8_t)q;
            if (a.codebooks_out) a.codebooks_out[(size_t)k * 16 + q] = (uint8_t)q;
        }
        m.n_escapes = 0;
        m.valid = 1;
        m.pad = 0;
    }
    if (a.hist_out && a.batch.segs == nullptr && a.batch.single.n_elems == 0)
        for (uint32_t i = threadIdx.x; i < 256; i += kThreads) a.hist_out[i] = 0;
}

// ------------------------------------------------------------- histogram
// The tiles of range blockIdx.x counted piece by piece (a piece = the
// range's tiles of one segment) by the block's kThreads threads, into the
// 256 x 32 lane columns s_hist (zeroed, and seg_cache filled, before);
// at the end of a piece its 256 counts are the difference of the column
// sums, added to the segment's counts, and kept when the piece opens or
// closes the range.  The block that completes a segment's tile count runs
// that segment's select.
// kAccum: the piece counts go to the caller's histograms instead (no range
// records, no completion count, no select).
template <bool kBatched, bool kAccum>
__device__ __forceinline__ void count_range(const HistArgs &a, uint32_t *s_hist, const SegCache &s_segc, SelShared &s_sel) {
    const Batch &batch = a.sel.batch;
    const uint32_t tid = threadIdx.x;
    const uint32_t col = smem_u32(s_hist) + (tid & 31) * 4;
    const uint64_t R = a.sel.range_tiles;
    const uint64_t t_begin = (uint64_t)blockIdx.x * R;
    const uint64_t t_end = umin64(t_begin + R, batch.n_tiles);

    uint32_t prev = 0;  // column sum of bin `tid` at the last piece boundary
    uint64_t t = t_begin;
    while (t < t_end) {
        const uint32_t k = find_segment(s_segc, batch, t);
        const sz_segment seg = load_segment(batch, k);
        const uint64_t n_seg_tiles = seg_tiles(batch, seg.n_elems);
        const uint64_t ps = t, pe = umin64(seg.tile_begin + n_seg_tiles, t_end);  // the piece [ps, pe)
        for (; t < pe; ++t) {
            const TileRef r = resolve_tile(batch, seg, k, t);
            const uint16_t *src = kBatched ? a.pages[seg.page_begin + r.page] + r.in_page : a.base + r.elem0;
            const bool ok = (reinterpret_cast<uintptr_t>(src) & 15) == 0;
            if (!ok && tid == 0) set_status(a.status ? a.status + k : nullptr, SZ_ERR_ALIGN);
            for (uint32_t sub = 0; ok && sub < r.n_subs; ++sub) {
                const uint16_t *p = src + sub * kSub;
                const uint32_t len = umin32(kSub, r.len - sub * kSub);
                // bulk prefetch of the next sub-tile into L2 while this one is
                // counted: inside the tile, or -- a single stream of one-sub-tile
                // tiles, where the next tile follows in memory -- the next tile's
                if (tid == 0) {
                    uint64_t rest = 0;
                    if (sub + 1 < r.n_subs) rest = r.len - (sub + 1) * kSub;
                    else if (!kBatched && batch.tile_subs == 1 && t + 1 < t_end) rest = r.n - (r.elem0 + r.len);
                    const uint32_t next = ((uint32_t)umin64(kSub, rest) * 2u) & ~15u;
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
        }
        __syncthreads();
        // fold the 32 columns of bin `tid`, starting at its own lane so a
        // warp's 32 reads fall in 32 different banks
        uint32_t sum = 0;
#pragma unroll 8
        for (uint32_t i = 0; i < 32; ++i) sum += s_hist[tid * 32 + ((i + tid) & 31)];
        const uint32_t acc = sum - prev;
        prev = sum;
        if (kAccum) {
            const size_t row = a.accum_index ? a.accum_index[k] : k;
            if (acc) atomicAdd(&a.accum[row * 256 + tid], acc);
            __syncthreads();  // folds done before the next piece's counts land
            continue;
        }
        if (ps == t_begin) a.rhist[rhist_at(gridDim.x, 0, tid, blockIdx.x)] = acc;
        else if (pe == t_end) a.rhist[rhist_at(gridDim.x, 1, tid, blockIdx.x)] = acc;
        if (acc) atomicAdd(&a.seg_hist[(size_t)k * 256 + tid], acc);
        __threadfence();
        __syncthreads();  // folds done before the next piece's counts land
        if (tid == 0) {
            const uint32_t add = (uint32_t)(pe - ps);
            s_sel.flag = atomicAdd(&a.seg_done[k], add) + add == (uint32_t)n_seg_tiles;
        }
        __syncthreads();
        if (s_sel.flag) {  // every other piece of segment k is counted and published
            __threadfence();
            select_segment(a.sel, k, nullptr, s_sel);
        }
    }
}


// ------------------------------------------------------------- histogram
// One block per range (count_range).  kSmallTiles: every tile is a single
// sub-tile (pages of at most 16,384 elements, or the one-sub-tile tiles of
// a short single stream); that build is given registers for 3 blocks per
// SM -- measured 0.70 -> 0.86 of the copy bandwidth on 16-token pages,
// while the same bound costs 8 % on 65,536-element tiles.  Those get a
// bound of 5 blocks per SM (at most 51 registers; unbounded, the compiler
// chose 32 and spilled): 0.706 -> 0.680 ms on the 64-tensor batch, with the
// largest shared-memory carveout holding 5 blocks.
template <bool kBatched, bool kSmallTiles, bool kAccum>
__global__ void __launch_bounds__(kThreads, kSmallTiles ? 3 : 5) hist_kernel(const HistArgs a) {
    extern __shared__ __align__(128) uint32_t s_hist[];  // kHistWords
    __shared__ SegCache s_segc;
    __shared__ SelShared s_sel;
    static_assert(kThreads == 256, "one thread per bin");
    allow_dependents();  // the encode kernel may start its prologue
    if (blockIdx.x == 0 && threadIdx.x == 0) {  // words only the next kernel reads
        if (a.reset_status) *a.reset_status = SZ_OK;
        if (a.reset_size) *a.reset_size = 0;
    }
    for (uint32_t i = threadIdx.x; i < kHistWords; i += kThreads) s_hist[i] = 0;
    seg_cache_fill(s_segc, a.sel.batch);  // ends with __syncthreads
    if (!kAccum && blockIdx.x == 0) empty_segments(a);
    count_range<kBatched, kAccum>(a, s_hist, s_segc, s_sel);
}

// Caller codebook for a single tensor: the select again with that codebook,
// unless it is the one the workspace already holds.  Also resets the
// encode's status, size and completion words.
__global__ void __launch_bounds__(kThreads) reselect_kernel(const ReselectArgs a) {
    __shared__ SelShared s_sel;
    __shared__ int s_same;
    if (threadIdx.x == 0) {
        *a.status = SZ_OK;
        *a.out_bytes = 0;
        *a.enc_done = 0;
        s_same = a.sel.meta[0].valid != 0;
    }
    __syncthreads();
    if (threadIdx.x < 16 && a.sel.meta[0].codebook[threadIdx.x] != a.codebook_in[threadIdx.x]) s_same = 0;
    __syncthreads();
    if (s_same) return;
    select_segment(a.sel, 0, a.codebook_in, s_sel);
}

// Codebook of each of a list of caller histograms (one block per
// histogram): the 16 exponents of rank 0..15 and, optionally, the escape
// count = the histogram's total - the codebook's counts.
__global__ void __launch_bounds__(kThreads) select_kernel(const uint32_t *hists, uint8_t *codebooks,
                                                          uint64_t *escapes) {
    __shared__ RankShared s_rank;
    __shared__ unsigned long long s_sum[2][kWarps];  // [0]: all counts, [1]: codebook counts
    const uint32_t tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const uint32_t c = hists[(size_t)blockIdx.x * 256 + tid];
    const uint32_t rank = exponent_rank(c, tid, s_rank);
    if (rank < 16) codebooks[(size_t)blockIdx.x * 16 + rank] = (uint8_t)tid;
    if (escapes == nullptr) return;
    unsigned long long all = c, top = rank < 16 ? c : 0u;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        all += __shfl_down_sync(0xFFFFFFFFu, all, d);
        top += __shfl_down_sync(0xFFFFFFFFu, top, d);
    }
    if (lane == 0) {
        s_sum[0][wid] = all;
        s_sum[1][wid] = top;
    }
    __syncthreads();
    if (tid == 0) {
        unsigned long long ta = 0, tt = 0;
        for (int w = 0; w < kWarps; ++w) {
            ta += s_sum[0][w];
            tt += s_sum[1][w];
        }
        escapes[blockIdx.x] = ta - tt;
    }
}

// ------------------------------------------------------------ launchers
template <bool kAccum>
void launch_hist_t(const HistArgs &a, bool batched, int grid, size_t smem, cudaStream_t s) {
    const bool small = a.sel.batch.page_elems <= kSub || a.sel.batch.tile_elems <= kSub;
    // 65,536-element tiles: the largest shared-memory carveout (64-tensor
    // batch right after a decode: 0.734 -> 0.678 ms; back to back with no
    // other kernel between it is 0.619 -> 0.671 ms, the cost of the smaller
    // L1).  The accumulate mode keeps the driver's carveout (0.115 -> 0.099
    // ms per 512 MiB prefill chunk), and so does the one-sub-tile build.
    if (batched && small) {
        hist_kernel<true, true, kAccum><<<grid, kThreads, smem, s>>>(a);
    } else if (batched) {
        if (!kAccum) prefer_max_shared<hist_kernel<true, false, kAccum>>();
        hist_kernel<true, false, kAccum><<<grid, kThreads, smem, s>>>(a);
    } else if (small) {
        hist_kernel<false, true, kAccum><<<grid, kThreads, smem, s>>>(a);
    } else {
        if (!kAccum) prefer_max_shared<hist_kernel<false, false, kAccum>>();
        hist_kernel<false, false, kAccum><<<grid, kThreads, smem, s>>>(a);
    }
}

// a.accum set: the accumulate mode
cudaError_t launch_hist(const HistArgs &a, bool batched, cudaStream_t s) {
    const int grid = (int)umax64(1, div_up(a.sel.batch.n_tiles, a.sel.range_tiles));
    const size_t smem = kHistWords * sizeof(uint32_t);
    if (a.accum != nullptr)
        launch_hist_t<true>(a, batched, grid, smem, s);
    else
        launch_hist_t<false>(a, batched, grid, smem, s);
    return cudaGetLastError();
}

cudaError_t launch_select(const uint32_t *hists, uint32_t n_hists, uint8_t *codebooks, uint64_t *escapes,
                          cudaStream_t s) {
    if (n_hists == 0) return cudaSuccess;
    select_kernel<<<n_hists, kThreads, 0, s>>>(hists, codebooks, escapes);
    return cudaGetLastError();
}

cudaError_t launch_reselect(const ReselectArgs &a, cudaStream_t s) {
    reselect_kernel<<<1, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace sz
