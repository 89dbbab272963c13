// sz_api.cu -- the C ABI declared in include/splitzip.h: argument checks,
// workspace layout and kernel launches.  Everything here is host code; it
// allocates nothing and never synchronises the caller's stream.
#include <atomic>
#include <mutex>

#include "sz_internal.cuh"

namespace sz {
cudaError_t launch_hist(const HistArgs &a, bool batched, cudaStream_t s);
cudaError_t launch_select(const uint32_t *hists, uint32_t n_hists, uint8_t *codebooks, uint64_t *escapes,
                          cudaStream_t s);
cudaError_t launch_reselect(const ReselectArgs &a, cudaStream_t s);
cudaError_t launch_encode(const EncodeArgs &a, bool batched, cudaStream_t s);
cudaError_t launch_encode_one_pass(const EncodeArgs &a, bool batched, cudaStream_t s);
cudaError_t launch_place(const PlaceArgs &a, bool batched, int sms, cudaStream_t s);
cudaError_t launch_small_encode(const uint16_t *in, uint64_t n, const SmallWs &w, uint8_t *out, uint64_t out_cap,
                                uint64_t *out_bytes, uint8_t *codebook_out, int32_t *status, cudaStream_t s);
cudaError_t launch_small_decode(const uint8_t *c, uint64_t cap, uint16_t *out, uint64_t n, int32_t *status,
                                cudaStream_t s);
cudaError_t launch_esc_index(const DecodeArgs &a, bool batched, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, bool batched, int grid, int sms, cudaStream_t s);
int decode_blocks_per_sm();
}  // namespace sz

using namespace sz;

namespace {

constexpr uint64_t kMaxElems = 0xFFFFFFFFull;  // largest n: positions are u32, n < 2^32
constexpr uint64_t kAlign = 256;
constexpr uint64_t kSmallEncodeMax = 1ull << 20;  // sz_compress: 4,096-element blocks up to this many elements (measured crossover 2-4 MiB)
constexpr uint64_t kSmallDecodeMax = 1ull << 17;  // sz_decode: one launch of 4,096-element blocks up to this (measured crossover 256-512 KiB)

std::atomic<uint64_t> g_wait_limit_ns{1000000000ull};
std::atomic<uint32_t> g_debug_flags{0};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

uint64_t round_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ---- workspace layout for S segments, T tiles and G = min(T, kMaxRanges)
// ranges (256-byte aligned parts)
//   seg_hist   u32[S][256]     exponent counts per segment      } zeroed together
//   seg_done   u32[S]          tiles counted so far per segment } by the histogram call
//   enc_done   u32[S]          tiles of complete encode pieces  } (and by the encode call)
//   meta       SegMeta[S]      codebook and escape count per segment
//   rhist      u32[2][256][G]  counts of each range's first and last piece (range-minor)
//   rrec       RangeRec[G]     escape placement of each range's pieces
//   sub_start  u32[ST + S]     first escape index of each sub-tile (decode; S = sub-tiles per tile)
struct Ws {
    uint64_t seg_hist, seg_done, enc_done, meta, rhist, rrec, sub_start, total;
};
Ws ws_layout(uint64_t n_segs, uint64_t n_tiles, uint64_t tile_subs) {
    const uint64_t g = umin64(n_tiles, kMaxRanges);
    Ws w;
    w.seg_hist = 0;
    w.seg_done = 1024 * n_segs;
    w.enc_done = 1028 * n_segs;
    w.meta = round_up(w.enc_done + 4 * n_segs, kAlign);
    w.rhist = round_up(w.meta + sizeof(SegMeta) * n_segs, kAlign);
    w.rrec = round_up(w.rhist + 2048 * g, kAlign);
    w.sub_start = round_up(w.rrec + sizeof(RangeRec) * g, kAlign);
    w.total = round_up(w.sub_start + 4 * (tile_subs * n_tiles + n_segs), kAlign);
    return w;
}

// ---- one-pass workspace for S segments, T tiles and G = min(T, kMaxRanges)
// ranges
//   ovf_count   u32               tiles listed for the rescan      } zeroed
//   blocks_done u32               rescan blocks finished           } per call
//   rcnt      RangeRec[G]         escapes of each range's first and last piece
//   seg_e     u32[S]              escape count of each segment
//   tile_cnt  u32[T]              escapes of each tile
//   ovf       OvfItem[T]          tiles whose records overflowed their slot
//   slots     u32[T][C]           each tile's first C = tile / 16 escape records
struct Ws1 {
    uint64_t ovf_count, blocks_done, rcnt, seg_e, tile_cnt, ovf, slots, total;
};
Ws1 ws1_layout(uint64_t n_segs, uint64_t n_tiles, uint64_t slot_cap) {
    const uint64_t g = umin64(n_tiles, kMaxRanges);
    Ws1 w;
    w.ovf_count = 0;
    w.blocks_done = 4;
    w.rcnt = kAlign;
    w.seg_e = round_up(w.rcnt + sizeof(RangeRec) * g, kAlign);
    w.tile_cnt = round_up(w.seg_e + 4 * n_segs, kAlign);
    w.ovf = round_up(w.tile_cnt + 4 * n_tiles, kAlign);
    w.slots = round_up(w.ovf + sizeof(OvfItem) * n_tiles, kAlign);
    w.total = round_up(w.slots + 4ull * slot_cap * n_tiles, kAlign);
    return w;
}

}  // namespace

namespace sz {

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }
uint32_t debug_flags() { return g_debug_flags.load(); }

sz_status device_info(DeviceInfo &out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SZ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SZ_ERR_INVALID;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SZ_ERR_CUDA;
        d.dec_occ = decode_blocks_per_sm();
        d.ready = true;
    }
    out = d;
    return SZ_OK;
}

Batch single_batch(uint64_t n) {
    Batch b{};
    b.segs = nullptr;
    b.n_segs = 1;
    b.page_elems = n > 0 ? n : 1;
    set_tiles(b, n < kSmallTileBelow ? 1u : kSubsPerTile);
    b.n_tiles = segment_tiles(n, b.page_elems, b.tile_shift);
    b.single.n_elems = n;
    b.single.page_begin = 0;
    b.single.out_offset = 0;
    b.single.tile_begin = 0;
    return b;
}

}  // namespace sz

namespace {

Batch make_batch(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles, uint64_t page_elems) {
    Batch b{};
    b.segs = d_segs;
    b.n_segs = n_segs;
    b.page_elems = page_elems;
    set_tiles(b, kSubsPerTile);
    b.n_tiles = n_tiles;
    return b;
}

// ---- sz_compress's short-stream scratch, for S = ceil(n / 4096) slices
//   [0, 1024) stream counts, [1024, 1028) slices counted, [1028, 1032)
//   slices encoded (zeroed together), [1280, 1312) SegMeta, [1536, ...)
//   first escape index per slice, then u32[S][256] counts per slice
struct WsSmall {
    uint64_t meta, block_off, block_hist, total;
};
WsSmall small_layout(uint64_t n) {
    const uint64_t nb = umax64(1, div_up(n, (uint64_t)kThreads * kChunk));
    WsSmall w;
    w.meta = 1280;
    w.block_off = 1536;
    w.block_hist = round_up(w.block_off + 4 * nb, kAlign);
    w.total = round_up(w.block_hist + 1024 * nb, kAlign);
    return w;
}

Ws single_ws(uint64_t n) {
    const Batch b = single_batch(n);
    Ws w = ws_layout(1, b.n_tiles, b.tile_subs);
    if (n <= kSmallEncodeMax) w.total = umax64(w.total, small_layout(n).total);
    return w;
}

template <class T>
T *at(void *ws, uint64_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

// The select's view of the workspace, with the range partition of this
// device (the histogram and encode calls of one batch derive the same one).
SelectCtx select_ctx(const Batch &b, void *ws, const Ws &w, const DeviceInfo &dev) {
    SelectCtx c{};
    c.batch = b;
    c.seg_hist = at<uint32_t>(ws, w.seg_hist);
    c.rhist = at<uint32_t>(ws, w.rhist);
    c.meta = at<SegMeta>(ws, w.meta);
    c.rrec = at<RangeRec>(ws, w.rrec);
    c.range_tiles = plan_ranges(b.n_tiles, (uint64_t)dev.sms).tiles;
    return c;
}

HistArgs hist_args(const SelectCtx &c, void *ws, const Ws &w) {
    HistArgs h{};
    h.sel = c;
    h.seg_hist = at<uint32_t>(ws, w.seg_hist);
    h.seg_done = at<uint32_t>(ws, w.seg_done);
    h.rhist = at<uint32_t>(ws, w.rhist);
    return h;
}

sz_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SZ_OK : SZ_ERR_CUDA; }

#define SZ_TRY_CUDA(call)                          \
    do {                                           \
        cudaError_t _e = (call);                   \
        if (_e != cudaSuccess) return SZ_ERR_CUDA; \
    } while (0)

// ---- one pass with the caller's codebook(s): encode, then escape placement
sz_status one_pass(const Batch &b, const uint16_t *const *d_pages, const uint16_t *d_in,
                          const uint8_t *d_codebooks, uint8_t *d_out, uint64_t out_cap, uint64_t *d_out_bytes,
                          int32_t *d_status, void *d_ws, const Ws1 &w, cudaStream_t s) {
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    const uint64_t ns = b.segs ? b.n_segs : 1;
    SZ_TRY_CUDA(cudaMemsetAsync(d_out_bytes, 0, 8 * ns, s));
    SZ_TRY_CUDA(cudaMemsetAsync(d_status, 0, 4 * ns, s));
    SZ_TRY_CUDA(cudaMemsetAsync(at<uint8_t>(d_ws, w.ovf_count), 0, 8, s));  // ovf_count, blocks_done
    EncodeArgs a{};
    a.batch = b;
    a.pages = d_pages;
    a.base = d_in;
    a.out = d_out;
    a.out_cap = out_cap;
    a.out_bytes = d_out_bytes;
    a.status = d_status;
    a.range_tiles = plan_ranges(b.n_tiles, (uint64_t)dev.sms).tiles;
    a.wait_limit_ns = wait_limit_ns();
    a.debug_flags = debug_flags();
    a.codebooks_in = d_codebooks;
    a.tile_cnt = at<uint32_t>(d_ws, w.tile_cnt);
    a.slots = at<uint32_t>(d_ws, w.slots);
    a.rcnt = at<RangeRec>(d_ws, w.rcnt);
    if (b.n_tiles > 0) SZ_TRY_CUDA(launch_encode_one_pass(a, b.segs != nullptr, s));
    PlaceArgs p{};
    p.batch = b;
    p.pages = d_pages;
    p.base = d_in;
    p.codebooks_in = d_codebooks;
    p.out = d_out;
    p.out_cap = out_cap;
    p.out_bytes = d_out_bytes;
    p.status = d_status;
    p.tile_cnt = a.tile_cnt;
    p.slots = a.slots;
    p.rcnt = a.rcnt;
    p.range_tiles = a.range_tiles;
    p.ovf_count = at<uint32_t>(d_ws, w.ovf_count);
    p.ovf = at<OvfItem>(d_ws, w.ovf);
    p.seg_e = at<uint32_t>(d_ws, w.seg_e);
    p.blocks_done = at<uint32_t>(d_ws, w.blocks_done);
    return cuda_status(launch_place(p, b.segs != nullptr, dev.sms, s));
}

}  // namespace

namespace sz {

sz_status compress_pipelined(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap,
                             uint64_t *d_out_bytes, uint8_t *d_codebook16_or_null, int32_t *d_status,
                             const CompressScratch &w, const DeviceInfo &dev, cudaStream_t s) {
    SZ_TRY_CUDA(cudaMemsetAsync(w.zero, 0, w.zero_bytes, s));  // seg_hist, seg_done, enc_done
    SelectCtx c{};
    c.batch = single_batch(n);
    c.seg_hist = w.seg_hist;
    c.rhist = w.rhist;
    c.meta = w.meta;
    c.rrec = w.rrec;
    c.range_tiles = plan_ranges(c.batch.n_tiles, (uint64_t)dev.sms).tiles;
    c.codebooks_out = d_codebook16_or_null;
    HistArgs h{};
    h.sel = c;
    h.base = d_in;
    h.seg_hist = w.seg_hist;
    h.seg_done = w.seg_done;
    h.rhist = w.rhist;
    EncodeArgs a{};  // the codebook the histogram kernel chose: no reselect
    a.batch = c.batch;
    a.base = d_in;
    a.out = d_out;
    a.out_cap = out_cap;
    a.out_bytes = d_out_bytes;
    a.status = d_status;
    a.meta = c.meta;
    a.rrec = c.rrec;
    a.range_tiles = c.range_tiles;
    a.enc_done = w.enc_done;
    a.wait_limit_ns = wait_limit_ns();
    a.debug_flags = debug_flags();
    h.reset_status = d_status;  // the histogram kernel sets no status on a single stream
    h.reset_size = d_out_bytes;
    SZ_TRY_CUDA(launch_hist(h, false, s));
    return cuda_status(launch_encode(a, false, s));
}

}  // namespace sz

extern "C" {

sz_status sz_plan(uint64_t n_elems, uint64_t *max_compressed_bytes, uint64_t *workspace_bytes) {
    if (!max_compressed_bytes || !workspace_bytes) return SZ_ERR_NULL;
    if (n_elems > kMaxElems) return SZ_ERR_TOO_LARGE;
    *max_compressed_bytes = SZ_MAX_BYTES(n_elems);
    *workspace_bytes = single_ws(n_elems).total;
    return SZ_OK;
}

sz_status sz_histogram_codebook(const uint16_t *d_in, uint64_t n, uint8_t *d_codebook16,
                                uint32_t *d_hist256_or_null, void *d_ws, uint64_t ws_bytes, void *stream) {
    if (!d_codebook16 || !d_ws || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    const Ws w = single_ws(n);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SZ_TRY_CUDA(cudaMemsetAsync(at<uint8_t>(d_ws, w.seg_hist), 0, w.meta - w.seg_hist, s));  // seg_hist, seg_done, enc_done
    SelectCtx c = select_ctx(single_batch(n), d_ws, w, dev);
    c.codebooks_out = d_codebook16;
    c.hist_out = d_hist256_or_null;
    HistArgs h = hist_args(c, d_ws, w);
    h.base = d_in;
    return cuda_status(launch_hist(h, false, s));
}

sz_status sz_encode(const uint16_t *d_in, uint64_t n, const uint8_t *d_codebook16, uint8_t *d_out,
                    uint64_t out_cap, uint64_t *d_out_bytes, int32_t *d_status, void *d_ws, uint64_t ws_bytes,
                    void *stream) {
    if (!d_codebook16 || !d_out || !d_out_bytes || !d_status || !d_ws || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_out) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    if (out_cap < container_size(n, 0)) return SZ_ERR_CAPACITY;
    const Ws w = single_ws(n);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // escape count and range records for this codebook, from the piece
    // counts sz_histogram_codebook left in the workspace (nothing to do when
    // it is the codebook chosen there); also resets *d_status, *d_out_bytes
    ReselectArgs ra{};
    ra.sel = select_ctx(single_batch(n), d_ws, w, dev);
    ra.codebook_in = d_codebook16;
    ra.status = d_status;
    ra.out_bytes = d_out_bytes;
    ra.enc_done = at<uint32_t>(d_ws, w.enc_done);
    SZ_TRY_CUDA(launch_reselect(ra, s));
    EncodeArgs a{};
    a.batch = ra.sel.batch;
    a.base = d_in;
    a.out = d_out;
    a.out_cap = out_cap;
    a.out_bytes = d_out_bytes;
    a.status = d_status;
    a.meta = ra.sel.meta;
    a.rrec = ra.sel.rrec;
    a.range_tiles = ra.sel.range_tiles;
    a.enc_done = ra.enc_done;
    a.wait_limit_ns = wait_limit_ns();
    a.debug_flags = debug_flags();
    return cuda_status(launch_encode(a, false, s));
}

sz_status sz_decode(const uint8_t *d_in, uint64_t in_bytes, uint16_t *d_out, uint64_t n, int32_t *d_status,
                    void *d_ws, uint64_t ws_bytes, void *stream) {
    if (!d_in || !d_status || !d_ws || (n > 0 && !d_out)) return SZ_ERR_NULL;
    if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
    if (!aligned16(d_in) || (n > 0 && !aligned16(d_out)) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    const Ws w = single_ws(n);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (n <= kSmallDecodeMax) {
        SZ_TRY_CUDA(cudaMemsetAsync(d_status, 0, sizeof(int32_t), s));
        return cuda_status(launch_small_decode(d_in, in_bytes, d_out, n, d_status, s));
    }
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    DecodeArgs a{};
    a.batch = single_batch(n);
    a.base = d_out;
    a.in = d_in;
    a.in_cap = in_bytes;
    a.status = d_status;
    a.sub_start = at<uint32_t>(d_ws, w.sub_start);
    a.wait_limit_ns = wait_limit_ns();
    a.debug_flags = debug_flags();
    SZ_TRY_CUDA(launch_esc_index(a, false, s));
    return cuda_status(launch_decode(a, false, dev.sms * dev.dec_occ, dev.sms, s));
}

sz_status sz_compress(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap, uint64_t *d_out_bytes,
                      uint8_t *d_codebook16_or_null, int32_t *d_status, void *d_ws, uint64_t ws_bytes, void *stream) {
    if (!d_out || !d_out_bytes || !d_status || !d_ws || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_out) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    if (out_cap < container_size(n, 0)) return SZ_ERR_CAPACITY;
    const Ws w = single_ws(n);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (n <= kSmallEncodeMax) {  // short stream: one memset, two launches over 4,096-element slices
        const WsSmall ws = small_layout(n);
        SZ_TRY_CUDA(cudaMemsetAsync(d_ws, 0, 1032, s));
        SmallWs sw;
        sw.seg_hist = at<uint32_t>(d_ws, 0);
        sw.done = at<uint32_t>(d_ws, 1024);
        sw.done2 = at<uint32_t>(d_ws, 1028);
        sw.meta = at<SegMeta>(d_ws, ws.meta);
        sw.block_off = at<uint32_t>(d_ws, ws.block_off);
        sw.block_hist = at<uint32_t>(d_ws, ws.block_hist);
        return cuda_status(
            launch_small_encode(d_in, n, sw, d_out, out_cap, d_out_bytes, d_codebook16_or_null, d_status, s));
    }
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    CompressScratch cs;
    cs.zero = at<uint8_t>(d_ws, w.seg_hist);
    cs.zero_bytes = w.meta - w.seg_hist;
    cs.seg_hist = at<uint32_t>(d_ws, w.seg_hist);
    cs.seg_done = at<uint32_t>(d_ws, w.seg_done);
    cs.enc_done = at<uint32_t>(d_ws, w.enc_done);
    cs.meta = at<SegMeta>(d_ws, w.meta);
    cs.rhist = at<uint32_t>(d_ws, w.rhist);
    cs.rrec = at<RangeRec>(d_ws, w.rrec);
    return compress_pipelined(d_in, n, d_out, out_cap, d_out_bytes, d_codebook16_or_null, d_status, cs, dev, s);
}

sz_status sz_plan_batched(uint32_t n_segs, const uint64_t *h_seg_elems, uint64_t page_elems, sz_segment *h_segs,
                          uint64_t *total_pages, uint64_t *n_tiles, uint64_t *out_bytes,
                          uint64_t *workspace_bytes) {
    if ((n_segs > 0 && (!h_seg_elems || !h_segs)) || !total_pages || !n_tiles || !out_bytes || !workspace_bytes)
        return SZ_ERR_NULL;
    if (page_elems == 0) return SZ_ERR_INVALID;
    uint64_t pages = 0, tiles = 0, out = 0;
    bool multi_page = false;
    for (uint32_t k = 0; k < n_segs; ++k) {
        const uint64_t n = h_seg_elems[k];
        if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
        multi_page |= n > page_elems;
        h_segs[k].n_elems = n;
        h_segs[k].page_begin = pages;
        h_segs[k].out_offset = out;
        h_segs[k].tile_begin = tiles;
        pages += div_up(n, page_elems);
        tiles += segment_tiles(n, page_elems, 16);
        out += round_up(SZ_MAX_BYTES(n), kAlign);
    }
    if (multi_page && page_elems % 64 != 0) return SZ_ERR_ALIGN;
    if (tiles > 0xFFFFFFFFull) return SZ_ERR_TOO_LARGE;
    *total_pages = pages;
    *n_tiles = tiles;
    *out_bytes = out;
    *workspace_bytes = ws_layout(n_segs, tiles, kSubsPerTile).total;
    return SZ_OK;
}

sz_status sz_histogram_codebook_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                                        const uint16_t *const *d_pages, uint64_t page_elems,
                                        uint8_t *d_codebooks_or_null, int32_t *d_status, void *d_ws,
                                        uint64_t ws_bytes, void *stream) {
    if (n_segs == 0) return SZ_OK;
    if (!d_segs || !d_status || !d_ws || (n_tiles > 0 && !d_pages)) return SZ_ERR_NULL;
    if (page_elems == 0) return SZ_ERR_INVALID;
    if (!aligned16(d_ws)) return SZ_ERR_ALIGN;
    const Ws w = ws_layout(n_segs, n_tiles, kSubsPerTile);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SZ_TRY_CUDA(cudaMemsetAsync(at<uint8_t>(d_ws, w.seg_hist), 0, w.meta - w.seg_hist, s));  // seg_hist, seg_done, enc_done
    SZ_TRY_CUDA(cudaMemsetAsync(d_status, 0, 4 * (uint64_t)n_segs, s));
    SelectCtx c = select_ctx(make_batch(n_segs, d_segs, n_tiles, page_elems), d_ws, w, dev);
    c.codebooks_out = d_codebooks_or_null;
    HistArgs h = hist_args(c, d_ws, w);
    h.pages = d_pages;
    h.status = d_status;
    return cuda_status(launch_hist(h, true, s));
}

sz_status sz_encode_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                            const uint16_t *const *d_pages, uint64_t page_elems, uint8_t *d_out, uint64_t out_cap,
                            uint64_t *d_out_bytes, int32_t *d_status, void *d_ws, uint64_t ws_bytes,
                            void *stream) {
    if (n_segs == 0) return SZ_OK;
    if (!d_segs || !d_out || !d_out_bytes || !d_status || !d_ws || (n_tiles > 0 && !d_pages)) return SZ_ERR_NULL;
    if (page_elems == 0) return SZ_ERR_INVALID;
    if (!aligned16(d_out) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    const Ws w = ws_layout(n_segs, n_tiles, kSubsPerTile);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SZ_TRY_CUDA(cudaMemsetAsync(d_out_bytes, 0, 8 * (uint64_t)n_segs, s));
    SZ_TRY_CUDA(cudaMemsetAsync(at<uint8_t>(d_ws, w.enc_done), 0, 4 * (uint64_t)n_segs, s));
    const SelectCtx c = select_ctx(make_batch(n_segs, d_segs, n_tiles, page_elems), d_ws, w, dev);
    EncodeArgs a{};
    a.batch = c.batch;
    a.pages = d_pages;
    a.out = d_out;
    a.out_cap = out_cap;
    a.out_bytes = d_out_bytes;
    a.status = d_status;
    a.meta = c.meta;
    a.rrec = c.rrec;
    a.range_tiles = c.range_tiles;
    a.enc_done = at<uint32_t>(d_ws, w.enc_done);
    a.wait_limit_ns = wait_limit_ns();
    a.debug_flags = debug_flags();
    return cuda_status(launch_encode(a, true, s));
}

sz_status sz_decode_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles, const uint8_t *d_in,
                            uint64_t in_cap, uint16_t *const *d_pages, uint64_t page_elems, int32_t *d_status,
                            void *d_ws, uint64_t ws_bytes, void *stream) {
    if (n_segs == 0) return SZ_OK;
    if (!d_segs || !d_in || !d_status || !d_ws || (n_tiles > 0 && !d_pages)) return SZ_ERR_NULL;
    if (page_elems == 0) return SZ_ERR_INVALID;
    if (!aligned16(d_in) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    const Ws w = ws_layout(n_segs, n_tiles, kSubsPerTile);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DecodeArgs a{};  // the index kernel writes every segment's status
    a.batch = make_batch(n_segs, d_segs, n_tiles, page_elems);
    a.pages = d_pages;
    a.in = d_in;
    a.in_cap = in_cap;
    a.status = d_status;
    a.sub_start = at<uint32_t>(d_ws, w.sub_start);
    a.wait_limit_ns = wait_limit_ns();
    a.debug_flags = debug_flags();
    SZ_TRY_CUDA(launch_esc_index(a, true, s));
    return cuda_status(launch_decode(a, true, dev.sms * dev.dec_occ, dev.sms, s));
}

sz_status sz_plan_one_pass(uint64_t n_elems, uint64_t *max_compressed_bytes, uint64_t *workspace_bytes) {
    if (!max_compressed_bytes || !workspace_bytes) return SZ_ERR_NULL;
    if (n_elems > kMaxElems) return SZ_ERR_TOO_LARGE;
    *max_compressed_bytes = container_size(n_elems, n_elems);
    const Batch b = single_batch(n_elems);
    *workspace_bytes = ws1_layout(1, b.n_tiles, slot_cap(b)).total;
    return SZ_OK;
}

sz_status sz_encode_one_pass(const uint16_t *d_in, uint64_t n, const uint8_t *d_codebook16, uint8_t *d_out,
                             uint64_t out_cap, uint64_t *d_out_bytes, int32_t *d_status, void *d_ws,
                             uint64_t ws_bytes, void *stream) {
    if (!d_codebook16 || !d_out || !d_out_bytes || !d_status || !d_ws || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_out) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    if (out_cap < container_size(n, 0)) return SZ_ERR_CAPACITY;
    const Batch b = single_batch(n);
    const Ws1 w = ws1_layout(1, b.n_tiles, slot_cap(b));
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    return one_pass(b, nullptr, d_in, d_codebook16, d_out, out_cap, d_out_bytes, d_status, d_ws, w,
                    static_cast<cudaStream_t>(stream));
}

sz_status sz_workspace_one_pass_batched(uint32_t n_segs, uint64_t n_tiles, uint64_t *workspace_bytes) {
    if (!workspace_bytes) return SZ_ERR_NULL;
    if (n_tiles > 0xFFFFFFFFull) return SZ_ERR_TOO_LARGE;
    *workspace_bytes = ws1_layout(n_segs, n_tiles, kTile / kSlotDiv).total;
    return SZ_OK;
}

sz_status sz_encode_one_pass_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                                     const uint16_t *const *d_pages, uint64_t page_elems,
                                     const uint8_t *d_codebooks, uint8_t *d_out, uint64_t out_cap,
                                     uint64_t *d_out_bytes, int32_t *d_status, void *d_ws, uint64_t ws_bytes,
                                     void *stream) {
    if (n_segs == 0) return SZ_OK;
    if (!d_segs || !d_codebooks || !d_out || !d_out_bytes || !d_status || !d_ws || (n_tiles > 0 && !d_pages))
        return SZ_ERR_NULL;
    if (page_elems == 0) return SZ_ERR_INVALID;
    if (n_tiles > 0xFFFFFFFFull) return SZ_ERR_TOO_LARGE;
    if (!aligned16(d_out) || !aligned16(d_ws)) return SZ_ERR_ALIGN;
    const Ws1 w = ws1_layout(n_segs, n_tiles, kTile / kSlotDiv);
    if (ws_bytes < w.total) return SZ_ERR_WORKSPACE;
    return one_pass(make_batch(n_segs, d_segs, n_tiles, page_elems), d_pages, nullptr, d_codebooks, d_out, out_cap,
                    d_out_bytes, d_status, d_ws, w, static_cast<cudaStream_t>(stream));
}

sz_status sz_histogram_accumulate(const uint16_t *d_in, uint64_t n, uint32_t *d_hist256, void *stream) {
    if (!d_hist256 || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > kMaxElems) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && !aligned16(d_in)) || (reinterpret_cast<uintptr_t>(d_hist256) & 3) != 0) return SZ_ERR_ALIGN;
    if (n == 0) return SZ_OK;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    HistArgs h{};
    h.sel.batch = single_batch(n);
    h.sel.range_tiles = plan_ranges(h.sel.batch.n_tiles, (uint64_t)dev.sms).tiles;
    h.base = d_in;
    h.accum = d_hist256;
    return cuda_status(launch_hist(h, false, static_cast<cudaStream_t>(stream)));
}

sz_status sz_histogram_accumulate_batched(uint32_t n_segs, const sz_segment *d_segs, uint64_t n_tiles,
                                          const uint16_t *const *d_pages, uint64_t page_elems,
                                          const uint32_t *d_hist_index_or_null, uint32_t *d_hists,
                                          int32_t *d_status, void *stream) {
    if (n_segs == 0) return SZ_OK;
    if (!d_segs || !d_hists || !d_status || (n_tiles > 0 && !d_pages)) return SZ_ERR_NULL;
    if (page_elems == 0) return SZ_ERR_INVALID;
    if (n_tiles > 0xFFFFFFFFull) return SZ_ERR_TOO_LARGE;
    if ((reinterpret_cast<uintptr_t>(d_hists) & 3) != 0) return SZ_ERR_ALIGN;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    SZ_TRY_CUDA(cudaMemsetAsync(d_status, 0, 4 * (uint64_t)n_segs, s));
    if (n_tiles == 0) return SZ_OK;
    HistArgs h{};
    h.sel.batch = make_batch(n_segs, d_segs, n_tiles, page_elems);
    h.sel.range_tiles = plan_ranges(n_tiles, (uint64_t)dev.sms).tiles;
    h.pages = d_pages;
    h.status = d_status;
    h.accum = d_hists;
    h.accum_index = d_hist_index_or_null;
    return cuda_status(launch_hist(h, true, s));
}

sz_status sz_select_codebook(const uint32_t *d_hist256, uint8_t *d_codebook16, uint64_t *d_escapes_or_null,
                             void *stream) {
    return sz_select_codebook_batched(1, d_hist256, d_codebook16, d_escapes_or_null, stream);
}

sz_status sz_select_codebook_batched(uint32_t n_hists, const uint32_t *d_hists, uint8_t *d_codebooks,
                                     uint64_t *d_escapes_or_null, void *stream) {
    if (n_hists == 0) return SZ_OK;
    if (!d_hists || !d_codebooks) return SZ_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(d_hists) & 3) != 0 || (reinterpret_cast<uintptr_t>(d_escapes_or_null) & 7) != 0)
        return SZ_ERR_ALIGN;
    return cuda_status(launch_select(d_hists, n_hists, d_codebooks, d_escapes_or_null,
                                     static_cast<cudaStream_t>(stream)));
}

sz_status sz_set_wait_limit_ns(uint64_t limit_ns) {
    g_wait_limit_ns.store(limit_ns);
    return SZ_OK;
}

sz_status sz_debug_set_flags(uint32_t flags) {
    g_debug_flags.store(flags);
    return SZ_OK;
}

uint64_t sz_tile_elems(void) { return kTile; }  // batched calls and single streams of 2^27 elements or more

const char *sz_version(void) { return "splitzip-b200 1.1 sm_100a"; }

}  // extern "C"
