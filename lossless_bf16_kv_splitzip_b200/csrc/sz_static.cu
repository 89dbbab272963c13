// sz_static.cu -- sz_encode_static: histogram, codebook and container of one
// tensor with no caller workspace and no allocation at all.
//
// Some callers cannot allocate device memory when they compress: code that
// runs inside a custom allocator or a memory-pool callback, a process whose
// device memory is fully reserved up front by a serving engine, or a
// pre-recorded sequence of work that must not touch the allocator.  For them
// the scratch this path needs lives in one file-scope __device__ array,
// loaded with the library: kStaticScratchBytes on every GPU that loads it,
// held until the process exits.  Inputs and outputs still come from the
// caller.
#include <mutex>

#include "sz_internal.cuh"

namespace sz {
cudaError_t launch_hist(const HistArgs &a, bool batched, cudaStream_t s);
cudaError_t launch_encode(const EncodeArgs &a, bool batched, cudaStream_t s);
}  // namespace sz

using namespace sz;

namespace {

// Scratch layout for one tensor of at most SZ_STATIC_MAX_ELEMS elements
// (4096 tiles, so at most kMaxRanges = 1024 ranges):
//   [0, 1024)      exponent counts of the tensor, u32[256]
//   [1024, 1028)   tiles counted so far
//   [1280, 1312)   SegMeta (codebook, escape count)
//   [1536, ...)    counts of each range's first and last piece, u32[1024][2][256]
//   then           escape placement of each range, RangeRec[1024]
constexpr uint64_t kMaxTiles = (SZ_STATIC_MAX_ELEMS + kTile - 1) / kTile;
constexpr uint64_t kRanges = kMaxTiles < kMaxRanges ? kMaxTiles : kMaxRanges;
constexpr uint64_t kOffSegHist = 0;
constexpr uint64_t kOffSegDone = 1024;
constexpr uint64_t kOffMeta = 1280;
constexpr uint64_t kOffRhist = 1536;
constexpr uint64_t kOffRrec = kOffRhist + 2048 * kRanges;
constexpr uint64_t kStaticScratchBytes = kOffRrec + sizeof(RangeRec) * kRanges;
static_assert(kStaticScratchBytes == SZ_STATIC_SCRATCH_BYTES, "header and layout agree");

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

struct StaticDevice {
    bool ready = false;
    uint8_t *scratch = nullptr;  // device address of g_static_scratch on that device
    int sms = 0;
};
std::mutex g_static_mu;
StaticDevice g_static_dev[64];

// Once per device, with that device current: the device address of the
// scratch array (in host code the array's name is not a device address).
bool static_device(StaticDevice &out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(g_static_mu);
    StaticDevice &d = g_static_dev[dev];
    if (!d.ready) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return false;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        d.scratch = static_cast<uint8_t *>(p);
        d.ready = true;
    }
    out = d;
    return true;
}

}  // namespace

extern "C" sz_status sz_encode_static(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap,
                                      uint64_t *d_out_bytes, uint8_t *d_codebook16_or_null, int32_t *d_status,
                                      void *stream) {
    if (!d_out || !d_out_bytes || !d_status || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > SZ_STATIC_MAX_ELEMS) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && (reinterpret_cast<uintptr_t>(d_in) & 15) != 0) || (reinterpret_cast<uintptr_t>(d_out) & 15) != 0)
        return SZ_ERR_ALIGN;
    if (out_cap < container_size(n, 0)) return SZ_ERR_CAPACITY;
    StaticDevice dev;
    if (!static_device(dev)) return SZ_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = dev.scratch;

    // The array keeps the previous call's contents: the tensor counts and
    // the tile count are accumulated with atomics and must start at zero;
    // everything else is overwritten before it is read.
    if (cudaMemsetAsync(ws + kOffSegHist, 0, 1028, s) != cudaSuccess) return SZ_ERR_CUDA;
    if (cudaMemsetAsync(d_out_bytes, 0, sizeof(uint64_t), s) != cudaSuccess) return SZ_ERR_CUDA;
    if (cudaMemsetAsync(d_status, 0, sizeof(int32_t), s) != cudaSuccess) return SZ_ERR_CUDA;

    Batch b{};
    b.segs = nullptr;
    b.n_segs = 1;
    b.page_elems = n > 0 ? n : 1;
    b.tiles_per_page = (uint32_t)tiles_per_page(b.page_elems);
    b.n_tiles = segment_tiles(n, b.page_elems);
    b.single.n_elems = n;

    HistArgs h{};
    h.sel.batch = b;
    h.sel.seg_hist = reinterpret_cast<uint32_t *>(ws + kOffSegHist);
    h.sel.rhist = reinterpret_cast<uint32_t *>(ws + kOffRhist);
    h.sel.meta = reinterpret_cast<SegMeta *>(ws + kOffMeta);
    h.sel.rrec = reinterpret_cast<RangeRec *>(ws + kOffRrec);
    h.sel.range_tiles = plan_ranges(b.n_tiles, (uint64_t)dev.sms).tiles;
    h.sel.codebooks_out = d_codebook16_or_null;
    h.base = d_in;
    h.seg_hist = reinterpret_cast<uint32_t *>(ws + kOffSegHist);
    h.seg_done = reinterpret_cast<uint32_t *>(ws + kOffSegDone);
    h.rhist = reinterpret_cast<uint32_t *>(ws + kOffRhist);
    if (launch_hist(h, false, s) != cudaSuccess) return SZ_ERR_CUDA;

    EncodeArgs a{};
    a.batch = b;
    a.base = d_in;
    a.out = d_out;
    a.out_cap = out_cap;
    a.out_bytes = d_out_bytes;
    a.status = d_status;
    a.meta = h.sel.meta;
    a.rrec = h.sel.rrec;
    a.range_tiles = h.sel.range_tiles;
    a.wait_limit_ns = 1000000000ull;
    a.debug_flags = 0;
    return launch_encode(a, false, s) == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}
