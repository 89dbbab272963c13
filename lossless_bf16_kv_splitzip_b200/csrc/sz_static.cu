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
cudaError_t launch_hist(const HistArgs &a, bool batched, int grid, cudaStream_t s);
cudaError_t launch_select(const SelectArgs &a, cudaStream_t s);
cudaError_t launch_encode(const EncodeArgs &a, bool batched, int grid, cudaStream_t s);
int hist_blocks_per_sm();
int encode_blocks_per_sm();
}  // namespace sz

using namespace sz;

namespace {

// Scratch layout for one tensor of at most SZ_STATIC_MAX_ELEMS elements:
//   [0, 1024)      exponent counts of the tensor, u32[256]
//   [1024, 1056)   SegMeta (codebook, escape count)
//   [1280, ...)    exponent counts of every 65,536-element tile, u32[T][256]
//   then           first escape index of every tile, u32[T]
constexpr uint64_t kMaxTiles = (SZ_STATIC_MAX_ELEMS + kTile - 1) / kTile;
constexpr uint64_t kOffSegHist = 0;
constexpr uint64_t kOffMeta = 1024;
constexpr uint64_t kOffTileHist = 1280;
constexpr uint64_t kOffTileOff = kOffTileHist + 1024 * kMaxTiles;
constexpr uint64_t kStaticScratchBytes = kOffTileOff + 4 * kMaxTiles;
static_assert(kStaticScratchBytes == SZ_STATIC_SCRATCH_BYTES, "header and layout agree");

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

struct StaticDevice {
    bool ready = false;
    uint8_t *scratch = nullptr;  // device address of g_static_scratch on that device
    int sms = 0, hist_occ = 1, enc_occ = 1;
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
        d.hist_occ = hist_blocks_per_sm();
        d.enc_occ = encode_blocks_per_sm();
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

    // The array keeps the previous call's contents: the tensor counts are
    // accumulated with atomics and must start at zero; everything else is
    // overwritten before it is read.
    if (cudaMemsetAsync(ws + kOffSegHist, 0, 1024, s) != cudaSuccess) return SZ_ERR_CUDA;
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
    h.batch = b;
    h.base = d_in;
    h.seg_hist = reinterpret_cast<uint32_t *>(ws + kOffSegHist);
    h.tile_hist = reinterpret_cast<uint32_t *>(ws + kOffTileHist);
    if (launch_hist(h, false, dev.sms * dev.hist_occ, s) != cudaSuccess) return SZ_ERR_CUDA;

    SelectArgs sa{};
    sa.batch = b;
    sa.seg_hist = h.seg_hist;
    sa.tile_hist = h.tile_hist;
    sa.meta = reinterpret_cast<SegMeta *>(ws + kOffMeta);
    sa.tile_off = reinterpret_cast<uint32_t *>(ws + kOffTileOff);
    sa.codebooks_out = d_codebook16_or_null;
    if (launch_select(sa, s) != cudaSuccess) return SZ_ERR_CUDA;

    EncodeArgs a{};
    a.batch = b;
    a.base = d_in;
    a.out = d_out;
    a.out_cap = out_cap;
    a.out_bytes = d_out_bytes;
    a.status = d_status;
    a.meta = sa.meta;
    a.tile_off = sa.tile_off;
    a.wait_limit_ns = 1000000000ull;
    a.debug_flags = 0;
    return launch_encode(a, false, dev.sms * dev.enc_occ, s) == cudaSuccess ? SZ_OK : SZ_ERR_CUDA;
}
