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

using namespace sz;

namespace {

// Scratch layout for one tensor of at most SZ_STATIC_MAX_ELEMS elements
// (at most kMaxRanges = 1024 ranges, whatever the tile size):
//   [0, 1024)      exponent counts of the tensor, u32[256]      } cleared
//   [1024, 1028)   tiles counted so far                         } by every
//   [1028, 1032)   tiles of complete encode pieces              } call
//   [1280, 1312)   SegMeta (codebook, escape count)
//   [1536, ...)    counts of each range's first and last piece, u32[1024][2][256]
//   then           escape placement of each range, RangeRec[1024]
constexpr uint64_t kRanges = kMaxRanges;
static_assert(SZ_STATIC_MAX_ELEMS / kTile >= kMaxRanges, "a stream at the limit may use every range");
constexpr uint64_t kOffSegHist = 0;
constexpr uint64_t kOffSegDone = 1024;
constexpr uint64_t kOffEncDone = 1028;
constexpr uint64_t kOffMeta = 1280;
constexpr uint64_t kOffRhist = 1536;
constexpr uint64_t kOffRrec = kOffRhist + 2048 * kRanges;
constexpr uint64_t kStaticScratchBytes = kOffRrec + sizeof(RangeRec) * kRanges;
static_assert(kStaticScratchBytes == SZ_STATIC_SCRATCH_BYTES, "header and layout agree");

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
uint8_t *g_static_addr[kMaxDevices];  // device address of g_static_scratch, per device

// Once per device, with that device current: the device address of the
// scratch array (in host code the array's name is not a device address).
sz_status static_scratch(uint8_t *&out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SZ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SZ_ERR_INVALID;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SZ_ERR_CUDA;
        g_static_addr[dev] = static_cast<uint8_t *>(p);
    }
    out = g_static_addr[dev];
    return SZ_OK;
}

}  // namespace

extern "C" sz_status sz_encode_static(const uint16_t *d_in, uint64_t n, uint8_t *d_out, uint64_t out_cap,
                                      uint64_t *d_out_bytes, uint8_t *d_codebook16_or_null, int32_t *d_status,
                                      void *stream) {
    if (!d_out || !d_out_bytes || !d_status || (n > 0 && !d_in)) return SZ_ERR_NULL;
    if (n > SZ_STATIC_MAX_ELEMS) return SZ_ERR_TOO_LARGE;
    if ((n > 0 && (reinterpret_cast<uintptr_t>(d_in) & 15) != 0) || (reinterpret_cast<uintptr_t>(d_out) & 15) != 0)
        return SZ_ERR_ALIGN;
    if (out_cap < 48 + n + (n + 1) / 2) return SZ_ERR_CAPACITY;
    uint8_t *ws = nullptr;
    if (const sz_status st = static_scratch(ws)) return st;
    DeviceInfo dev;
    if (const sz_status st = device_info(dev)) return st;
    // The array keeps the previous call's contents: the tensor counts and
    // the two completion counts are cleared first; everything else is
    // overwritten before it is read.
    CompressScratch cs;
    cs.zero = ws + kOffSegHist;
    cs.zero_bytes = kOffEncDone + 4;
    cs.seg_hist = reinterpret_cast<uint32_t *>(ws + kOffSegHist);
    cs.seg_done = reinterpret_cast<uint32_t *>(ws + kOffSegDone);
    cs.enc_done = reinterpret_cast<uint32_t *>(ws + kOffEncDone);
    cs.meta = reinterpret_cast<SegMeta *>(ws + kOffMeta);
    cs.rhist = reinterpret_cast<uint32_t *>(ws + kOffRhist);
    cs.rrec = reinterpret_cast<RangeRec *>(ws + kOffRrec);
    return compress_pipelined(d_in, n, d_out, out_cap, d_out_bytes, d_codebook16_or_null, d_status, cs, dev,
                              static_cast<cudaStream_t>(stream));
}
