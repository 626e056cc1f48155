// s12_noalloc.cu -- s12_gemv_noalloc: the fused decode-GEMV for callers that
// cannot allocate device memory.
//
// s12_gemv needs a small device workspace (the stream-K partial sums and the
// per-row-group arrival counters).  Some callers have no way to provide one:
// a plugin inside an inference engine whose allocator owns every byte of
// device memory, code that runs under a fixed memory budget, or a latency-
// critical path where cudaMalloc's implicit device synchronisation is not
// acceptable.  This entry point serves them with a workspace that is part of
// the library image itself: a file-scope __device__ array, reserved when the
// library's module is loaded on a device and held until the process exits.
//
// Limits (checked on every call, S12_ERR_CAPACITY beyond them):
//   - at most kMaxSms streaming multiprocessors on the device (B200: 148),
//   - at most kMaxRows rows in the container.
// The array is 2,883,584 bytes (2.75 MiB) on every device that loads the
// library.
#include <mutex>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace {

constexpr int kMaxSms = 160;
constexpr uint64_t kMaxRows = 1ull << 20;
constexpr int kWarpsPerSm = 16;       // warps per CTA of the GEMV kernel
constexpr uint64_t kSlotBytes = 512;  // one stream-K partial: 32 lanes x 4 floats
constexpr uint64_t kPartBytes = static_cast<uint64_t>(kMaxSms) * kWarpsPerSm * 2 * kSlotBytes;
constexpr uint64_t kCntBytes = (kMaxRows / 16) * sizeof(uint32_t);
constexpr uint64_t kScratchBytes = kPartBytes + kCntBytes;

// The workspace.  Host code must not use the name as an address (on the host
// it names a stand-in object, not device memory); the device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_gemv_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of g_gemv_scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return S12_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || !p) return S12_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return S12_OK;
}

}  // namespace
}  // namespace s12

using namespace s12;

extern "C" int s12_gemv_noalloc(const s12_view *v, const uint16_t *x, int B, float *y, uint32_t *err_flag,
                                void *stream) {
    if (!v || !x || !y) return S12_ERR_ARG;
    if (v->rows > kMaxRows) return S12_ERR_CAPACITY;
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    if (sms > kMaxSms) return S12_ERR_CAPACITY;
    const size_t need = s12_gemv_ws_bytes(v, B);
    if (need == 0) return S12_ERR_SHAPE;  // invalid view or batch: s12_gemv reports which
    if (need > kScratchBytes) return S12_ERR_CAPACITY;
    void *ws = nullptr;
    int rc = scratch_address(&ws);
    if (rc != S12_OK) return rc;
    // The arrival counters (the workspace's tail) must start at zero.  A
    // completed call leaves them zero, but one cut short by an error may not:
    // clear this call's counters first (an asynchronous memset, no
    // allocation).  The partial sums need no clearing.
    const uint64_t cnt = align_up(((v->rows + 15) / 16) * sizeof(uint32_t), kAlign);
    if (cudaMemsetAsync(static_cast<uint8_t *>(ws) + (need - cnt), 0, cnt,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return S12_ERR_CUDA;
    return s12_gemv(v, x, B, y, ws, need, err_flag, stream);
}
