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

#include <cudaTypedefs.h>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace {

constexpr int kMaxSms = 160;
constexpr uint64_t kMaxRows = 1ull << 20;
// the same partial-sum and counter regions s12_gemv_ws_bytes sizes, for the
// largest device and container this array serves
constexpr uint64_t kPartBytes = gemv_part_bytes(kMaxSms);
constexpr uint64_t kCntBytes = gemv_cnt_bytes(kMaxRows / 16);
constexpr uint64_t kScratchBytes = kPartBytes + kCntBytes;
static_assert(kScratchBytes == 2883584, "the documented size of the static workspace");

// The workspace.  Host code must not use the name as an address (on the host
// it names a stand-in object, not device memory); the device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_gemv_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};
CUcontext g_ctx[kMaxDevices] = {};
PFN_cuCtxGetCurrent_v4000 g_get_ctx = nullptr;
std::once_flag g_get_ctx_once;

// Device address of g_gemv_scratch for the current device, looked up with
// that device current the first time it is needed and cached.  The cache is
// keyed on the current context as well as the device: after cudaDeviceReset
// (or with another context current) the module lives elsewhere, so the
// address is looked up again.
int scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return S12_ERR_CUDA;
    std::call_once(g_get_ctx_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    });
    if (!g_get_ctx) return S12_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (g_get_ctx(&ctx) != CUDA_SUCCESS) return S12_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!ctx || !g_addr[dev] || g_ctx[dev] != ctx) {
        // (the lookup also makes the runtime's context current on this
        // thread if no CUDA call has done so yet)
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess || !p) return S12_ERR_CUDA;
        if (g_get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return S12_ERR_CUDA;
        g_addr[dev] = p;
        g_ctx[dev] = ctx;
    }
    *out = g_addr[dev];
    return S12_OK;
}

}  // namespace
}  // namespace s12

using namespace s12;

extern "C" int s12_gemv_noalloc(const s12_view *v, const uint16_t *x, int B, float *y, uint32_t *err_flag,
                                void *stream) {
    // the same argument checks and status codes as s12_gemv, first
    void *out[1] = {y};
    int rc = gemv_check(v, 1, &x, B, out, nullptr, err_flag);
    if (rc != S12_OK) return rc;
    if (v->rows > kMaxRows) return S12_ERR_CAPACITY;
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    if (sms > kMaxSms) return S12_ERR_CAPACITY;
    const size_t part = gemv_part_bytes(sms);
    const size_t cnt = gemv_cnt_bytes((v->rows + 15) / 16);
    const size_t need = s12_gemv_ws_bytes(v, B);
    if (need != part + cnt || need > kScratchBytes) return S12_ERR_CAPACITY;
    void *ws = nullptr;
    rc = scratch_address(&ws);
    if (rc != S12_OK) return rc;
    // The arrival counters (the workspace's tail) must start at zero.  Every
    // call leaves them zero, a call whose waits gave up included; clearing
    // this call's counters first (an asynchronous memset, no allocation)
    // also covers a previous call that never ran to its end.  The partial
    // sums need no clearing.
    if (cudaMemsetAsync(static_cast<uint8_t *>(ws) + part, 0, cnt, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return S12_ERR_CUDA;
    return s12_gemv(v, x, B, y, ws, need, err_flag, stream);
}
