// s12_load.cu -- whole-tensor load with fallback to the original BF16
// weights.
//
// "Lossless LLM Weight Compression vs 8-bit GGUF", section "A 14-day
// production-readiness pilot": keep the original BF16 weights beside the
// compressed ones, check what was loaded, and serve a tensor that fails a
// check from its original copy instead of from a wrong decode.  This call is
// that step for one tensor: host validation and plane hashes first, then the
// device decode with its err_flag, and the caller's BF16 copy (or a
// rejection the caller can act on, for instance by reloading) when any check
// fails.
#include <cstring>

#include "s12_device.cuh"
#include "s12_launch.h"

using namespace s12;

namespace {

// Host checks: validation and, if given, the expected plane hashes.
void host_checks(const void *container, size_t bytes, const uint64_t *expected, s12_load_result *res) {
    s12_report rep;
    if (s12_validate_host(container, bytes, &rep) != S12_OK) {
        res->problem = rep.problem ? rep.problem : S12_BAD_HEADER;
        return;
    }
    if (expected) {
        uint64_t h[5];
        if (s12_plane_hashes_host(container, bytes, h) != S12_OK) {
            res->problem = S12_BAD_HEADER;
            return;
        }
        for (int i = 0; i < 5; ++i)
            if (h[i] != expected[i]) res->hash_mismatch |= 1u << i;
    }
}

}  // namespace

extern "C" int s12_load_bf16(const void *container, size_t bytes, const uint64_t *expected_hashes,
                             const uint16_t *fallback, uint64_t rows, uint64_t cols, void *dev_container,
                             size_t dev_cap, uint16_t *dev_out, uint32_t *dev_err, s12_load_result *res,
                             void *stream) {
    if (!container || !res || !dev_container || !dev_out || !dev_err || rows == 0 || cols == 0)
        return S12_ERR_ARG;
    if (cols % kTile) return S12_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(dev_container) & 255) || (reinterpret_cast<uintptr_t>(dev_out) & 15) ||
        (reinterpret_cast<uintptr_t>(dev_err) & 3))
        return S12_ERR_ALIGN;
    std::memset(res, 0, sizeof *res);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t out_bytes = static_cast<size_t>(rows) * cols * 2;

    host_checks(container, bytes, expected_hashes, res);
    bool ok = res->problem == 0 && res->hash_mismatch == 0;
    if (ok) {
        // the header (valid by now) must describe the tensor the caller expects
        uint64_t shape[2];
        std::memcpy(shape, static_cast<const uint8_t *>(container) + 8, sizeof shape);
        if (shape[0] != rows || shape[1] != cols) {
            res->problem = S12_BAD_HEADER;
            ok = false;
        }
    }
    if (ok) {
        if (bytes > dev_cap) return S12_ERR_CAPACITY;
        // (s12_open reads the header back through the legacy default stream:
        // the copy must have landed first)
        if (cudaMemcpyAsync(dev_container, container, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemsetAsync(dev_err, 0, 4, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
            return S12_ERR_CUDA;
        s12_view v;
        int rc = s12_open(dev_container, bytes, &v);
        if (rc != S12_OK) return rc;
        rc = s12_decode(&v, dev_out, dev_err, stream);
        if (rc != S12_OK) return rc;
        uint32_t flags = 0;
        if (cudaMemcpyAsync(&flags, dev_err, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess)
            return S12_ERR_CUDA;
        res->device_flags = flags;
        if (flags == 0) {
            res->outcome = S12_LOAD_DECODED;
            return S12_OK;
        }
    }
    if (!fallback) {
        res->outcome = S12_LOAD_REJECTED;
        return S12_OK;
    }
    if (cudaMemcpyAsync(dev_out, fallback, out_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return S12_ERR_CUDA;
    res->outcome = S12_LOAD_FALLBACK;
    return S12_OK;
}
