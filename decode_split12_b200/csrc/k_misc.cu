// k_misc.cu -- the plain BF16 GEMV used as the uncompressed comparison point
// (the exponent histogram of s12_stats runs on the decode kernel, k_decode.cu).
#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

// ---------------------------------------------------------------------------
// Plain BF16 GEMV (uncompressed baseline).  One warp per row, 128-bit loads
// of 8 weights per lane, four loads in flight per lane, x read through the
// read-only cache, FP32 accumulation and a shuffle reduction.
template <int B>
__global__ void __launch_bounds__(256) bf16_gemv_kernel(const uint16_t *__restrict__ w, int64_t R, int64_t K,
                                                        const uint16_t *__restrict__ x, float *__restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t K8 = K / 8;
    for (int64_t row = warp; row < R; row += n_warps) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(w + row * K);
        float acc[B];
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = 0.f;
        for (int64_t k8 = lane; k8 < K8; k8 += 32 * 4) {
            uint4 wv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                wv[u] = (k8 + 32 * u < K8) ? __ldcs(wr + k8 + 32 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (k8 + 32 * u >= K8) break;
                const uint32_t ww[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + b * K) + k8 + 32 * u);
                    const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[b] = fmaf(__uint_as_float(ww[q] << 16), __uint_as_float(xx[q] << 16), acc[b]);
                        acc[b] = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), __uint_as_float(xx[q] & 0xFFFF0000u),
                                      acc[b]);
                    }
                }
            }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float v = acc[b];
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, d);
            if (lane == 0) y[b * R + row] = v;
        }
    }
}

template <int B>
static cudaError_t run_bf16(const uint16_t *w, int64_t R, int64_t K, const uint16_t *x, float *y,
                            cudaStream_t stream) {
    int sms = 0, per_sm = 0;
    cudaError_t e = device_sms(&sms);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bf16_gemv_kernel<B>, 256, 0);
    if (e != cudaSuccess) return e;
    int64_t grid = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
    const int64_t need = (R + 7) / 8;
    if (grid > need) grid = need;
    bf16_gemv_kernel<B><<<static_cast<unsigned>(grid), 256, 0, stream>>>(w, R, K, x, y);
    return cudaGetLastError();
}

int launch_bf16_gemv(const uint16_t *w, int64_t rows, int64_t cols, const uint16_t *x, int B, float *y,
                     cudaStream_t stream) {
    cudaError_t e;
    switch (B) {
        case 1: e = run_bf16<1>(w, rows, cols, x, y, stream); break;
        case 2: e = run_bf16<2>(w, rows, cols, x, y, stream); break;
        case 3: e = run_bf16<3>(w, rows, cols, x, y, stream); break;
        case 4: e = run_bf16<4>(w, rows, cols, x, y, stream); break;
        case 5: e = run_bf16<5>(w, rows, cols, x, y, stream); break;
        case 6: e = run_bf16<6>(w, rows, cols, x, y, stream); break;
        case 7: e = run_bf16<7>(w, rows, cols, x, y, stream); break;
        default: e = run_bf16<8>(w, rows, cols, x, y, stream); break;
    }
    return e == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace s12
