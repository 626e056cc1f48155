// k_misc.cu -- exponent-histogram kernel for s12_stats and the plain BF16
// GEMV used as the uncompressed comparison point.
#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

// ---------------------------------------------------------------------------
// Exponent histogram of the decoded weights ("你的 bf16 模型,有 5 個 bit 是廢的",
// section 1: the exponent field carries about 2.6 of its 8 bits).  Decodes
// 16 weights per lane exactly as s12_decode does and counts their exponent
// fields in a per-CTA shared histogram.
__global__ void __launch_bounds__(256) exp_hist_kernel(s12_view v, unsigned long long *hist) {
    __shared__ uint32_t s_hist[256];
    s_hist[threadIdx.x] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const uint64_t n16 = v.rows * v.cols / 16;
    const uint64_t warp = (static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const uint64_t n_warps = (static_cast<uint64_t>(gridDim.x) * blockDim.x) >> 5;
    for (uint64_t wc = warp; wc < (n16 + 31) / 32; wc += n_warps) {
        const uint64_t q = wc * 32 + lane;
        const bool active = q < n16;
        uint4 raw = make_uint4(0, 0, 0, 0);
        uint2 code = make_uint2(0, 0);
        uint32_t b = 0, lo = 0, hi = 0;
        if (active) {
            raw = __ldg(reinterpret_cast<const uint4 *>(v.raw) + q);
            code = __ldg(reinterpret_cast<const uint2 *>(v.code) + q);
            b = __ldg(v.base + (q >> 3));
            lo = __ldg(v.esc_off + (q >> 3));
            hi = __ldg(v.esc_off + (q >> 3) + 1);
        }
        const uint32_t B4 = b * 0x01010101u;
        const uint32_t m0 = escape_nibbles(code.x), m1 = escape_nibbles(code.y);
        uint32_t w[8];
        decode16(raw, code, B4, w);
        if (__ballot_sync(0xFFFFFFFFu, (m0 | m1) != 0))
            fix_escapes(w, raw, code, B4, m0, m1, lo, hi, active, v.n_esc, v.esc, nullptr);
        if (active) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                atomicAdd(&s_hist[(w[k] >> 7) & 0xFFu], 1u);
                atomicAdd(&s_hist[(w[k] >> 23) & 0xFFu], 1u);
            }
        }
    }
    __syncthreads();
    if (s_hist[threadIdx.x]) atomicAdd(hist + threadIdx.x, static_cast<unsigned long long>(s_hist[threadIdx.x]));
}

int launch_stats_hist(const s12_view *v, unsigned long long *hist, cudaStream_t stream) {
    if (v->version != 1) return S12_ERR_ARG;
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    if (cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned long long), stream) != cudaSuccess) return S12_ERR_CUDA;
    const uint64_t need = (v->rows * v->cols / 16 + 255) / 256;
    uint64_t grid = static_cast<uint64_t>(sms) * 4;
    if (grid > need) grid = need;
    if (grid == 0) grid = 1;
    exp_hist_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(*v, hist);
    return cudaGetLastError() == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

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
