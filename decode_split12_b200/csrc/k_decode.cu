// k_decode.cu -- standalone Split12 decode: container -> BF16 matrix.
//
// Each lane owns 16 consecutive weights (one 128-bit raw load, one 64-bit
// code load, two 128-bit stores); a warp covers 512 weights = 4 tiles.  The
// exponent is base + code, a byte-wise integer ADD ("GPU 友善 12 位無損 BF16
// 壓縮格式", key points); code-15 weights take their exact value from the
// escape stream, located by the tile's prefix offset and the weight's rank
// among the tile's escapes.  HBM-bound: it reads 1.5 bytes per weight plus
// 5 bytes per tile plus 2 bytes per escape and writes 2 bytes per weight.
#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

struct DecodeParams {
    const uint8_t *__restrict__ raw;
    const uint8_t *__restrict__ code;
    const uint8_t *__restrict__ base;
    const uint32_t *__restrict__ esc_off;
    const uint16_t *__restrict__ esc;
    uint64_t n_esc;
    uint64_t n16;  // number of 16-weight chunks = rows*cols/16
    uint16_t *__restrict__ out;
    uint32_t *err;
};

constexpr int kDecodeUnroll = 2;

__global__ void __launch_bounds__(256) decode_kernel(DecodeParams p) {
    const int lane = threadIdx.x & 31;
    const uint64_t warp = (static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const uint64_t n_warps = (static_cast<uint64_t>(gridDim.x) * blockDim.x) >> 5;
    const uint64_t n_wchunks = (p.n16 + 31) / 32;

    for (uint64_t wc = warp; wc < n_wchunks; wc += n_warps * kDecodeUnroll) {
        uint4 raw[kDecodeUnroll];
        uint2 code[kDecodeUnroll];
        uint32_t b[kDecodeUnroll], lo[kDecodeUnroll], hi[kDecodeUnroll];
        bool active[kDecodeUnroll];
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            const uint64_t q = (wc + u * n_warps) * 32 + lane;
            active[u] = q < p.n16;
            raw[u] = make_uint4(0, 0, 0, 0);
            code[u] = make_uint2(0, 0);
            b[u] = 0;
            lo[u] = hi[u] = 0;
            if (active[u]) {
                raw[u] = __ldcs(reinterpret_cast<const uint4 *>(p.raw) + q);
                code[u] = __ldcs(reinterpret_cast<const uint2 *>(p.code) + q);
                const uint64_t t = q >> 3;
                b[u] = __ldg(p.base + t);
                lo[u] = __ldg(p.esc_off + t);
                hi[u] = __ldg(p.esc_off + t + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kDecodeUnroll; ++u) {
            if (wc + u * n_warps >= n_wchunks) break;  // warp-uniform
            const uint64_t q = (wc + u * n_warps) * 32 + lane;
            if (b[u] > kMaxBase) raise_flag(p.err, S12_FLAG_BASE);
            const uint32_t B4 = b[u] * 0x01010101u;
            const uint32_t m0 = escape_nibbles(code[u].x), m1 = escape_nibbles(code[u].y);
            uint32_t w[8];
            decode16(raw[u], code[u], B4, w);
            const bool any = (m0 | m1) != 0;
            if (__ballot_sync(0xFFFFFFFFu, any)) {
                fix_escapes(w, raw[u], code[u], B4, m0, m1, lo[u], hi[u], active[u], p.n_esc, p.esc, p.err);
            } else if (active[u] && lo[u] != hi[u]) {
                raise_flag(p.err, S12_FLAG_ESC_COUNT);
            }
            if (active[u]) {
                uint4 *o = reinterpret_cast<uint4 *>(p.out) + 2 * q;
                __stcs(o, make_uint4(w[0], w[1], w[2], w[3]));
                __stcs(o + 1, make_uint4(w[4], w[5], w[6], w[7]));
            }
        }
    }
}

int launch_decode(const s12_view *v, uint16_t *out, uint32_t *err, cudaStream_t stream) {
    if (v->version != 1) return S12_ERR_ARG;
    DecodeParams p;
    p.raw = v->raw;
    p.code = v->code;
    p.base = v->base;
    p.esc_off = v->esc_off;
    p.esc = v->esc;
    p.n_esc = v->n_esc;
    p.n16 = v->rows * v->cols / 16;
    p.out = out;
    p.err = err;
    int sms = 0, per_sm = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel, 256, 0) != cudaSuccess)
        return S12_ERR_CUDA;
    const uint64_t need = (p.n16 + 255) / 256;
    uint64_t grid = static_cast<uint64_t>(sms) * (per_sm > 0 ? per_sm : 1);
    if (grid > need) grid = need;
    if (grid == 0) grid = 1;
    decode_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace s12
