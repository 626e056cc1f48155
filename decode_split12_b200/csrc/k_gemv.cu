// k_gemv.cu -- fused Split12 decode-GEMV for batch 1..8 on sm_100a.
//
//   y[b][n] = sum_k W[n][k] * x[b][k]
//
// The weights stay compressed in HBM; the exact BF16 values are rebuilt in
// registers and used at once in the product ("Lossless LLM Weight
// Compression vs 8-bit GGUF", section "What does 'lossless' mean for LLM
// weights?": decode into registers or shared memory and multiply
// immediately).  The kernel is HBM-bound: it must move the compressed planes
// (1.5 bytes per weight + 5 bytes per tile + 2 bytes per escape) at close to
// the copy bandwidth.
//
// Work: a CTA owns a contiguous range of rows (one persistent CTA per SM).
// Each row is cut into passes of up to 4 tiles (512 columns); the CTA's
// passes, in row-major order, are dealt to its NW warps in contiguous, equal
// ranges, so every warp streams the same number of bytes and no warp waits
// for another.  The activations x are staged once per CTA in shared memory
// by the TMA engine (a bulk copy per batch row).
//
// A warp streams its range U passes at a time: every lane first issues the
// loads of its 16 weights of each of the U passes (one 128-bit load of raw
// bytes, one 64-bit load of codes, the tile's base byte and escape offsets;
// streaming cache policy), then decodes them -- a byte-wise base + code ADD
// and byte permutes into BF16 pairs -- and multiplies them with the BF16
// activations by FMAs that take BF16 inputs and accumulate in FP32, one
// accumulator set per pass.  Many warps per SM keep enough loads in flight
// to cover the HBM latency.  The passes' sums are then folded into rows:
// when the row changes the warp reduces with shuffles; rows wholly inside
// its range go straight to y, the at most two rows it shares with
// neighbouring warps are combined at the end in warp order, so y is
// deterministic.  Code-15 weights take their exact value from the escape
// stream (rare, out-of-line path).
//
// Launched with programmatic dependent launch: the weight loads of a CTA's
// first passes may start before the previous kernel in the stream has
// finished; x and y wait for it.
#include <algorithm>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

constexpr int kPassTiles = 4;   // tiles per pass
constexpr int kU = 4;           // passes whose loads are in flight together
constexpr int kMaxWarps = 32;   // warps per CTA at most

struct GemvParams {
    const uint8_t *__restrict__ raw;
    const uint8_t *__restrict__ code;
    const uint8_t *__restrict__ base;
    const uint32_t *__restrict__ esc_off;
    const uint16_t *__restrict__ esc;
    uint64_t n_esc;
    const uint16_t *__restrict__ x;
    float *__restrict__ y;
    uint32_t *err;
    int R, K, T, SPR;  // rows, columns, tiles per row, passes per row
    int NW;            // warps per CTA
    int x_smem;        // 1: x staged in shared memory
    uint32_t x_off, part_off;
};

// Boundary partial sums: the first and last rows of a warp's range that
// other warps share.
template <int B>
struct Part {
    int row[2];
    float v[2][B];
};

// Consumer warps per CTA for batch B: enough warps to hide the HBM latency
// within the register budget of the batch's accumulators.
template <int B>
constexpr int warps_for_batch() {
    return B == 1 ? 32 : (B <= 3 ? 16 : 8);
}

// acc0 += lo(w) * lo(x), acc1 += hi(w) * hi(x): BF16 operands, FP32 accumulate.
__device__ __forceinline__ void fma_bf16x2(float &acc0, float &acc1, uint32_t w, uint32_t x) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(w), "r"(x));
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// A position in this CTA's pass sequence: CTA-relative row and pass in row.
struct PassPos {
    int r, j;
};

template <int B>
__global__ void __launch_bounds__(32 * warps_for_batch<B>(), 1) gemv_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.R, K = p.K, T = p.T, SPR = p.SPR, NW = p.NW;
    const int r0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * R / gridDim.x);
    const int r1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * R / gridDim.x);
    const int n_pass = (r1 - r0) * SPR;
    // this warp's passes [pa, pb)
    const int pa = static_cast<int>(static_cast<int64_t>(warp) * n_pass / NW);
    const int pb = static_cast<int>(static_cast<int64_t>(warp + 1) * n_pass / NW);
    uint64_t *xbar = reinterpret_cast<uint64_t *>(smem);
    Part<B> *parts = reinterpret_cast<Part<B> *>(smem + p.part_off);

    if (threadIdx.x == 0) {
        mbar_init(xbar, 1);
        fence_barrier_init();
        grid_launch_dependents();
    }
    if (lane == 0) parts[warp].row[0] = parts[warp].row[1] = -1;
    __syncthreads();
    if (threadIdx.x == 0) {
        grid_dependency_wait();  // x may be written by the previous kernel in the stream
        if (p.x_smem) {
            mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(B * K * 2));
            for (int b = 0; b < B; ++b)
                tma_load_1d(smem + p.x_off + static_cast<size_t>(b) * K * 2, p.x + static_cast<size_t>(b) * K,
                            static_cast<uint32_t>(K * 2), xbar, policy_evict_last());
        } else {
            mbar_arrive(xbar);
        }
    }
    const bool x_ok = mbar_wait(xbar, 0, p.err);
    grid_dependency_wait();  // y may be read by earlier kernels

    const uint32_t g = static_cast<uint32_t>(lane >> 3);         // tile of the pass this lane decodes
    const uint32_t wofs = static_cast<uint32_t>(lane & 7) * 16;  // first weight of the lane in its tile
    const uint32_t x_lane = smem_addr(smem + p.x_off) + (g * 128 + wofs) * 2;  // lane's x in pass 0 of a row
    const uint16_t *xg_lane = p.x + g * 128 + wofs;
    const bool check = p.err != nullptr;

    float acc[B][2];  // running partial of row cur_rr
#pragma unroll
    for (int b = 0; b < B; ++b) acc[b][0] = acc[b][1] = 0.f;
    PassPos q = {pa / SPR, pa - (pa / SPR) * SPR};  // next pass
    int cur_rr = q.r;

    auto flush = [&](int rr) {  // reduce this warp's partial of CTA row rr and publish it
        float v[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float t = acc[b][0] + acc[b][1];
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, d);
            v[b] = t;
            acc[b][0] = acc[b][1] = 0.f;
        }
        if (lane == 0) {
            const bool starts_before = rr * SPR < pa, ends_after = (rr + 1) * SPR > pb;
            if (!starts_before && !ends_after) {
#pragma unroll
                for (int b = 0; b < B; ++b) p.y[static_cast<size_t>(b) * R + r0 + rr] = v[b];
            } else {
                const int e = starts_before ? 0 : 1;
                parts[warp].row[e] = rr;
#pragma unroll
                for (int b = 0; b < B; ++b) parts[warp].v[e][b] = v[b];
            }
        }
    };

    for (int P0 = pa; P0 < pb && x_ok; P0 += kU) {
        // positions of the U passes
        PassPos qp[kU];
        qp[0] = q;
#pragma unroll
        for (int i = 1; i < kU; ++i) {
            qp[i] = qp[i - 1];
            if (++qp[i].j == SPR) {
                qp[i].j = 0;
                ++qp[i].r;
            }
        }
        // issue every load of the U passes first
        uint4 raw[kU];
        uint2 code[kU];
        uint32_t bse[kU], lo[kU], hi[kU];
        bool act[kU];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            const int tcol = kPassTiles * qp[i].j + static_cast<int>(g);
            act[i] = (P0 + i < pb) && (tcol < T);
            raw[i] = make_uint4(0, 0, 0, 0);
            code[i] = make_uint2(0, 0);
            bse[i] = lo[i] = hi[i] = 0;
            if (act[i]) {
                const uint64_t t = static_cast<uint64_t>(r0 + qp[i].r) * T + tcol;
                raw[i] = __ldcs(reinterpret_cast<const uint4 *>(p.raw + t * 128 + wofs));
                code[i] = __ldcs(reinterpret_cast<const uint2 *>(p.code + t * 64 + wofs / 2));
                bse[i] = __ldg(p.base + t);
                lo[i] = __ldg(p.esc_off + t);
                hi[i] = __ldg(p.esc_off + t + 1);
            }
        }
        float accp[kU][B][2];
#pragma unroll
        for (int i = 0; i < kU; ++i) {
#pragma unroll
            for (int b = 0; b < B; ++b) accp[i][b][0] = accp[i][b][1] = 0.f;
            const uint32_t col_off = static_cast<uint32_t>(kPassTiles * qp[i].j) * 256u;  // bytes of x before the pass
            uint32_t xv[B][8];
#pragma unroll
            for (int b = 0; b < B; ++b) {
                uint4 a = make_uint4(0, 0, 0, 0), a2 = make_uint4(0, 0, 0, 0);
                if (act[i]) {
                    if (p.x_smem) {
                        const uint32_t xa = x_lane + col_off + static_cast<uint32_t>(b * K) * 2;
                        a = lds128(xa);
                        a2 = lds128(xa + 16);
                    } else {
                        const uint4 *xp = reinterpret_cast<const uint4 *>(xg_lane + col_off / 2 + static_cast<size_t>(b) * K);
                        a = __ldg(xp);
                        a2 = __ldg(xp + 1);
                    }
                }
                xv[b][0] = a.x; xv[b][1] = a.y; xv[b][2] = a.z; xv[b][3] = a.w;
                xv[b][4] = a2.x; xv[b][5] = a2.y; xv[b][6] = a2.z; xv[b][7] = a2.w;
            }
            const uint32_t B4 = bse[i] * 0x01010101u;
            uint32_t w[8];
            decode16(raw[i], code[i], B4, w);
            const uint32_t m0 = escape_nibbles(code[i].x), m1 = escape_nibbles(code[i].y);
            if (check && bse[i] > kMaxBase) raise_flag(p.err, S12_FLAG_BASE);
            if (__ballot_sync(0xFFFFFFFFu, (m0 | m1) != 0 || lo[i] != hi[i]))
                fix_escapes(w, raw[i], code[i], B4, m0, m1, lo[i], hi[i], act[i], p.n_esc, p.esc, p.err);
#pragma unroll
            for (int qq = 0; qq < 8; ++qq)
#pragma unroll
                for (int b = 0; b < B; ++b) fma_bf16x2(accp[i][b][0], accp[i][b][1], w[qq], xv[b][qq]);
        }
        // fold the passes into rows
#pragma unroll
        for (int i = 0; i < kU; ++i) {
            if (P0 + i < pb) {
                if (qp[i].r != cur_rr) {
                    flush(cur_rr);
                    cur_rr = qp[i].r;
                }
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    acc[b][0] += accp[i][b][0];
                    acc[b][1] += accp[i][b][1];
                }
            }
        }
        q = qp[kU - 1];
        if (++q.j == SPR) {
            q.j = 0;
            ++q.r;
        }
    }
    if (x_ok && pa < pb) flush(cur_rr);
    __syncthreads();
    // rows shared by neighbouring warps: sum the partials in warp order
    if (warp == 0 && lane < B) {
        int row = -1;
        float sum = 0.f;
        for (int w = 0; w < NW; ++w) {
            for (int e = 0; e < 2; ++e) {
                const int rr = parts[w].row[e];
                if (rr < 0) continue;
                if (rr != row) {
                    if (row >= 0) p.y[static_cast<size_t>(lane) * R + r0 + row] = sum;
                    row = rr;
                    sum = 0.f;
                }
                sum += parts[w].v[e][lane];
            }
        }
        if (row >= 0) p.y[static_cast<size_t>(lane) * R + r0 + row] = sum;
    }
}

// ---------------------------------------------------------------------------
// Host side.

namespace {

constexpr uint32_t kSmemLimit = 227 * 1024;

template <int B>
cudaError_t run(const s12_view *v, const uint16_t *x, float *y, uint32_t *err, int sms, cudaStream_t stream) {
    GemvParams p;
    p.raw = v->raw;
    p.code = v->code;
    p.base = v->base;
    p.esc_off = v->esc_off;
    p.esc = v->esc;
    p.n_esc = v->n_esc;
    p.x = x;
    p.y = y;
    p.err = err;
    p.R = static_cast<int>(v->rows);
    p.K = static_cast<int>(v->cols);
    p.T = p.K / kTile;
    p.SPR = (p.T + kPassTiles - 1) / kPassTiles;
    p.NW = warps_for_batch<B>();
    p.part_off = 128;
    p.x_off = static_cast<uint32_t>(align_up(p.part_off + sizeof(Part<B>) * kMaxWarps, 128));
    const uint64_t xbytes = static_cast<uint64_t>(B) * p.K * 2;
    p.x_smem = (p.x_off + xbytes <= kSmemLimit) ? 1 : 0;
    const uint32_t smem = p.x_off + (p.x_smem ? static_cast<uint32_t>(xbytes) : 0);
    auto kern = gemv_kernel<B>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(std::min(sms, p.R));
    cfg.blockDim = dim3(32 * p.NW);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int launch_gemv(const s12_view *v, const uint16_t *x, int B, float *y, uint32_t *err, cudaStream_t stream) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    cudaError_t e;
    switch (B) {
        case 1: e = run<1>(v, x, y, err, sms, stream); break;
        case 2: e = run<2>(v, x, y, err, sms, stream); break;
        case 3: e = run<3>(v, x, y, err, sms, stream); break;
        case 4: e = run<4>(v, x, y, err, sms, stream); break;
        case 5: e = run<5>(v, x, y, err, sms, stream); break;
        case 6: e = run<6>(v, x, y, err, sms, stream); break;
        case 7: e = run<7>(v, x, y, err, sms, stream); break;
        default: e = run<8>(v, x, y, err, sms, stream); break;
    }
    return e == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace s12
