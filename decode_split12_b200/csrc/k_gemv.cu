// k_gemv.cu -- fused Split12 decode-GEMV for batch 1..8 on sm_100a.
//
//   y[b][n] = sum_k W[n][k] * x[b][k]
//
// The weights stay compressed in HBM; the exact BF16 values are rebuilt in
// registers from shared-memory tiles and used at once in the product
// ("Lossless LLM Weight Compression vs 8-bit GGUF", section "What does
// 'lossless' mean for LLM weights?": decode into registers or shared memory
// and multiply immediately).  The kernel is HBM-bound: it must move the
// compressed planes (1.5 bytes per weight + 5 bytes per tile + 2 bytes per
// escape) at close to the copy bandwidth.
//
// Structure (one persistent CTA per SM, rows split evenly between CTAs):
//   * warp 8 is the producer.  Lane 0 issues TMA bulk copies
//     (cp.async.bulk) of each stage -- SR rows x KC columns of the raw,
//     code, base and esc_off planes -- into a ring of NSTAGE shared-memory
//     slots, plus the activations x for the current column chunk.  All 32
//     lanes then reduce the consumers' per-stage partial sums in a fixed
//     order and write y, so y is deterministic.
//   * warps 0..7 are consumers, laid out as WK x WR: warp (wk, wr) handles
//     the 512-weight column slots wk, wk+WK, ... of stage rows wr, wr+WR, ...
//     Each lane decodes 16 weights per row per slot (byte-wise base+code ADD
//     and byte permutes), multiplies them by x in FP32, and at the end of the
//     stage the warp reduces with shuffles and publishes one partial per
//     (row, batch) before releasing the slot.
//   * When B*K*2 bytes of x exceed the shared-memory budget, K is split into
//     phases of KC columns with a double-buffered x chunk; phase c > 0 adds
//     into y.
#include <algorithm>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

constexpr int kConsumerWarps = 8;
constexpr int kGemvThreads = 32 * (kConsumerWarps + 1);
constexpr int kMaxStages = 8;
constexpr uint32_t kBarrierBytes = 256;

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
    int R, K, T;
    int KC, n_phase, n_xbuf, SR, WK, WR, NSTAGE;
    uint32_t stage_bytes, off_code, off_hb, off_ho, hb_stride, ho_stride;
    uint32_t part_off, xbuf_off, ring_off;
};

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

template <int B, int RPW>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const __grid_constant__ GemvParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + kMaxStages;
    uint64_t *xfull = empty + kMaxStages;
    float *part = reinterpret_cast<float *>(smem + p.part_off);
    uint8_t *xbuf = smem + p.xbuf_off;
    uint8_t *ring = smem + p.ring_off;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.R / gridDim.x);
    const int r1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.R / gridDim.x);
    const int nrows = r1 - r0;
    const int n_groups = (nrows + p.SR - 1) / p.SR;
    const int n_stages = n_groups * p.n_phase;
    const int n_active = p.WK * p.WR;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.NSTAGE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], n_active);
        }
        mbar_init(&xfull[0], 1);
        mbar_init(&xfull[1], 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (n_stages == 0) return;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        int released = 0;
        bool ok = true;
        auto release_one = [&]() {
            const int j = released;
            const int s = j % p.NSTAGE;
            if (ok) ok = mbar_wait(&empty[s], (j / p.NSTAGE) & 1, p.err);
            ok = __all_sync(0xFFFFFFFFu, ok);
            const int c = j / n_groups, g = j % n_groups;
            const int sr = min(p.SR, nrows - g * p.SR);
            const float *ps = part + static_cast<size_t>(s) * p.WK * p.SR * B;
            if (ok) {
                for (int idx = lane; idx < sr * B; idx += 32) {
                    const int i = idx / B, b = idx - (idx / B) * B;
                    float v = 0.f;
                    for (int wk = 0; wk < p.WK; ++wk) v += ps[(wk * p.SR + i) * B + b];
                    float *yp = p.y + static_cast<size_t>(b) * p.R + (r0 + g * p.SR + i);
                    if (c == 0)
                        *yp = v;
                    else
                        *yp += v;
                }
            }
            __syncwarp();
            ++released;
        };
        int issued = 0;
        for (int j = 0; j < n_stages && ok; ++j) {
            const int c = j / n_groups, g = j % n_groups, s = j % p.NSTAGE;
            if (j >= p.NSTAGE) release_one();
            const int k0 = c * p.KC;
            const int kc = min(p.KC, p.K - k0);
            if (g == 0) {
                if (c >= p.n_xbuf)
                    while (ok && released < (c - p.n_xbuf + 1) * n_groups) release_one();
                if (lane == 0 && ok) {
                    uint64_t *xb = &xfull[c % p.n_xbuf];
                    mbar_arrive_expect_tx(xb, static_cast<uint32_t>(B * kc * 2));
                    for (int b = 0; b < B; ++b)
                        tma_load_1d(xbuf + (static_cast<size_t>(c % p.n_xbuf) * B + b) * p.KC * 2,
                                    p.x + static_cast<size_t>(b) * p.K + k0, static_cast<uint32_t>(kc * 2), xb,
                                    pol_x);
                }
            }
            if (lane == 0 && ok) {
                const int sr = min(p.SR, nrows - g * p.SR);
                uint8_t *st = ring + static_cast<size_t>(s) * p.stage_bytes;
                const int nt = kc / kTile;
                uint32_t bytes = 0;
                for (int i = 0; i < sr; ++i) {
                    const uint64_t row = static_cast<uint64_t>(r0 + g * p.SR + i);
                    const uint64_t t0 = row * p.T + k0 / kTile;
                    const uintptr_t ba = reinterpret_cast<uintptr_t>(p.base + t0) & ~uintptr_t(15);
                    const uintptr_t be = (reinterpret_cast<uintptr_t>(p.base + t0 + nt) + 15) & ~uintptr_t(15);
                    const uintptr_t oa = reinterpret_cast<uintptr_t>(p.esc_off + t0) & ~uintptr_t(15);
                    const uintptr_t oe = (reinterpret_cast<uintptr_t>(p.esc_off + t0 + nt + 1) + 15) & ~uintptr_t(15);
                    bytes += kc + kc / 2 + static_cast<uint32_t>(be - ba) + static_cast<uint32_t>(oe - oa);
                }
                mbar_arrive_expect_tx(&full[s], bytes);
                for (int i = 0; i < sr; ++i) {
                    const uint64_t row = static_cast<uint64_t>(r0 + g * p.SR + i);
                    const uint64_t w0 = row * p.K + k0;
                    const uint64_t t0 = row * p.T + k0 / kTile;
                    tma_load_1d(st + static_cast<size_t>(i) * p.KC, p.raw + w0, kc, &full[s], pol_w);
                    tma_load_1d(st + p.off_code + static_cast<size_t>(i) * (p.KC / 2), p.code + w0 / 2, kc / 2,
                                &full[s], pol_w);
                    const uintptr_t ba = reinterpret_cast<uintptr_t>(p.base + t0) & ~uintptr_t(15);
                    const uintptr_t be = (reinterpret_cast<uintptr_t>(p.base + t0 + nt) + 15) & ~uintptr_t(15);
                    tma_load_1d(st + p.off_hb + static_cast<size_t>(i) * p.hb_stride, reinterpret_cast<const void *>(ba),
                                static_cast<uint32_t>(be - ba), &full[s], pol_w);
                    const uintptr_t oa = reinterpret_cast<uintptr_t>(p.esc_off + t0) & ~uintptr_t(15);
                    const uintptr_t oe = (reinterpret_cast<uintptr_t>(p.esc_off + t0 + nt + 1) + 15) & ~uintptr_t(15);
                    tma_load_1d(st + p.off_ho + static_cast<size_t>(i) * p.ho_stride, reinterpret_cast<const void *>(oa),
                                static_cast<uint32_t>(oe - oa), &full[s], pol_w);
                }
            }
            if (ok) issued = j + 1;
        }
        while (ok && released < n_stages) release_one();
        if (!ok) {
            // Unwind after a timeout: let every copy already issued land
            // (bounded) before the CTA's shared memory goes away.
            for (int j = max(0, issued - p.NSTAGE); j < issued; ++j)
                mbar_wait(&full[j % p.NSTAGE], (j / p.NSTAGE) & 1, nullptr);
            if (issued > 0) {
                const int c_last = (issued - 1) / n_groups;
                for (int c = max(0, c_last - p.n_xbuf + 1); c <= c_last; ++c)
                    mbar_wait(&xfull[c % p.n_xbuf], (c / p.n_xbuf) & 1, nullptr);
            }
        }
        return;
    }
    if (warp >= n_active) return;

    // -------------------------------------------------------------- consumers
    const int wk = warp % p.WK, wr = warp / p.WK;
    for (int j = 0; j < n_stages; ++j) {
        const int c = j / n_groups, g = j % n_groups, s = j % p.NSTAGE;
        const int sr = min(p.SR, nrows - g * p.SR);
        const int k0 = c * p.KC;
        const int kc = min(p.KC, p.K - k0);
        bool ok = true;
        if (g == 0) ok = mbar_wait(&xfull[c % p.n_xbuf], (c / p.n_xbuf) & 1, p.err);
        if (ok) ok = mbar_wait(&full[s], (j / p.NSTAGE) & 1, p.err);
        if (!__all_sync(0xFFFFFFFFu, ok)) return;

        const uint8_t *st = ring + static_cast<size_t>(s) * p.stage_bytes;
        const uint8_t *xb = xbuf + static_cast<size_t>(c % p.n_xbuf) * B * p.KC * 2;
        float2 acc[RPW][B];
#pragma unroll
        for (int ii = 0; ii < RPW; ++ii)
#pragma unroll
            for (int b = 0; b < B; ++b) acc[ii][b] = make_float2(0.f, 0.f);

        // shared-memory header rows (shifted by the 16-byte rounding of the copy)
        const uint8_t *hb[RPW];
        const uint32_t *ho[RPW];
#pragma unroll
        for (int ii = 0; ii < RPW; ++ii) {
            const int i = wr + ii * p.WR;
            const uint64_t row = static_cast<uint64_t>(r0 + g * p.SR + (i < sr ? i : 0));
            const uint64_t t0 = row * p.T + k0 / kTile;
            const uint32_t sb = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(p.base + t0) & 15);
            const uint32_t so = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(p.esc_off + t0) & 15);
            hb[ii] = st + p.off_hb + static_cast<size_t>(i) * p.hb_stride + sb;
            ho[ii] = reinterpret_cast<const uint32_t *>(st + p.off_ho + static_cast<size_t>(i) * p.ho_stride + so);
        }

        const int n_slots = (kc + 511) / 512;
        for (int ks = wk; ks < n_slots; ks += p.WK) {
            const int kl = ks * 512 + lane * 16;
            const bool active = kl < kc;
            uint32_t xv[B][8];
#pragma unroll
            for (int b = 0; b < B; ++b) {
                uint4 a = make_uint4(0, 0, 0, 0), bb = make_uint4(0, 0, 0, 0);
                if (active) {
                    const uint4 *xp = reinterpret_cast<const uint4 *>(xb + (static_cast<size_t>(b) * p.KC + kl) * 2);
                    a = xp[0];
                    bb = xp[1];
                }
                xv[b][0] = a.x; xv[b][1] = a.y; xv[b][2] = a.z; xv[b][3] = a.w;
                xv[b][4] = bb.x; xv[b][5] = bb.y; xv[b][6] = bb.z; xv[b][7] = bb.w;
            }
#pragma unroll
            for (int ii = 0; ii < RPW; ++ii) {
                const int i = wr + ii * p.WR;
                if (i >= sr) break;  // warp-uniform
                uint4 raw = make_uint4(0, 0, 0, 0);
                uint2 code = make_uint2(0, 0);
                uint32_t bse = 0, lo = 0, hi = 0;
                if (active) {
                    raw = *reinterpret_cast<const uint4 *>(st + static_cast<size_t>(i) * p.KC + kl);
                    code = *reinterpret_cast<const uint2 *>(st + p.off_code + static_cast<size_t>(i) * (p.KC / 2) + kl / 2);
                    const int tl = kl >> 7;
                    bse = hb[ii][tl];
                    lo = ho[ii][tl];
                    hi = ho[ii][tl + 1];
                }
                if (bse > kMaxBase) raise_flag(p.err, S12_FLAG_BASE);
                const uint32_t B4 = bse * 0x01010101u;
                const uint32_t m0 = escape_nibbles(code.x), m1 = escape_nibbles(code.y);
                uint32_t w[8];
                decode16(raw, code, B4, w);
                if (__ballot_sync(0xFFFFFFFFu, (m0 | m1) != 0)) {
                    fix_escapes(w, raw, code, B4, m0, m1, lo, hi, active, p.n_esc, p.esc, p.err);
                } else if (active && (lane & 7) == 0 && lo != hi) {
                    raise_flag(p.err, S12_FLAG_ESC_COUNT);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float wl = bf16lo(w[q]), wh = bf16hi(w[q]);
#pragma unroll
                    for (int b = 0; b < B; ++b) {
                        acc[ii][b].x = fmaf(wl, bf16lo(xv[b][q]), acc[ii][b].x);
                        acc[ii][b].y = fmaf(wh, bf16hi(xv[b][q]), acc[ii][b].y);
                    }
                }
            }
        }
        // warp reduction -> one partial per (row, batch) for this slot class
        float *ps = part + static_cast<size_t>(s) * p.WK * p.SR * B;
#pragma unroll
        for (int ii = 0; ii < RPW; ++ii) {
            const int i = wr + ii * p.WR;
            if (i >= sr) break;
#pragma unroll
            for (int b = 0; b < B; ++b) {
                float v = acc[ii][b].x + acc[ii][b].y;
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, d);
                if (lane == 0) ps[(wk * p.SR + i) * B + b] = v;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

// ---------------------------------------------------------------------------
// Host side: pick the stage shape for (R, K, B) and launch.

namespace {

constexpr uint32_t kSmemLimit = 227 * 1024;
constexpr uint32_t kXBudget = 96 * 1024;
constexpr uint32_t kRingBudget = 120 * 1024;

struct GemvPlan {
    GemvParams p;
    int rpw;
    uint32_t smem;
    int grid;
};

int pick_wk(int n_slots) {
    if (n_slots >= kConsumerWarps) {
        for (int wk = kConsumerWarps; wk >= 5; --wk)
            if (n_slots % wk == 0) return wk;
        return kConsumerWarps;
    }
    // fewer slots than warps: one warp per slot, the rest split the rows
    int wk = 1;
    while (wk * 2 <= n_slots) wk *= 2;
    return wk;
}

int plan_gemv(const s12_view *v, int B, int sms, GemvPlan *out) {
    GemvParams &p = out->p;
    const int K = static_cast<int>(v->cols);
    p.R = static_cast<int>(v->rows);
    p.K = K;
    p.T = K / kTile;
    // column chunking so that the activations fit
    if (static_cast<uint64_t>(B) * K * 2 <= kXBudget) {
        p.KC = K;
        p.n_xbuf = 1;
    } else {
        int kc = static_cast<int>(kXBudget / 2 / (B * 2));
        kc = kc / 512 * 512;
        if (kc < 512) kc = 512;
        p.KC = kc;
        p.n_xbuf = 2;
    }
    p.n_phase = (K + p.KC - 1) / p.KC;
    const int n_slots = (p.KC + 511) / 512;
    p.WK = pick_wk(n_slots);
    p.WR = kConsumerWarps / p.WK;
    // rows per warp per stage: reuse x over more rows as B grows, and keep a
    // stage near 8-24 KB of compressed weights
    const double row_bytes = 1.5 * p.KC;
    int rpw = (B >= 4) ? 4 : (B >= 2 ? 2 : 2);
    while (rpw > 1 && row_bytes * rpw * p.WR > 24576.0) rpw /= 2;
    p.SR = rpw * p.WR;
    out->rpw = rpw;
    const int nt = p.KC / kTile;
    p.hb_stride = static_cast<uint32_t>(align_up(nt + 32, 16));
    p.ho_stride = static_cast<uint32_t>(align_up(4 * (nt + 1) + 32, 16));
    p.off_code = static_cast<uint32_t>(p.SR) * p.KC;
    p.off_hb = p.off_code + static_cast<uint32_t>(p.SR) * (p.KC / 2);
    p.off_ho = p.off_hb + static_cast<uint32_t>(p.SR) * p.hb_stride;
    p.stage_bytes = static_cast<uint32_t>(align_up(p.off_ho + static_cast<uint32_t>(p.SR) * p.ho_stride, 128));
    const uint32_t xbytes = static_cast<uint32_t>(p.n_xbuf) * B * p.KC * 2;
    const uint32_t part_bytes_per_stage = static_cast<uint32_t>(p.WK * p.SR * B * 4);
    uint32_t fixed = kBarrierBytes + xbytes;
    int nst = kMaxStages;
    while (nst > 2 && (nst * p.stage_bytes > kRingBudget ||
                       fixed + nst * (p.stage_bytes + part_bytes_per_stage) + 1024 > kSmemLimit))
        --nst;
    p.NSTAGE = nst;
    p.part_off = kBarrierBytes;
    p.xbuf_off = static_cast<uint32_t>(align_up(p.part_off + nst * part_bytes_per_stage, 128));
    p.ring_off = static_cast<uint32_t>(align_up(p.xbuf_off + xbytes, 128));
    out->smem = p.ring_off + nst * p.stage_bytes;
    if (out->smem > kSmemLimit) return S12_ERR_SHAPE;
    out->grid = std::min(sms, p.R);
    return S12_OK;
}

template <int B, int RPW>
cudaError_t run(const GemvPlan &pl, cudaStream_t stream) {
    auto kern = gemv_kernel<B, RPW>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return e;
    kern<<<pl.grid, kGemvThreads, pl.smem, stream>>>(pl.p);
    return cudaGetLastError();
}

template <int B>
cudaError_t run_b(const GemvPlan &pl, cudaStream_t stream) {
    switch (pl.rpw) {
        case 1: return run<B, 1>(pl, stream);
        case 2: return run<B, 2>(pl, stream);
        default: return run<B, 4>(pl, stream);
    }
}

}  // namespace

int launch_gemv(const s12_view *v, const uint16_t *x, int B, float *y, uint32_t *err, cudaStream_t stream) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    GemvPlan pl;
    int rc = plan_gemv(v, B, sms, &pl);
    if (rc != S12_OK) return rc;
    GemvParams &p = pl.p;
    p.raw = v->raw;
    p.code = v->code;
    p.base = v->base;
    p.esc_off = v->esc_off;
    p.esc = v->esc;
    p.n_esc = v->n_esc;
    p.x = x;
    p.y = y;
    p.err = err;
    cudaError_t e;
    switch (B) {
        case 1: e = run_b<1>(pl, stream); break;
        case 2: e = run_b<2>(pl, stream); break;
        case 3: e = run_b<3>(pl, stream); break;
        case 4: e = run_b<4>(pl, stream); break;
        case 5: e = run_b<5>(pl, stream); break;
        case 6: e = run_b<6>(pl, stream); break;
        case 7: e = run_b<7>(pl, stream); break;
        default: e = run_b<8>(pl, stream); break;
    }
    return e == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace s12
