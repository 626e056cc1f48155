// k_decode.cu -- standalone Split12 decode (container -> BF16 matrix) and the
// exponent histogram of s12_stats, for container versions 1 and 2.
//
// The exponent is base + code, a byte-wise integer ADD ("GPU 友善 12 位無損
// BF16 壓縮格式", key points); code-15 weights take their exact value from
// the escape stream, located by the tile's offset and the weight's rank
// among the tile's escapes.  The kernel is HBM-bound: it reads 1.5 bytes per
// weight plus the tile headers and escapes, and writes 2 bytes per weight.
//
// The stream is cut into chunks of 32 tiles (4096 weights: 4 KB raw, 2 KB
// code, 8 KB out), all contiguous in memory.  Four CTAs per SM (four
// independent streams hide each other's waits better than one deep one), each:
//   warp 0       producer: per chunk it writes each tile's base and first
//                escape offset into the stage (loaded six chunks ahead), then
//                one lane starts bulk copies of the raw bytes, the codes and
//                the chunk's whole escape span into the stage, completing on
//                the stage's mbarrier.
//   warps 1..8   decode: each takes 4 tiles of the chunk, 16 weights per
//                lane; the decoded words go to the warp's staging buffer in
//                shared memory, escaped weights are overwritten there from
//                the staged escape span, and one lane writes the 1 KB back
//                with a bulk shared-to-global copy (double-buffered).
// Up to 1,024 escapes per chunk are staged (more than 20 % of its weights);
// only beyond that does an escape cost a read of the stream.
// Every wait is bounded (about a second) and raises S12_FLAG_TIMEOUT.
#include <algorithm>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace dec {

constexpr int kChunkTiles = 32;
constexpr int kDecWarps = 8;
constexpr int kThreads = 32 * (kDecWarps + 1);
constexpr int kStages = 4;
constexpr int kCtasPerSm = 4;
constexpr uint32_t kRawB = kChunkTiles * 128;
constexpr uint32_t kCodeB = kChunkTiles * 64;
constexpr uint32_t kMetaB = 2 * 4 * (kChunkTiles + 1) + 8;  // base[33], off[33] as u32, aligned to 16
constexpr uint32_t kEscCap = 1024;  // escapes staged per chunk (more are read from the stream directly)
constexpr uint32_t kEscB = 2 * kEscCap + 16;                // + alignment slack of the bulk copy
constexpr uint32_t kStageB = kRawB + kCodeB + kMetaB + kEscB;
constexpr uint32_t kOffMeta = kRawB + kCodeB, kOffEsc = kOffMeta + kMetaB;
constexpr uint32_t kSlotB = 4 * 256;  // one warp's 4 decoded tiles
static_assert(kStageB % 16 == 0 && kOffEsc % 16 == 0, "bulk copies need 16-byte alignment");

struct Params {
    const uint8_t *raw;
    const uint8_t *code;
    const void *meta;       // version 1: base u8[n_tiles]; version 2: tmeta u16[n_tiles]
    const uint32_t *off;    // version 1: esc_off u32[n_tiles + 1]; version 2: row_esc u32[rows + 1]
    const uint16_t *esc;
    uint32_t n_esc;
    long long n_tiles;
    int T;                  // tiles per row
    uint16_t *out;          // rows x cols BF16 (decode) or null (histogram)
    unsigned long long *hist;  // 256 counters (histogram) or null
    uint32_t *err;
};

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles) return false;
    return true;
}
// 1-D bulk copy global -> shared, completing on bar (16-byte aligned, size a
// multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// 1-D bulk copy shared -> global, in this thread's current bulk group.
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Chunk range of CTA c: [c*n/G, (c+1)*n/G).
__device__ __forceinline__ long long chunk_start(long long c, long long n, int G) { return c * n / G; }

template <int V, bool HIST>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sb = (smem_addr(smem_raw) + 127u) & ~127u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full = sb, empty = sb + 8 * kStages;
    const uint32_t stages = sb + 256;
    const uint32_t slots = stages + kStages * kStageB;           // 2 per decode warp
    __shared__ uint32_t s_hist[256];  // histogram mode
    __shared__ uint32_t s_tab[32];    // version 4: the symbol table
    const long long n_chunks = (p.n_tiles + kChunkTiles - 1) / kChunkTiles;
    const long long c0 = chunk_start(blockIdx.x, n_chunks, gridDim.x), c1 = chunk_start(blockIdx.x + 1, n_chunks, gridDim.x);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(full + 8 * s, 1);
            bar_init(empty + 8 * s, kDecWarps);
        }
        fence_barrier_init();
    }
    if (HIST)
        for (int i = threadIdx.x; i < 256; i += kThreads) s_hist[i] = 0;
    if (V == 4 && threadIdx.x < 32) s_tab[threadIdx.x] = __ldg(static_cast<const uint16_t *>(p.meta) + threadIdx.x);
    __syncthreads();

    if (warp == 0) {
        // ---- producer
        // metadata of chunk c for this lane's tile: base, first escape
        // offset (version 1) or escape count (version 2); lane 31 of version
        // 1 also the end of the chunk's span
        auto load = [&](long long c, uint32_t &mb, uint32_t &mo, uint32_t &me) {
            const long long t0 = c * kChunkTiles, t = t0 + lane;
            const int nt = static_cast<int>(min(static_cast<long long>(kChunkTiles), p.n_tiles - t0));
            mb = mo = me = 0;
            if (lane < nt) {
                if (V != 2) {
                    mb = V == 4 ? 0u : __ldg(static_cast<const uint8_t *>(p.meta) + t);
                    mo = __ldg(p.off + t);
                } else {
                    const uint32_t w = __ldg(static_cast<const uint16_t *>(p.meta) + t);
                    mb = w & 0xFFu;
                    mo = w >> 8;
                }
            }
            if (V != 2 && lane == 31) me = __ldg(p.off + t0 + nt);
        };
        // version 2: escapes before the first tile of the range
        uint32_t carry = 0;
        if (V == 2 && c0 < c1) {
            const long long t0 = c0 * kChunkTiles, r0 = t0 / p.T;
            uint32_t s = 0;
            for (long long t = r0 * p.T + lane; t < t0; t += 32) s += __ldg(static_cast<const uint16_t *>(p.meta) + t) >> 8;
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, d);
            carry = __ldg(p.off + r0) + s;
        }
        // a ring of the next kAhead chunks' metadata in registers, so each
        // chunk's loads have several chunks of time to land
        constexpr int kAhead = 6;
        uint32_t rb[kAhead], ro[kAhead], re[kAhead];
#pragma unroll
        for (int j = 0; j < kAhead; ++j) {
            rb[j] = ro[j] = re[j] = 0;
            if (c0 + j < c1) load(c0 + j, rb[j], ro[j], re[j]);
        }
        bool ok = true;
        long long k = 0;
        for (long long c = c0; c < c1; ++c, ++k) {
            const int s = static_cast<int>(k % kStages);
            const uint32_t round = static_cast<uint32_t>(k / kStages);
            if (!__all_sync(0xFFFFFFFFu, bar_wait(empty + 8 * s, (round & 1u) ^ 1u))) {
                raise_flag(p.err, S12_FLAG_TIMEOUT);
                ok = false;
                break;
            }
            const long long t0 = c * kChunkTiles;
            const int nt = static_cast<int>(min(static_cast<long long>(kChunkTiles), p.n_tiles - t0));
            const uint32_t mb = rb[0], mo = ro[0], me = re[0];
#pragma unroll
            for (int j = 0; j + 1 < kAhead; ++j) {
                rb[j] = rb[j + 1];
                ro[j] = ro[j + 1];
                re[j] = re[j + 1];
            }
            rb[kAhead - 1] = ro[kAhead - 1] = re[kAhead - 1] = 0;
            if (c + kAhead < c1) load(c + kAhead, rb[kAhead - 1], ro[kAhead - 1], re[kAhead - 1]);
            // first escape of each tile, and the chunk's span [e0, e1)
            uint32_t first, e1;
            if (V != 2) {
                first = mo;
                e1 = __shfl_sync(0xFFFFFFFFu, me, 31);
            } else {
                uint32_t incl = mo;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                    if (lane >= d) incl += v;
                }
                first = carry + incl - mo;
                e1 = carry + __shfl_sync(0xFFFFFFFFu, incl, 31);
                carry = e1;
            }
            const uint32_t e0 = __shfl_sync(0xFFFFFFFFu, first, 0);
            const uint32_t st = stages + s * kStageB;
            sts32(st + kOffMeta + 4 * lane, mb);
            sts32(st + kOffMeta + 4 * (kChunkTiles + 1) + 4 * lane, first);
            if (lane == 0) sts32(st + kOffMeta + 4 * (kChunkTiles + 1) + 4 * kChunkTiles, e1);
            // the escape span to stage: clamped to the stream and to kEscCap
            // values (the decoders read any further escapes of the chunk
            // from the stream itself, and flag reads outside the chunk's span)
            const uint32_t ec1 = min(e1, p.n_esc), ec0 = min(e0, ec1);
            const uint32_t n_stage = min(ec1 - ec0, kEscCap);
            const uint32_t a0 = (2u * ec0) & ~15u, a1 = (2u * (ec0 + n_stage) + 15u) & ~15u;
            if (lane == 0) {
                sts32(st + kOffMeta + 8 * (kChunkTiles + 1), ec0);
                sts32(st + kOffMeta + 8 * (kChunkTiles + 1) + 4, ec0 + n_stage);
            }
            __syncwarp();
            if (lane == 0) {
                const uint32_t esc_bytes = n_stage ? a1 - a0 : 0u;
                bar_expect_tx(full + 8 * s, nt * 192u + esc_bytes);
                if (V == 3) {
                    // the pair plane: a tile's raw bytes and codes, 192 bytes
                    bulk_load(st, p.raw + t0 * 192, nt * 192u, full + 8 * s);
                } else {
                    bulk_load(st, p.raw + t0 * 128, nt * 128u, full + 8 * s);
                    bulk_load(st + kRawB, p.code + t0 * 64, nt * 64u, full + 8 * s);
                }
                if (esc_bytes)
                    bulk_load(st + kOffEsc, reinterpret_cast<const uint8_t *>(p.esc) + a0, esc_bytes, full + 8 * s);
            }
        }
        if (!ok && lane == 0) {
            // let the copies already started land before the CTA exits
            for (long long j = (k >= kStages ? k - kStages : 0); j < k; ++j)
                bar_wait(full + 8 * static_cast<uint32_t>(j % kStages), static_cast<uint32_t>(j / kStages) & 1u);
        }
    } else {
        // ---- decode warps: warp w takes tiles 4(w-1) .. +3 of each chunk,
        // lane l the 16 weights 16 (l % 8) .. of tile l / 8
        const int dw = warp - 1;
        const int tl = 4 * dw + (lane >> 3), piece = lane & 7;
        long long k = 0;
        for (long long c = c0; c < c1; ++c, ++k) {
            const int s = static_cast<int>(k % kStages);
            const uint32_t slot = slots + static_cast<uint32_t>(2 * dw + (HIST ? 0 : (k & 1))) * kSlotB;
            if (!HIST) {
                // the slot's store from two chunks ago has read it
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
            }
            if (!__all_sync(0xFFFFFFFFu, bar_wait(full + 8 * s, static_cast<uint32_t>(k / kStages) & 1u))) {
                raise_flag(p.err, S12_FLAG_TIMEOUT);
                break;
            }
            const long long t0 = c * kChunkTiles;
            const int nt = static_cast<int>(min(static_cast<long long>(kChunkTiles), p.n_tiles - t0));
            const bool active = tl < nt;
            const uint32_t st = stages + s * kStageB, meta = st + kOffMeta;
            const uint32_t sl = lds32(meta + 8 * (kChunkTiles + 1)), sh = lds32(meta + 8 * (kChunkTiles + 1) + 4);
            uint4 raw = make_uint4(0, 0, 0, 0);
            uint2 code = make_uint2(0, 0);
            uint32_t base = 0, lo = 0, hi = 0;
            if (active) {
                if (V == 3) {
                    // 8 pairs of 3 bytes: raw, raw, two codes; regrouped
                    // into the 16 raw bytes and 8 code bytes of version 1
                    uint32_t q[6];
                    const uint32_t a = st + tl * 192 + piece * 24;
#pragma unroll
                    for (int h = 0; h < 3; ++h)
                        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                     : "=r"(q[2 * h]), "=r"(q[2 * h + 1])
                                     : "r"(a + 8 * h));
                    raw.x = prmt(q[0], q[1], 0x4310u);  // bytes 0 1 3 4
                    raw.y = prmt(q[1], q[2], 0x6532u);  // bytes 6 7 9 10
                    raw.z = prmt(q[3], q[4], 0x4310u);  // bytes 12 13 15 16
                    raw.w = prmt(q[4], q[5], 0x6532u);  // bytes 18 19 21 22
                    code.x = prmt(prmt(q[0], q[1], 0x0052u), q[2], 0x7410u);  // bytes 2 5 8 11
                    code.y = prmt(prmt(q[3], q[4], 0x0052u), q[5], 0x7410u);  // bytes 14 17 20 23
                } else {
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(raw.x), "=r"(raw.y), "=r"(raw.z), "=r"(raw.w)
                                 : "r"(st + tl * 128 + piece * 16));
                    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                 : "=r"(code.x), "=r"(code.y)
                                 : "r"(st + kRawB + tl * 64 + piece * 8));
                }
                base = lds32(meta + 4 * tl);
                lo = lds32(meta + 4 * (kChunkTiles + 1) + 4 * tl);
                // the tile's span ends where the next one starts (the chunk's
                // last tile: at the chunk's end)
                hi = lds32(meta + 4 * (kChunkTiles + 1) + 4 * (tl + 1 < nt ? tl + 1 : kChunkTiles));
            }
            uint32_t m0, m1;
            uint32_t w[8];
            if (V == 4) {
                // code = nibble << 1 | raw bit 7; the weight is table[code] << 7
                // | mantissa, or an escape (code 31, flagged like a version 1
                // escape nibble: bit 4j+3 of m0 / m1)
                m0 = m1 = 0;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint32_t rw = j < 4 ? raw.x : j < 8 ? raw.y : j < 12 ? raw.z : raw.w;
                    const uint32_t r = (rw >> (8 * (j & 3))) & 0xFFu;
                    const uint32_t nib = ((j < 8 ? code.x : code.y) >> (4 * (j & 7))) & 0xFu;
                    const uint32_t cd = (nib << 1) | (r >> 7);
                    uint32_t v = 0;
                    if (cd == 31u) {
                        if (j < 8)
                            m0 |= 8u << (4 * j);
                        else
                            m1 |= 8u << (4 * (j - 8));
                    } else {
                        const uint32_t sym = s_tab[cd];
                        if (sym > 511u) raise_flag(p.err, S12_FLAG_BASE);  // an unused table entry
                        v = ((sym & 0x1FFu) << 7) | (r & 0x7Fu);
                    }
                    if (j & 1)
                        w[j >> 1] |= v << 16;
                    else
                        w[j >> 1] = v;
                }
            } else {
                if (base > static_cast<uint32_t>(kMaxBase)) raise_flag(p.err, S12_FLAG_BASE);
                m0 = escape_nibbles(code.x);
                m1 = escape_nibbles(code.y);
            }
            // rank of the lane's first escape within its tile (8 lanes per tile)
            const uint32_t cnt = __popc(m0) + __popc(m1);
            uint32_t incl = cnt;
#pragma unroll
            for (int d = 1; d < 8; d <<= 1) {
                const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d, 8);
                if (piece >= d) incl += v;
            }
            if (active && piece == 7 && incl != hi - lo) raise_flag(p.err, S12_FLAG_ESC_COUNT);
            // with escape nibbles cleared, base + code never carries out of its byte
            if (V != 4)
                decode16(raw, (m0 | m1) ? make_uint2(clear_escapes(code.x, m0), clear_escapes(code.y, m1)) : code,
                         base * 0x01010101u, w);
            const uint32_t mine = slot + static_cast<uint32_t>(lane) * 32u;  // tile-major: the output order
            if (active) {
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(mine), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                             "r"(w[3])
                             : "memory");
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(mine + 16), "r"(w[4]), "r"(w[5]),
                             "r"(w[6]), "r"(w[7])
                             : "memory");
                // escaped weights: their exact values from the staged span
                uint64_t mm = (static_cast<uint64_t>(m1) << 32) | m0;
                uint32_t i = lo + incl - cnt;
                const uint32_t esc_s = st + kOffEsc + ((2u * sl) & 15u);
                while (mm) {
                    const int j = (__ffsll(static_cast<long long>(mm)) - 1) >> 2;
                    mm &= mm - 1;
                    uint16_t v = 0;
                    if (i >= sl && i < sh && i < hi)
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(esc_s + 2u * (i - sl)) : "memory");
                    else if (i >= lo && i < hi && i < p.n_esc)
                        v = __ldg(p.esc + i);
                    else
                        raise_flag(p.err, S12_FLAG_ESC_RANGE);
                    ++i;
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(mine + 2u * j), "h"(v) : "memory");
                }
            }
            // the stage is no longer needed
            __syncwarp();
            if (lane == 0) bar_arrive(empty + 8 * s);
            const int ntw = min(4, nt - 4 * dw);  // this warp's tiles in the chunk
            if (HIST) {
                if (active) {
                    uint4 a, b;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w)
                                 : "r"(mine)
                                 : "memory");
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                                 : "r"(mine + 16)
                                 : "memory");
                    const uint32_t ww[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        atomicAdd(&s_hist[(ww[e] >> 7) & 0xFFu], 1u);
                        atomicAdd(&s_hist[(ww[e] >> 23) & 0xFFu], 1u);
                    }
                }
                __syncwarp();
            } else if (ntw > 0) {
                // generic-proxy writes must be visible to the bulk copy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) bulk_store(p.out + (t0 + 4 * dw) * kTile, slot, static_cast<uint32_t>(ntw) * 256u);
            }
        }
        if (!HIST && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    if (HIST) {
        __syncthreads();
        for (int i = threadIdx.x; i < 256; i += kThreads)
            if (s_hist[i]) atomicAdd(p.hist + i, static_cast<unsigned long long>(s_hist[i]));
    }
}

}  // namespace dec

namespace {

template <int V, bool HIST>
int run_decode(const s12_view *v, uint16_t *out, unsigned long long *hist, uint32_t *err, cudaStream_t stream) {
    dec::Params p;
    p.raw = v->raw;
    p.code = v->code;
    p.meta = V == 4   ? static_cast<const void *>(v->symtab)
             : V != 2 ? static_cast<const void *>(v->base)
                      : static_cast<const void *>(v->tmeta);
    p.off = V != 2 ? v->esc_off : v->row_esc;
    p.esc = v->esc;
    p.n_esc = static_cast<uint32_t>(v->n_esc);
    p.n_tiles = static_cast<long long>(v->n_tiles);
    p.T = static_cast<int>(v->cols / kTile);
    p.out = out;
    p.hist = hist;
    p.err = err;
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    const long long n_chunks = (p.n_tiles + dec::kChunkTiles - 1) / dec::kChunkTiles;
    const int grid = static_cast<int>(std::max(1LL, std::min<long long>(static_cast<long long>(dec::kCtasPerSm) * sms,
                                                                         n_chunks)));
    const uint32_t smem = 128 + 256 + dec::kStages * dec::kStageB + 2 * dec::kDecWarps * dec::kSlotB;
    auto kern = dec::decode_kernel<V, HIST>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return S12_ERR_CUDA;
    kern<<<grid, dec::kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace

int launch_decode(const s12_view *v, uint16_t *out, uint32_t *err, cudaStream_t stream) {
    if (v->version == 4) return run_decode<4, false>(v, out, nullptr, err, stream);
    if (v->version == 3) return run_decode<3, false>(v, out, nullptr, err, stream);
    return v->version == 1 ? run_decode<1, false>(v, out, nullptr, err, stream)
                           : run_decode<2, false>(v, out, nullptr, err, stream);
}

int launch_stats_hist(const s12_view *v, unsigned long long *hist, cudaStream_t stream) {
    if (cudaMemsetAsync(hist, 0, 256 * sizeof(unsigned long long), stream) != cudaSuccess) return S12_ERR_CUDA;
    if (v->version == 4) return run_decode<4, true>(v, nullptr, hist, nullptr, stream);
    if (v->version == 3) return run_decode<3, true>(v, nullptr, hist, nullptr, stream);
    return v->version == 1 ? run_decode<1, true>(v, nullptr, hist, nullptr, stream)
                           : run_decode<2, true>(v, nullptr, hist, nullptr, stream);
}

}  // namespace s12
