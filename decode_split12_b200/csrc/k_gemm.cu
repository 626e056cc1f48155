// k_gemm.cu -- fused Split12 decode-skinny-GEMM on the tcgen05 tensor cores
// (sm_100a), for the decode phase with 16..256 token rows:
//
//   Y[m][n] = sum_k X[m][k] * W[n][k]      X: M x K bf16,  W: N x K Split12
//
// computed as Y^T = W * X^T so that the compressed matrix is the tensor
// core's A operand (UMMA M = 128 rows of W) and the token rows are its
// N (16..256).  This is the decode-phase case where the product is a real
// dense contraction ("Lossless LLM Weight Compression vs 8-bit GGUF",
// section "How does this compare with prior lossless systems?": fused
// decompression-GEMM; "GPU 友善 12 位無損 BF16 壓縮格式", key points: the
// integer-ADD decode feeding tensor-core kernels).
//
// One CTA per SM, eighteen warps with fixed roles:
//   warp 0      TMA producer: per 64-column chunk of a 128-row tile, the raw
//               plane (128 x 64 bytes), the code plane (128 x 32 bytes) and
//               the X chunk (M x 64 bf16, 128-byte swizzle) into a ring of
//               stages, completing on the stage's mbarrier.
//   warp 1      TMEM owner and MMA issuer: one lane issues four
//               tcgen05.mma.kind::f16 (K = 16 each) per chunk, A = the
//               decoded W chunk in shared memory, B = the X chunk, FP32
//               accumulators in TMEM (128 lanes x M columns), and releases
//               stages and A buffers with tcgen05.commit.
//   warps 2..17 decode: each thread owns 16 weights of one row per chunk,
//               rebuilds the exact BF16 values (byte-wise base + code ADD,
//               escapes patched from the escape stream) and stores them in
//               the canonical K-major 128-byte-swizzled layout the tensor
//               core reads; then, at the end of each tile, the epilogue:
//               tcgen05.ld of the accumulators and the stores of Y.
//
// Work split (stream-K): the (tile, chunk) units are dealt to the CTAs in
// equal contiguous ranges.  A tile covered whole by one CTA goes straight to
// Y; a tile shared by several CTAs is finished by the last of them to
// arrive, which adds the partials in CTA order (deterministic) from the
// workspace and resets the tile's counter to zero.
//
// Every wait is bounded (about a second); a wait that gives up raises
// S12_FLAG_TIMEOUT and the CTA unwinds, waiting (bounded) for its copies in
// flight and freeing its TMEM before it exits.
#include <algorithm>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace gemm {

constexpr int kRows = 128;         // W rows per tile (UMMA M)
constexpr int kChunk = 64;         // K columns per chunk (one 128-byte swizzle atom of bf16)
constexpr int kDecodeWarps = 16;
constexpr int kThreads = 32 * (2 + kDecodeWarps);
constexpr uint32_t kRawBytes = kRows * kChunk;       // 8 KB
constexpr uint32_t kCodeBytes = kRows * kChunk / 2;  // 4 KB
constexpr uint32_t kABytes = kRows * kChunk * 2;     // 16 KB decoded chunk
constexpr int kABufs = 3;
constexpr int kMaxStages = 6;

struct __align__(64) Params {
    CUtensorMap tm_raw;   // u8 [N][K], box 64 x 128
    CUtensorMap tm_code;  // u8 [N][K/2], box 32 x 128
    CUtensorMap tm_x;     // bf16 [M][K], box 64 x Mp, 128-byte swizzle
    const uint8_t *base;
    const uint32_t *esc_off;
    const uint16_t *esc;
    const uint8_t *code;  // the code plane in global memory (escape ranking)
    uint64_t n_esc;
    float *y;             // M x N fp32
    float *part;          // workspace: [grid][2][Mp][kRows] partial tiles
    uint32_t *cnt;        // workspace: one arrival counter per tile (zero between calls)
    uint32_t *err;
    int N, K, T, M, Mp;   // Mp = M rounded up to a multiple of 16
    int n_tiles, n_chunks;  // tiles of 128 rows; 64-column chunks per row
    long long n_units;      // n_tiles * n_chunks
    int stages;
    uint32_t stage_bytes;   // X chunk + raw + code, multiple of 1024
    uint32_t x_bytes;       // Mp * 128
    uint32_t tmem_cols;     // power of two >= max(32, Mp)
};

// ---------------------------------------------------------------------------
// PTX wrappers (tcgen05, TMA, mbarriers).

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Bounded wait for phase `parity`; false after about a second.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_hint(bar, parity, 1000u))  // the thread may sleep up to 1 us per try
        if (clock64() - t0 > kWaitCycles) return false;
    return true;
}

__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap *tm, int c0, int c1, uint32_t bar,
                                      uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(tm), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem] for one 128 x N x 16 step, BF16 -> FP32.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 TMEM lanes x 8 consecutive 32-bit columns into 8 registers per thread.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
}

// 32 TMEM lanes x 4 consecutive 32-bit columns into 4 registers per thread.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes in 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);       // start address
    d |= static_cast<uint64_t>(1u) << 16;                     // leading byte offset (unused for this layout)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;             // stride byte offset: 8 rows
    d |= static_cast<uint64_t>(1u) << 46;                     // descriptor version for sm_100
    d |= static_cast<uint64_t>(2u) << 61;                     // 128-byte swizzle
    return d;
}

// Instruction descriptor: BF16 x BF16 -> FP32, both operands K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t instr_desc(int n) {
    return (1u << 4)                                  // D format FP32
           | (1u << 7)                                // A format BF16
           | (1u << 10)                               // B format BF16
           | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(kRows >> 4) << 24);  // M / 16
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ void sts16(uint32_t a, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}

__device__ __forceinline__ long long unit_start(long long c, long long n, int grid) { return c * n / grid; }

__device__ __forceinline__ long long cta_of_unit(long long b, long long n, int grid) {
    return ((b + 1) * grid + n - 1) / n - 1;
}

}  // namespace gemm
}  // namespace s12

namespace s12 {
namespace gemm {

// Shared-memory layout (offsets from the 1024-aligned base).
struct Layout {
    uint32_t full, empty, a_full, a_empty, acc_full, acc_empty, done;  // mbarriers
    uint32_t tmem_slot, xchg;                                     // 4-byte words
    uint32_t stages, abuf;                                        // data regions
};

__device__ __forceinline__ Layout layout(uint32_t sb, const Params &p) {
    Layout L;
    L.full = sb;
    L.empty = sb + 8 * kMaxStages;
    L.a_full = sb + 16 * kMaxStages;
    L.a_empty = L.a_full + 8 * kABufs;
    L.acc_full = L.a_empty + 8 * kABufs;
    L.acc_empty = L.acc_full + 8;
    L.done = L.acc_empty + 8;
    L.tmem_slot = L.done + 8;
    L.xchg = L.tmem_slot + 4;
    L.stages = sb + 1024;
    L.abuf = L.stages + static_cast<uint32_t>(p.stages) * p.stage_bytes;
    return L;
}

// Decode one 16-weight piece (row r of the tile, columns 16*q4 .. +15 of
// the chunk) from the stage into the A buffer, patching escapes.  Called by
// whole quads (the four lanes of a quad share the row).
// Per-tile metadata of one row: base and escape offsets.
struct RowMeta {
    uint32_t base, lo, hi;
    uint32_t fv0, fv1;  // the tile row's first two escape values (fetched one unit ahead)
};

__device__ __forceinline__ void fetch_escapes(const Params &p, RowMeta &m) {
    m.fv0 = m.fv1 = 0;
    if (m.lo < m.hi && m.lo < p.n_esc) m.fv0 = __ldg(p.esc + m.lo);
    if (m.lo + 1 < m.hi && m.lo + 1 < p.n_esc) m.fv1 = __ldg(p.esc + m.lo + 1);
}

// Rows past the end (zeros from the copy engine) read the last row's
// metadata but report no escapes.
__device__ __forceinline__ RowMeta load_row_meta(const Params &p, long long unit, int r) {
    const int tile = static_cast<int>(unit / p.n_chunks), j = static_cast<int>(unit % p.n_chunks) >> 1;
    const int n = tile * kRows + r;
    const size_t t = static_cast<size_t>(min(n, p.N - 1)) * p.T + j;
    RowMeta m;
    m.base = __ldg(p.base + t);
    m.lo = __ldg(p.esc_off + t);
    m.hi = __ldg(p.esc_off + t + 1);
    if (n >= p.N) m.hi = m.lo;
    m.fv0 = m.fv1 = 0;
    return m;
}

// `carry` holds, after a first-half chunk of a tile row with escapes, that
// half's escape count for the row (all four lanes of the quad); the
// second-half chunk that follows uses it instead of re-reading the codes.
template <bool CHECK>
__device__ __forceinline__ void decode_piece(const Params &p, uint32_t st_raw, uint32_t st_code, uint32_t abuf,
                                             int tile, int chunk, int r, int q4, unsigned full_mask,
                                             const RowMeta &rm, uint32_t &carry, bool carry_ok) {
    const int n = tile * kRows + r;
    const int j = chunk >> 1, h = chunk & 1;
    const int nc = min(n, p.N - 1);
    const uint32_t base = rm.base, lo = rm.lo, hi = rm.hi;
    const uint4 raw = lds128(st_raw + r * 64 + q4 * 16);
    uint2 code = lds64(st_code + r * 32 + q4 * 8);
    const uint32_t rowa = abuf + static_cast<uint32_t>(r) * 128u, sw = static_cast<uint32_t>(r & 7);
    uint2 m = make_uint2(0, 0);
    bool esc = lo != hi;
    if (CHECK) {
        m = make_uint2(escape_nibbles(code.x), escape_nibbles(code.y));
        if ((m.x | m.y) && !esc) raise_flag(p.err, S12_FLAG_ESC_COUNT);
        if (base > static_cast<uint32_t>(kMaxBase)) raise_flag(p.err, S12_FLAG_BASE);
    }
    const unsigned quads = __ballot_sync(full_mask, esc);
    uint32_t rank = 0;
    if (esc) {
        if (!CHECK) m = make_uint2(escape_nibbles(code.x), escape_nibbles(code.y));
        code = make_uint2(clear_escapes(code.x, m.x), clear_escapes(code.y, m.y));  // no carry out of a byte
        const uint32_t cnt = __popc(m.x) + __popc(m.y);
        uint32_t incl = cnt;
#pragma unroll
        for (int d = 1; d < 4; d <<= 1) {
            const uint32_t v = __shfl_up_sync(quads, incl, d, 4);
            if (q4 >= d) incl += v;
        }
        uint32_t before = 0;  // escapes of this tile row in the first half (columns 0..63)
        if (h == 1 && carry_ok) {
            before = carry;
        } else if (h == 1) {
            const uint2 c0 = __ldg(reinterpret_cast<const uint2 *>(p.code + static_cast<size_t>(nc) * (p.K / 2) +
                                                                   static_cast<size_t>(j) * 64 + q4 * 8));
            uint32_t n0 = __popc(escape_nibbles(c0.x)) + __popc(escape_nibbles(c0.y));
            n0 += __shfl_xor_sync(quads, n0, 1, 4);
            n0 += __shfl_xor_sync(quads, n0, 2, 4);
            before = n0;
        }
        const uint32_t total_half = __shfl_sync(quads, incl, 3, 4);
        if (h == 0) carry = total_half;
        if (h == 1 && q4 == 0 && before + total_half != hi - lo) raise_flag(p.err, S12_FLAG_ESC_COUNT);
        if (h == 0 && q4 == 0 && total_half > hi - lo) raise_flag(p.err, S12_FLAG_ESC_COUNT);
        rank = lo + before + incl - cnt;
    }
    uint32_t w[8];
    decode16(raw, code, base * 0x01010101u, w);
    sts128(rowa + (((2u * q4) ^ sw) << 4), w[0], w[1], w[2], w[3]);
    sts128(rowa + (((2u * q4 + 1u) ^ sw) << 4), w[4], w[5], w[6], w[7]);
    if (esc && (m.x | m.y)) {
        const uint32_t limit = lo <= hi ? static_cast<uint32_t>(hi < p.n_esc ? hi : p.n_esc) : 0u;
        uint64_t mm = (static_cast<uint64_t>(m.y) << 32) | m.x;
        uint32_t idx = rank;
        while (mm) {
            const int jj = (__ffsll(static_cast<long long>(mm)) - 1) >> 2;  // weight within the piece
            mm &= mm - 1;
            uint16_t v = 0;
            if (idx < limit)
                v = idx == lo ? static_cast<uint16_t>(rm.fv0)
                              : (idx == lo + 1 ? static_cast<uint16_t>(rm.fv1) : __ldg(p.esc + idx));
            else
                raise_flag(p.err, S12_FLAG_ESC_RANGE);
            ++idx;
            const uint32_t kl = static_cast<uint32_t>(q4 * 16 + jj);  // column within the chunk
            sts16(rowa + ((((kl >> 3) ^ sw)) << 4) + (kl & 7u) * 2u, v);
        }
    }
}

}  // namespace gemm
}  // namespace s12

namespace s12 {
namespace gemm {

// Epilogue for tile `tile` (the accumulators are final for this CTA's part
// of it): store Y directly, or hand the partial to the stream-K fix-up.
// Run by the 512 decode threads (warps 2..17); ew = warp - 2.
__device__ __forceinline__ void epilogue(const Params &p, uint32_t tmem, const Layout &L, int tile, long long u0,
                                         long long u1, int ew, int lane) {
    const int warp = ew + 2;
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31 are this warp's
    const int row = quad * 32 + lane;          // row within the tile
    const int n = tile * kRows + row;
    const int part_cols = p.Mp / 4, c_begin = (ew >> 2) * part_cols;  // four warps share a lane quadrant
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const long long t0 = static_cast<long long>(tile) * p.n_chunks, t1 = t0 + p.n_chunks;
    const bool whole = t0 >= u0 && t1 <= u1;
    const int cta = blockIdx.x;
    const int slot = (tile == static_cast<int>(u0 / p.n_chunks)) ? 0 : 1;
    float *mine = p.part + (static_cast<size_t>(cta) * 2 + slot) * static_cast<size_t>(p.Mp) * kRows;
    for (int c = c_begin; c < c_begin + part_cols; c += 4) {
        uint32_t v[4];
        tmem_ld4(taddr + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = c + i;
            if (whole) {
                if (m < p.M && n < p.N) p.y[static_cast<size_t>(m) * p.N + n] = __uint_as_float(v[i]);
            } else {
                __stcg(mine + static_cast<size_t>(m) * kRows + row, __uint_as_float(v[i]));
            }
        }
    }
    if (whole) return;
    // stream-K fix-up: the last contributor of the tile adds the partials in
    // CTA order and writes Y
    __threadfence();
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeWarps) : "memory");
    const long long n_units = p.n_units;
    const int grid = gridDim.x;
    const long long cf = cta_of_unit(t0, n_units, grid), cl = cta_of_unit(t1 - 1, n_units, grid);
    if (ew == 0 && lane == 0) {
        uint32_t n_contrib = 0;
        for (long long c = cf; c <= cl; ++c)
            if (unit_start(c, n_units, grid) < unit_start(c + 1, n_units, grid)) ++n_contrib;
        const uint32_t prev = atomicAdd(p.cnt + tile, 1u);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(L.xchg), "r"(prev + 1 == n_contrib ? 1u : 0u) : "memory");
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeWarps) : "memory");
    uint32_t last;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(last) : "r"(L.xchg) : "memory");
    if (!last) return;
    __threadfence();
    for (int idx = ew * 32 + lane; idx < p.Mp * kRows; idx += 32 * kDecodeWarps) {
        const int m = idx / kRows, r = idx - m * kRows;
        float s = 0.f;
        for (long long c = cf; c <= cl; ++c) {
            const long long cs = unit_start(c, n_units, grid);
            if (cs >= unit_start(c + 1, n_units, grid)) continue;
            const int sl = (tile == static_cast<int>(cs / p.n_chunks)) ? 0 : 1;
            s += __ldcg(p.part + (static_cast<size_t>(c) * 2 + sl) * static_cast<size_t>(p.Mp) * kRows +
                        static_cast<size_t>(idx));
        }
        const int nn = tile * kRows + r;
        if (m < p.M && nn < p.N) p.y[static_cast<size_t>(m) * p.N + nn] = s;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeWarps) : "memory");
    if (ew == 0 && lane == 0) atomicExch(p.cnt + tile, 0u);
}

template <bool CHECK>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sb = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const Layout L = layout(sb, p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long u0 = unit_start(blockIdx.x, p.n_units, gridDim.x);
    const long long u1 = unit_start(blockIdx.x + 1, p.n_units, gridDim.x);
    const int S = p.stages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            bar_init(L.full + 8 * s, 1);
            bar_init(L.empty + 8 * s, kDecodeWarps + 1);
        }
        for (int a = 0; a < kABufs; ++a) {
            bar_init(L.a_full + 8 * a, kDecodeWarps);
            bar_init(L.a_empty + 8 * a, 1);
        }
        bar_init(L.acc_full, 1);
        bar_init(L.acc_empty, kDecodeWarps);
        bar_init(L.done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(L.tmem_slot, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t tmem;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(tmem) : "r"(L.tmem_slot) : "memory");
    if (warp == 0) {
        // ---- TMA producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            int s = 0;
            uint32_t round = 0;
            long long issued = 0;
            for (long long u = u0; u < u1; ++u) {
                const int tile = static_cast<int>(u / p.n_chunks), chunk = static_cast<int>(u % p.n_chunks);
                if (!bar_wait(L.empty + 8 * s, (round & 1u) ^ 1u)) {
                    raise_flag(p.err, S12_FLAG_TIMEOUT);
                    break;
                }
                const uint32_t st = L.stages + static_cast<uint32_t>(s) * p.stage_bytes;
                bar_expect_tx(L.full + 8 * s, p.x_bytes + kRawBytes + kCodeBytes);
                tma2d(st, &p.tm_x, chunk * kChunk, 0, L.full + 8 * s, pol_x);
                tma2d(st + p.x_bytes, &p.tm_raw, chunk * kChunk, tile * kRows, L.full + 8 * s, pol_w);
                tma2d(st + p.x_bytes + kRawBytes, &p.tm_code, chunk * (kChunk / 2), tile * kRows, L.full + 8 * s,
                      pol_w);
                ++issued;
                if (++s == S) {
                    s = 0;
                    ++round;
                }
            }
            // let every copy this CTA started land before it exits (already
            // true when the consumers ran to the end)
            for (long long i = issued > S ? issued - S : 0; i < issued; ++i)
                bar_wait(L.full + 8 * static_cast<uint32_t>(i % S), static_cast<uint32_t>((i / S) & 1));
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = instr_desc(p.Mp);
            int s = 0, a = 0;
            uint32_t round = 0, around = 0, tiles = 0;
            for (long long u = u0; u < u1; ++u) {
                const int chunk = static_cast<int>(u % p.n_chunks);
                const bool first = (u == u0) || chunk == 0;
                const bool last = (u + 1 == u1) || chunk == p.n_chunks - 1;
                bool w = bar_wait(L.full + 8 * s, round & 1u) && bar_wait(L.a_full + 8 * a, around & 1u);
                if (w && first) w = bar_wait(L.acc_empty, (tiles & 1u) ^ 1u);
                if (!w) {
                    raise_flag(p.err, S12_FLAG_TIMEOUT);
                    break;
                }
                if (first) ++tiles;
                tc_fence_after();
                const uint32_t xa = L.stages + static_cast<uint32_t>(s) * p.stage_bytes;
                const uint32_t aa = L.abuf + static_cast<uint32_t>(a) * kABytes;
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    umma_bf16(tmem, smem_desc_sw128(aa + kk * 32), smem_desc_sw128(xa + kk * 32), idesc,
                              (first && kk == 0) ? 0u : 1u);
                umma_commit(L.empty + 8 * s);
                umma_commit(L.a_empty + 8 * a);
                if (last) umma_commit(L.acc_full);
                if (++s == S) {
                    s = 0;
                    ++round;
                }
                if (++a == kABufs) {
                    a = 0;
                    ++around;
                }
            }
            // every product issued has completed before TMEM is freed
            umma_commit(L.done);
            bar_wait(L.done, 0);
        }
    } else {
        // ---- decode warps (and the epilogue)
        const int ew = warp - 2;
        const int t = ew * 32 + lane;
        const int q4 = t & 3, r = t >> 2;  // row r of each chunk, columns 16*q4 .. +15
        int s = 0, a = 0;
        uint32_t round = 0, around = 0, tiles = 0;
        // the row metadata of the next two units is in flight while a unit is decoded
        RowMeta m0 = {0, 0, 0, 0, 0}, m1 = {0, 0, 0, 0, 0};
        if (u0 < u1) {
            m0 = load_row_meta(p, u0, r);
            fetch_escapes(p, m0);
        }
        if (u0 + 1 < u1) m1 = load_row_meta(p, u0 + 1, r);
        uint32_t carry = 0;
        for (long long u = u0; u < u1; ++u) {
            const int tile = static_cast<int>(u / p.n_chunks), chunk = static_cast<int>(u % p.n_chunks);
            const bool last = (u + 1 == u1) || chunk == p.n_chunks - 1;
            RowMeta m2 = m1;
            if (u + 2 < u1) m2 = load_row_meta(p, u + 2, r);
            if (u + 1 < u1) fetch_escapes(p, m1);  // m1's offsets arrived during the previous unit
            const bool w = bar_wait(L.full + 8 * s, round & 1u) && bar_wait(L.a_empty + 8 * a, (around & 1u) ^ 1u);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                raise_flag(p.err, S12_FLAG_TIMEOUT);
                break;
            }
            const uint32_t st = L.stages + static_cast<uint32_t>(s) * p.stage_bytes;
            const uint32_t aa = L.abuf + static_cast<uint32_t>(a) * kABytes;
            decode_piece<CHECK>(p, st + p.x_bytes, st + p.x_bytes + kRawBytes, aa, tile, chunk, r, q4, 0xFFFFFFFFu, m0,
                                carry, u > u0);
            m0 = m1;
            m1 = m2;
            // generic-proxy stores must be visible to the tensor core
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                bar_arrive(L.a_full + 8 * a);
                bar_arrive(L.empty + 8 * s);
            }
            if (++s == S) {
                s = 0;
                ++round;
            }
            if (++a == kABufs) {
                a = 0;
                ++around;
            }
            if (last) {
                const bool wa = bar_wait(L.acc_full, tiles & 1u);
                if (!__all_sync(0xFFFFFFFFu, wa)) {
                    raise_flag(p.err, S12_FLAG_TIMEOUT);
                    break;
                }
                ++tiles;
                tc_fence_after();
                epilogue(p, tmem, L, tile, u0, u1, ew, lane);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) bar_arrive(L.acc_empty);
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

}  // namespace gemm

// ---------------------------------------------------------------------------
// Host side.

namespace {

constexpr uint32_t kSmemLimit = 227 * 1024;

struct Plan {
    int Mp, n_tiles, n_chunks, grid, stages;
    long long n_units;
    uint32_t x_bytes, stage_bytes, tmem_cols, smem;
    size_t part_bytes, cnt_bytes;
};

Plan plan(const s12_view *v, int M, int sms) {
    Plan pl;
    pl.Mp = (M + 15) / 16 * 16;
    pl.n_tiles = static_cast<int>((v->rows + gemm::kRows - 1) / gemm::kRows);
    pl.n_chunks = static_cast<int>(v->cols / gemm::kChunk);
    pl.n_units = static_cast<long long>(pl.n_tiles) * pl.n_chunks;
    pl.grid = static_cast<int>(std::max(1LL, std::min<long long>(sms, pl.n_units)));
    pl.x_bytes = static_cast<uint32_t>(pl.Mp) * 128u;
    pl.stage_bytes = pl.x_bytes + gemm::kRawBytes + gemm::kCodeBytes;
    const uint32_t fixed = 1024 + 1024 + gemm::kABufs * gemm::kABytes;  // alignment slack, barriers, A buffers
    pl.stages = static_cast<int>(std::min<uint32_t>(gemm::kMaxStages, (kSmemLimit - fixed) / pl.stage_bytes));
    pl.smem = fixed + static_cast<uint32_t>(pl.stages) * pl.stage_bytes;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(pl.Mp)) cols <<= 1;
    pl.tmem_cols = cols;
    // sized for the largest grid so one workspace fits every call with this M
    pl.part_bytes = align_up(static_cast<uint64_t>(sms) * 2 * pl.Mp * gemm::kRows * sizeof(float), kAlign);
    pl.cnt_bytes = align_up(static_cast<uint64_t>(pl.n_tiles) * sizeof(uint32_t), kAlign);
    return pl;
}

}  // namespace

size_t gemm_ws_bytes(const s12_view *v, int M) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return 0;
    const Plan pl = plan(v, M, sms);
    return pl.part_bytes + pl.cnt_bytes;
}

int launch_gemm(const s12_view *v, const uint16_t *x, int M, float *y, void *ws, size_t ws_bytes, uint32_t *err,
                cudaStream_t stream) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    const Plan pl = plan(v, M, sms);
    if (!ws || ws_bytes < pl.part_bytes + pl.cnt_bytes) return S12_ERR_CAPACITY;
    if (pl.stages < 2) return S12_ERR_SHAPE;
    gemm::Params p = {};
    const uint64_t N = v->rows, K = v->cols;
    if (make_tmap_u8_2d(&p.tm_raw, v->raw, K, N, K, gemm::kChunk, gemm::kRows, false) != S12_OK) return S12_ERR_CUDA;
    if (make_tmap_u8_2d(&p.tm_code, v->code, K / 2, N, K / 2, gemm::kChunk / 2, gemm::kRows, false) != S12_OK)
        return S12_ERR_CUDA;
    if (make_tmap_bf16_2d(&p.tm_x, x, K, static_cast<uint64_t>(M), K * 2, gemm::kChunk, static_cast<uint32_t>(pl.Mp),
                          true) != S12_OK)
        return S12_ERR_CUDA;
    p.base = v->base;
    p.esc_off = v->esc_off;
    p.esc = v->esc;
    p.code = v->code;
    p.n_esc = v->n_esc;
    p.y = y;
    p.part = static_cast<float *>(ws);
    p.cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + pl.part_bytes);
    p.err = err;
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.T = p.K / kTile;
    p.M = M;
    p.Mp = pl.Mp;
    p.n_tiles = pl.n_tiles;
    p.n_chunks = pl.n_chunks;
    p.n_units = pl.n_units;
    p.stages = pl.stages;
    p.stage_bytes = pl.stage_bytes;
    p.x_bytes = pl.x_bytes;
    p.tmem_cols = pl.tmem_cols;
    auto kern = err ? gemm::gemm_tc_kernel<true> : gemm::gemm_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess)
        return S12_ERR_CUDA;
    kern<<<pl.grid, gemm::kThreads, pl.smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace s12
