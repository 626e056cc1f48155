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
//   warp 0      TMA producer: per unit (a 128-row tile x one 128-column tile
//               column), the raw plane (128 x 128 bytes, 128-byte swizzle),
//               the code plane (128 x 64 bytes) and the X columns (M x 128
//               bf16 as two 128-byte-swizzled atoms) into a ring of stages,
//               completing on the stage's mbarrier.
//   warp 1      TMEM owner and MMA issuer: one lane issues eight
//               tcgen05.mma.kind::f16 (K = 16 each) per unit, A = the
//               decoded W unit in shared memory, B = the X columns, FP32
//               accumulators in TMEM (128 lanes x M columns), and releases
//               stages and A buffers with tcgen05.commit.
//   warps 2..17 decode: each thread owns 32 weights of one row per unit,
//               rebuilds the exact BF16 values (byte-wise base + code ADD,
//               escapes patched from the escape stream) and stores them in
//               the canonical K-major 128-byte-swizzled layout the tensor
//               core reads; then, at the end of each tile, the epilogue:
//               tcgen05.ld of the accumulators and the stores of Y.
//
// A call may hold up to S12_GEMM_MAX_PROBLEMS matrices (s12_gemm_skinny_multi,
// for instance the experts of a mixture-of-experts block), each with its own
// shape, token rows and output; they share the tensor core's N (the largest
// M rounded up to 16), and their units are numbered matrix after matrix.
//
// Work split (stream-K): the (tile, tile column) units are dealt to the CTAs in
// equal contiguous ranges.  A tile covered whole by one CTA goes straight to
// Y; a tile shared by several CTAs is finished by the last of them to
// arrive, which adds the partials in CTA order (deterministic) from the
// workspace and resets the tile's counter to zero.
//
// Every wait is bounded (about a second); a wait that gives up raises
// S12_FLAG_TIMEOUT and the CTA unwinds, waiting (bounded) for its copies in
// flight and freeing its TMEM before it exits.  An unwinding CTA still
// arrives on the counter of every shared tile it had not yet finished, so
// the counters return to zero (Y is then not valid; the flag says so).
//
// Both container versions are read: version 1 keeps per tile a base byte and
// an escape offset; version 2 (compact header) keeps per tile one u16 of
// base | escape count and per row one escape offset, and each decode thread
// carries its row's running offset from tile column to tile column.  Y is
// written as FP32 or, for callers whose next step takes BF16, rounded to
// BF16 (nearest even).
#include <algorithm>

#include <cuda_bf16.h>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace gemm {

constexpr int kRows = 128;         // W rows per tile (UMMA M)
constexpr int kChunk = 128;        // K columns per unit: one whole tile row
constexpr int kAtom = 64;          // bf16 columns per 128-byte swizzle atom
constexpr int kDecodeWarps = 16;
constexpr int kThreads = 32 * (2 + kDecodeWarps);
constexpr uint32_t kRawBytes = kRows * kChunk;       // 16 KB
constexpr uint32_t kCodeBytes = kRows * kChunk / 2;  // 8 KB
constexpr uint32_t kAtomBytes = kRows * kAtom * 2;   // 16 KB: one swizzle atom of the decoded unit
constexpr uint32_t kABytes = 2 * kAtomBytes;         // 32 KB
constexpr int kMaxABufs = 3;
constexpr int kMaxStages = 6;
constexpr int kMaxProblems = S12_GEMM_MAX_PROBLEMS;

// One matrix of a call (a grouped call has several, with their own shapes,
// token rows and outputs).
struct __align__(64) Problem {
    CUtensorMap tm_raw;   // u8 [N][K], box 128 x 128, 128-byte swizzle
    CUtensorMap tm_code;  // u8 [N][K/2], box 64 x 128
    CUtensorMap tm_x;     // bf16 [M][K], box 64 x Mp, 128-byte swizzle (rows >= M read as 0)
    const void *meta;       // version 1: base u8[n_tiles]; version 2: (base | count << 8) u16[n_tiles]
    const uint32_t *off;    // version 1: esc_off u32[n_tiles + 1]; version 2: row_esc u32[N + 1]
    const uint16_t *esc;
    uint64_t n_esc;
    void *y;                // M x N, fp32 (out 0) or bf16 (out 1)
    int out;
    long long unit0;        // first unit of this matrix in the call's numbering
    int N, K, T, M;
    int n_tiles, n_chunks;  // tiles of 128 rows; 128-column units per row (= tiles per row)
    int tile0;              // first tile of this matrix in the call's numbering (counters)
};

template <int NP>
struct __align__(64) Params {
    Problem prob[NP];
    float *part;          // workspace: [grid][2][Mp][kRows] partial tiles
    uint32_t *cnt;        // workspace: one arrival counter per tile (zero between calls)
    uint32_t *err;
    int n_problems;
    int Mp;               // the largest M of the call rounded up to a multiple of 16
    long long n_units;    // all matrices' units
    int stages;
    uint32_t stage_bytes;   // X chunk + raw + code, multiple of 1024
    uint32_t x_bytes;       // Mp * 256: the unit's X columns as two swizzle atoms
    uint32_t x_atom;        // Mp * 128
    int a_bufs;             // decoded-unit buffers, 1 or 2
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
    while (!mbar_try_wait(bar, parity))
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
    uint32_t tmem_slot, xchg, abort, n_done;                      // 4-byte words
    uint32_t stages, abuf;                                        // data regions
};

template <int NP>
__device__ __forceinline__ Layout layout(uint32_t sb, const Params<NP> &p) {
    Layout L;
    L.full = sb;
    L.empty = sb + 8 * kMaxStages;
    L.a_full = sb + 16 * kMaxStages;
    L.a_empty = L.a_full + 8 * kMaxABufs;
    L.acc_full = L.a_empty + 8 * kMaxABufs;
    L.acc_empty = L.acc_full + 8;
    L.done = L.acc_empty + 8;
    L.tmem_slot = L.done + 8;
    L.xchg = L.tmem_slot + 4;
    L.abort = L.xchg + 4;   // set when a wait of this CTA gave up
    L.n_done = L.abort + 4; // tiles of this CTA whose counter arrival is done (or not needed)
    L.stages = sb + 1024;
    L.abuf = L.stages + static_cast<uint32_t>(p.stages) * p.stage_bytes;
    return L;
}

// Decode one 16-weight piece (row r of the tile, columns 16*q4 .. +15 of
// the chunk) from the stage into the A buffer, patching escapes.  Called by
// whole quads (the four lanes of a quad share the row).
// Per-tile metadata of one row: base and escape offsets.
// (Escape values are read when a unit needs them: fetching a row's first
// two one unit ahead cost more per unit than it hid, 6 % at M = 16.)
// The words as loaded (any arithmetic on them at load time would make the
// thread wait for the load there):
//   version 1:  w0 = base, w1 = esc_off[t], w2 = esc_off[t+1]
//   version 2:  w0 = tmeta[t], w1 = row_esc[n] on a row's first tile column
struct RowMeta {
    uint32_t w0, w1, w2;
    int pi;  // the matrix the unit belongs to
};

// Base and escape span [lo, hi) of a row's tile; `run` carries the row's
// escape offset (version 2) from one tile column to the next.
struct RowSpan {
    uint32_t base, lo, hi;
};

template <int V>
__device__ __forceinline__ RowSpan row_span(const RowMeta &m, int chunk, uint32_t &run) {
    if (V == 1) return RowSpan{m.w0, m.w1, m.w2};
    if (chunk == 0) run = m.w1;
    const RowSpan s{m.w0 & 0xFFu, run, run + (m.w0 >> 8)};
    run = s.hi;
    return s;
}

// Rows past the end (zeros from the copy engine) read the last row's
// metadata but report no escapes.
// A unit's position: matrix, 128-row tile and tile column, advanced without
// division (units run tile-major within a matrix, matrices in call order).
struct UPos {
    int p, tile, chunk;
};

// (with one matrix, NP = 1, the matrix index stays a compile-time 0)
template <int NP>
__device__ __forceinline__ void next(UPos &q, const Params<NP> &P) {
    if (++q.chunk == P.prob[NP == 1 ? 0 : q.p].n_chunks) {
        q.chunk = 0;
        ++q.tile;
        if (NP > 1 && q.tile == P.prob[q.p].n_tiles) {
            q.tile = 0;
            if (q.p + 1 < P.n_problems) ++q.p;
        }
    }
}

// Position of unit u (one division, once per CTA).
template <int NP>
__device__ __forceinline__ UPos locate(const Params<NP> &P, long long u) {
    int i = 0;
    if (NP > 1)
        while (i + 1 < P.n_problems && u >= P.prob[i + 1].unit0) ++i;
    const long long lu = u - P.prob[i].unit0;
    UPos q;
    q.p = i;
    q.tile = static_cast<int>(lu / P.prob[i].n_chunks);
    q.chunk = static_cast<int>(lu - static_cast<long long>(q.tile) * P.prob[i].n_chunks);
    return q;
}

template <int V, int NP>
__device__ __forceinline__ RowMeta load_row_meta(const Params<NP> &P, UPos q, int r) {
    const Problem &p = P.prob[q.p];
    const int tile = q.tile, j = q.chunk;  // a unit is one whole tile column
    const int n = tile * kRows + r;
    const int nc = min(n, p.N - 1);
    const size_t t = static_cast<size_t>(nc) * p.T + j;
    RowMeta m;
    if (V == 1) {
        m.w0 = __ldg(static_cast<const uint8_t *>(p.meta) + t);
        m.w1 = __ldg(p.off + t);
        m.w2 = n < p.N ? __ldg(p.off + t + 1) : m.w1;
    } else {
        const uint32_t w = __ldg(static_cast<const uint16_t *>(p.meta) + t);
        m.w0 = n < p.N ? w : (w & 0xFFu);  // rows past the end: no escapes
        m.w1 = j == 0 ? __ldg(p.off + nc) : 0u;
        m.w2 = 0u;
    }
    m.pi = q.p;
    return m;
}

// Version 2: escape offset of row r of the unit at q before its tile column
// (row_esc plus the counts of the row's earlier tiles), summed by the four
// lanes that share the row (lanes l, l^8, l^16, l^24; lane q4 takes tiles
// q4, q4 + 4, ...).
template <int NP>
__device__ __forceinline__ uint32_t row_offset_v2(const Params<NP> &P, UPos q, int r, int q4) {
    const Problem &p = P.prob[q.p];
    const int nc = min(q.tile * kRows + r, p.N - 1);
    const uint16_t *tm = static_cast<const uint16_t *>(p.meta) + static_cast<size_t>(nc) * p.T;
    uint32_t s = 0;
    for (int k = q4; k < q.chunk; k += 4) s += __ldg(tm + k) >> 8;
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 8);
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 16);
    return s + __ldg(p.off + nc);
}

// Decode the lane's 32 weights of one tile row (row r of the unit, columns
// 32*q4 .. +31, as two 16-weight chunks) from the stage into the A buffer,
// patching escapes.  Called by all 32 lanes; the four lanes of a quad share
// the row, and escapes are ranked within the row with quad shuffles (chunk
// order: lane q4 = 0..3, first chunk then second).
template <bool CHECK>
__device__ __forceinline__ void decode_row(const Problem &p, uint32_t *err, uint32_t st_raw, uint32_t st_code,
                                           uint32_t abuf, int r, int q4, const RowSpan &rm) {
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    const uint32_t lo = rm.lo, hi = rm.hi;
    const uint4 rw0 = lds128(st_raw + r * 128 + (((2u * q4) ^ sw) << 4));  // raw rows are 128-byte swizzled
    const uint4 rw1 = lds128(st_raw + r * 128 + (((2u * q4 + 1u) ^ sw) << 4));
    uint4 code = lds128(st_code + r * 64 + 16 * (static_cast<uint32_t>(q4) ^ ((static_cast<uint32_t>(r) >> 1) & 3u)));
    bool esc = lo != hi;
    uint2 m0 = make_uint2(0, 0), m1 = make_uint2(0, 0);
    if (CHECK) {
        m0 = make_uint2(escape_nibbles(code.x), escape_nibbles(code.y));
        m1 = make_uint2(escape_nibbles(code.z), escape_nibbles(code.w));
        if ((m0.x | m0.y | m1.x | m1.y) && !esc) raise_flag(err, S12_FLAG_ESC_COUNT);
        if (rm.base > static_cast<uint32_t>(kMaxBase)) raise_flag(err, S12_FLAG_BASE);
    }
    const unsigned quads = __ballot_sync(0xFFFFFFFFu, esc);
    uint32_t s0 = 0, s1 = 0;
    if (esc) {
        if (!CHECK) {
            m0 = make_uint2(escape_nibbles(code.x), escape_nibbles(code.y));
            m1 = make_uint2(escape_nibbles(code.z), escape_nibbles(code.w));
        }
        // clear the escape nibbles so base + code never carries out of a byte
        code = make_uint4(clear_escapes(code.x, m0.x), clear_escapes(code.y, m0.y), clear_escapes(code.z, m1.x),
                          clear_escapes(code.w, m1.y));
        const uint32_t n0 = __popc(m0.x) + __popc(m0.y), n = n0 + __popc(m1.x) + __popc(m1.y);
        uint32_t incl = n;
#pragma unroll
        for (int d = 1; d < 4; d <<= 1) {
            const uint32_t v = __shfl_up_sync(quads, incl, 8 * d);
            if (q4 >= d) incl += v;
        }
        const uint32_t tot = __shfl_sync(quads, incl, 24 + (r & 7));
        if (q4 == 0 && tot != hi - lo) raise_flag(err, S12_FLAG_ESC_COUNT);
        s0 = lo + incl - n;
        s1 = s0 + n0;
    }
    // columns 32*q4 .. +31 lie in atom q4 / 2, at 16-byte pieces pb .. pb + 3
    const uint32_t row = abuf + static_cast<uint32_t>(q4 >> 1) * kAtomBytes + static_cast<uint32_t>(r) * 128u;
    const uint32_t pb = 4u * static_cast<uint32_t>(q4 & 1);
    const uint32_t B4 = rm.base * 0x01010101u;
    uint32_t w[8];
    decode16(rw0, make_uint2(code.x, code.y), B4, w);
    sts128(row + (((pb + 0u) ^ sw) << 4), w[0], w[1], w[2], w[3]);
    sts128(row + (((pb + 1u) ^ sw) << 4), w[4], w[5], w[6], w[7]);
    decode16(rw1, make_uint2(code.z, code.w), B4, w);
    sts128(row + (((pb + 2u) ^ sw) << 4), w[0], w[1], w[2], w[3]);
    sts128(row + (((pb + 3u) ^ sw) << 4), w[4], w[5], w[6], w[7]);
    if (esc) {
        const uint32_t limit = lo <= hi ? static_cast<uint32_t>(hi < p.n_esc ? hi : p.n_esc) : 0u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint2 m = h ? m1 : m0;
            uint64_t mm = (static_cast<uint64_t>(m.y) << 32) | m.x;
            uint32_t idx = h ? s1 : s0;
            while (mm) {
                const uint32_t jj = static_cast<uint32_t>((__ffsll(static_cast<long long>(mm)) - 1) >> 2);
                mm &= mm - 1;
                uint16_t v = 0;
                if (idx < limit)
                    v = __ldg(p.esc + idx);
                else
                    raise_flag(err, S12_FLAG_ESC_RANGE);
                ++idx;
                const uint32_t kl = 8u * pb + 16u * h + jj;  // column within the atom
                sts16(row + (((kl >> 3) ^ sw) << 4) + (kl & 7u) * 2u, v);
            }
        }
    }
}

}  // namespace gemm
}  // namespace s12

namespace s12 {
namespace gemm {

__device__ __forceinline__ void store_y(const Problem &pr, size_t o, float v) {
    if (pr.out == 1)
        static_cast<uint16_t *>(pr.y)[o] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    else
        static_cast<float *>(pr.y)[o] = v;
}

// One more tile of this CTA has its counter arrival behind it (or needs none).
__device__ __forceinline__ void note_done(const Layout &L) {
    uint32_t n;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(n) : "r"(L.n_done) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(L.n_done), "r"(n + 1) : "memory");
}

// A wait gave up: raise the flag and mark the CTA as unwinding.
template <int NP>
__device__ __forceinline__ void give_up(const Params<NP> &p, const Layout &L) {
    raise_flag(p.err, S12_FLAG_TIMEOUT);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(L.abort), "r"(1u) : "memory");
}

// Number of CTAs whose unit range meets tile units [t0, t1).
__device__ __forceinline__ uint32_t contributors(long long t0, long long t1, long long n_units, int grid) {
    const long long cf = cta_of_unit(t0, n_units, grid), cl = cta_of_unit(t1 - 1, n_units, grid);
    uint32_t n = 0;
    for (long long c = cf; c <= cl; ++c)
        if (unit_start(c, n_units, grid) < unit_start(c + 1, n_units, grid)) ++n;
    return n;
}

// After an unwinding CTA's threads have all stopped: arrive on the counter of
// every tile of its range that it shares with other CTAs and had not yet
// finished, resetting the counter when this arrival is the last.  Run by one
// thread.
template <int NP>
__device__ void abort_arrivals(const Params<NP> &p, const Layout &L, long long u0, long long u1) {
    uint32_t n_done;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(n_done) : "r"(L.n_done) : "memory");
    UPos q = locate(p, u0);
    uint32_t k = 0;
    for (long long u = u0; u < u1; ++k) {
        const Problem &pr = p.prob[q.p];
        const long long t0 = pr.unit0 + static_cast<long long>(q.tile) * pr.n_chunks, t1 = t0 + pr.n_chunks;
        if (k >= n_done && !(t0 >= u0 && t1 <= u1)) {
            const uint32_t gtile = static_cast<uint32_t>(pr.tile0 + q.tile);
            const uint32_t prev = atomicAdd(p.cnt + gtile, 1u);
            if (prev + 1 == contributors(t0, t1, p.n_units, gridDim.x)) atomicExch(p.cnt + gtile, 0u);
        }
        u = t1;
        q.chunk = 0;
        if (++q.tile == pr.n_tiles) {
            q.tile = 0;
            ++q.p;
        }
    }
}

// Epilogue for tile `tile` of matrix pr (the accumulators are final for this
// CTA's part of it): store Y directly, or hand the partial to the stream-K
// fix-up.  gtile is the tile's index in the call's numbering (its counter),
// [t0, t1) its units.  A CTA's first tile uses partial slot 0, any later one
// slot 1; the CTA whose range starts at unit cs therefore used slot 0 for
// this tile exactly when cs >= t0.  Run by the 512 decode threads (warps
// 2..17); ew = warp - 2.
template <int NP>
__device__ __forceinline__ void epilogue(const Params<NP> &p, const Problem &pr, uint32_t tmem, const Layout &L,
                                         int tile, int gtile, long long t0, long long u0, long long u1, int ew,
                                         int lane) {
    const int warp = ew + 2;
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31 are this warp's
    const int row = quad * 32 + lane;          // row within the tile
    const int n = tile * kRows + row;
    const int part_cols = p.Mp / 4, c_begin = (ew >> 2) * part_cols;  // four warps share a lane quadrant
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const long long t1 = t0 + pr.n_chunks;
    const bool whole = t0 >= u0 && t1 <= u1;
    const int cta = blockIdx.x;
    const int slot = u0 >= t0 ? 0 : 1;
    float *mine = p.part + (static_cast<size_t>(cta) * 2 + slot) * static_cast<size_t>(p.Mp) * kRows;
    for (int c = c_begin; c < c_begin + part_cols; c += 4) {
        uint32_t v[4];
        tmem_ld4(taddr + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = c + i;
            if (whole) {
                if (m < pr.M && n < pr.N) store_y(pr, static_cast<size_t>(m) * pr.N + n, __uint_as_float(v[i]));
            } else {
                __stcg(mine + static_cast<size_t>(m) * kRows + row, __uint_as_float(v[i]));
            }
        }
    }
    if (whole) {
        if (ew == 0 && lane == 0) note_done(L);
        return;
    }
    // stream-K fix-up: the last contributor of the tile adds the partials in
    // CTA order and writes Y
    __threadfence();
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeWarps) : "memory");
    const long long n_units = p.n_units;
    const int grid = gridDim.x;
    const long long cf = cta_of_unit(t0, n_units, grid), cl = cta_of_unit(t1 - 1, n_units, grid);
    if (ew == 0 && lane == 0) {
        const uint32_t n_contrib = contributors(t0, t1, n_units, grid);
        const uint32_t prev = atomicAdd(p.cnt + gtile, 1u);
        note_done(L);
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
            const int sl = cs >= t0 ? 0 : 1;
            s += __ldcg(p.part + (static_cast<size_t>(c) * 2 + sl) * static_cast<size_t>(p.Mp) * kRows +
                        static_cast<size_t>(idx));
        }
        const int nn = tile * kRows + r;
        if (m < pr.M && nn < pr.N) store_y(pr, static_cast<size_t>(m) * pr.N + nn, s);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecodeWarps) : "memory");
    if (ew == 0 && lane == 0) atomicExch(p.cnt + gtile, 0u);
}

template <bool CHECK, int NP, int V>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params<NP> p) {
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
        for (int a = 0; a < p.a_bufs; ++a) {
            bar_init(L.a_full + 8 * a, kDecodeWarps);
            bar_init(L.a_empty + 8 * a, 1);
        }
        bar_init(L.acc_full, 1);
        bar_init(L.acc_empty, kDecodeWarps);
        bar_init(L.done, 1);
        asm volatile("st.shared.v2.u32 [%0], {%1, %1};" ::"r"(L.abort), "r"(0u) : "memory");
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
    const UPos q0 = u0 < u1 ? locate(p, u0) : UPos{0, 0, 0};
    if (warp == 0) {
        // ---- TMA producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            int s = 0;
            uint32_t round = 0;
            long long issued = 0;
            UPos q = q0;
            for (long long u = u0; u < u1; ++u, next(q, p)) {
                const Problem &pr = p.prob[q.p];
                const int tile = q.tile, chunk = q.chunk;
                if (!bar_wait(L.empty + 8 * s, (round & 1u) ^ 1u)) {
                    give_up(p, L);
                    break;
                }
                const uint32_t st = L.stages + static_cast<uint32_t>(s) * p.stage_bytes;
                bar_expect_tx(L.full + 8 * s, p.x_bytes + kRawBytes + kCodeBytes);
                tma2d(st, &pr.tm_x, chunk * kChunk, 0, L.full + 8 * s, pol_x);
                tma2d(st + p.x_atom, &pr.tm_x, chunk * kChunk + kAtom, 0, L.full + 8 * s, pol_x);
                tma2d(st + p.x_bytes, &pr.tm_raw, chunk * kChunk, tile * kRows, L.full + 8 * s, pol_w);
                tma2d(st + p.x_bytes + kRawBytes, &pr.tm_code, chunk * (kChunk / 2), tile * kRows, L.full + 8 * s,
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
            UPos q = q0;
            for (long long u = u0; u < u1; ++u, next(q, p)) {
                const bool first = (u == u0) || q.chunk == 0;
                const bool last = (u + 1 == u1) || q.chunk == p.prob[q.p].n_chunks - 1;
                bool w = bar_wait(L.full + 8 * s, round & 1u) && bar_wait(L.a_full + 8 * a, around & 1u);
                if (w && first) w = bar_wait(L.acc_empty, (tiles & 1u) ^ 1u);
                if (!w) {
                    give_up(p, L);
                    break;
                }
                if (first) ++tiles;
                tc_fence_after();
                const uint32_t xa = L.stages + static_cast<uint32_t>(s) * p.stage_bytes;
                const uint32_t aa = L.abuf + static_cast<uint32_t>(a) * kABytes;
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk) {
                    const uint32_t atom = static_cast<uint32_t>(kk >> 2), sub = static_cast<uint32_t>(kk & 3) * 32u;
                    umma_bf16(tmem, smem_desc_sw128(aa + atom * kAtomBytes + sub),
                              smem_desc_sw128(xa + atom * p.x_atom + sub), idesc, (first && kk == 0) ? 0u : 1u);
                }
                umma_commit(L.empty + 8 * s);
                umma_commit(L.a_empty + 8 * a);
                if (last) umma_commit(L.acc_full);
                if (++s == S) {
                    s = 0;
                    ++round;
                }
                if (++a == p.a_bufs) {
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
        const int q4 = lane >> 3, r = 8 * ew + (lane & 7);  // row r of each unit, columns 32*q4 .. +31
        int s = 0, a = 0;
        uint32_t round = 0, around = 0, tiles = 0;
        // the row metadata of the next two units is in flight while a unit is decoded
        RowMeta m0 = {0, 0, 0, 0}, m1 = {0, 0, 0, 0};
        UPos q = q0;
        UPos qm = q;  // the unit whose metadata is loaded next
        if (u0 < u1) m0 = load_row_meta<V>(p, qm, r);
        next(qm, p);
        if (u0 + 1 < u1) m1 = load_row_meta<V>(p, qm, r);
        next(qm, p);
        // version 2: the row's escape offset at the current tile column
        uint32_t run = 0;
        if (V == 2 && u0 < u1 && q0.chunk > 0) run = row_offset_v2(p, q0, r, q4);
        for (long long u = u0; u < u1; ++u, next(q, p)) {
            const Problem &pr = p.prob[q.p];
            const int tile = q.tile, chunk = q.chunk;
            const bool last = (u + 1 == u1) || chunk == pr.n_chunks - 1;
            RowMeta m2 = m1;
            if (u + 2 < u1) {
                m2 = load_row_meta<V>(p, qm, r);
                next(qm, p);
            }
            const bool w = bar_wait(L.full + 8 * s, round & 1u) && bar_wait(L.a_empty + 8 * a, (around & 1u) ^ 1u);
            if (!__all_sync(0xFFFFFFFFu, w)) {
                give_up(p, L);
                break;
            }
            const uint32_t st = L.stages + static_cast<uint32_t>(s) * p.stage_bytes;
            const uint32_t aa = L.abuf + static_cast<uint32_t>(a) * kABytes;
            decode_row<CHECK>(pr, p.err, st + p.x_bytes, st + p.x_bytes + kRawBytes, aa, r, q4,
                              row_span<V>(m0, chunk, run));
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
            if (++a == p.a_bufs) {
                a = 0;
                ++around;
            }
            if (last) {
                const bool wa = bar_wait(L.acc_full, tiles & 1u);
                if (!__all_sync(0xFFFFFFFFu, wa)) {
                    give_up(p, L);
                    break;
                }
                ++tiles;
                tc_fence_after();
                const long long t0 = pr.unit0 + static_cast<long long>(tile) * pr.n_chunks;
                epilogue(p, pr, tmem, L, tile, pr.tile0 + tile, t0, u0, u1, ew, lane);
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
    if (warp == 2 && lane == 0) {
        uint32_t ab;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(ab) : "r"(L.abort) : "memory");
        if (ab) abort_arrivals(p, L, u0, u1);
    }
}

}  // namespace gemm

// ---------------------------------------------------------------------------
// Host side.

namespace {

constexpr uint32_t kSmemLimit = 227 * 1024;

struct Plan {
    int Mp, n_tiles, grid, stages;
    long long n_units;
    uint32_t x_bytes, x_atom, stage_bytes, tmem_cols, smem;
    int a_bufs;
    size_t part_bytes, cnt_bytes;
};

// One plan for `count` matrices with token rows M[i]; they share Mp, the
// largest M rounded up to 16.
Plan plan(const s12_view *views, int count, const int *M, int sms) {
    Plan pl;
    int mmax = 0;
    pl.n_tiles = 0;
    pl.n_units = 0;
    for (int i = 0; i < count; ++i) {
        mmax = std::max(mmax, M[i]);
        const int tiles = static_cast<int>((views[i].rows + gemm::kRows - 1) / gemm::kRows);
        pl.n_tiles += tiles;
        pl.n_units += static_cast<long long>(tiles) * static_cast<long long>(views[i].cols / gemm::kChunk);
    }
    pl.Mp = (mmax + 15) / 16 * 16;
    pl.grid = static_cast<int>(std::max(1LL, std::min<long long>(sms, pl.n_units)));
    pl.x_atom = static_cast<uint32_t>(pl.Mp) * 128u;
    pl.x_bytes = 2 * pl.x_atom;
    pl.stage_bytes = pl.x_bytes + gemm::kRawBytes + gemm::kCodeBytes;
    // three decoded-unit buffers when three stages still fit beside them, else fewer
    pl.a_bufs = gemm::kMaxABufs;
    uint32_t fixed = 0;
    for (;; --pl.a_bufs) {
        fixed = 1024 + 1024 + static_cast<uint32_t>(pl.a_bufs) * gemm::kABytes;  // slack, barriers, A buffers
        pl.stages = static_cast<int>(std::min<uint32_t>(gemm::kMaxStages, (kSmemLimit - fixed) / pl.stage_bytes));
        if (pl.stages >= (pl.a_bufs == 3 ? 3 : 2) || pl.a_bufs == 1) break;
    }
    pl.smem = fixed + static_cast<uint32_t>(pl.stages) * pl.stage_bytes;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(pl.Mp)) cols <<= 1;
    pl.tmem_cols = cols;
    // sized for the largest grid so one workspace fits every call with this Mp
    pl.part_bytes = align_up(static_cast<uint64_t>(sms) * 2 * pl.Mp * gemm::kRows * sizeof(float), kAlign);
    pl.cnt_bytes = align_up(static_cast<uint64_t>(pl.n_tiles) * sizeof(uint32_t), kAlign);
    return pl;
}

template <bool CHECK, int NP, int V>
int run_gemm(const s12_view *views, int count, const uint16_t *const *x, const int *M, void *const *y,
             const int *out, void *ws, uint32_t *err, const Plan &pl, cudaStream_t stream) {
    gemm::Params<NP> p = {};
    long long unit0 = 0;
    int tile0 = 0;
    for (int i = 0; i < count; ++i) {
        const s12_view *v = views + i;
        gemm::Problem &q = p.prob[i];
        const uint64_t N = v->rows, K = v->cols;
        if (make_tmap_u8_2d(&q.tm_raw, v->raw, K, N, K, gemm::kChunk, gemm::kRows, 128) != S12_OK)
            return S12_ERR_CUDA;
        if (make_tmap_u8_2d(&q.tm_code, v->code, K / 2, N, K / 2, gemm::kChunk / 2, gemm::kRows, 64) != S12_OK)
            return S12_ERR_CUDA;
        if (make_tmap_bf16_2d(&q.tm_x, x[i], K, static_cast<uint64_t>(M[i]), K * 2, gemm::kAtom,
                              static_cast<uint32_t>(pl.Mp), 128) != S12_OK)
            return S12_ERR_CUDA;
        q.meta = V == 1 ? static_cast<const void *>(v->base) : static_cast<const void *>(v->tmeta);
        q.off = V == 1 ? v->esc_off : v->row_esc;
        q.esc = v->esc;
        q.n_esc = v->n_esc;
        q.y = y[i];
        q.out = out ? out[i] : 0;
        q.N = static_cast<int>(N);
        q.K = static_cast<int>(K);
        q.T = q.K / kTile;
        q.M = M[i];
        q.n_tiles = static_cast<int>((N + gemm::kRows - 1) / gemm::kRows);
        q.n_chunks = static_cast<int>(K / gemm::kChunk);
        q.unit0 = unit0;
        q.tile0 = tile0;
        unit0 += static_cast<long long>(q.n_tiles) * q.n_chunks;
        tile0 += q.n_tiles;
    }
    p.part = static_cast<float *>(ws);
    p.cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + pl.part_bytes);
    p.err = err;
    p.n_problems = count;
    p.Mp = pl.Mp;
    p.n_units = pl.n_units;
    p.stages = pl.stages;
    p.stage_bytes = pl.stage_bytes;
    p.x_bytes = pl.x_bytes;
    p.x_atom = pl.x_atom;
    p.a_bufs = pl.a_bufs;
    p.tmem_cols = pl.tmem_cols;
    auto kern = gemm::gemm_tc_kernel<CHECK, NP, V>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess)
        return S12_ERR_CUDA;
    kern<<<pl.grid, gemm::kThreads, pl.smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace

size_t gemm_ws_bytes(const s12_view *views, int count, const int *M) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return 0;
    const Plan pl = plan(views, count, M, sms);
    return pl.part_bytes + pl.cnt_bytes;
}

int launch_gemm(const s12_view *views, int count, const uint16_t *const *x, const int *M, void *const *y,
                const int *out, void *ws, size_t ws_bytes, uint32_t *err, cudaStream_t stream) {
    // one container version per call
    const uint32_t version = views[0].version;
    for (int i = 0; i < count; ++i) {
        if (views[i].version != version || (version != 1 && version != 2)) return S12_ERR_ARG;
        if (out && out[i] != 0 && out[i] != 1) return S12_ERR_ARG;
    }
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    const Plan pl = plan(views, count, M, sms);
    if (!ws || ws_bytes < pl.part_bytes + pl.cnt_bytes) return S12_ERR_CAPACITY;
    if (pl.stages < 2) return S12_ERR_SHAPE;
    // a one-matrix call takes the small parameter block
    constexpr int kG = gemm::kMaxProblems;
    if (version == 1) {
        if (count == 1)
            return err ? run_gemm<true, 1, 1>(views, count, x, M, y, out, ws, err, pl, stream)
                       : run_gemm<false, 1, 1>(views, count, x, M, y, out, ws, err, pl, stream);
        return err ? run_gemm<true, kG, 1>(views, count, x, M, y, out, ws, err, pl, stream)
                   : run_gemm<false, kG, 1>(views, count, x, M, y, out, ws, err, pl, stream);
    }
    if (count == 1)
        return err ? run_gemm<true, 1, 2>(views, count, x, M, y, out, ws, err, pl, stream)
                   : run_gemm<false, 1, 2>(views, count, x, M, y, out, ws, err, pl, stream);
    return err ? run_gemm<true, kG, 2>(views, count, x, M, y, out, ws, err, pl, stream)
               : run_gemm<false, kG, 2>(views, count, x, M, y, out, ws, err, pl, stream);
}

}  // namespace s12
