// k_gemv.cu -- fused Split12 decode-GEMV for batch 1..8 on sm_100a.
//
//   y[b][n] = sum_k W[n][k] * x[b][k]
//
// The weights stay compressed in HBM; the exact BF16 values are rebuilt in
// registers and used at once in the product ("Lossless LLM Weight
// Compression vs 8-bit GGUF", section "What does 'lossless' mean for LLM
// weights?": decode into registers or shared memory and multiply
// immediately).  The kernel is HBM-bound and must move the compressed planes
// (1.5 bytes per weight + 5 bytes per tile + 2 bytes per escape) at close to
// the copy bandwidth, so the work per weight has to stay at a few integer
// instructions.
//
// Shape of the work.  A "block" is 16 rows x one 128-weight tile column.  A
// warp decodes a block straight into the A-operand registers of the warp-level
// tensor-core product mma.m16n8k16 (BF16 in, FP32 accumulate).  Lane (g, q)
// (g = lane / 4, q = lane % 4) owns rows g and g+8 and the 32 columns
// 32q .. 32q+31 of the tile, as two 16-weight chunks (halves h = 0, 1).  A
// chunk is decoded with a byte-wise base + code ADD and byte permutes into
// eight BF16 pairs that feed four products; the B operand is the matching
// slice of x for batch row g.  The tensor core does the multiplies and the
// reduction across the quad, so the decode is nearly all the arithmetic.
//
// Data movement.  Every warp owns a ring of shared-memory stages.  One lane
// fills a stage with two TMA tensor copies (raw plane: 16 rows x 128 bytes
// with the 128-byte swizzle, so the lanes' 16-byte reads hit distinct banks;
// code plane: 16 rows x 64 bytes), completing on the stage's mbarrier, and
// refills it as soon as the lanes have read it into registers.  The ring
// keeps several blocks in flight per warp at no register cost, so 16 warps
// fit on an SM.  The per-tile base and escape offsets are read with plain
// loads two blocks ahead.  Escape values are read when a block needs them:
// prefetching each tile's first escape one block ahead cost more in
// per-block work and registers than the load it hid (the layer ran 7.5 %
// slower with it).
//
// Work split (stream-K).  Blocks are numbered row-group-major (16-row group,
// then tile column) and dealt to all warps of the grid in equal contiguous
// ranges, so every warp streams the same number of bytes.  A warp keeps the
// accumulators of its current row group in registers; a group it covers
// whole goes straight to y.  A group shared by several warps is finished by
// the last of them to arrive: each contributor writes its partial to the
// workspace and bumps the group's counter; the one that completes the count
// adds the partials in warp order (so y is the same on every call) and
// resets the counter to zero for the next call.
//
// Launched with programmatic dependent launch: the weight copies start before
// the previous kernel in the stream has finished; x, y and the workspace wait
// for it.
#include <algorithm>

#include <cuda_bf16.h>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace gemv {

constexpr int kRowsPerGroup = 16;
constexpr int kSlotFloats = 128;  // one partial: 32 lanes x 4 accumulators
#ifndef S12_GEMV_WARPS
#define S12_GEMV_WARPS 16
#endif
constexpr int kWarps = S12_GEMV_WARPS;  // warps per CTA, one CTA per SM
constexpr int kMaxStages = 4;
constexpr int kMaxProblems = S12_GEMV_MAX_PROBLEMS;
constexpr uint32_t kRawBytes = 16 * 128;   // raw plane of one block
constexpr uint32_t kCodeBytes = 16 * 64;   // code plane of one block
constexpr uint32_t kStageBytes = kRawBytes + kCodeBytes;
constexpr uint32_t kRingOff = 1024;        // rings start 1024-aligned (128-byte swizzle atom)

// One matrix of a grouped call.
struct __align__(64) Problem {
    CUtensorMap tm_raw;   // u8 [R][K], box 128 x 16, 128-byte swizzle
    CUtensorMap tm_code;  // u8 [R][K/2], box 64 x 16
    const uint8_t *base;
    const uint32_t *esc_off;
    const uint16_t *esc;
    const uint16_t *x;    // B x K bf16
    float *y;             // B x R fp32 (act = 0)
    uint16_t *h;          // B x R/2 bf16 (act = 1)
    uint64_t n_esc;
    long long block0;     // first block of this matrix in the grouped numbering
    int R, K, T, n_groups;
    int group0;           // first row group of this matrix in the grouped numbering
    int act;              // epilogue: 0 = y fp32; 1 = SwiGLU of interleaved gate/up rows into h
};

struct __align__(64) Params {
    Problem prob[kMaxProblems];
    uint32_t *err;
    float *part;    // workspace: [n_units][2][kSlotFloats] partials
    uint32_t *cnt;  // workspace: one arrival counter per row group (zero between calls)
    long long n_blocks;
    int n_problems, B;
    int n_units;    // warps in the grid
    int stages;     // ring depth per warp, 2..kMaxStages
};

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// d += A * B for one m16n8k16 product, BF16 operands, FP32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mbar_init_s(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx_s(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Wait for phase `parity` of the barrier; false after about a second.
__device__ __forceinline__ bool mbar_wait_s(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles) return false;
    return true;
}

// 2-D TMA copy of one box into this CTA's shared memory, completing on bar.
__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap *tm, int c0, int c1, uint32_t bar,
                                      uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(tm), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
        : "memory");
}

// Position of a block: matrix, 16-row group and tile column.
struct Pos {
    int p, grp, j;
};

__device__ __forceinline__ void advance(Pos &ps, const Params &pr) {
    if (++ps.j == pr.prob[ps.p].T) {
        ps.j = 0;
        if (++ps.grp == pr.prob[ps.p].n_groups) {
            ps.grp = 0;
            ++ps.p;
        }
    }
}

// Position of grouped block b (b < n_blocks).
__device__ __forceinline__ Pos locate(const Params &pr, long long b) {
    int p = 0;
    while (p + 1 < pr.n_problems && pr.prob[p + 1].block0 <= b) ++p;
    const long long local = b - pr.prob[p].block0;
    const int T = pr.prob[p].T;
    return Pos{p, static_cast<int>(local / T), static_cast<int>(local % T)};
}

// Grouped row-group index of a position (the arrival-counter index).
__device__ __forceinline__ long long group_id(const Params &pr, Pos ps) { return pr.prob[ps.p].group0 + ps.grp; }

// Per-tile metadata of the lane's two rows for one block.
struct Meta {
    uint32_t baseA, baseB, loA, hiA, loB, hiB;
};

// Rows past the end (the TMA copies read them as zeros) read the last row's
// metadata but report no escapes.
__device__ __forceinline__ Meta load_meta(const Problem &m_, Pos ps, int g) {
    const int rA = ps.grp * kRowsPerGroup + g, rB = rA + 8;
    const size_t tA = static_cast<size_t>(min(rA, m_.R - 1)) * m_.T + ps.j;
    const size_t tB = static_cast<size_t>(min(rB, m_.R - 1)) * m_.T + ps.j;
    Meta m;
    m.baseA = __ldg(m_.base + tA);
    m.baseB = __ldg(m_.base + tB);
    m.loA = __ldg(m_.esc_off + tA);
    m.hiA = __ldg(m_.esc_off + tA + 1);
    m.loB = __ldg(m_.esc_off + tB);
    m.hiB = __ldg(m_.esc_off + tB + 1);
    if (rA >= m_.R) m.hiA = m.loA;
    if (rB >= m_.R) m.hiB = m.loB;
    return m;
}

// Metadata of the block after `prev` in the same row group (ps.j > 0): a
// tile's first escape offset is the previous tile's end, so only the base
// and the new end are read.
__device__ __forceinline__ Meta load_meta_next(const Problem &m_, Pos ps, int g, const Meta &prev) {
    const int rA = ps.grp * kRowsPerGroup + g, rB = rA + 8;
    const size_t tA = static_cast<size_t>(min(rA, m_.R - 1)) * m_.T + ps.j;
    const size_t tB = static_cast<size_t>(min(rB, m_.R - 1)) * m_.T + ps.j;
    Meta m;
    m.baseA = __ldg(m_.base + tA);
    m.baseB = __ldg(m_.base + tB);
    m.loA = prev.hiA;
    m.loB = prev.hiB;
    m.hiA = rA < m_.R ? __ldg(m_.esc_off + tA + 1) : m.loA;
    m.hiB = rB < m_.R ? __ldg(m_.esc_off + tB + 1) : m.loB;
    return m;
}

// First block of warp unit u's range.
__device__ __forceinline__ long long unit_start(long long u, long long n_blocks, int n_units) {
    return u * n_blocks / n_units;
}

__device__ __forceinline__ long long unit_of_block(long long b, long long n, int nu) {
    return ((b + 1) * nu + n - 1) / n - 1;
}

}  // namespace gemv
}  // namespace s12

namespace s12 {
namespace gemv {

// Write the accumulators of row group `grp` of matrix m to its y: lane
// (g, q) holds D[g][2q], D[g][2q+1], D[g+8][2q], D[g+8][2q+1] (row of W,
// batch row).
__device__ __forceinline__ void store_y(const Problem &m, int B, const float (&a)[4], int grp, int g, int q) {
    if (m.act) {
        // SwiGLU epilogue.  The matrix interleaves the gate and up
        // projections in blocks of 8 rows (rows 16i .. 16i+7 are gate rows
        // 8i .. 8i+7, rows 16i+8 .. 16i+15 the up rows with the same
        // indices), so this lane holds gate row f and up row f of the same
        // batch columns: h[b][f] = silu(gate) * up, rounded to BF16.
        const int f = grp * 8 + g, F = m.R >> 1;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int b = 2 * q + i;
            if (f < F && b < B) {
                const float gt = a[i], up = a[2 + i];
                const float hv = gt / (1.f + expf(-gt)) * up;
                m.h[static_cast<size_t>(b) * F + f] = __bfloat16_as_ushort(__float2bfloat16_rn(hv));
            }
        }
        return;
    }
    const int rA = grp * kRowsPerGroup + g;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = rA + (i >= 2 ? 8 : 0);
        const int b = 2 * q + (i & 1);
        if (r < m.R && b < B) m.y[static_cast<size_t>(b) * m.R + r] = a[i];
    }
}

// The warp's accumulators of the row group at `ps` are complete for its part
// of the group: store them, or hand them to the stream-K fix-up.  G0 is the
// grouped index of the warp's first row group.
__device__ __noinline__ void finish_group(const Params &pr, float4 a4, Pos ps, long long u, long long ub0,
                                          long long ub1, long long G0, int lane) {
    const float acc[4] = {a4.x, a4.y, a4.z, a4.w};
    const int g = lane >> 2, q = lane & 3;
    const Problem &m = pr.prob[ps.p];
    const long long n = pr.n_blocks;
    const long long gb0 = m.block0 + static_cast<long long>(ps.grp) * m.T, gb1 = gb0 + m.T;
    if (gb0 >= ub0 && gb1 <= ub1) {
        store_y(m, pr.B, acc, ps.grp, g, q);
        return;
    }
    const long long G = m.group0 + ps.grp;
    const int slot = G == G0 ? 0 : 1;
    float4 *mine = reinterpret_cast<float4 *>(pr.part + (static_cast<size_t>(u) * 2 + slot) * kSlotFloats) + lane;
    __stcg(mine, a4);
    __threadfence();
    __syncwarp();
    const long long uf = unit_of_block(gb0, n, pr.n_units), ul = unit_of_block(gb1 - 1, n, pr.n_units);
    uint32_t n_contrib = 0;
    for (long long v = uf; v <= ul; ++v)
        if (unit_start(v, n, pr.n_units) < unit_start(v + 1, n, pr.n_units)) ++n_contrib;
    uint32_t prev = 0;
    if (lane == 0) prev = atomicAdd(pr.cnt + G, 1u);
    prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
    if (prev + 1 != n_contrib) return;
    __threadfence();
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (long long v = uf; v <= ul; ++v) {
        const long long vs = unit_start(v, n, pr.n_units);
        if (vs >= unit_start(v + 1, n, pr.n_units)) continue;
        const int sl = group_id(pr, locate(pr, vs)) == G ? 0 : 1;
        const float4 t =
            __ldcg(reinterpret_cast<const float4 *>(pr.part + (static_cast<size_t>(v) * 2 + sl) * kSlotFloats) + lane);
        s[0] += t.x;
        s[1] += t.y;
        s[2] += t.z;
        s[3] += t.w;
    }
    store_y(m, pr.B, s, ps.grp, g, q);
    if (lane == 0) atomicExch(pr.cnt + G, 0u);
}

// Escapes of one tile row for this lane (set up only for rows whose tile has
// escapes): the stream index of the first escape of each of the lane's two
// chunks, the end of the tile's escapes, and which chunks have any.
struct EscRow {
    uint32_t s0, s1, limit, has;  // has: bit h set if chunk h holds an escape
};

__device__ __forceinline__ uint32_t count2(uint2 m) { return __popc(m.x) + __popc(m.y); }

__device__ __forceinline__ uint2 esc_mask(uint2 c) { return make_uint2(escape_nibbles(c.x), escape_nibbles(c.y)); }

// Called by whole quads (the lanes of `quads`, a union of complete quads that
// share a tile row).  Chunk order within a tile row: lane q = 0..3, half 0
// then half 1 (chunk 2q + h covers columns 32q + 16h .. +15).  The tile's
// code-15 count is checked against its esc_off span.
__device__ __forceinline__ EscRow prepare_row(uint4 c, uint32_t lo, uint32_t hi, uint64_t n_esc, uint32_t *err,
                                              unsigned quads, int q) {
    const uint32_t n0 = count2(esc_mask(make_uint2(c.x, c.y))), n1 = count2(esc_mask(make_uint2(c.z, c.w)));
    const uint32_t n = n0 + n1;
    uint32_t incl = n;
#pragma unroll
    for (int d = 1; d < 4; d <<= 1) {
        const uint32_t v = __shfl_up_sync(quads, incl, d, 4);
        if (q >= d) incl += v;
    }
    const uint32_t tot = __shfl_sync(quads, incl, 3, 4);
    EscRow e;
    e.s0 = lo + incl - n;
    e.s1 = e.s0 + n0;
    e.limit = lo <= hi ? static_cast<uint32_t>(hi < n_esc ? hi : n_esc) : 0u;
    e.has = (n0 ? 1u : 0u) | (n1 ? 2u : 0u);
    if (q == 0 && tot != hi - lo) raise_flag(err, S12_FLAG_ESC_COUNT);
    return e;
}

// A chunk with escapes: put the exact value of each escaped weight in place,
// reading the stream from index `idx`; reads at or past the tile's end are
// skipped and flagged.  The decoded words go through the lane's 32-byte
// shared-memory scratch `sc`, so a weight is replaced by one 16-bit store
// at its position.  With base <= 240, base + 15 stays inside its byte and
// the other weights of the chunk are already right; a base of 241 could
// carry into the next byte, so such chunks are decoded again with the
// escape nibbles cleared first.
__device__ __forceinline__ void fix_chunk(uint32_t (&w)[8], uint4 raw, uint2 code, uint32_t base, uint32_t idx,
                                          uint32_t limit, const uint16_t *__restrict__ esc, uint32_t *err,
                                          uint32_t sc) {
    const uint2 m = esc_mask(code);
    if (base > static_cast<uint32_t>(kMaxBase - 1))
        decode16(raw, make_uint2(clear_escapes(code.x, m.x), clear_escapes(code.y, m.y)), base * 0x01010101u, w);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sc), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                 : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sc + 16), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                 "r"(w[7])
                 : "memory");
    // nibble j of the chunk is 15  <=>  bit 4j+3 of the 64-bit mask
    uint64_t mm = (static_cast<uint64_t>(m.y) << 32) | m.x;
    while (mm) {
        const int j = (__ffsll(static_cast<long long>(mm)) - 1) >> 2;
        mm &= mm - 1;
        uint32_t v = 0;
        if (idx < limit)
            v = __ldg(esc + idx);
        else
            raise_flag(err, S12_FLAG_ESC_RANGE);
        ++idx;
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(sc + 2u * j), "h"(static_cast<uint16_t>(v)) : "memory");
    }
    uint4 a, b;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w) : "r"(sc)
                 : "memory");
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "r"(sc + 16)
                 : "memory");
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

__device__ __forceinline__ float4 sum_halves(const float (&acc)[2][4]) {
    return make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
}

// The lane's 16 activations (batch row gx, columns j*128 + 32q + 16h ..),
// read through the L1 cache.
__device__ __forceinline__ void load_x(uint32_t (&xw)[8], const uint16_t *xl, int j, int h) {
    const uint4 *src = reinterpret_cast<const uint4 *>(xl + static_cast<size_t>(j) * kTile + h * 16);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
    xw[4] = b.x; xw[5] = b.y; xw[6] = b.z; xw[7] = b.w;
}

// One half of a block: four m16n8k16 products of rows g / g+8 with x.
__device__ __forceinline__ void half_mma(float (&acc)[4], const uint32_t (&wa)[8], const uint32_t (&wb)[8],
                                         const uint32_t (&xw)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) mma16816(acc, wa[2 * i], wb[2 * i], wa[2 * i + 1], wb[2 * i + 1], xw[2 * i], xw[2 * i + 1]);
}

}  // namespace gemv
}  // namespace s12

namespace s12 {
namespace gemv {

// Start the copies of the block at `ps` into stage st (completing on bar).
__device__ __forceinline__ void copy_block(const Params &pr, Pos ps, uint32_t st, uint32_t bar, uint64_t pol) {
    const Problem &m = pr.prob[ps.p];
    mbar_expect_tx_s(bar, kStageBytes);
    tma2d(st, &m.tm_raw, ps.j * 128, ps.grp * kRowsPerGroup, bar, pol);
    tma2d(st + kRawBytes, &m.tm_code, ps.j * 64, ps.grp * kRowsPerGroup, bar, pol);
}

template <bool CHECK>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_tma_kernel(const __grid_constant__ Params pr) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sb = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const long long n = pr.n_blocks;
    const long long u = static_cast<long long>(blockIdx.x) * kWarps + warp;
    const long long ub0 = unit_start(u, n, pr.n_units), ub1 = unit_start(u + 1, n, pr.n_units);
    const int nb = static_cast<int>(ub1 - ub0);
    const int S = pr.stages;
    const uint32_t bars = sb + static_cast<uint32_t>(warp) * kMaxStages * 8u;
    const uint32_t ring = sb + kRingOff + static_cast<uint32_t>(warp * S) * kStageBytes;
    const uint32_t scr = sb + kRingOff + static_cast<uint32_t>(kWarps * S) * kStageBytes + threadIdx.x * 32u;
    if (threadIdx.x == 0) grid_launch_dependents();

    // The weights are never written by other kernels: start the copies
    // before waiting for the previous grid.
    const Pos p0 = nb > 0 ? locate(pr, ub0) : Pos{0, 0, 0};
    Pos pi = p0;  // next block to copy
    uint64_t pol = 0;
    if (lane == 0) {
        pol = policy_evict_first();
        for (int s = 0; s < S; ++s) mbar_init_s(bars + 8u * s, 1);
        fence_barrier_init();
        for (int s = 0; s < S && s < nb; ++s) {
            copy_block(pr, pi, ring + s * kStageBytes, bars + 8u * s, pol);
            advance(pi, pr);
        }
    }
    __syncwarp();
    if (nb == 0) return;
    grid_dependency_wait();  // x, y and the workspace may belong to earlier kernels
    const int gx = g < pr.B ? g : 0;  // batch rows past B repeat row 0; their outputs are dropped
    // lane's shared-memory offsets inside a stage (raw rows are 128-byte swizzled)
    const uint32_t oA0 = g * 128 + (((2 * q) ^ g) << 4), oA1 = g * 128 + (((2 * q + 1) ^ g) << 4);
    const uint32_t oB0 = oA0 + 8 * 128, oB1 = oA1 + 8 * 128;
    const uint32_t oCA = kRawBytes + g * 64 + 16 * q, oCB = oCA + 8 * 64;

    Pos pc = p0;  // block being computed
    Pos pm = p0;  // block whose metadata is loaded (two ahead)
    Meta m0 = load_meta(pr.prob[pm.p], pm, g), m1 = m0;
    advance(pm, pr);
    if (nb > 1) m1 = load_meta(pr.prob[pm.p], pm, g);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // one chain per half
    Pos cur = p0;
    const long long G0 = group_id(pr, p0);
    int s = 0;
    uint32_t parity = 0;
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
        // metadata two blocks ahead
        Meta m2 = m1;
        if (i + 2 < nb) {
            advance(pm, pr);
            m2 = pm.j > 0 ? load_meta_next(pr.prob[pm.p], pm, g, m1) : load_meta(pr.prob[pm.p], pm, g);
        }
        if (pc.grp != cur.grp || pc.p != cur.p) {
            finish_group(pr, sum_halves(acc), cur, u, ub0, ub1, G0, lane);
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[0][k] = acc[1][k] = 0.f;
            cur = pc;
        }
        const uint32_t bar = bars + 8u * s;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_s(bar, parity))) {
            raise_flag(pr.err, S12_FLAG_TIMEOUT);
            ok = false;
            break;
        }
        const uint32_t st = ring + s * kStageBytes;
        bool esc = (m0.loA != m0.hiA) || (m0.loB != m0.hiB);
        if (CHECK) {
            const uint4 cA = lds128(st + oCA), cB = lds128(st + oCB);
            esc = esc || (escape_nibbles(cA.x) | escape_nibbles(cA.y) | escape_nibbles(cA.z) | escape_nibbles(cA.w) |
                          escape_nibbles(cB.x) | escape_nibbles(cB.y) | escape_nibbles(cB.z) | escape_nibbles(cB.w)) != 0;
            if (m0.baseA > static_cast<uint32_t>(kMaxBase) || m0.baseB > static_cast<uint32_t>(kMaxBase))
                raise_flag(pr.err, S12_FLAG_BASE);
        }
        const Problem &mp = pr.prob[pc.p];
        const uint16_t *xl = mp.x + static_cast<size_t>(gx) * mp.K + 32 * q;
        const uint4 rA0 = lds128(st + oA0), rA1 = lds128(st + oA1), rB0 = lds128(st + oB0), rB1 = lds128(st + oB1);
        const uint4 cA = lds128(st + oCA), cB = lds128(st + oCB);
        // the stage is in registers: hand it back to the copy engine
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && i + S < nb) copy_block(pr, pi, st, bar, pol);
        const uint32_t B4A = m0.baseA * 0x01010101u, B4B = m0.baseB * 0x01010101u;
        uint32_t xw[8], wa[8], wb[8];
        if (!__any_sync(0xFFFFFFFFu, esc)) {
            // no escapes in the block: straight decode and products
            load_x(xw, xl, pc.j, 0);
            decode16(rA0, make_uint2(cA.x, cA.y), B4A, wa);
            decode16(rB0, make_uint2(cB.x, cB.y), B4B, wb);
            half_mma(acc[0], wa, wb, xw);
            load_x(xw, xl, pc.j, 1);
            decode16(rA1, make_uint2(cA.z, cA.w), B4A, wa);
            decode16(rB1, make_uint2(cB.z, cB.w), B4B, wb);
            half_mma(acc[1], wa, wb, xw);
        } else {
            // some tile row of the block has escapes: rank them per row (quad
            // shuffles), decode, patch the escaped weights, multiply
            const bool escA = m0.loA != m0.hiA || (escape_nibbles(cA.x) | escape_nibbles(cA.y) |
                                                   escape_nibbles(cA.z) | escape_nibbles(cA.w)) != 0;
            const bool escB = m0.loB != m0.hiB || (escape_nibbles(cB.x) | escape_nibbles(cB.y) |
                                                   escape_nibbles(cB.z) | escape_nibbles(cB.w)) != 0;
            const unsigned qA = __ballot_sync(0xFFFFFFFFu, escA), qB = __ballot_sync(0xFFFFFFFFu, escB);
            EscRow eA = {0, 0, 0, 0}, eB = {0, 0, 0, 0};
            if (escA) eA = prepare_row(cA, m0.loA, m0.hiA, mp.n_esc, pr.err, qA, q);
            if (escB) eB = prepare_row(cB, m0.loB, m0.hiB, mp.n_esc, pr.err, qB, q);
            load_x(xw, xl, pc.j, 0);
            decode16(rA0, make_uint2(cA.x, cA.y), B4A, wa);
            decode16(rB0, make_uint2(cB.x, cB.y), B4B, wb);
            if (eA.has & 1u)
                fix_chunk(wa, rA0, make_uint2(cA.x, cA.y), m0.baseA, eA.s0, eA.limit, mp.esc, pr.err, scr);
            if (eB.has & 1u)
                fix_chunk(wb, rB0, make_uint2(cB.x, cB.y), m0.baseB, eB.s0, eB.limit, mp.esc, pr.err, scr);
            half_mma(acc[0], wa, wb, xw);
            load_x(xw, xl, pc.j, 1);
            decode16(rA1, make_uint2(cA.z, cA.w), B4A, wa);
            decode16(rB1, make_uint2(cB.z, cB.w), B4B, wb);
            if (eA.has & 2u)
                fix_chunk(wa, rA1, make_uint2(cA.z, cA.w), m0.baseA, eA.s1, eA.limit, mp.esc, pr.err, scr);
            if (eB.has & 2u)
                fix_chunk(wb, rB1, make_uint2(cB.z, cB.w), m0.baseB, eB.s1, eB.limit, mp.esc, pr.err, scr);
            half_mma(acc[1], wa, wb, xw);
        }
        if (i + S < nb) advance(pi, pr);

        advance(pc, pr);
        m0 = m1;
        m1 = m2;
        if (++s == S) {
            s = 0;
            parity ^= 1u;
        }
    }
    if (ok) {
        finish_group(pr, sum_halves(acc), cur, u, ub0, ub1, G0, lane);
    } else if (lane == 0) {
        // a wait gave up: let the copies still in flight land before exiting
        for (int k = 0; k < S; ++k) mbar_wait_s(bars + 8u * k, parity ^ (k < s ? 1u : 0u));
    }
}

}  // namespace gemv

// ---------------------------------------------------------------------------
// Host side.

namespace {

constexpr uint32_t kSmemLimit = 227 * 1024;

struct Plan {
    long long n_blocks, n_groups;
    int grid, n_units;
    size_t part_bytes, cnt_bytes;
};

Plan plan(const s12_view *views, int count, int sms) {
    Plan pl;
    pl.n_blocks = pl.n_groups = 0;
    for (int i = 0; i < count; ++i) {
        const long long groups =
            static_cast<long long>((views[i].rows + gemv::kRowsPerGroup - 1) / gemv::kRowsPerGroup);
        pl.n_groups += groups;
        pl.n_blocks += groups * static_cast<long long>(views[i].cols / kTile);
    }
    const long long want = (pl.n_blocks + gemv::kWarps - 1) / gemv::kWarps;
    pl.grid = static_cast<int>(std::max(1LL, std::min<long long>(sms, want)));
    pl.n_units = pl.grid * gemv::kWarps;
    // sized for the largest grid so one workspace fits every call on the device
    pl.part_bytes =
        align_up(static_cast<uint64_t>(sms) * gemv::kWarps * 2 * gemv::kSlotFloats * sizeof(float), kAlign);
    pl.cnt_bytes = align_up(static_cast<uint64_t>(pl.n_groups) * sizeof(uint32_t), kAlign);
    return pl;
}

template <bool CHECK>
int run(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *act,
        void *ws, uint32_t *err, const Plan &pl, cudaStream_t stream) {
    gemv::Params pr = {};
    long long block0 = 0;
    int group0 = 0;
    for (int i = 0; i < count; ++i) {
        const s12_view *v = views + i;
        gemv::Problem &m = pr.prob[i];
        const uint64_t R = v->rows, K = v->cols;
        if (make_tmap_u8_2d(&m.tm_raw, v->raw, K, R, K, 128, gemv::kRowsPerGroup, 128) != S12_OK)
            return S12_ERR_CUDA;
        if (make_tmap_u8_2d(&m.tm_code, v->code, K / 2, R, K / 2, 64, gemv::kRowsPerGroup, 0) != S12_OK)
            return S12_ERR_CUDA;
        m.base = v->base;
        m.esc_off = v->esc_off;
        m.esc = v->esc;
        m.x = x[i];
        m.act = act ? act[i] : 0;
        m.y = m.act ? nullptr : static_cast<float *>(y[i]);
        m.h = m.act ? static_cast<uint16_t *>(y[i]) : nullptr;
        m.n_esc = v->n_esc;
        m.R = static_cast<int>(R);
        m.K = static_cast<int>(K);
        m.T = m.K / kTile;
        m.n_groups = (m.R + gemv::kRowsPerGroup - 1) / gemv::kRowsPerGroup;
        m.block0 = block0;
        m.group0 = group0;
        block0 += static_cast<long long>(m.n_groups) * m.T;
        group0 += m.n_groups;
    }
    pr.err = err;
    pr.part = static_cast<float *>(ws);
    pr.cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + pl.part_bytes);
    pr.n_blocks = pl.n_blocks;
    pr.n_problems = count;
    pr.B = B;
    pr.n_units = pl.n_units;
    pr.stages = gemv::kMaxStages;
    // 1 KB alignment slack, barriers, the warps' rings, 32 bytes of escape
    // scratch per lane
    const uint32_t smem = 1024 + gemv::kRingOff + gemv::kWarps * pr.stages * gemv::kStageBytes + gemv::kWarps * 32 * 32;
    if (smem > kSmemLimit) return S12_ERR_CUDA;
    auto kern = gemv::gemv_tma_kernel<CHECK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return S12_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(32 * gemv::kWarps);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, pr) == cudaSuccess ? S12_OK : S12_ERR_CUDA;
}

}  // namespace

size_t gemv_ws_bytes(const s12_view *views, int count) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return 0;
    const Plan pl = plan(views, count, sms);
    return pl.part_bytes + pl.cnt_bytes;
}

int launch_gemv(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *act,
                void *ws, size_t ws_bytes, uint32_t *err, cudaStream_t stream) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    const Plan pl = plan(views, count, sms);
    if (ws_bytes < pl.part_bytes + pl.cnt_bytes) return S12_ERR_CAPACITY;
    return err ? run<true>(views, count, x, B, y, act, ws, err, pl, stream)
               : run<false>(views, count, x, B, y, act, ws, err, pl, stream);
}

}  // namespace s12
