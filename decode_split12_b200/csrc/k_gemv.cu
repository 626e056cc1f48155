// k_gemv.cu -- fused Split12 decode-GEMV for batch 1..8 on sm_100a.
//
//   y[b][n] = sum_k W[n][k] * x[b][k]
//
// The weights stay compressed in HBM; the exact BF16 values are rebuilt in
// registers and used at once in the product ("Lossless LLM Weight
// Compression vs 8-bit GGUF", section "What does 'lossless' mean for LLM
// weights?": decode into registers or shared memory and multiply
// immediately).  The kernel is HBM-bound: it must move the compressed planes
// (1.5 bytes per weight plus the tile headers and escapes) at close to the
// copy bandwidth, so the work per weight has to stay at a few integer
// instructions and the copies must keep the memory system busy.
//
// Shape of the work.  A "block" is 16 rows x one 128-weight tile.  A warp
// decodes a block straight into the A-operand registers of the warp-level
// tensor-core product mma.m16n8k16 (BF16 in, FP32 accumulate).  Lane (g, q)
// (g = lane / 4, q = lane % 4) owns rows g and g+8 and the 32 columns
// 32q .. 32q+31 of the tile, as two 16-weight halves.  A half is decoded with
// a byte-wise base + code ADD and byte permutes into eight BF16 pairs that
// feed four products; the B operand is the matching slice of x for batch row
// g.  The tensor core does the multiplies and the reduction across the quad.
//
// Data movement.  Every warp owns a ring of two shared-memory stages.  A stage
// is TWO consecutive tiles of the warp's 16 rows, brought in by two 3-D TMA
// copies (raw plane: 16 rows x 2 x 128 bytes, 128-byte swizzled so the lanes'
// 16-byte reads hit distinct banks; code plane: 16 rows x 2 x 64 bytes).  Each
// row of a copy is then 256 (raw) or 128 (code) contiguous bytes.  Measured
// on B200 with the copies alone, that streams at the copy bandwidth, while
// one tile per copy (128- and 64-byte row pieces) stays near 65 % of it.
//
// Per-tile metadata.  The four lanes of a quad share a row, so each lane
// fetches one metadata word of its two rows per stage and the quad exchanges
// them with shuffles: for a version 1 container the bases and escape-offset
// ends of the stage's two tiles, for version 2 the two (base | count) words.
// The escape stream is walked with a running offset per row, so a tile with
// no escapes (nearly all of them) costs no offset arithmetic, and the
// decision "does this block hold an escape" comes from the metadata, not from
// scanning the code nibbles (which the checked variant still does).
//
// Escapes.  A block whose tiles all have empty escape spans takes the straight
// path.  Otherwise each affected row ranks its escapes across the quad with
// shuffles, and each half that holds one is patched through a 32-byte
// per-lane shared scratch: the decoded words are stored, every escaped weight
// is overwritten by one 16-bit store of its exact value, and the words are
// read back.  With a tile base of 241, base + 15 would carry into the next
// byte, so such halves are decoded again with the escape nibbles cleared.
//
// Work split (stream-K).  Blocks are numbered row-group-major (16-row group,
// then tile) across all matrices of the call and dealt to all warps of the
// grid in equal contiguous ranges, so every warp streams the same number of
// bytes.  A warp keeps the accumulators of its current row group in
// registers; a group it covers whole goes straight to y.  A group shared by
// several warps is finished by the last of them to arrive: each contributor
// writes its partial to the workspace and bumps the group's counter; the one
// that completes the count adds the partials in warp order (so y is the same
// on every call) and resets the counter to zero for the next call.  A warp
// whose bounded wait gives up still arrives on every group it was to
// contribute to, so the counters return to zero even then.
//
// Launched with programmatic dependent launch: the weight copies and the
// metadata loads start before the previous kernel in the stream has
// finished; x, y and the workspace wait for it.
#include <algorithm>

#include <cuda_bf16.h>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace gemv {

constexpr int kRowsPerGroup = 16;
constexpr int kNT = 2;       // tiles per stage
constexpr int kStages = 2;   // stages per warp ring
constexpr int kWarps = kGemvWarps;
constexpr int kSlotFloats = static_cast<int>(kGemvSlotBytes / 4);
constexpr int kMaxProblems = S12_GEMV_MAX_PROBLEMS;
constexpr uint32_t kRawTile = kRowsPerGroup * 128;   // raw plane of one block
constexpr uint32_t kCodeTile = kRowsPerGroup * 64;   // code plane of one block
constexpr uint32_t kRawStage = kNT * kRawTile;
constexpr uint32_t kStageBytes = kNT * (kRawTile + kCodeTile);
constexpr uint32_t kRingOff = 1024;  // rings start 1024-aligned (128-byte swizzle atom)
static_assert(kSlotFloats == 128, "one partial is 32 lanes x 4 accumulators");
static_assert(kStageBytes % 1024 == 0, "stages keep the swizzle atom alignment");

constexpr int kOutF32 = kGemvOutF32, kOutSwiglu = kGemvOutSwiglu, kOutBf16 = kGemvOutBf16;

// One matrix of a grouped call.
struct __align__(64) Problem {
    CUtensorMap tm_raw;   // u8 {128, R, T} (strides K, 128), box {128, 16, 2}, 128-byte swizzle
    CUtensorMap tm_code;  // u8 {64, R, T} (strides K/2, 64), box {64, 16, 2}
    const void *meta;     // version 1: base u8[n_tiles]; version 2: (base | count << 8) u16[n_tiles]
    const uint32_t *off;  // version 1: esc_off u32[n_tiles + 1]; version 2: row_esc u32[R + 1]
    const uint16_t *esc;
    const uint16_t *x;    // B x K bf16
    void *y;              // kOutF32: B x R fp32; kOutBf16: B x R bf16; kOutSwiglu: B x R/2 bf16
    uint32_t n_esc;
    int R, K, T, n_groups;
    int out;              // kOutF32, kOutSwiglu or kOutBf16
    long long block0;     // first block of this matrix in the grouped numbering
    int group0;           // first row group of this matrix in the grouped numbering
};

struct __align__(64) Params {
    Problem prob[kMaxProblems];
    uint32_t *err;
    float *part;    // workspace: [n_units][2][kSlotFloats] partials
    uint32_t *cnt;  // workspace: one arrival counter per row group (zero between calls)
    long long n_blocks;
    int n_problems, B;
    int n_units;    // warps in the grid
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

// 3-D TMA copy of one box into this CTA's shared memory, completing on bar.
__device__ __forceinline__ void tma3d(uint32_t dst, const CUtensorMap *tm, int c0, int c1, int c2, uint32_t bar,
                                      uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(tm), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(policy)
        : "memory");
}

// A stage position: matrix, 16-row group, first tile, and the number of
// blocks of the warp's range from here on (0: past the range).
struct Cur {
    int p, grp, j, left;
};

// Tiles in the stage starting at c: up to kNT, never past the row or the
// warp's range (requires c.left > 0).
__device__ __forceinline__ int stage_len(const Params &pr, const Cur &c) {
    const int n = min(pr.prob[c.p].T - c.j, c.left);
    return n < kNT ? n : kNT;
}

__device__ __forceinline__ void advance(Cur &c, int len, const Params &pr) {
    c.left -= len;
    c.j += len;
    if (c.j == pr.prob[c.p].T) {
        c.j = 0;
        if (++c.grp == pr.prob[c.p].n_groups) {
            c.grp = 0;
            ++c.p;
        }
    }
}

// Position of grouped block b (b < n_blocks), with `left` blocks to go.
__device__ __forceinline__ Cur locate(const Params &pr, long long b, int left) {
    int p = 0;
    while (p + 1 < pr.n_problems && pr.prob[p + 1].block0 <= b) ++p;
    const long long local = b - pr.prob[p].block0;
    const int T = pr.prob[p].T;
    return Cur{p, static_cast<int>(local / T), static_cast<int>(local % T), left};
}

// First block of warp unit u's range.
__device__ __forceinline__ long long unit_start(long long u, long long n_blocks, int n_units) {
    return u * n_blocks / n_units;
}

__device__ __forceinline__ long long unit_of_block(long long b, long long n, int nu) {
    return ((b + 1) * nu + n - 1) / n - 1;
}

// Start the copies of the stage at c into stage buffer st (completing on bar).
__device__ __forceinline__ void issue(const Params &pr, const Cur &c, uint32_t st, uint32_t bar) {
    const Problem &m = pr.prob[c.p];
    const uint64_t pol = policy_evict_first();
    mbar_expect_tx_s(bar, kStageBytes);
    tma3d(st, &m.tm_raw, 0, c.grp * kRowsPerGroup, c.j, bar, pol);
    tma3d(st + kRawStage, &m.tm_code, 0, c.grp * kRowsPerGroup, c.j, bar, pol);
}

// ---------------------------------------------------------------------------
// Metadata.  Per stage the lane loads one word for each of its rows (row r of
// matrix m, tiles j .. j+len-1); the quad's four words are, by lane q:
//   version 1:  base[t], base[t+1], esc_off[t+1], esc_off[t+2]   (t = r*T + j)
//   version 2:  tmeta[t], tmeta[t+1], -, -
// Rows past the end read as 0 (no escapes).
template <int V>
__device__ __forceinline__ uint32_t load_item(const Problem &m, int r, int j, int len, int q) {
    if (r >= m.R) return 0;
    const size_t t0 = static_cast<size_t>(r) * m.T + j;
    if (V == 1) {
        if (q < 2) return q < len ? static_cast<uint32_t>(__ldg(static_cast<const uint8_t *>(m.meta) + t0 + q)) : 0u;
        return q - 2 < len ? __ldg(m.off + t0 + 1 + (q - 2)) : 0u;
    }
    return q < len ? static_cast<uint32_t>(__ldg(static_cast<const uint16_t *>(m.meta) + t0 + q)) : 0u;
}

// Escapes before tile (r, j) in the stream, for a segment that starts at
// tile j (version 2: only the row start; the caller adds the earlier tiles'
// counts when j > 0).
template <int V>
__device__ __forceinline__ uint32_t load_start(const Problem &m, int r, int j) {
    if (r >= m.R) return 0;
    if (V == 1) return __ldg(m.off + static_cast<size_t>(r) * m.T + j);
    return __ldg(m.off + r);
}

// Escape counts of tiles 0 .. j-1 of row r (version 2), summed across the
// quad (every lane of the warp calls it; lane q takes tiles q, q+4, ...).
__device__ __forceinline__ uint32_t prefix_count_v2(const Problem &m, int r, int j, int q) {
    uint32_t s = 0;
    if (r < m.R) {
        const uint16_t *tm = static_cast<const uint16_t *>(m.meta) + static_cast<size_t>(r) * m.T;
        for (int k = q; k < j; k += 4) s += __ldg(tm + k) >> 8;
    }
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
    return s;
}

struct Meta {
    uint32_t a, b;    // the lane's words for rows g and g+8
    uint32_t sa, sb;  // escapes before the stage's first tile (segment starts only)
};

template <int V>
__device__ __forceinline__ Meta load_meta(const Problem &m, const Cur &c, int len, int g, int q, bool seg_start) {
    const int rA = c.grp * kRowsPerGroup + g, rB = rA + 8;
    Meta r;
    r.a = load_item<V>(m, rA, c.j, len, q);
    r.b = load_item<V>(m, rB, c.j, len, q);
    r.sa = seg_start ? load_start<V>(m, rA, c.j) : 0u;
    r.sb = seg_start ? load_start<V>(m, rB, c.j) : 0u;
    return r;
}

// Base and escape-span end of tile t of the stage for one row, from the
// quad's words (w = the lane's word for that row, off = the running offset).
template <int V>
__device__ __forceinline__ void tile_meta(uint32_t w, int qb, int t, uint32_t off, uint32_t &base, uint32_t &end) {
    const uint32_t v = __shfl_sync(0xFFFFFFFFu, w, qb + t);
    base = v & 0xFFu;
    if (V == 1)
        end = __shfl_sync(0xFFFFFFFFu, w, qb + 2 + t);
    else
        end = off + (v >> 8);
}

// ---------------------------------------------------------------------------
// Escapes.

__device__ __forceinline__ uint2 esc_mask(uint32_t a, uint32_t b) {
    return make_uint2(escape_nibbles(a), escape_nibbles(b));
}

// Escapes of one tile row for this lane: the masks of its two halves, the
// stream index of its first escape in each, and the end of the row's span.
// Called by all 32 lanes; the four lanes of a quad share the row and rank
// their escapes in chunk order (lane q = 0..3, half 0 then half 1).  The
// tile's code-15 count is checked against its span.
struct EscRow {
    uint2 m0, m1;
    uint32_t s0, s1, limit;
};

__device__ __forceinline__ EscRow prepare_row(uint4 c, uint32_t lo, uint32_t hi, uint32_t n_esc, uint32_t *err,
                                              int q) {
    EscRow e;
    e.m0 = esc_mask(c.x, c.y);
    e.m1 = esc_mask(c.z, c.w);
    const uint32_t n0 = __popc(e.m0.x) + __popc(e.m0.y);
    const uint32_t n = n0 + __popc(e.m1.x) + __popc(e.m1.y);
    uint32_t incl = n;
#pragma unroll
    for (int d = 1; d < 4; d <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d, 4);
        if (q >= d) incl += v;
    }
    const uint32_t tot = __shfl_sync(0xFFFFFFFFu, incl, 3, 4);
    e.s0 = lo + incl - n;
    e.s1 = e.s0 + n0;
    e.limit = lo <= hi ? min(hi, n_esc) : 0u;
    if (q == 0 && tot != hi - lo) raise_flag(err, S12_FLAG_ESC_COUNT);
    return e;
}

// A half with escapes: put the exact value of each escaped weight in place,
// reading the stream from index `idx`; reads at or past `limit` are skipped
// and flagged.  The decoded words go through the lane's 32-byte shared
// scratch `sc`, so a weight is replaced by one 16-bit store at its position.
// With base <= 240, base + 15 stays inside its byte and the other weights of
// the half are already right; a base of 241 could carry into the next byte,
// so such halves are decoded again with the escape nibbles cleared first.
__device__ __forceinline__ void fix_half(uint32_t (&w)[8], uint4 raw, uint2 code, uint2 m, uint32_t base, uint32_t idx,
                                      uint32_t limit, const uint16_t *__restrict__ esc, uint32_t *err, uint32_t sc) {
    if (base > static_cast<uint32_t>(kMaxBase - 1))
        decode16(raw, make_uint2(clear_escapes(code.x, m.x), clear_escapes(code.y, m.y)), base * 0x01010101u, w);
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sc), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                 : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sc + 16), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                 "r"(w[7])
                 : "memory");
    // nibble j of the half is 15  <=>  bit 4j+3 of the 64-bit mask
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

// ---------------------------------------------------------------------------
// Products.

// The lane's 16 activations of half h (batch row of xl, columns 32q + 16h ..
// of the tile at xl), read through the L1 cache.
__device__ __forceinline__ void load_x(uint32_t (&xw)[8], const uint16_t *xl, int h) {
    const uint4 *src = reinterpret_cast<const uint4 *>(xl + h * 16);
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

// ---------------------------------------------------------------------------
// Results.

// Write the accumulators of row group `grp` of matrix m: lane (g, q) holds
// D[g][2q], D[g][2q+1], D[g+8][2q], D[g+8][2q+1] (row of W, batch row).
__device__ __forceinline__ void store_y(const Problem &m, int B, const float (&a)[4], int grp, int g, int q) {
    if (m.out == kOutSwiglu) {
        // SwiGLU epilogue.  The matrix interleaves the gate and up
        // projections in blocks of 8 rows (rows 16i .. 16i+7 are gate rows
        // 8i .. 8i+7, rows 16i+8 .. 16i+15 the up rows with the same
        // indices), so this lane holds gate row f and up row f of the same
        // batch columns: h[b][f] = silu(gate) * up, rounded to BF16.
        const int f = grp * 8 + g, F = m.R >> 1;
        uint16_t *h = static_cast<uint16_t *>(m.y);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int b = 2 * q + i;
            if (f < F && b < B) {
                const float gt = a[i], up = a[2 + i];
                const float hv = gt / (1.f + expf(-gt)) * up;
                h[static_cast<size_t>(b) * F + f] = __bfloat16_as_ushort(__float2bfloat16_rn(hv));
            }
        }
        return;
    }
    const int rA = grp * kRowsPerGroup + g;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = rA + (i >= 2 ? 8 : 0);
        const int b = 2 * q + (i & 1);
        if (r < m.R && b < B) {
            const size_t o = static_cast<size_t>(b) * m.R + r;
            if (m.out == kOutBf16)
                static_cast<uint16_t *>(m.y)[o] = __bfloat16_as_ushort(__float2bfloat16_rn(a[i]));
            else
                static_cast<float *>(m.y)[o] = a[i];
        }
    }
}

__device__ __forceinline__ int group_id(const Params &pr, int p, int grp) { return pr.prob[p].group0 + grp; }

// The warp's accumulators of row group (p, grp) are complete for its part of
// the group: store them, or hand them to the stream-K fix-up.  G0 is the
// grouped index of the warp's first row group.
__device__ __noinline__ void finish_group(const Params &pr, float4 a4, int p, int grp, int G0) {
    const float acc[4] = {a4.x, a4.y, a4.z, a4.w};
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const Problem &m = pr.prob[p];
    const long long n = pr.n_blocks;
    const long long u = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
    const long long ub0 = unit_start(u, n, pr.n_units), ub1 = unit_start(u + 1, n, pr.n_units);
    const long long gb0 = m.block0 + static_cast<long long>(grp) * m.T, gb1 = gb0 + m.T;
    if (gb0 >= ub0 && gb1 <= ub1) {
        store_y(m, pr.B, acc, grp, g, q);
        return;
    }
    const int G = m.group0 + grp;
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
        const Cur cv = locate(pr, vs, 0);
        const int sl = group_id(pr, cv.p, cv.grp) == G ? 0 : 1;
        const float4 t =
            __ldcg(reinterpret_cast<const float4 *>(pr.part + (static_cast<size_t>(v) * 2 + sl) * kSlotFloats) + lane);
        s[0] += t.x;
        s[1] += t.y;
        s[2] += t.z;
        s[3] += t.w;
    }
    store_y(m, pr.B, s, grp, g, q);
    if (lane == 0) atomicExch(pr.cnt + G, 0u);
}

__device__ __forceinline__ float4 sum_halves(const float (&acc)[2][4]) {
    return make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
}

// ---------------------------------------------------------------------------
// The kernel.  CHECK: an error word was given (every tile's escape count and
// base are verified).  V: the container version.

template <bool CHECK, int V>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_kernel(const __grid_constant__ Params pr) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sb = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3, qb = lane & ~3;
    const uint32_t bars = sb + static_cast<uint32_t>(warp) * kStages * 8u;
    const uint32_t ring = sb + kRingOff + static_cast<uint32_t>(warp) * kStages * kStageBytes;
    if (threadIdx.x == 0) grid_launch_dependents();
    Cur cc;  // the stage being computed
    {
        const long long u = static_cast<long long>(blockIdx.x) * kWarps + warp;
        const long long ub0 = unit_start(u, pr.n_blocks, pr.n_units);
        const int nb = static_cast<int>(unit_start(u + 1, pr.n_blocks, pr.n_units) - ub0);
        if (nb <= 0) return;
        cc = locate(pr, ub0, nb);
    }

    // The weights are never written by other kernels: start the copies and
    // the metadata loads before waiting for the previous grid.
    Cur pc = cc;     // next stage to copy
    int issued = 0;  // stages copied so far
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init_s(bars + 8u * s, 1);
        fence_barrier_init();
    }
    __syncwarp();
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
        if (pc.left > 0) {
            const int len = stage_len(pr, pc);
            if (lane == 0) issue(pr, pc, ring + s * kStageBytes, bars + 8u * s);
            advance(pc, len, pr);
            ++issued;
        }
    }

    int lenc = stage_len(pr, cc);
    Meta mc = load_meta<V>(pr.prob[cc.p], cc, lenc, g, q, true);
    if (V == 2 && cc.j > 0) {
        mc.sa += prefix_count_v2(pr.prob[cc.p], cc.grp * kRowsPerGroup + g, cc.j, q);
        mc.sb += prefix_count_v2(pr.prob[cc.p], cc.grp * kRowsPerGroup + g + 8, cc.j, q);
    }
    Cur cn = cc;  // the stage after it
    advance(cn, lenc, pr);
    int gp = cc.p, ggrp = cc.grp;  // the row group being accumulated
    uint32_t offA = mc.sa, offB = mc.sb;
    const int G0 = group_id(pr, gp, ggrp);
    grid_dependency_wait();  // x, y and the workspace may belong to earlier kernels
    const int gx = g < pr.B ? g : 0;  // batch rows past B repeat row 0; their outputs are dropped
    // the lane's shared-memory offsets inside a tile (raw rows are 128-byte swizzled)
    const uint32_t oA0 = g * 128 + (((2 * q) ^ g) << 4), oA1 = g * 128 + (((2 * q + 1) ^ g) << 4);
    const uint32_t oCA = kRawStage + g * 64 + 16 * q;

    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // one chain per half
    int consumed = 0;  // stages consumed so far
    bool ok = true;
    while (cc.left > 0) {
        // metadata of the next stage, one stage ahead
        int lenn = 0;
        Meta mn = {0u, 0u, 0u, 0u};
        if (cn.left > 0) {
            lenn = stage_len(pr, cn);
            mn = load_meta<V>(pr.prob[cn.p], cn, lenn, g, q, cn.j == 0);
        }
        if (cc.p != gp || cc.grp != ggrp) {
            finish_group(pr, sum_halves(acc), gp, ggrp, G0);
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[0][k] = acc[1][k] = 0.f;
            gp = cc.p;
            ggrp = cc.grp;
            offA = mc.sa;
            offB = mc.sb;
        }
        const int s = consumed & 1;
        const uint32_t bar = bars + 8u * s;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_s(bar, static_cast<uint32_t>(consumed >> 1) & 1u))) {
            raise_flag(pr.err, S12_FLAG_TIMEOUT);
            ok = false;
            break;
        }
        const Problem &m = pr.prob[cc.p];
        const uint32_t st = ring + s * kStageBytes;
        const uint16_t *xrow = m.x + static_cast<size_t>(gx) * m.K + 32 * q + static_cast<size_t>(cc.j) * kTile;
#pragma unroll
        for (int t = 0; t < kNT; ++t) {
            if (t >= lenc) break;
            const uint32_t tt = st + t * kRawTile, tc = st + t * kCodeTile;
            const uint4 rA0 = lds128(tt + oA0), rA1 = lds128(tt + oA1);
            const uint4 rB0 = lds128(tt + oA0 + 8 * 128), rB1 = lds128(tt + oA1 + 8 * 128);
            const uint4 cA = lds128(tc + oCA), cB = lds128(tc + oCA + 8 * 64);
            if (t == lenc - 1) {
                // the stage is in registers: hand it back to the copy engine
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (pc.left > 0) {
                    const int len = stage_len(pr, pc);
                    if (lane == 0) issue(pr, pc, st, bar);
                    advance(pc, len, pr);
                    ++issued;
                }
            }
            uint32_t bA, eA, bB, eB;
            tile_meta<V>(mc.a, qb, t, offA, bA, eA);
            tile_meta<V>(mc.b, qb, t, offB, bB, eB);
            bool esc = (eA != offA) || (eB != offB);
            if (CHECK) {
                esc = esc || (escape_nibbles(cA.x) | escape_nibbles(cA.y) | escape_nibbles(cA.z) | escape_nibbles(cA.w) |
                              escape_nibbles(cB.x) | escape_nibbles(cB.y) | escape_nibbles(cB.z) |
                              escape_nibbles(cB.w)) != 0;
                if (bA > static_cast<uint32_t>(kMaxBase) || bB > static_cast<uint32_t>(kMaxBase))
                    raise_flag(pr.err, S12_FLAG_BASE);
            }
            const uint16_t *xl = xrow + t * kTile;
            const uint32_t B4A = bA * 0x01010101u, B4B = bB * 0x01010101u;
            uint32_t xw[8], wa[8], wb[8];
            if (!__any_sync(0xFFFFFFFFu, esc)) {
                // no escapes in the block: straight decode and products
                load_x(xw, xl, 0);
                decode16(rA0, make_uint2(cA.x, cA.y), B4A, wa);
                decode16(rB0, make_uint2(cB.x, cB.y), B4B, wb);
                half_mma(acc[0], wa, wb, xw);
                load_x(xw, xl, 1);
                decode16(rA1, make_uint2(cA.z, cA.w), B4A, wa);
                decode16(rB1, make_uint2(cB.z, cB.w), B4B, wb);
                half_mma(acc[1], wa, wb, xw);
            } else {
                // some row of the block has escapes: rank them per row (quad
                // shuffles), decode, patch the escaped weights, multiply
                const uint32_t scr = sb + kRingOff + kWarps * kStages * kStageBytes + threadIdx.x * 32u;
                const EscRow xa = prepare_row(cA, offA, eA, m.n_esc, pr.err, q);
                const EscRow xb = prepare_row(cB, offB, eB, m.n_esc, pr.err, q);
                load_x(xw, xl, 0);
                decode16(rA0, make_uint2(cA.x, cA.y), B4A, wa);
                decode16(rB0, make_uint2(cB.x, cB.y), B4B, wb);
                if (xa.m0.x | xa.m0.y)
                    fix_half(wa, rA0, make_uint2(cA.x, cA.y), xa.m0, bA, xa.s0, xa.limit, m.esc, pr.err, scr);
                if (xb.m0.x | xb.m0.y)
                    fix_half(wb, rB0, make_uint2(cB.x, cB.y), xb.m0, bB, xb.s0, xb.limit, m.esc, pr.err, scr);
                half_mma(acc[0], wa, wb, xw);
                load_x(xw, xl, 1);
                decode16(rA1, make_uint2(cA.z, cA.w), B4A, wa);
                decode16(rB1, make_uint2(cB.z, cB.w), B4B, wb);
                if (xa.m1.x | xa.m1.y)
                    fix_half(wa, rA1, make_uint2(cA.z, cA.w), xa.m1, bA, xa.s1, xa.limit, m.esc, pr.err, scr);
                if (xb.m1.x | xb.m1.y)
                    fix_half(wb, rB1, make_uint2(cB.z, cB.w), xb.m1, bB, xb.s1, xb.limit, m.esc, pr.err, scr);
                half_mma(acc[1], wa, wb, xw);
            }
            offA = eA;
            offB = eB;
        }
        ++consumed;
        cc = cn;
        lenc = lenn;
        mc = mn;
        if (lenn > 0) advance(cn, lenn, pr);
    }
    if (ok) {
        finish_group(pr, sum_halves(acc), gp, ggrp, G0);
        return;
    }
    // A wait gave up (the error word says so; y is not valid).  Still arrive
    // on the current row group and every later one this warp shares, so each
    // group's counter returns to zero, then let the copies still in flight
    // land before the warp exits.
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int left = cc.left + (cc.j > 0 ? cc.j : 0);;) {
        finish_group(pr, z, gp, ggrp, G0);
        // blocks of this warp's range after the group just finished
        left -= pr.prob[gp].T;
        if (left <= 0) break;
        if (++ggrp == pr.prob[gp].n_groups) {
            ggrp = 0;
            if (++gp == pr.n_problems) break;
        }
    }
    if (lane == 0)
        for (int k = consumed; k < issued; ++k) mbar_wait_s(bars + 8u * (k & 1), static_cast<uint32_t>(k >> 1) & 1u);
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
    pl.part_bytes = gemv_part_bytes(sms);
    pl.cnt_bytes = gemv_cnt_bytes(static_cast<uint64_t>(pl.n_groups));
    return pl;
}

template <bool CHECK, int V>
int run(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *out,
        void *ws, uint32_t *err, const Plan &pl, cudaStream_t stream) {
    gemv::Params pr = {};
    long long block0 = 0;
    int group0 = 0;
    for (int i = 0; i < count; ++i) {
        const s12_view *v = views + i;
        gemv::Problem &m = pr.prob[i];
        const uint64_t R = v->rows, K = v->cols, T = K / kTile;
        if (make_tmap_u8_3d(&m.tm_raw, v->raw, 128, R, T, K, 128, 128, gemv::kRowsPerGroup, gemv::kNT, 128) !=
            S12_OK)
            return S12_ERR_CUDA;
        if (make_tmap_u8_3d(&m.tm_code, v->code, 64, R, T, K / 2, 64, 64, gemv::kRowsPerGroup, gemv::kNT, 0) !=
            S12_OK)
            return S12_ERR_CUDA;
        m.meta = V == 1 ? static_cast<const void *>(v->base) : static_cast<const void *>(v->tmeta);
        m.off = V == 1 ? v->esc_off : v->row_esc;
        m.esc = v->esc;
        m.x = x[i];
        m.y = y[i];
        m.out = out ? out[i] : gemv::kOutF32;
        m.n_esc = static_cast<uint32_t>(v->n_esc);
        m.R = static_cast<int>(R);
        m.K = static_cast<int>(K);
        m.T = static_cast<int>(T);
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
    // 1 KB alignment slack, barriers, the warps' rings, 32 bytes of escape
    // scratch per lane
    const uint32_t smem =
        1024 + gemv::kRingOff + gemv::kWarps * gemv::kStages * gemv::kStageBytes + gemv::kWarps * 32 * 32;
    if (smem > kSmemLimit) return S12_ERR_CUDA;
    auto kern = gemv::gemv_kernel<CHECK, V>;
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

int launch_gemv(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *out,
                void *ws, size_t ws_bytes, uint32_t *err, cudaStream_t stream) {
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    const Plan pl = plan(views, count, sms);
    if (ws_bytes < pl.part_bytes + pl.cnt_bytes) return S12_ERR_CAPACITY;
    const uint32_t version = views[0].version;
    for (int i = 1; i < count; ++i)
        if (views[i].version != version) return S12_ERR_ARG;
    if (version == 1)
        return err ? run<true, 1>(views, count, x, B, y, out, ws, err, pl, stream)
                   : run<false, 1>(views, count, x, B, y, out, ws, err, pl, stream);
    return err ? run<true, 2>(views, count, x, B, y, out, ws, err, pl, stream)
               : run<false, 2>(views, count, x, B, y, out, ws, err, pl, stream);
}

}  // namespace s12
