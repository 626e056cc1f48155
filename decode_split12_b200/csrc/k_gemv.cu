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
// Per-tile metadata.  Each lane loads, a stage ahead, the metadata of its
// tile for its two rows, as loaded words (arithmetic on them at load time
// would make the warp wait there): for a version 1 container the base and
// the tile's escape span from esc_off, for version 2 the stage's two
// (base | count) words and, at a row group's first stage, the row's escape
// offset, from which the spans follow as a running offset per row.  The
// decision "does this stage hold an escape" comes from the spans, not from
// scanning the code nibbles (which the checked variant still does).
//
// Escapes.  A stage whose tile rows all have empty escape spans takes the
// straight path, one loop-free body.  Otherwise the stage goes through one
// compact loop over its chunks: the first half of a tile row finds its
// first escape at the span's start, the second half counts back from the
// span's end (its escapes are the row's last), and each chunk with an escape
// is patched through a 32-byte per-lane shared scratch: the decoded words
// are stored, every escaped weight is overwritten by one 16-bit store of its
// exact value, and the words are read back.  With a tile base of 241,
// base + 15 would carry into the next byte, so such chunks are decoded again
// with the escape nibbles cleared.
//
// Work split (stream-K).  Blocks are numbered row-group-major (16-row group,
// then tile) across all matrices of the call and dealt to all warps of the
// grid in equal contiguous ranges, so every warp streams the same number of
// bytes (a CTA's warps hold consecutive ranges).  A warp keeps the
// accumulators of its current row group in registers; a group it covers
// whole goes straight to y.  A warp's first and last groups may be shared
// with its neighbours: their sums wait in registers until the warp is done,
// then go to its (by then free) ring in shared memory, and after a block
// barrier the warp holding a shared group's first block in this CTA adds the
// parts of the warps it spans, in warp order.  A group that stays inside the
// CTA is then stored; one that crosses into another CTA is finished across
// CTAs by the last CTA to arrive: each writes its part to the workspace and
// bumps the group's counter, and the one that completes the count adds the
// parts in CTA order (so y is the same on every call) and resets the counter
// to zero for the next call.  Small matrices, where a 16-row group spans
// many warps, so need no global fence or atomic for most groups.  A warp
// whose bounded wait gives up still hands in (zero) parts, so every counter
// sees all its arrivals and returns to zero even then.
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
    CUtensorMap tm_raw;   // u8 {128, T, R} (strides 128, K), box {128, 2, 16}, 128-byte swizzle
    CUtensorMap tm_code;  // u8 {64, T, R} (strides 64, K/2), box {64, 2, 16}, 64-byte swizzle
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
    float *part;    // workspace: [CTAs][2][kSlotFloats] partials of row groups shared by CTAs
    uint32_t *cnt;  // workspace: one arrival counter per row group (zero between calls)
    long long n_blocks;
    int n_problems, B;
    int n_units;    // warps in the grid
};

__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

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

// Position of grouped block b (b < n_blocks), with `left` blocks to go.  (A
// matrix has fewer than 2^32 / 2048 blocks, so 32-bit division serves.)
__device__ __forceinline__ Cur locate(const Params &pr, long long b, int left) {
    int p = 0;
    while (p + 1 < pr.n_problems && pr.prob[p + 1].block0 <= b) ++p;
    const uint32_t local = static_cast<uint32_t>(b - pr.prob[p].block0);
    const uint32_t T = static_cast<uint32_t>(pr.prob[p].T);
    const uint32_t grp = local / T;
    return Cur{p, static_cast<int>(grp), static_cast<int>(local - grp * T), left};
}

// First block of warp unit u's range: floor(u * n_blocks / n_units), from a
// double-precision quotient (the product is below 2^53) corrected to the
// exact floor; cheaper than a 64-bit integer division.
__device__ __forceinline__ long long unit_start(long long u, long long n_blocks, int n_units) {
    const long long x = u * n_blocks;
    long long q = static_cast<long long>(static_cast<double>(x) / static_cast<double>(n_units));
    if (q * n_units > x)
        --q;
    else if ((q + 1) * n_units <= x)
        ++q;
    return q;
}


// Start the copies of the stage at c into stage buffer st (completing on bar).
__device__ __forceinline__ void issue(const Params &pr, const Cur &c, uint32_t st, uint32_t bar) {
    const Problem &m = pr.prob[c.p];
    const uint64_t pol = policy_evict_first();
    mbar_expect_tx_s(bar, kStageBytes);
    tma3d(st, &m.tm_raw, 0, c.j, c.grp * kRowsPerGroup, bar, pol);
    tma3d(st + kRawStage, &m.tm_code, 0, c.j, c.grp * kRowsPerGroup, bar, pol);
}

// ---------------------------------------------------------------------------
// Metadata.  Lane (g, q) of a stage works on tile tq = q / 2 of the stage
// (its columns 64 (q % 2) .. +63 of that tile) for rows g and g+8, so it needs
// per row one base and the tile row's escape span [s, e).  They are loaded a
// stage ahead into a Meta (rows past the end and lanes past the stage's last
// tile read as base 0 with an empty span):
//   version 1:  base[t], esc_off[t], esc_off[t+1]     (t = r*T + j + tq)
//   version 2:  tmeta of the stage's two tiles, and the row's escape offset
//               row_esc[r] when the stage starts a row group; the spans
//               follow from a running offset per row.
struct Meta {
    uint32_t a0, a1, a2;  // row g
    uint32_t b0, b1, b2;  // row g + 8
};

// (the loaded words are kept as they are: any arithmetic on them here would
// make the warp wait for the loads a stage early)
template <int V>
__device__ __forceinline__ void load_row_meta(const Problem &m, int r, int j, int len, int tq, bool seg_start,
                                              uint32_t &w0, uint32_t &w1, uint32_t &w2) {
    w0 = w1 = w2 = 0u;
    if (r >= m.R) return;
    const size_t t0 = static_cast<size_t>(r) * m.T + j;
    if (V == 1) {
        if (tq < len) {
            w0 = __ldg(static_cast<const uint8_t *>(m.meta) + t0 + tq);
            w1 = __ldg(m.off + t0 + tq);
            w2 = __ldg(m.off + t0 + tq + 1);
        }
    } else {
        const uint16_t *tm = static_cast<const uint16_t *>(m.meta) + t0;
        w0 = __ldg(tm);
        if (len > 1) w1 = __ldg(tm + 1);
        if (seg_start) w2 = __ldg(m.off + r);
    }
}

template <int V>
__device__ __forceinline__ Meta load_meta(const Problem &m, const Cur &c, int len, int g, int tq, bool seg_start) {
    const int rA = c.grp * kRowsPerGroup + g;
    Meta r;
    load_row_meta<V>(m, rA, c.j, len, tq, seg_start, r.a0, r.a1, r.a2);
    load_row_meta<V>(m, rA + 8, c.j, len, tq, seg_start, r.b0, r.b1, r.b2);
    return r;
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

// A row's base and escape span [s, e) for the lane's tile; `run` is the
// row's escape offset at the stage's first tile (version 2), advanced past
// the stage.
template <int V>
__device__ __forceinline__ void row_span(uint32_t w0, uint32_t w1, uint32_t w2, int tq, uint32_t &run, uint32_t &base,
                                         uint32_t &s, uint32_t &e) {
    if (V == 1) {
        base = w0;
        s = w1;
        e = w2;
    } else {
        const uint32_t c0 = w0 >> 8, c1 = w1 >> 8;
        base = (tq ? w1 : w0) & 0xFFu;
        s = run + (tq ? c0 : 0u);
        e = s + (tq ? c1 : c0);
        run += c0 + c1;
    }
}

// ---------------------------------------------------------------------------
// Escapes.

// Escape-nibble counts of the lane's four 16-weight chunks of one row, one
// byte each (code words cw[0..3]: chunk c is cw[c/2].{x,y} or .{z,w}).
__device__ __forceinline__ uint32_t chunk_counts(uint4 c01, uint4 c23) {
    return __popc(escape_nibbles(c01.x) | (escape_nibbles(c01.y) >> 1)) |
           (__popc(escape_nibbles(c01.z) | (escape_nibbles(c01.w) >> 1)) << 8) |
           (__popc(escape_nibbles(c23.x) | (escape_nibbles(c23.y) >> 1)) << 16) |
           (__popc(escape_nibbles(c23.z) | (escape_nibbles(c23.w) >> 1)) << 24);
}

// A chunk with escapes: put the exact value of each escaped weight in place,
// taking stream index `idx` on; reads at or past `limit` are skipped and
// flagged.  The decoded words go through the lane's 32-byte shared scratch
// `sc`, so a weight is replaced by one 16-bit store at its position.  With
// base <= 240, base + 15 stays inside its byte and the other weights of the
// chunk are already right; a base of 241 could carry into the next byte, so
// such chunks are decoded again with the escape nibbles cleared first.
__device__ __forceinline__ void fix_chunk(uint32_t (&w)[8], uint4 raw, uint2 code, uint2 m, uint32_t base,
                                          uint32_t idx, uint32_t limit, const uint16_t *__restrict__ esc,
                                          uint32_t *err, uint32_t sc) {
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

// ---------------------------------------------------------------------------
// Products.

// The lane's 16 activations of chunk c (batch row and first column at xl),
// read through the L1 cache.
__device__ __forceinline__ void load_x(uint32_t (&xw)[8], const uint16_t *xl, int c) {
    const uint4 *src = reinterpret_cast<const uint4 *>(xl + c * 16);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
    xw[4] = b.x; xw[5] = b.y; xw[6] = b.z; xw[7] = b.w;
}

// One chunk: four m16n8k16 products of rows g / g+8 with x.
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

// First block of CTA c's range (its warps' ranges in order).
__device__ __forceinline__ long long cta_start(const Params &pr, long long c) {
    return unit_start(c * kWarps, pr.n_blocks, pr.n_units);
}

// Row group (p, grp) holds blocks [gb0, gb1) of the grouped numbering.
__device__ __forceinline__ void group_blocks(const Params &pr, int p, int grp, long long &gb0, long long &gb1) {
    gb0 = pr.prob[p].block0 + static_cast<long long>(grp) * pr.prob[p].T;
    gb1 = gb0 + pr.prob[p].T;
}

// The partial sums of a row group shared by several CTAs: this CTA's part
// goes to the workspace (slot 0 for the CTA's first group, 1 for its last),
// and the last CTA to arrive adds all parts in CTA order, stores y and
// resets the group's counter.  Run by one warp.
__device__ __noinline__ void cta_fixup(const Params &pr, float4 a4, int p, int grp) {
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const Problem &m = pr.prob[p];
    const int n_ctas = gridDim.x;
    const long long c = blockIdx.x, c0 = cta_start(pr, c);
    long long gb0, gb1;
    group_blocks(pr, p, grp, gb0, gb1);
    const int G = m.group0 + grp;
    float4 *mine = reinterpret_cast<float4 *>(pr.part + (static_cast<size_t>(c) * 2 + (gb0 <= c0 ? 0 : 1)) *
                                                            kSlotFloats) + lane;
    __stcg(mine, a4);
    __threadfence();
    __syncwarp();
    // the CTAs whose ranges meet the group (a CTA's range is never empty)
    long long cf = c, cl = c;
    while (cf > 0 && cta_start(pr, cf) > gb0) --cf;
    while (cl + 1 < n_ctas && cta_start(pr, cl + 1) < gb1) ++cl;
    uint32_t prev = 0;
    if (lane == 0) prev = atomicAdd(pr.cnt + G, 1u);
    prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
    if (prev + 1 != static_cast<uint32_t>(cl - cf + 1)) return;
    __threadfence();
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (long long v = cf; v <= cl; ++v) {
        const int sl = gb0 <= cta_start(pr, v) ? 0 : 1;
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

// After every warp of the CTA has put the sums of its split row groups in
// its partial slots (slot 0: its first group, slot 1: its last; in its own
// ring, which is free by then): each split group is completed by the warp
// whose range holds the group's first block inside this CTA, adding the
// parts of the warps it spans in warp order, then storing y or handing the
// CTA's part to the fix-up across CTAs.
__device__ __noinline__ void cta_combine(const Params &pr, uint32_t slots0) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const long long u = static_cast<long long>(blockIdx.x) * kWarps;
    // the CTA's warp boundaries, lane i holding the start of warp i's range
    const long long bnd = unit_start(u + (lane <= kWarps ? lane : kWarps), pr.n_blocks, pr.n_units);
    auto boundary = [&](int i) { return static_cast<long long>(__shfl_sync(0xFFFFFFFFu, bnd, i)); };
    const long long c0 = boundary(0), c1 = boundary(kWarps);
    const long long wb = boundary(warp), we = boundary(warp + 1);
    if (wb >= we) return;
    const Cur first = locate(pr, wb, 0), last = locate(pr, we - 1, 0);
    for (int k = 0; k < 2; ++k) {
        const Cur cg = k ? last : first;
        if (k && cg.p == first.p && cg.grp == first.grp) break;
        long long gb0, gb1;
        group_blocks(pr, cg.p, cg.grp, gb0, gb1);
        if (gb0 >= wb && gb1 <= we) continue;  // whole in this warp: stored already
        if ((gb0 > c0 ? gb0 : c0) < wb) continue;  // an earlier warp completes it
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        for (int v = warp; v < kWarps; ++v) {
            const long long vb = boundary(v), ve = boundary(v + 1);
            if (vb >= gb1) break;
            if (vb >= ve) continue;
            const uint32_t sl = gb0 <= vb ? 0u : 1u;  // the group is warp v's first or last
            const uint4 t = lds128(slots0 + static_cast<uint32_t>(v) * kStages * kStageBytes + sl * kGemvSlotBytes +
                                   16u * lane);
            s[0] += __uint_as_float(t.x);
            s[1] += __uint_as_float(t.y);
            s[2] += __uint_as_float(t.z);
            s[3] += __uint_as_float(t.w);
        }
        if (gb0 >= c0 && gb1 <= c1)
            store_y(pr.prob[cg.p], pr.B, s, cg.grp, g, q);
        else
            cta_fixup(pr, make_float4(s[0], s[1], s[2], s[3]), cg.p, cg.grp);
    }
}

__device__ __forceinline__ float4 sum_halves(const float (&acc)[2][4]) {
    return make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
}

// Store the sums of a row group held whole by this warp.
__device__ __forceinline__ void store_whole(const Params &pr, int p, int grp, const float (&acc)[2][4], int g,
                                            int q) {
    const float a[4] = {acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]};
    store_y(pr.prob[p], pr.B, a, grp, g, q);
}

// ---------------------------------------------------------------------------
// The kernel.  CHECK: an error word was given (every tile's escape count and
// base are verified).  V: the container version.

template <bool CHECK, int V>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_kernel(const __grid_constant__ Params pr) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sb = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3, tq = q >> 1, qh = q & 1;
    const uint32_t bars = sb + static_cast<uint32_t>(warp) * kStages * 8u;
    const uint32_t ring = sb + kRingOff + static_cast<uint32_t>(warp) * kStages * kStageBytes;
    if (threadIdx.x == 0) grid_launch_dependents();
    const long long u = static_cast<long long>(blockIdx.x) * kWarps + warp;
    const long long ub0 = unit_start(u, pr.n_blocks, pr.n_units);
    const int nb = static_cast<int>(unit_start(u + 1, pr.n_blocks, pr.n_units) - ub0);
    // The warp's range, then the row groups it shares with other warps
    // completed together (a lambda, so that its early exits still reach the
    // block barrier below).
    auto body = [&]() {
    Cur cc = locate(pr, ub0, nb);  // the stage being computed

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
    Meta mc = load_meta<V>(pr.prob[cc.p], cc, lenc, g, tq, true);
    uint32_t runA = 0, runB = 0;  // version 2: the rows' escape offsets at the current stage
    if (V == 2) {
        runA = mc.a2;
        runB = mc.b2;
        if (cc.j > 0) {
            runA += prefix_count_v2(pr.prob[cc.p], cc.grp * kRowsPerGroup + g, cc.j, q);
            runB += prefix_count_v2(pr.prob[cc.p], cc.grp * kRowsPerGroup + g + 8, cc.j, q);
        }
    }
    Cur cn = cc;  // the stage after it
    advance(cn, lenc, pr);

    int gp = cc.p, ggrp = cc.grp;  // the row group being accumulated
    const int G0 = group_id(pr, gp, ggrp);
    // the sums of the warp's first row group when other warps share it
    float4 first_part = make_float4(0.f, 0.f, 0.f, 0.f);
    grid_dependency_wait();  // x, y and the workspace may belong to earlier kernels
    const int gx = g < pr.B ? g : 0;  // batch rows past B repeat row 0; their outputs are dropped
    // The lane's shared-memory places (stage layout [row][tile][bytes]): raw
    // row g of its tile at oR (row g+8 2048 bytes on), 16-byte chunk k of it
    // at ((k ^ rsw) << 4); code row g at oC (row g+8 1024 bytes on), 16-byte
    // piece k at ((k ^ csw) << 4).  With the copy engine's 128-byte (raw) and
    // 64-byte (code) swizzles, every 16-byte read of a quarter warp hits its
    // own banks.
    const uint32_t oR = static_cast<uint32_t>(2 * g + tq) * 128u, rsw = static_cast<uint32_t>(2 * g + tq) & 7u;
    const uint32_t oC = kRawStage + static_cast<uint32_t>(2 * g + tq) * 64u, csw = static_cast<uint32_t>(g) & 3u;
    const uint32_t oC0 = oC + ((static_cast<uint32_t>(2 * qh) ^ csw) << 4);
    const uint32_t oC1 = oC + ((static_cast<uint32_t>(2 * qh + 1) ^ csw) << 4);

    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // two chains
    int consumed = 0;  // stages consumed so far
    bool ok = true;
    while (cc.left > 0) {
        // metadata of the next stage, one stage ahead
        int lenn = 0;
        Meta mn = {0u, 0u, 0u, 0u, 0u, 0u};
        if (cn.left > 0) {
            lenn = stage_len(pr, cn);
            mn = load_meta<V>(pr.prob[cn.p], cn, lenn, g, tq, cn.j == 0);
        }
        if (cc.p != gp || cc.grp != ggrp) {
            // a group ends inside the range: the warp's whole group is stored,
            // its first group (if another warp has part of it) is kept
            long long gb0, gb1;
            group_blocks(pr, gp, ggrp, gb0, gb1);
            if (gb0 >= ub0)
                store_whole(pr, gp, ggrp, acc, g, q);
            else
                first_part = sum_halves(acc);
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[0][k] = acc[1][k] = 0.f;
            gp = cc.p;
            ggrp = cc.grp;
            if (V == 2) {
                runA = mc.a2;
                runB = mc.b2;
            }
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
        const bool live = tq < lenc;  // the lane's tile belongs to this stage
        uint32_t bA, sA, eA, bB, sB, eB;
        row_span<V>(mc.a0, mc.a1, mc.a2, tq, runA, bA, sA, eA);
        row_span<V>(mc.b0, mc.b1, mc.b2, tq, runB, bB, sB, eB);

        uint4 cA0 = make_uint4(0, 0, 0, 0), cA1 = cA0, cB0 = cA0, cB1 = cA0;
        if (live) {
            cA0 = lds128(st + oC0);
            cA1 = lds128(st + oC1);
            cB0 = lds128(st + oC0 + 1024);
            cB1 = lds128(st + oC1 + 1024);
        }
        bool esc = (eA != sA) || (eB != sB);
        if (CHECK) {
            // every tile row's code-15 count against its span (the two lanes
            // of a pair hold the row's two halves)
            const uint32_t ccA = chunk_counts(cA0, cA1), ccB = chunk_counts(cB0, cB1);
            const uint32_t totA = (ccA * 0x01010101u) >> 24, totB = (ccB * 0x01010101u) >> 24;
            const uint32_t pairA = __shfl_xor_sync(0xFFFFFFFFu, totA, 1), pairB = __shfl_xor_sync(0xFFFFFFFFu, totB, 1);
            if (live && qh == 0 && (totA + pairA != eA - sA || totB + pairB != eB - sB))
                raise_flag(pr.err, S12_FLAG_ESC_COUNT);
            esc = esc || (ccA | ccB) != 0;
            if (bA > static_cast<uint32_t>(kMaxBase) || bB > static_cast<uint32_t>(kMaxBase))
                raise_flag(pr.err, S12_FLAG_BASE);
        }
        const bool anyesc = __any_sync(0xFFFFFFFFu, esc);
        const uint32_t B4A = bA * 0x01010101u, B4B = bB * 0x01010101u;
        const uint16_t *xl = m.x + static_cast<size_t>(gx) * m.K + static_cast<size_t>(cc.j + tq) * kTile + 64 * qh;
        const uint32_t oRA = st + oR, oRB = oRA + 2048;
        if (!anyesc) {
            // no escapes in the stage: straight decode and products, the
            // loop unrolled (this is the hot code)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 rA = make_uint4(0, 0, 0, 0), rB = rA;
                if (live) {
                    rA = lds128(oRA + ((static_cast<uint32_t>(4 * qh + c) ^ rsw) << 4));
                    rB = lds128(oRB + ((static_cast<uint32_t>(4 * qh + c) ^ rsw) << 4));
                }
                if (c == 3) {
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
                uint32_t xw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if (live) load_x(xw, xl, c);
                const uint4 kA4 = c < 2 ? cA0 : cA1, kB4 = c < 2 ? cB0 : cB1;
                const uint2 kA = (c & 1) ? make_uint2(kA4.z, kA4.w) : make_uint2(kA4.x, kA4.y);
                const uint2 kB = (c & 1) ? make_uint2(kB4.z, kB4.w) : make_uint2(kB4.x, kB4.y);
                uint32_t wa[8], wb[8];
                decode16(rA, kA, B4A, wa);
                decode16(rB, kB, B4B, wb);
                half_mma(acc[c & 1], wa, wb, xw);
            }
        } else {
            // some tile row of the stage has escapes: one compact loop over
            // the chunks (rare code, kept small), the stage held until its end
            const uint32_t ccA = chunk_counts(cA0, cA1), ccB = chunk_counts(cB0, cB1);
            // the lane's first escape in each row: the first half of a tile
            // row counts from the span's start, the second half back from its
            // end (its escapes are the row's last ones)
            uint32_t iA = qh ? eA - ((ccA * 0x01010101u) >> 24) : sA;
            uint32_t iB = qh ? eB - ((ccB * 0x01010101u) >> 24) : sB;
            const uint32_t limA = sA <= eA ? min(eA, m.n_esc) : 0u, limB = sB <= eB ? min(eB, m.n_esc) : 0u;
            const uint32_t scr = sb + kRingOff + kWarps * kStages * kStageBytes + threadIdx.x * 32u;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint4 rA = make_uint4(0, 0, 0, 0), rB = rA;
                uint2 kA = make_uint2(0, 0), kB = kA;
                uint32_t xw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                if (live) {
                    rA = lds128(oRA + ((static_cast<uint32_t>(4 * qh + c) ^ rsw) << 4));
                    rB = lds128(oRB + ((static_cast<uint32_t>(4 * qh + c) ^ rsw) << 4));
                    // chunk c's 8 code bytes: 16-byte piece c / 2 (swizzled), half c % 2
                    const uint32_t piece = st + oC + ((static_cast<uint32_t>(2 * qh + (c >> 1)) ^ csw) << 4) + 8u * (c & 1);
                    kA = lds64(piece);
                    kB = lds64(piece + 1024);
                    load_x(xw, xl, c);
                }
                uint32_t wa[8], wb[8];
                decode16(rA, kA, B4A, wa);
                decode16(rB, kB, B4B, wb);
                const uint2 mA = make_uint2(escape_nibbles(kA.x), escape_nibbles(kA.y));
                const uint2 mB = make_uint2(escape_nibbles(kB.x), escape_nibbles(kB.y));
                if (mA.x | mA.y) fix_chunk(wa, rA, kA, mA, bA, iA, limA, m.esc, pr.err, scr);
                if (mB.x | mB.y) fix_chunk(wb, rB, kB, mB, bB, iB, limB, m.esc, pr.err, scr);
                iA += (ccA >> (8 * c)) & 0xFFu;
                iB += (ccB >> (8 * c)) & 0xFFu;
                if (c & 1)
                    half_mma(acc[1], wa, wb, xw);
                else
                    half_mma(acc[0], wa, wb, xw);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (pc.left > 0) {
                const int len = stage_len(pr, pc);
                if (lane == 0) issue(pr, pc, st, bar);
                advance(pc, len, pr);
                ++issued;
            }
        }
        ++consumed;
        cc = cn;
        lenc = lenn;
        mc = mn;
        if (lenn > 0) advance(cn, lenn, pr);
    }
    // the last group: whole in the range, or shared (its part goes to slot
    // 0 when it is also the first group, else to slot 1)
    long long gb0, gb1;
    group_blocks(pr, gp, ggrp, gb0, gb1);
    const long long ub1 = ub0 + nb;
    float4 last_part = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ok) {
        if (gb0 >= ub0 && gb1 <= ub1)
            store_whole(pr, gp, ggrp, acc, g, q);
        else if (group_id(pr, gp, ggrp) == G0)
            first_part = sum_halves(acc);
        else
            last_part = sum_halves(acc);
    } else {
        // A wait gave up (the error word says so; y is not valid): the
        // shared groups get zero parts, so every counter still sees all its
        // arrivals; the copies still in flight land first.
        first_part = last_part = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0)
            for (int k = consumed; k < issued; ++k)
                mbar_wait_s(bars + 8u * (k & 1), static_cast<uint32_t>(k >> 1) & 1u);
        __syncwarp();
    }
    // the ring is free now: the two parts go to its first 1 KB
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(ring + 16u * lane), "f"(first_part.x),
                 "f"(first_part.y), "f"(first_part.z), "f"(first_part.w)
                 : "memory");
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(ring + kGemvSlotBytes + 16u * lane),
                 "f"(last_part.x), "f"(last_part.y), "f"(last_part.z), "f"(last_part.w)
                 : "memory");
    };
    if (nb > 0) body();
    __syncthreads();
    grid_dependency_wait();
    cta_combine(pr, sb + kRingOff);
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
        if (make_tmap_u8_3d(&m.tm_raw, v->raw, 128, T, R, 128, K, 128, gemv::kNT, gemv::kRowsPerGroup, 128) !=
            S12_OK)
            return S12_ERR_CUDA;
        if (make_tmap_u8_3d(&m.tm_code, v->code, 64, T, R, 64, K / 2, 64, gemv::kNT, gemv::kRowsPerGroup, 64) !=
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
