// s12_device.cuh -- device-side building blocks shared by the Split12 kernels
// (sm_100a only): container geometry, PTX wrappers for mbarriers and TMA bulk
// copies, bounded waits, and the register-level decode of 16 weights.
//
// Format (restated from the pages; see include/s12.h for the byte layout):
// a BF16 weight is 1 sign, 8 exponent and 7 mantissa bits ("你的 bf16 模型,
// 有 5 個 bit 是廢的", section 1 table).  It is stored as a raw byte
// (sign | mantissa) plus a 4-bit exponent code relative to the base of its
// 128-weight tile; code 15 means the whole value sits in the escape stream
// ("GPU 友善 12 位無損 BF16 壓縮格式", key points and technical deep dive:
// one integer ADD decodes, escapes live in a separate buffer).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "s12.h"

namespace s12 {

constexpr int kTile = 128;           // weights per tile (along K)
constexpr int kMaxBase = 241;        // base + 14 <= 255
constexpr uint32_t kAlign = 256;     // plane alignment inside a container
constexpr uint32_t kHeaderBytes = 256;

__host__ __device__ inline uint64_t align_up(uint64_t n, uint64_t a) { return (n + a - 1) / a * a; }

// Plane offsets of a container with the given shape and escape count.
struct Geometry {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_raw, off_code, off_base, off_esc_off, off_esc, total;
};

__host__ __device__ inline Geometry geometry(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    Geometry g;
    g.rows = rows;
    g.cols = cols;
    g.n_tiles = rows * (cols / kTile);
    g.n_esc = n_esc;
    g.off_raw = kHeaderBytes;
    g.off_code = g.off_raw + align_up(rows * cols, kAlign);
    g.off_base = g.off_code + align_up(rows * cols / 2, kAlign);
    g.off_esc_off = g.off_base + align_up(g.n_tiles, kAlign);
    g.off_esc = g.off_esc_off + align_up(4 * (g.n_tiles + 1), kAlign);
    g.total = g.off_esc + align_up(2 * n_esc, kAlign);
    return g;
}

// Plane offsets of a version 2 container (compact tile header): the raw,
// code and escape planes as in version 1, and in place of the base and
// offset planes one u16 per tile (base | escape count << 8) and one u32 per
// row (escapes in the rows before it; the last entry is n_esc).
struct Geometry2 {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_raw, off_code, off_tmeta, off_row_esc, off_esc, total;
};

__host__ __device__ inline Geometry2 geometry2(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    Geometry2 g;
    g.rows = rows;
    g.cols = cols;
    g.n_tiles = rows * (cols / kTile);
    g.n_esc = n_esc;
    g.off_raw = kHeaderBytes;
    g.off_code = g.off_raw + align_up(rows * cols, kAlign);
    g.off_tmeta = g.off_code + align_up(rows * cols / 2, kAlign);
    g.off_row_esc = g.off_tmeta + align_up(2 * g.n_tiles, kAlign);
    g.off_esc = g.off_row_esc + align_up(4 * (rows + 1), kAlign);
    g.total = g.off_esc + align_up(2 * n_esc, kAlign);
    return g;
}

// Plane offsets of a version 3 container (packed 24-bit pairs): weights 2i
// and 2i+1 stored as raw(2i), raw(2i+1), code(2i) | code(2i+1) << 4 in one
// pair plane, then the base, offset and escape planes of version 1.
struct Geometry3 {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_pair, off_base, off_esc_off, off_esc, total;
};

__host__ __device__ inline Geometry3 geometry3(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    Geometry3 g;
    g.rows = rows;
    g.cols = cols;
    g.n_tiles = rows * (cols / kTile);
    g.n_esc = n_esc;
    g.off_pair = kHeaderBytes;
    g.off_base = g.off_pair + align_up(rows * cols / 2 * 3, kAlign);
    g.off_esc_off = g.off_base + align_up(g.n_tiles, kAlign);
    g.off_esc = g.off_esc_off + align_up(4 * (g.n_tiles + 1), kAlign);
    g.total = g.off_esc + align_up(2 * n_esc, kAlign);
    return g;
}

// Plane offsets of a version 4 container (sign-and-exponent symbol codes):
// the symbol table u16[32], then raw, code, esc_off and esc as version 1
// (no base plane).
struct Geometry4 {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_table, off_raw, off_code, off_esc_off, off_esc, total;
};

__host__ __device__ inline Geometry4 geometry4(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    Geometry4 g;
    g.rows = rows;
    g.cols = cols;
    g.n_tiles = rows * (cols / kTile);
    g.n_esc = n_esc;
    g.off_table = kHeaderBytes;
    g.off_raw = g.off_table + kAlign;  // 64 bytes used
    g.off_code = g.off_raw + align_up(rows * cols, kAlign);
    g.off_esc_off = g.off_code + align_up(rows * cols / 2, kAlign);
    g.off_esc = g.off_esc_off + align_up(4 * (g.n_tiles + 1), kAlign);
    g.total = g.off_esc + align_up(2 * n_esc, kAlign);
    return g;
}

// ---------------------------------------------------------------------------
// Bounded waiting.  Every spin in these kernels gives up after about a second
// at full clock, sets S12_FLAG_TIMEOUT and lets the caller unwind.
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ void raise_flag(uint32_t *err, uint32_t bits) {
    if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Programmatic dependent launch: wait until the grids this one depends on
// have completed (and their writes are visible); allow the next grid in the
// stream to begin launching.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// L2 policy for data read exactly once (weights): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------
// Byte permute and register-level decode.

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Four weights: raw bytes R = [r0 r1 r2 r3] and exponents E = [e0 e1 e2 e3]
// (one per byte) give the BF16 pairs (w0, w1) and (w2, w3).  The BF16 high
// byte is sign | exponent >> 1, the low byte is (exponent & 1) << 7 | mantissa.
__device__ __forceinline__ void assemble4(uint32_t R, uint32_t E, uint32_t &p01, uint32_t &p23) {
    const uint32_t M = 0x80808080u;
    const uint32_t hi = ((E >> 1) & ~M) | (R & M);
    const uint32_t lo = ((E << 7) & M) | (R & ~M);
    p01 = prmt(lo, hi, 0x5140u);  // [lo0 hi0 lo1 hi1]
    p23 = prmt(lo, hi, 0x7362u);  // [lo2 hi2 lo3 hi3]
}

// Eight weights from two raw words and one code word (byte j of C holds the
// codes of weights 2j (low nibble) and 2j+1 (high nibble)); B4 = base in
// every byte.  Exponent = base + code, one byte-wise integer ADD: no carry
// leaves a byte because base <= 241 and code <= 14 on this path (escape
// nibbles are cleared before this call whenever the word has any).
__device__ __forceinline__ void decode8(uint32_t R0, uint32_t R1, uint32_t C, uint32_t B4, uint32_t out[4]) {
    const uint32_t ce = (C & 0x0F0F0F0Fu) + B4;         // e0 e2 e4 e6
    const uint32_t co = ((C >> 4) & 0x0F0F0F0Fu) + B4;  // e1 e3 e5 e7
    const uint32_t E0 = prmt(ce, co, 0x5140u);          // e0 e1 e2 e3
    const uint32_t E1 = prmt(ce, co, 0x7362u);          // e4 e5 e6 e7
    assemble4(R0, E0, out[0], out[1]);
    assemble4(R1, E1, out[2], out[3]);
}

// Sixteen weights: raw = 16 raw bytes, code = 8 code bytes; out[j] holds the
// BF16 pair (w_2j, w_2j+1), low half first.
__device__ __forceinline__ void decode16(uint4 raw, uint2 code, uint32_t B4, uint32_t out[8]) {
    decode8(raw.x, raw.y, code.x, B4, out);
    decode8(raw.z, raw.w, code.y, B4, out + 4);
}

// Bit 4j+3 set iff nibble j of C equals 15 (an escape).
__device__ __forceinline__ uint32_t escape_nibbles(uint32_t C) {
    return ((C & 0x77777777u) + 0x11111111u) & C & 0x88888888u;
}

// Clear every escape nibble (so the byte-wise ADD cannot carry).
__device__ __forceinline__ uint32_t clear_escapes(uint32_t C, uint32_t m) {
    return C & ~(m | (m >> 1) | (m >> 2) | (m >> 3));
}

}  // namespace s12
