// s12_validate.cu -- host-side container validation and per-plane hashes.
//
// "Lossless LLM Weight Compression vs 8-bit GGUF", section "A 14-day
// production-readiness pilot": inject corruption and confirm that it is
// detected rather than decoded into wrong weights.  The kernels already raise
// err_flag bits when they meet inconsistent escape data; these calls check a
// whole container in host memory before it is trusted (for instance after it
// is read from disk), and give 64-bit hashes of its planes so that bytes
// without redundancy (raw bytes, escape values) can be checked against hashes
// stored at encode time.
//
// A container is valid when the header is well formed, the bytes cover every
// plane, esc_off starts at 0 and ends at n_esc, and every tile has
// non-decreasing offsets within the stream, a base of at most 241 and exactly
// as many code-15 nibbles as its offsets span.  Non-zero padding does not
// make a container invalid (nothing reads it); it is reported as a note.
#include <cstring>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {
namespace {

uint32_t rd32(const uint8_t *p) {
    return uint32_t(p[0]) | uint32_t(p[1]) << 8 | uint32_t(p[2]) << 16 | uint32_t(p[3]) << 24;
}
uint64_t rd64(const uint8_t *p) { return uint64_t(rd32(p)) | uint64_t(rd32(p + 4)) << 32; }

// FNV-1a, 64-bit: offset basis 0xcbf29ce484222325, prime 0x100000001b3.
uint64_t fnv1a64(const uint8_t *p, uint64_t n) {
    uint64_t h = 0xcbf29ce484222325ull;
    for (uint64_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 0x100000001b3ull;
    }
    return h;
}

bool any_nonzero(const uint8_t *p, uint64_t n) {
    for (uint64_t i = 0; i < n; ++i)
        if (p[i]) return true;
    return false;
}

// Header checks shared by both calls; fills the geometry.
int parse_header(const uint8_t *c, size_t bytes, Geometry *g) {
    if (bytes < kHeaderBytes) return S12_BAD_SIZE;
    if (std::memcmp(c, "S12\0", 4) != 0 || rd32(c + 4) != 1 || rd32(c + 24) != static_cast<uint32_t>(kTile) ||
        rd32(c + 28) != 0)
        return S12_BAD_HEADER;
    for (int i = 40; i < 64; ++i)
        if (c[i]) return S12_BAD_HEADER;
    const uint64_t rows = rd64(c + 8), cols = rd64(c + 16), n_esc = rd64(c + 32);
    if (rows == 0 || cols == 0 || cols % kTile) return S12_BAD_HEADER;
    if (rows >= (uint64_t(1) << 32) || cols >= (uint64_t(1) << 32) || rows * cols >= (uint64_t(1) << 32))
        return S12_BAD_HEADER;
    if (n_esc > rows * cols) return S12_BAD_HEADER;
    *g = geometry(rows, cols, n_esc);
    if (g->total > bytes) return S12_BAD_SIZE;
    return 0;
}

}  // namespace
}  // namespace s12

using namespace s12;

extern "C" uint64_t s12_fnv1a64(const void *data, size_t bytes) {
    return data ? fnv1a64(static_cast<const uint8_t *>(data), bytes) : fnv1a64(nullptr, 0);
}

extern "C" int s12_validate_host(const void *container, size_t bytes, s12_report *out) {
    if (!container || !out) return S12_ERR_ARG;
    std::memset(out, 0, sizeof *out);
    const uint8_t *c = static_cast<const uint8_t *>(container);
    Geometry g;
    const int bad = parse_header(c, bytes, &g);
    if (bad) {
        out->problem = static_cast<uint32_t>(bad);
        return S12_ERR_CORRUPT;
    }
    const uint8_t *code = c + g.off_code, *base = c + g.off_base, *off = c + g.off_esc_off;
    if (rd32(off) != 0 || rd32(off + 4 * g.n_tiles) != g.n_esc) {
        out->problem = S12_BAD_OFFSETS;
        return S12_ERR_CORRUPT;
    }
    for (uint64_t t = 0; t < g.n_tiles; ++t) {
        const uint32_t lo = rd32(off + 4 * t), hi = rd32(off + 4 * (t + 1));
        uint32_t n15 = 0;
        for (int k = 0; k < kTile / 2; ++k) {
            const uint8_t b = code[t * (kTile / 2) + k];
            n15 += ((b & 0x0F) == 0x0F) + ((b >> 4) == 0x0F);
        }
        out->n_esc_counted += n15;
        uint32_t problem = 0;
        if (hi < lo || hi > g.n_esc)
            problem = S12_BAD_TILE_OFFSETS;
        else if (base[t] > kMaxBase)
            problem = S12_BAD_BASE;
        else if (n15 != hi - lo)
            problem = S12_BAD_ESC_COUNT;
        if (problem) {
            out->problem = problem;
            out->tile = t;
            return S12_ERR_CORRUPT;
        }
    }
    // padding after the 64 header bytes in use and after every plane
    const uint64_t ends[6][2] = {{64, g.off_raw},
                                 {g.off_raw + g.rows * g.cols, g.off_code},
                                 {g.off_code + g.rows * g.cols / 2, g.off_base},
                                 {g.off_base + g.n_tiles, g.off_esc_off},
                                 {g.off_esc_off + 4 * (g.n_tiles + 1), g.off_esc},
                                 {g.off_esc + 2 * g.n_esc, g.total}};
    for (const auto &e : ends)
        if (any_nonzero(c + e[0], e[1] - e[0])) out->notes |= S12_NOTE_PADDING;
    return S12_OK;
}

extern "C" int s12_plane_hashes_host(const void *container, size_t bytes, uint64_t out[5]) {
    if (!container || !out) return S12_ERR_ARG;
    const uint8_t *c = static_cast<const uint8_t *>(container);
    Geometry g;
    if (parse_header(c, bytes, &g)) return S12_ERR_CORRUPT;
    out[0] = fnv1a64(c + g.off_raw, g.rows * g.cols);
    out[1] = fnv1a64(c + g.off_code, g.rows * g.cols / 2);
    out[2] = fnv1a64(c + g.off_base, g.n_tiles);
    out[3] = fnv1a64(c + g.off_esc_off, 4 * (g.n_tiles + 1));
    out[4] = fnv1a64(c + g.off_esc, 2 * g.n_esc);
    return S12_OK;
}

// ---------------------------------------------------------------------------
// Container version 2 (a compact tile header) as a storage format.  Same
// raw, code and escape planes; per tile one u16 = base | escape count << 8
// and per row one u32 escape offset, instead of a u8 base and a u32 offset
// per tile: 2 bytes per tile + 4 per row instead of 5 per tile, toward the
// 24.967 % payload reduction of "Lossless LLM Weight Compression vs 8-bit
// GGUF" (English edition, opening summary).  The kernels read both
// versions; these calls convert between them in host memory, for storage or
// transfer.

namespace s12 {
namespace {

void wr32(uint8_t *p, uint32_t v) {
    for (int i = 0; i < 4; ++i) p[i] = static_cast<uint8_t>(v >> (8 * i));
}

}  // namespace
}  // namespace s12

extern "C" int s12_to_v2_host(const void *v1, size_t v1_bytes, void *dst, size_t dst_cap, size_t *bytes_out) {
    if (!v1 || !bytes_out) return S12_ERR_ARG;
    s12_report rep;
    const int rc = s12_validate_host(v1, v1_bytes, &rep);
    if (rc != S12_OK) return rc;
    const uint8_t *c = static_cast<const uint8_t *>(v1);
    const Geometry g = geometry(rd64(c + 8), rd64(c + 16), rd64(c + 32));
    const Geometry2 g2 = geometry2(g.rows, g.cols, g.n_esc);
    *bytes_out = g2.total;
    if (!dst) return S12_OK;
    if (dst_cap < g2.total) return S12_ERR_CAPACITY;
    uint8_t *d = static_cast<uint8_t *>(dst);
    std::memset(d, 0, g2.total);
    std::memcpy(d, c, 64);
    wr32(d + 4, 2);
    std::memcpy(d + g2.off_raw, c + g.off_raw, g.rows * g.cols);
    std::memcpy(d + g2.off_code, c + g.off_code, g.rows * g.cols / 2);
    std::memcpy(d + g2.off_esc, c + g.off_esc, 2 * g.n_esc);
    const uint8_t *off = c + g.off_esc_off;
    const uint64_t T = g.cols / kTile;
    for (uint64_t t = 0; t < g.n_tiles; ++t) {
        const uint32_t count = rd32(off + 4 * (t + 1)) - rd32(off + 4 * t);  // <= 128 in a valid container
        d[g2.off_tmeta + 2 * t] = c[g.off_base + t];
        d[g2.off_tmeta + 2 * t + 1] = static_cast<uint8_t>(count);
    }
    for (uint64_t r = 0; r <= g.rows; ++r) wr32(d + g2.off_row_esc + 4 * r, rd32(off + 4 * (r * T)));
    return S12_OK;
}

extern "C" int s12_from_v2_host(const void *v2, size_t v2_bytes, void *dst, size_t dst_cap, size_t *bytes_out) {
    if (!v2 || !bytes_out) return S12_ERR_ARG;
    const uint8_t *c = static_cast<const uint8_t *>(v2);
    if (v2_bytes < kHeaderBytes || std::memcmp(c, "S12\0", 4) != 0 || rd32(c + 4) != 2 ||
        rd32(c + 24) != static_cast<uint32_t>(kTile) || rd32(c + 28) != 0)
        return S12_ERR_CORRUPT;
    for (int i = 40; i < 64; ++i)
        if (c[i]) return S12_ERR_CORRUPT;
    const uint64_t rows = rd64(c + 8), cols = rd64(c + 16), n_esc = rd64(c + 32);
    if (rows == 0 || cols == 0 || cols % kTile || rows >= (uint64_t(1) << 32) || cols >= (uint64_t(1) << 32) ||
        rows * cols >= (uint64_t(1) << 32) || n_esc > rows * cols)
        return S12_ERR_CORRUPT;
    const Geometry2 g2 = geometry2(rows, cols, n_esc);
    if (g2.total > v2_bytes) return S12_ERR_CORRUPT;
    const Geometry g = geometry(rows, cols, n_esc);
    // the row offsets and tile counts must describe the escape stream exactly
    const uint8_t *row_esc = c + g2.off_row_esc, *tmeta = c + g2.off_tmeta;
    const uint64_t T = cols / kTile;
    if (rd32(row_esc) != 0 || rd32(row_esc + 4 * rows) != n_esc) return S12_ERR_CORRUPT;
    for (uint64_t r = 0; r < rows; ++r) {
        uint64_t k = rd32(row_esc + 4 * r);
        for (uint64_t j = 0; j < T; ++j) k += tmeta[2 * (r * T + j) + 1];
        if (k != rd32(row_esc + 4 * (r + 1))) return S12_ERR_CORRUPT;
    }
    *bytes_out = g.total;
    if (!dst) return S12_OK;
    if (dst_cap < g.total) return S12_ERR_CAPACITY;
    uint8_t *d = static_cast<uint8_t *>(dst);
    std::memset(d, 0, g.total);
    std::memcpy(d, c, 64);
    wr32(d + 4, 1);
    std::memcpy(d + g.off_raw, c + g2.off_raw, rows * cols);
    std::memcpy(d + g.off_code, c + g2.off_code, rows * cols / 2);
    std::memcpy(d + g.off_esc, c + g2.off_esc, 2 * n_esc);
    uint64_t k = 0;
    for (uint64_t t = 0; t < g.n_tiles; ++t) {
        if (t % T == 0) k = rd32(row_esc + 4 * (t / T));
        d[g.off_base + t] = tmeta[2 * t];
        wr32(d + g.off_esc_off + 4 * t, static_cast<uint32_t>(k));
        k += tmeta[2 * t + 1];
    }
    wr32(d + g.off_esc_off + 4 * g.n_tiles, static_cast<uint32_t>(n_esc));
    return S12_OK;
}

// ---------------------------------------------------------------------------
// Container version 3 (packed 24-bit pairs) as a storage format: version 1
// with the raw and code planes regrouped into one pair plane (weights 2i and
// 2i+1 as raw, raw, code | code << 4; "GPU 友善 12 位無損 BF16 壓縮格式",
// technical deep dive: two 12-bit weights per 3-byte word).  The metadata
// and escape planes are version 1's, byte for byte.

extern "C" int s12_to_v3_host(const void *v1, size_t v1_bytes, void *dst, size_t dst_cap, size_t *bytes_out) {
    if (!v1 || !bytes_out) return S12_ERR_ARG;
    s12_report rep;
    const int rc = s12_validate_host(v1, v1_bytes, &rep);
    if (rc != S12_OK) return rc;
    const uint8_t *c = static_cast<const uint8_t *>(v1);
    const Geometry g = geometry(rd64(c + 8), rd64(c + 16), rd64(c + 32));
    const Geometry3 g3 = geometry3(g.rows, g.cols, g.n_esc);
    *bytes_out = g3.total;
    if (!dst) return S12_OK;
    if (dst_cap < g3.total) return S12_ERR_CAPACITY;
    uint8_t *d = static_cast<uint8_t *>(dst);
    std::memset(d, 0, g3.total);
    std::memcpy(d, c, 64);
    wr32(d + 4, 3);
    const uint8_t *raw = c + g.off_raw, *code = c + g.off_code;
    uint8_t *pair = d + g3.off_pair;
    for (uint64_t i = 0; i < g.rows * g.cols / 2; ++i) {
        pair[3 * i] = raw[2 * i];
        pair[3 * i + 1] = raw[2 * i + 1];
        pair[3 * i + 2] = code[i];
    }
    std::memcpy(d + g3.off_base, c + g.off_base, g.n_tiles);
    std::memcpy(d + g3.off_esc_off, c + g.off_esc_off, 4 * (g.n_tiles + 1));
    std::memcpy(d + g3.off_esc, c + g.off_esc, 2 * g.n_esc);
    return S12_OK;
}

extern "C" int s12_from_v3_host(const void *v3, size_t v3_bytes, void *dst, size_t dst_cap, size_t *bytes_out) {
    if (!v3 || !bytes_out) return S12_ERR_ARG;
    const uint8_t *c = static_cast<const uint8_t *>(v3);
    if (v3_bytes < kHeaderBytes || std::memcmp(c, "S12\0", 4) != 0 || rd32(c + 4) != 3 ||
        rd32(c + 24) != static_cast<uint32_t>(kTile) || rd32(c + 28) != 0)
        return S12_ERR_CORRUPT;
    for (int i = 40; i < 64; ++i)
        if (c[i]) return S12_ERR_CORRUPT;
    const uint64_t rows = rd64(c + 8), cols = rd64(c + 16), n_esc = rd64(c + 32);
    if (rows == 0 || cols == 0 || cols % kTile || rows >= (uint64_t(1) << 32) || cols >= (uint64_t(1) << 32) ||
        rows * cols >= (uint64_t(1) << 32) || n_esc > rows * cols)
        return S12_ERR_CORRUPT;
    const Geometry3 g3 = geometry3(rows, cols, n_esc);
    if (g3.total > v3_bytes) return S12_ERR_CORRUPT;
    const Geometry g = geometry(rows, cols, n_esc);
    *bytes_out = g.total;
    if (!dst) return S12_OK;
    if (dst_cap < g.total) return S12_ERR_CAPACITY;
    uint8_t *d = static_cast<uint8_t *>(dst);
    std::memset(d, 0, g.total);
    std::memcpy(d, c, 64);
    wr32(d + 4, 1);
    const uint8_t *pair = c + g3.off_pair;
    for (uint64_t i = 0; i < rows * cols / 2; ++i) {
        d[g.off_raw + 2 * i] = pair[3 * i];
        d[g.off_raw + 2 * i + 1] = pair[3 * i + 1];
        d[g.off_code + i] = pair[3 * i + 2];
    }
    std::memcpy(d + g.off_base, c + g3.off_base, g.n_tiles);
    std::memcpy(d + g.off_esc_off, c + g3.off_esc_off, 4 * (g.n_tiles + 1));
    std::memcpy(d + g.off_esc, c + g3.off_esc, 2 * n_esc);
    // the result must be a valid version 1 container (offsets, counts, bases)
    s12_report rep;
    const int rc = s12_validate_host(d, g.total, &rep);
    return rc == S12_OK ? S12_OK : S12_ERR_CORRUPT;
}
