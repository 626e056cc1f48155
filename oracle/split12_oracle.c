/*
 * split12_oracle.c -- CPU oracle for the Split12 lossless BF16 weight format.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded,
 * obviously-correct statement of what the GPU library computes.  Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may load
 * it.  It shares no code, header, table or constant with the CUDA library:
 * every layout constant below is restated here from the format definition.
 *
 * Sources (web pages, cited by title and section):
 *   [W]  "Lossless LLM Weight Compression vs 8-bit GGUF: What Is Ready for
 *        Production?" (wavect.io blog; English edition, with Chinese and
 *        German editions of the same article).
 *   [M]  "你的 bf16 模型,有 5 個 bit 是廢的" (meowlab blog, 2026-10-04).
 *   [T]  "GPU 友善 12 位無損 BF16 壓縮格式" (setupai.cc digest of a Reddit
 *        post on a GPU-friendly 12-bit lossless BF16 format, "Turbo-Lossless").
 *
 * What the pages fix, restated:
 *   - A BF16 value is 1 sign bit, 8 exponent bits, 7 mantissa bits
 *     ([M] section 1, bit-field table; [W] "What did the GLM-5.2 experiment
 *     actually prove?").
 *   - Trained weights use a narrow set of exponents; common symbols get short
 *     fixed codes and rare ones go, exactly, to an escape stream ([W] same
 *     section; [M] section 1 entropy table).
 *   - The format is a fixed 12-bit rate, 1.33x smaller than BF16 ([T] key
 *     points), decoded for almost all weights by one integer ADD ([T] key
 *     points), with blocks of 128 weights sharing a base ([T] technical deep
 *     dive) and the escape table in a separate buffer ([T] technical deep dive).
 *   - Lossless means the round trip reproduces every bit ([W] "What does
 *     'lossless' mean for LLM weights?").
 *
 * Where the pages leave the container open, this oracle takes the following
 * readings (the same readings the library documents):
 *   - Each weight w (16 bits) is split into a raw byte
 *         raw = ((w >> 8) & 0x80) | (w & 0x7F)      (sign + 7 mantissa bits)
 *     and a 4-bit exponent code.  With e = (w >> 7) & 0xFF and the tile base b,
 *     code = e - b when b <= e <= b + 14, else code = 15 (escape).
 *   - Tile = 128 consecutive weights of one row along the column (K) axis;
 *     tile t = r * (cols / 128) + j covers w[r][128 j .. 128 j + 127].
 *   - The base b of a tile is the smallest b in [0, 241] that maximises the
 *     number of the tile's exponents inside [b, b + 14].
 *   - The raw byte is stored for every weight, escapes included; escapes
 *     carry the full 16-bit value in the escape stream, in row-major order;
 *     esc_off[t] = number of escapes in tiles before t.
 *   - Two codes per byte, the even-indexed weight in the low nibble.
 *   - Container (all integers little-endian; every part starts at a multiple
 *     of 256 bytes from the start and is zero-padded to one):
 *        header (64 bytes used, padded to 256):
 *          0..3  magic "S12\0"     4..7  u32 version = 1
 *          8..15 u64 rows         16..23 u64 cols
 *          24..27 u32 tile = 128  28..31 u32 flags = 0
 *          32..39 u64 n_esc       40..255 zero
 *        raw     u8 [rows*cols]
 *        code    u8 [rows*cols/2]
 *        base    u8 [n_tiles]
 *        esc_off u32[n_tiles + 1]
 *        esc     u16[n_esc]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_SHAPE (-2)
#define ORACLE_ERR_CAPACITY (-3)
#define ORACLE_ERR_CORRUPT (-4)

#define ORACLE_TILE 128u
#define ORACLE_WINDOW 15u       /* exponents b .. b+14 get codes 0..14 */
#define ORACLE_ESCAPE_CODE 15u
#define ORACLE_MAX_BASE 241u    /* b + 14 <= 255 */
#define ORACLE_ALIGN 256u
#define ORACLE_HEADER_USED 64u

/* ---------------------------------------------------------------------- */
/* little-endian helpers (the oracle does not assume host byte order)     */

static void put_u32(uint8_t *p, uint32_t v) {
    for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_u64(uint8_t *p, uint64_t v) {
    for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get_u32(const uint8_t *p) {
    uint32_t v = 0;
    for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
    return v;
}
static uint64_t get_u64(const uint8_t *p) {
    uint64_t v = 0;
    for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
    return v;
}
static uint16_t get_u16(const uint8_t *p) {
    return (uint16_t)(p[0] | (p[1] << 8));
}


static uint64_t pad_to_align(uint64_t n) {
    return (n + ORACLE_ALIGN - 1) / ORACLE_ALIGN * ORACLE_ALIGN;
}

/* ---------------------------------------------------------------------- */
/* BF16 fields ([M] section 1 bit-field table: 1 sign, 8 exponent, 7 mantissa) */

uint32_t oracle_bf16_sign(uint16_t w) { return (w >> 15) & 1u; }
uint32_t oracle_bf16_exponent(uint16_t w) { return (w >> 7) & 0xFFu; }
uint32_t oracle_bf16_mantissa(uint16_t w) { return w & 0x7Fu; }

/* Exact value of a BF16 pattern: BF16 is the upper half of an IEEE binary32,
 * so widening by 16 zero bits gives the same number, which a double holds
 * exactly (NaN and infinities included). */
double oracle_bf16_to_double(uint16_t w) {
    uint32_t bits = (uint32_t)w << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------------- */
/* Container geometry                                                      */

typedef struct {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_raw, off_code, off_base, off_esc_off, off_esc, total;
} oracle_layout;

static int layout_for(uint64_t rows, uint64_t cols, uint64_t n_esc, oracle_layout *L) {
    if (cols == 0 || cols % ORACLE_TILE != 0) return ORACLE_ERR_SHAPE;
    if (rows == 0) return ORACLE_ERR_SHAPE;
    if (rows > (UINT64_C(1) << 40) / cols) return ORACLE_ERR_SHAPE;
    L->rows = rows;
    L->cols = cols;
    L->n_tiles = rows * (cols / ORACLE_TILE);
    L->n_esc = n_esc;
    L->off_raw = pad_to_align(ORACLE_HEADER_USED);
    L->off_code = L->off_raw + pad_to_align(rows * cols);
    L->off_base = L->off_code + pad_to_align(rows * cols / 2);
    L->off_esc_off = L->off_base + pad_to_align(L->n_tiles);
    L->off_esc = L->off_esc_off + pad_to_align(4 * (L->n_tiles + 1));
    L->total = L->off_esc + pad_to_align(2 * n_esc);
    return ORACLE_OK;
}

/* Closed-form container size for given shape and escape count, or a
 * negative error code. */
int64_t oracle_container_bytes(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    oracle_layout L;
    int rc = layout_for(rows, cols, n_esc, &L);
    if (rc != ORACLE_OK) return rc;
    return (int64_t)L.total;
}

/* ---------------------------------------------------------------------- */
/* Per-tile base selection ([T] technical deep dive: a block of 128 weights
 * shares a base; [W] "What did the GLM-5.2 experiment actually prove?":
 * common exponent symbols get short codes).  The histogram of the tile's
 * exponent fields is taken, every admissible window [b, b+14] is counted,
 * and the smallest b with the largest count wins.  Returns the number of
 * the tile's weights that fall outside the window (its escapes).           */
int oracle_tile_base(const uint16_t *w, uint32_t *base_out, uint32_t *in_window_out) {
    if (!w || !base_out) return ORACLE_ERR_ARG;
    uint32_t hist[256];
    memset(hist, 0, sizeof hist);
    for (uint32_t i = 0; i < ORACLE_TILE; i++) hist[oracle_bf16_exponent(w[i])]++;
    uint32_t best_b = 0, best_count = 0;
    int have = 0;
    for (uint32_t b = 0; b <= ORACLE_MAX_BASE; b++) {
        uint32_t c = 0;
        for (uint32_t e = b; e < b + ORACLE_WINDOW; e++) c += hist[e];
        if (!have || c > best_count) {
            best_count = c;
            best_b = b;
            have = 1;
        }
    }
    *base_out = best_b;
    if (in_window_out) *in_window_out = best_count;
    return (int)(ORACLE_TILE - best_count);
}

/* ---------------------------------------------------------------------- */
/* One tile of the encoder (both container versions): the raw byte and code
 * nibble of every weight at row-major position t * 128 + i, and the escapes
 * appended to the stream at *written.  Returns the tile's escape count. */
static uint32_t pack_tile(const uint16_t *tw, uint32_t b, uint64_t t, uint8_t *raw, uint8_t *code, uint8_t *esc,
                          uint64_t *written) {
    uint32_t count = 0;
    for (uint32_t i = 0; i < ORACLE_TILE; i++) {
        uint64_t pos = t * ORACLE_TILE + i; /* row-major position */
        uint16_t v = tw[i];
        uint32_t e = oracle_bf16_exponent(v);
        uint32_t c;
        raw[pos] = (uint8_t)((oracle_bf16_sign(v) << 7) | oracle_bf16_mantissa(v));
        if (e >= b && e <= b + ORACLE_WINDOW - 1) {
            c = e - b;
        } else {
            c = ORACLE_ESCAPE_CODE;
            esc[2 * *written] = (uint8_t)(v & 0xFF);
            esc[2 * *written + 1] = (uint8_t)(v >> 8);
            (*written)++;
            count++;
        }
        if (pos % 2 == 0)
            code[pos / 2] = (uint8_t)c;               /* low nibble: even index */
        else
            code[pos / 2] |= (uint8_t)(c << 4);       /* high nibble: odd index */
    }
    return count;
}

/* ---------------------------------------------------------------------- */
/* Encoder.  With dst == NULL only *bytes_out is computed.                 */
int oracle_encode(const uint16_t *w, uint64_t rows, uint64_t cols, uint8_t *dst,
                  uint64_t cap, uint64_t *bytes_out) {
    if (!w || !bytes_out) return ORACLE_ERR_ARG;
    oracle_layout L;
    int rc = layout_for(rows, cols, 0, &L);
    if (rc != ORACLE_OK) return rc;

    /* pass 1: count escapes tile by tile */
    uint64_t n_esc = 0;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        uint32_t b;
        n_esc += (uint64_t)oracle_tile_base(w + t * ORACLE_TILE, &b, NULL);
    }
    if (n_esc > 0xFFFFFFFFull) return ORACLE_ERR_SHAPE; /* esc_off is u32 */
    layout_for(rows, cols, n_esc, &L);
    *bytes_out = L.total;
    if (!dst) return ORACLE_OK;
    if (cap < L.total) return ORACLE_ERR_CAPACITY;

    memset(dst, 0, L.total);
    memcpy(dst, "S12\0", 4);
    put_u32(dst + 4, 1);
    put_u64(dst + 8, rows);
    put_u64(dst + 16, cols);
    put_u32(dst + 24, ORACLE_TILE);
    put_u32(dst + 28, 0);
    put_u64(dst + 32, n_esc);

    uint8_t *raw = dst + L.off_raw;
    uint8_t *code = dst + L.off_code;
    uint8_t *base = dst + L.off_base;
    uint8_t *esc_off = dst + L.off_esc_off;
    uint8_t *esc = dst + L.off_esc;

    uint64_t written = 0;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        const uint16_t *tw = w + t * ORACLE_TILE;
        uint32_t b;
        oracle_tile_base(tw, &b, NULL);
        base[t] = (uint8_t)b;
        put_u32(esc_off + 4 * t, (uint32_t)written);
        pack_tile(tw, b, t, raw, code, esc, &written);
    }
    put_u32(esc_off + 4 * L.n_tiles, (uint32_t)written);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Container parsing and validation ([W] "A 14-day production-readiness
 * pilot", step 2: corruption must be detected, not silently decoded).      */
typedef struct {
    oracle_layout L;
    const uint8_t *raw, *code, *base, *esc_off, *esc;
} oracle_view;

static int open_view(const uint8_t *blob, uint64_t bytes, oracle_view *V) {
    if (!blob) return ORACLE_ERR_ARG;
    if (bytes < ORACLE_HEADER_USED) return ORACLE_ERR_CORRUPT;
    if (memcmp(blob, "S12\0", 4) != 0) return ORACLE_ERR_CORRUPT;
    if (get_u32(blob + 4) != 1) return ORACLE_ERR_CORRUPT;
    if (get_u32(blob + 24) != ORACLE_TILE) return ORACLE_ERR_CORRUPT;
    if (get_u32(blob + 28) != 0) return ORACLE_ERR_CORRUPT;
    for (int i = 40; i < 64; i++)
        if (blob[i] != 0) return ORACLE_ERR_CORRUPT;
    uint64_t rows = get_u64(blob + 8), cols = get_u64(blob + 16), n_esc = get_u64(blob + 32);
    if (layout_for(rows, cols, n_esc, &V->L) != ORACLE_OK) return ORACLE_ERR_CORRUPT;
    if (n_esc > rows * cols) return ORACLE_ERR_CORRUPT;
    if (bytes < V->L.total) return ORACLE_ERR_CORRUPT;
    V->raw = blob + V->L.off_raw;
    V->code = blob + V->L.off_code;
    V->base = blob + V->L.off_base;
    V->esc_off = blob + V->L.off_esc_off;
    V->esc = blob + V->L.off_esc;
    if (get_u32(V->esc_off) != 0) return ORACLE_ERR_CORRUPT;
    if (get_u32(V->esc_off + 4 * V->L.n_tiles) != n_esc) return ORACLE_ERR_CORRUPT;
    return ORACLE_OK;
}

static uint32_t code_at(const oracle_view *V, uint64_t pos) {
    uint8_t byte = V->code[pos / 2];
    return (pos % 2 == 0) ? (byte & 0x0Fu) : (uint32_t)(byte >> 4);
}

/* Decode one tile ([T] key points: one integer ADD of code and base gives
 * the exponent; code 15 takes the exact value from the escape stream). */
static int decode_tile(const oracle_view *V, uint64_t t, uint16_t *out) {
    uint32_t b = V->base[t];
    uint32_t lo = get_u32(V->esc_off + 4 * t);
    uint32_t hi = get_u32(V->esc_off + 4 * (t + 1));
    if (hi < lo || hi > V->L.n_esc || b > ORACLE_MAX_BASE) return ORACLE_ERR_CORRUPT;
    uint32_t k = 0; /* escapes seen so far in this tile */
    for (uint32_t i = 0; i < ORACLE_TILE; i++) {
        uint64_t pos = t * ORACLE_TILE + i;
        uint32_t c = code_at(V, pos);
        uint8_t r = V->raw[pos];
        if (c < ORACLE_ESCAPE_CODE) {
            uint32_t e = b + c;
            out[i] = (uint16_t)(((uint32_t)(r & 0x80) << 8) | (e << 7) | (r & 0x7Fu));
        } else {
            if (lo + k >= hi) return ORACLE_ERR_CORRUPT;
            out[i] = get_u16(V->esc + 2 * (uint64_t)(lo + k));
            k++;
        }
    }
    if (lo + k != hi) return ORACLE_ERR_CORRUPT;
    return ORACLE_OK;
}

int oracle_decode(const uint8_t *blob, uint64_t bytes, uint16_t *out) {
    if (!out) return ORACLE_ERR_ARG;
    oracle_view V;
    int rc = open_view(blob, bytes, &V);
    if (rc != ORACLE_OK) return rc;
    for (uint64_t t = 0; t < V.L.n_tiles; t++) {
        rc = decode_tile(&V, t, out + t * ORACLE_TILE);
        if (rc != ORACLE_OK) return rc;
    }
    return ORACLE_OK;
}

/* Decode a list of whole rows; out holds n_rows * cols values. */
int oracle_decode_rows(const uint8_t *blob, uint64_t bytes, const int64_t *row_idx,
                       int64_t n_rows, uint16_t *out) {
    if (!out || !row_idx || n_rows < 0) return ORACLE_ERR_ARG;
    oracle_view V;
    int rc = open_view(blob, bytes, &V);
    if (rc != ORACLE_OK) return rc;
    uint64_t tiles_per_row = V.L.cols / ORACLE_TILE;
    for (int64_t i = 0; i < n_rows; i++) {
        if (row_idx[i] < 0 || (uint64_t)row_idx[i] >= V.L.rows) return ORACLE_ERR_ARG;
        for (uint64_t j = 0; j < tiles_per_row; j++) {
            rc = decode_tile(&V, (uint64_t)row_idx[i] * tiles_per_row + j,
                             out + (uint64_t)i * V.L.cols + j * ORACLE_TILE);
            if (rc != ORACLE_OK) return rc;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Container version 2: a compact tile header.  [W] (English edition,
 * opening summary) reports a 24.967 % payload reduction for the byte split,
 * close to the bare 25 % of a 12-bit rate, which leaves little room for
 * per-tile metadata.  Version 1 spends 5 bytes per tile (u8 base + u32
 * offset, 0.3125 bit per weight); version 2 keeps the raw, code and escape
 * planes byte for byte and replaces the base and offset planes by
 *     tmeta   u16[n_tiles]   base (low byte) | escape count (high byte)
 *     row_esc u32[rows + 1]  escapes in the rows before r; row_esc[rows] = n_esc
 * so a tile's first escape is row_esc[r] plus the counts of the row's earlier
 * tiles: 2 bytes per tile plus 4 per row.  Header as version 1 with
 * version = 2; every plane starts on a 256-byte boundary. */
typedef struct {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_raw, off_code, off_tmeta, off_row_esc, off_esc, total;
} oracle_layout2;

static int layout2_for(uint64_t rows, uint64_t cols, uint64_t n_esc, oracle_layout2 *L) {
    if (cols == 0 || cols % ORACLE_TILE != 0 || rows == 0) return ORACLE_ERR_SHAPE;
    if (rows > (UINT64_C(1) << 40) / cols) return ORACLE_ERR_SHAPE;
    L->rows = rows;
    L->cols = cols;
    L->n_tiles = rows * (cols / ORACLE_TILE);
    L->n_esc = n_esc;
    L->off_raw = pad_to_align(ORACLE_HEADER_USED);
    L->off_code = L->off_raw + pad_to_align(rows * cols);
    L->off_tmeta = L->off_code + pad_to_align(rows * cols / 2);
    L->off_row_esc = L->off_tmeta + pad_to_align(2 * L->n_tiles);
    L->off_esc = L->off_row_esc + pad_to_align(4 * (rows + 1));
    L->total = L->off_esc + pad_to_align(2 * L->n_esc);
    return ORACLE_OK;
}

int64_t oracle_container_bytes_v2(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    oracle_layout2 L;
    int rc = layout2_for(rows, cols, n_esc, &L);
    if (rc != ORACLE_OK) return rc;
    return (int64_t)L.total;
}

/* Encoder, version 2 (same base choice and codes as version 1). */
int oracle_encode_v2(const uint16_t *w, uint64_t rows, uint64_t cols, uint8_t *dst, uint64_t cap,
                     uint64_t *bytes_out) {
    if (!w || !bytes_out) return ORACLE_ERR_ARG;
    oracle_layout2 L;
    int rc = layout2_for(rows, cols, 0, &L);
    if (rc != ORACLE_OK) return rc;
    uint64_t n_esc = 0;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        uint32_t b;
        n_esc += (uint64_t)oracle_tile_base(w + t * ORACLE_TILE, &b, NULL);
    }
    if (n_esc > 0xFFFFFFFFull) return ORACLE_ERR_SHAPE; /* row_esc is u32 */
    layout2_for(rows, cols, n_esc, &L);
    *bytes_out = L.total;
    if (!dst) return ORACLE_OK;
    if (cap < L.total) return ORACLE_ERR_CAPACITY;

    memset(dst, 0, L.total);
    memcpy(dst, "S12\0", 4);
    put_u32(dst + 4, 2);
    put_u64(dst + 8, rows);
    put_u64(dst + 16, cols);
    put_u32(dst + 24, ORACLE_TILE);
    put_u32(dst + 28, 0);
    put_u64(dst + 32, n_esc);
    uint8_t *raw = dst + L.off_raw, *code = dst + L.off_code, *tmeta = dst + L.off_tmeta;
    uint8_t *row_esc = dst + L.off_row_esc, *esc = dst + L.off_esc;
    const uint64_t tiles_per_row = cols / ORACLE_TILE;
    uint64_t written = 0;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        if (t % tiles_per_row == 0) put_u32(row_esc + 4 * (t / tiles_per_row), (uint32_t)written);
        const uint16_t *tw = w + t * ORACLE_TILE;
        uint32_t b;
        oracle_tile_base(tw, &b, NULL);
        const uint32_t count = pack_tile(tw, b, t, raw, code, esc, &written);
        tmeta[2 * t] = (uint8_t)b;
        tmeta[2 * t + 1] = (uint8_t)count; /* at most 128 */
    }
    put_u32(row_esc + 4 * rows, (uint32_t)written);
    return ORACLE_OK;
}

/* Decoder, version 2, with the container checks of version 1 restated for
 * this layout: row offsets start at 0, end at n_esc and never decrease; each
 * row's tile counts add up to its offset span; each tile's code-15 count
 * equals its stored count; bases are at most 241. */
int oracle_decode_v2(const uint8_t *blob, uint64_t bytes, uint16_t *out) {
    if (!blob || !out) return ORACLE_ERR_ARG;
    if (bytes < ORACLE_HEADER_USED || memcmp(blob, "S12\0", 4) != 0) return ORACLE_ERR_CORRUPT;
    if (get_u32(blob + 4) != 2 || get_u32(blob + 24) != ORACLE_TILE || get_u32(blob + 28) != 0)
        return ORACLE_ERR_CORRUPT;
    for (int i = 40; i < 64; i++)
        if (blob[i] != 0) return ORACLE_ERR_CORRUPT;
    uint64_t rows = get_u64(blob + 8), cols = get_u64(blob + 16), n_esc = get_u64(blob + 32);
    oracle_layout2 L;
    if (layout2_for(rows, cols, n_esc, &L) != ORACLE_OK) return ORACLE_ERR_CORRUPT;
    if (n_esc > rows * cols || bytes < L.total) return ORACLE_ERR_CORRUPT;
    const uint8_t *raw = blob + L.off_raw, *code = blob + L.off_code, *tmeta = blob + L.off_tmeta;
    const uint8_t *row_esc = blob + L.off_row_esc, *esc = blob + L.off_esc;
    if (get_u32(row_esc) != 0 || get_u32(row_esc + 4 * rows) != n_esc) return ORACLE_ERR_CORRUPT;
    const uint64_t tiles_per_row = cols / ORACLE_TILE;
    for (uint64_t r = 0; r < rows; r++) {
        uint64_t lo = get_u32(row_esc + 4 * r), hi = get_u32(row_esc + 4 * (r + 1));
        if (hi < lo || hi > n_esc) return ORACLE_ERR_CORRUPT;
        uint64_t k = lo; /* next escape of this row */
        for (uint64_t j = 0; j < tiles_per_row; j++) {
            uint64_t t = r * tiles_per_row + j;
            uint32_t b = tmeta[2 * t], count = tmeta[2 * t + 1], seen = 0;
            if (b > ORACLE_MAX_BASE || count > ORACLE_TILE) return ORACLE_ERR_CORRUPT;
            for (uint32_t i = 0; i < ORACLE_TILE; i++) {
                uint64_t pos = t * ORACLE_TILE + i;
                uint32_t c = (pos % 2 == 0) ? (code[pos / 2] & 0x0Fu) : (uint32_t)(code[pos / 2] >> 4);
                uint8_t rb = raw[pos];
                if (c < ORACLE_ESCAPE_CODE) {
                    out[pos] = (uint16_t)(((uint32_t)(rb & 0x80) << 8) | ((b + c) << 7) | (rb & 0x7Fu));
                } else {
                    if (k >= hi) return ORACLE_ERR_CORRUPT;
                    out[pos] = get_u16(esc + 2 * k);
                    k++;
                    seen++;
                }
            }
            if (seen != count) return ORACLE_ERR_CORRUPT;
        }
        if (k != hi) return ORACLE_ERR_CORRUPT;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Container version 3: packed 24-bit pairs.  [T] technical deep dive says
 * the 12-bit representation is packed into 3-byte words, two weights per
 * word.  Reading (the plainest one with the 12-bit split above): weights
 * 2i and 2i+1 (row-major, always in the same tile) form pair i, stored as
 * three consecutive bytes
 *     byte 3i     raw(w[2i])
 *     byte 3i+1   raw(w[2i+1])
 *     byte 3i+2   code(w[2i]) | code(w[2i+1]) << 4
 * in one pair plane u8[rows*cols*3/2] that takes the place of the raw and
 * code planes.  Base choice, codes, escapes, the base and esc_off planes and
 * the header (version = 3) are those of version 1; every plane starts on a
 * 256-byte boundary. */
typedef struct {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_pair, off_base, off_esc_off, off_esc, total;
} oracle_layout3;

static int layout3_for(uint64_t rows, uint64_t cols, uint64_t n_esc, oracle_layout3 *L) {
    if (cols == 0 || cols % ORACLE_TILE != 0 || rows == 0) return ORACLE_ERR_SHAPE;
    if (rows > (UINT64_C(1) << 40) / cols) return ORACLE_ERR_SHAPE;
    L->rows = rows;
    L->cols = cols;
    L->n_tiles = rows * (cols / ORACLE_TILE);
    L->n_esc = n_esc;
    L->off_pair = pad_to_align(ORACLE_HEADER_USED);
    L->off_base = L->off_pair + pad_to_align(rows * cols / 2 * 3);
    L->off_esc_off = L->off_base + pad_to_align(L->n_tiles);
    L->off_esc = L->off_esc_off + pad_to_align(4 * (L->n_tiles + 1));
    L->total = L->off_esc + pad_to_align(2 * L->n_esc);
    return ORACLE_OK;
}

int64_t oracle_container_bytes_v3(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    oracle_layout3 L;
    int rc = layout3_for(rows, cols, n_esc, &L);
    if (rc != ORACLE_OK) return rc;
    return (int64_t)L.total;
}

/* Encoder, version 3. */
int oracle_encode_v3(const uint16_t *w, uint64_t rows, uint64_t cols, uint8_t *dst, uint64_t cap,
                     uint64_t *bytes_out) {
    if (!w || !bytes_out) return ORACLE_ERR_ARG;
    oracle_layout3 L;
    int rc = layout3_for(rows, cols, 0, &L);
    if (rc != ORACLE_OK) return rc;
    uint64_t n_esc = 0;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        uint32_t b;
        n_esc += (uint64_t)oracle_tile_base(w + t * ORACLE_TILE, &b, NULL);
    }
    if (n_esc > 0xFFFFFFFFull) return ORACLE_ERR_SHAPE; /* esc_off is u32 */
    layout3_for(rows, cols, n_esc, &L);
    *bytes_out = L.total;
    if (!dst) return ORACLE_OK;
    if (cap < L.total) return ORACLE_ERR_CAPACITY;

    memset(dst, 0, L.total);
    memcpy(dst, "S12\0", 4);
    put_u32(dst + 4, 3);
    put_u64(dst + 8, rows);
    put_u64(dst + 16, cols);
    put_u32(dst + 24, ORACLE_TILE);
    put_u32(dst + 28, 0);
    put_u64(dst + 32, n_esc);
    uint8_t *pair = dst + L.off_pair, *base = dst + L.off_base, *off = dst + L.off_esc_off, *esc = dst + L.off_esc;
    uint64_t written = 0;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        const uint16_t *tw = w + t * ORACLE_TILE;
        uint32_t b;
        oracle_tile_base(tw, &b, NULL);
        base[t] = (uint8_t)b;
        put_u32(off + 4 * t, (uint32_t)written);
        /* the tile's raw bytes and codes as version 1 lays them out, then
         * regrouped into 3-byte pairs */
        uint8_t raw_t[ORACLE_TILE], code_t[ORACLE_TILE / 2];
        pack_tile(tw, b, 0, raw_t, code_t, esc, &written);
        uint8_t *pt = pair + 3 * (t * ORACLE_TILE / 2);
        for (uint32_t i = 0; i < ORACLE_TILE / 2; i++) {
            pt[3 * i] = raw_t[2 * i];
            pt[3 * i + 1] = raw_t[2 * i + 1];
            pt[3 * i + 2] = code_t[i];
        }
    }
    put_u32(off + 4 * L.n_tiles, (uint32_t)written);
    return ORACLE_OK;
}

/* Decoder, version 3, with the checks of version 1: offsets start at 0,
 * end at n_esc and never decrease; each tile's code-15 count equals its
 * offset span; bases are at most 241. */
int oracle_decode_v3(const uint8_t *blob, uint64_t bytes, uint16_t *out) {
    if (!blob || !out) return ORACLE_ERR_ARG;
    if (bytes < ORACLE_HEADER_USED || memcmp(blob, "S12\0", 4) != 0) return ORACLE_ERR_CORRUPT;
    if (get_u32(blob + 4) != 3 || get_u32(blob + 24) != ORACLE_TILE || get_u32(blob + 28) != 0)
        return ORACLE_ERR_CORRUPT;
    for (int i = 40; i < 64; i++)
        if (blob[i] != 0) return ORACLE_ERR_CORRUPT;
    uint64_t rows = get_u64(blob + 8), cols = get_u64(blob + 16), n_esc = get_u64(blob + 32);
    oracle_layout3 L;
    if (layout3_for(rows, cols, n_esc, &L) != ORACLE_OK) return ORACLE_ERR_CORRUPT;
    if (n_esc > rows * cols || bytes < L.total) return ORACLE_ERR_CORRUPT;
    const uint8_t *pair = blob + L.off_pair, *base = blob + L.off_base, *off = blob + L.off_esc_off;
    const uint8_t *esc = blob + L.off_esc;
    if (get_u32(off) != 0 || get_u32(off + 4 * L.n_tiles) != n_esc) return ORACLE_ERR_CORRUPT;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        const uint64_t lo = get_u32(off + 4 * t), hi = get_u32(off + 4 * (t + 1));
        const uint32_t b = base[t];
        if (hi < lo || hi > n_esc || b > ORACLE_MAX_BASE) return ORACLE_ERR_CORRUPT;
        uint64_t k = lo;
        for (uint32_t i = 0; i < ORACLE_TILE; i++) {
            const uint64_t pos = t * ORACLE_TILE + i, p = pos / 2;
            const uint8_t rb = pair[3 * p + (pos % 2)];
            const uint32_t c = (pos % 2 == 0) ? (pair[3 * p + 2] & 0x0Fu) : (uint32_t)(pair[3 * p + 2] >> 4);
            if (c < ORACLE_ESCAPE_CODE) {
                out[pos] = (uint16_t)(((uint32_t)(rb & 0x80) << 8) | ((b + c) << 7) | (rb & 0x7Fu));
            } else {
                if (k >= hi) return ORACLE_ERR_CORRUPT;
                out[pos] = get_u16(esc + 2 * k);
                k++;
            }
        }
        if (k != hi) return ORACLE_ERR_CORRUPT;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Container version 4: sign-and-exponent symbol codes.  [W] "What did the
 * GLM-5.2 experiment actually prove?" describes short fixed codes for the
 * common sign-and-exponent symbols of a tensor, with rare symbols sent
 * through an escape stream.  Reading (the plainest one that keeps a 12-bit
 * rate beside the 7 mantissa bits): the symbol of w is its top 9 bits,
 * s = w >> 7 (sign and exponent); the tensor's table holds its 31 most
 * frequent symbols (count descending, ties to the smaller symbol; unused
 * entries 0xFFFF); code = the symbol's index in the table, or 31 (escape).
 * The 5-bit code and the mantissa are split like version 1's fields:
 *     raw byte = (code & 1) << 7 | mantissa          (u8 per weight)
 *     nibble   = code >> 1                           (two per byte, low first)
 * so w = table[code] << 7 | (raw & 0x7F) for code < 31.  Escapes, their
 * row-major order and the per-tile offsets are those of version 1 (tile =
 * 128 weights of a row).  Container: header (version = 4), then
 *     table   u16[32]        the 31 symbols and one zero entry
 *     raw     u8 [rows*cols]
 *     code    u8 [rows*cols/2]
 *     esc_off u32[n_tiles + 1]
 *     esc     u16[n_esc]
 * each part on a 256-byte boundary. */
#define ORACLE_SYM_CODES 31u
#define ORACLE_SYM_ESCAPE 31u
#define ORACLE_SYM_UNUSED 0xFFFFu

typedef struct {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t off_table, off_raw, off_code, off_esc_off, off_esc, total;
} oracle_layout4;

static int layout4_for(uint64_t rows, uint64_t cols, uint64_t n_esc, oracle_layout4 *L) {
    if (cols == 0 || cols % ORACLE_TILE != 0 || rows == 0) return ORACLE_ERR_SHAPE;
    if (rows > (UINT64_C(1) << 40) / cols) return ORACLE_ERR_SHAPE;
    L->rows = rows;
    L->cols = cols;
    L->n_tiles = rows * (cols / ORACLE_TILE);
    L->n_esc = n_esc;
    L->off_table = pad_to_align(ORACLE_HEADER_USED);
    L->off_raw = L->off_table + pad_to_align(2 * 32);
    L->off_code = L->off_raw + pad_to_align(rows * cols);
    L->off_esc_off = L->off_code + pad_to_align(rows * cols / 2);
    L->off_esc = L->off_esc_off + pad_to_align(4 * (L->n_tiles + 1));
    L->total = L->off_esc + pad_to_align(2 * L->n_esc);
    return ORACLE_OK;
}

int64_t oracle_container_bytes_v4(uint64_t rows, uint64_t cols, uint64_t n_esc) {
    oracle_layout4 L;
    int rc = layout4_for(rows, cols, n_esc, &L);
    if (rc != ORACLE_OK) return rc;
    return (int64_t)L.total;
}

/* The symbol table of a tensor: its 31 most frequent symbols, count
 * descending, ties to the smaller symbol; table[i] = 0xFFFF past the number
 * of distinct symbols.  Returns the number of weights outside the table. */
uint64_t oracle_symbol_table(const uint16_t *w, uint64_t n, uint16_t table[32]) {
    uint64_t count[512];
    memset(count, 0, sizeof count);
    for (uint64_t i = 0; i < n; i++) count[w[i] >> 7]++;
    uint8_t taken[512];
    memset(taken, 0, sizeof taken);
    uint64_t covered = 0;
    for (uint32_t k = 0; k < 32; k++) table[k] = ORACLE_SYM_UNUSED;
    for (uint32_t k = 0; k < ORACLE_SYM_CODES; k++) {
        int best = -1;
        for (int s = 0; s < 512; s++) {
            if (taken[s] || count[s] == 0) continue;
            if (best < 0 || count[s] > count[best]) best = s; /* strictly more: ties keep the smaller */
        }
        if (best < 0) break;
        taken[best] = 1;
        table[k] = (uint16_t)best;
        covered += count[best];
    }
    table[31] = 0;
    return n - covered;
}

static uint32_t symbol_code(const uint16_t table[32], uint16_t w) {
    const uint16_t s = (uint16_t)(w >> 7);
    for (uint32_t k = 0; k < ORACLE_SYM_CODES; k++)
        if (table[k] == s) return k;
    return ORACLE_SYM_ESCAPE;
}

/* Encoder, version 4. */
int oracle_encode_v4(const uint16_t *w, uint64_t rows, uint64_t cols, uint8_t *dst, uint64_t cap,
                     uint64_t *bytes_out) {
    if (!w || !bytes_out) return ORACLE_ERR_ARG;
    oracle_layout4 L;
    int rc = layout4_for(rows, cols, 0, &L);
    if (rc != ORACLE_OK) return rc;
    uint16_t table[32];
    const uint64_t n_esc = oracle_symbol_table(w, rows * cols, table);
    if (n_esc > 0xFFFFFFFFull) return ORACLE_ERR_SHAPE; /* esc_off is u32 */
    layout4_for(rows, cols, n_esc, &L);
    *bytes_out = L.total;
    if (!dst) return ORACLE_OK;
    if (cap < L.total) return ORACLE_ERR_CAPACITY;

    memset(dst, 0, L.total);
    memcpy(dst, "S12\0", 4);
    put_u32(dst + 4, 4);
    put_u64(dst + 8, rows);
    put_u64(dst + 16, cols);
    put_u32(dst + 24, ORACLE_TILE);
    put_u32(dst + 28, 0);
    put_u64(dst + 32, n_esc);
    uint8_t *tab = dst + L.off_table, *raw = dst + L.off_raw, *code = dst + L.off_code;
    uint8_t *off = dst + L.off_esc_off, *esc = dst + L.off_esc;
    for (uint32_t k = 0; k < 32; k++) {
        tab[2 * k] = (uint8_t)(table[k] & 0xFF);
        tab[2 * k + 1] = (uint8_t)(table[k] >> 8);
    }
    uint64_t written = 0;
    for (uint64_t pos = 0; pos < rows * cols; pos++) {
        if (pos % ORACLE_TILE == 0) put_u32(off + 4 * (pos / ORACLE_TILE), (uint32_t)written);
        const uint16_t v = w[pos];
        const uint32_t c = symbol_code(table, v);
        raw[pos] = (uint8_t)(((c & 1u) << 7) | oracle_bf16_mantissa(v));
        const uint32_t nib = c >> 1;
        if (pos % 2 == 0)
            code[pos / 2] = (uint8_t)nib;
        else
            code[pos / 2] |= (uint8_t)(nib << 4);
        if (c == ORACLE_SYM_ESCAPE) {
            esc[2 * written] = (uint8_t)(v & 0xFF);
            esc[2 * written + 1] = (uint8_t)(v >> 8);
            written++;
        }
    }
    put_u32(off + 4 * L.n_tiles, (uint32_t)written);
    return ORACLE_OK;
}

/* Decoder, version 4, with the checks: the table's used entries are valid
 * 9-bit symbols, no code points at an unused entry, offsets start at 0, end
 * at n_esc and never decrease, and each tile's escape count equals its
 * offset span. */
int oracle_decode_v4(const uint8_t *blob, uint64_t bytes, uint16_t *out) {
    if (!blob || !out) return ORACLE_ERR_ARG;
    if (bytes < ORACLE_HEADER_USED || memcmp(blob, "S12\0", 4) != 0) return ORACLE_ERR_CORRUPT;
    if (get_u32(blob + 4) != 4 || get_u32(blob + 24) != ORACLE_TILE || get_u32(blob + 28) != 0)
        return ORACLE_ERR_CORRUPT;
    for (int i = 40; i < 64; i++)
        if (blob[i] != 0) return ORACLE_ERR_CORRUPT;
    uint64_t rows = get_u64(blob + 8), cols = get_u64(blob + 16), n_esc = get_u64(blob + 32);
    oracle_layout4 L;
    if (layout4_for(rows, cols, n_esc, &L) != ORACLE_OK) return ORACLE_ERR_CORRUPT;
    if (n_esc > rows * cols || bytes < L.total) return ORACLE_ERR_CORRUPT;
    const uint8_t *tab = blob + L.off_table, *raw = blob + L.off_raw, *code = blob + L.off_code;
    const uint8_t *off = blob + L.off_esc_off, *esc = blob + L.off_esc;
    uint16_t table[32];
    for (uint32_t k = 0; k < 32; k++) table[k] = get_u16(tab + 2 * k);
    for (uint32_t k = 0; k < ORACLE_SYM_CODES; k++)
        if (table[k] != ORACLE_SYM_UNUSED && table[k] > 511) return ORACLE_ERR_CORRUPT;
    if (get_u32(off) != 0 || get_u32(off + 4 * L.n_tiles) != n_esc) return ORACLE_ERR_CORRUPT;
    for (uint64_t t = 0; t < L.n_tiles; t++) {
        const uint64_t lo = get_u32(off + 4 * t), hi = get_u32(off + 4 * (t + 1));
        if (hi < lo || hi > n_esc) return ORACLE_ERR_CORRUPT;
        uint64_t k = lo;
        for (uint32_t i = 0; i < ORACLE_TILE; i++) {
            const uint64_t pos = t * ORACLE_TILE + i;
            const uint32_t nib = (pos % 2 == 0) ? (code[pos / 2] & 0x0Fu) : (uint32_t)(code[pos / 2] >> 4);
            const uint32_t c = (nib << 1) | (uint32_t)(raw[pos] >> 7);
            if (c < ORACLE_SYM_CODES) {
                if (table[c] == ORACLE_SYM_UNUSED) return ORACLE_ERR_CORRUPT;
                out[pos] = (uint16_t)(((uint32_t)table[c] << 7) | (raw[pos] & 0x7Fu));
            } else {
                if (k >= hi) return ORACLE_ERR_CORRUPT;
                out[pos] = get_u16(esc + 2 * k);
                k++;
            }
        }
        if (k != hi) return ORACLE_ERR_CORRUPT;
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Dense product in FP64: y[m][n] = sum_k W[n][k] * x[m][k], and the
 * tolerance scale s[m][n] = sum_k |W[n][k] * x[m][k]|.  Every BF16 operand
 * converts exactly; the product of two BF16 values is exact in FP64.  This
 * is the plain definition of the matrix product that [W] "What does
 * 'lossless' mean for LLM weights?" says the decoded weights feed. */
int oracle_matmul_f64(const uint16_t *w, uint64_t rows, uint64_t cols, const uint16_t *x,
                      int64_t m, double *y, double *s) {
    if (!w || !x || !y || m <= 0) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < m; i++) {
        for (uint64_t n = 0; n < rows; n++) {
            double acc = 0.0, mag = 0.0;
            for (uint64_t k = 0; k < cols; k++) {
                double p = oracle_bf16_to_double(w[n * cols + k]) *
                           oracle_bf16_to_double(x[(uint64_t)i * cols + k]);
                acc += p;
                mag += fabs(p);
            }
            y[(uint64_t)i * rows + n] = acc;
            if (s) s[(uint64_t)i * rows + n] = mag;
        }
    }
    return ORACLE_OK;
}

/* Fused-path reference: decode the container, then the dense FP64 product.
 * y and s are m x rows, row-major. */
int oracle_gemv_f64(const uint8_t *blob, uint64_t bytes, const uint16_t *x, int64_t m,
                    double *y, double *s) {
    oracle_view V;
    int rc = open_view(blob, bytes, &V);
    if (rc != ORACLE_OK) return rc;
    uint16_t *w = (uint16_t *)malloc(sizeof(uint16_t) * V.L.rows * V.L.cols);
    if (!w) return ORACLE_ERR_CAPACITY;
    rc = oracle_decode(blob, bytes, w);
    if (rc == ORACLE_OK) rc = oracle_matmul_f64(w, V.L.rows, V.L.cols, x, m, y, s);
    free(w);
    return rc;
}

/* Same as oracle_gemv_f64 for a sample of output rows: y and s are
 * m x n_rows, column i belonging to row_idx[i]. */
int oracle_gemv_rows_f64(const uint8_t *blob, uint64_t bytes, const uint16_t *x, int64_t m,
                         const int64_t *row_idx, int64_t n_rows, double *y, double *s) {
    oracle_view V;
    int rc = open_view(blob, bytes, &V);
    if (rc != ORACLE_OK) return rc;
    uint16_t *w = (uint16_t *)malloc(sizeof(uint16_t) * (uint64_t)n_rows * V.L.cols);
    if (!w) return ORACLE_ERR_CAPACITY;
    rc = oracle_decode_rows(blob, bytes, row_idx, n_rows, w);
    if (rc == ORACLE_OK) rc = oracle_matmul_f64(w, (uint64_t)n_rows, V.L.cols, x, m, y, s);
    free(w);
    return rc;
}

/* Gated-MLP activation for the SwiGLU epilogue of the fused GEMV: with
 * g = W_gate x and u = W_up x computed as above (in FP64),
 *     h = silu(g) * u,   silu(t) = t / (1 + exp(-t)),
 * elementwise over n values.  The pages name fused epilogues for decode
 * kernels but not an activation; this is the standard gated-MLP form. */
int oracle_silu_mul_f64(const double *g, const double *u, int64_t n, double *h) {
    if (!g || !u || !h || n < 0) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; i++) h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------- */
/* Statistics ([M] section 1: exponent and mantissa entropy of BF16 weights;
 * [T] key points: 12-bit rate, escape rate).                               */
typedef struct {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t container_bytes, payload_bytes, header_bytes, escape_bytes;
    double escape_rate;          /* n_esc / (rows * cols) */
    double bits_per_weight;      /* 8 * container_bytes / (rows * cols) */
    double ratio_vs_bf16;        /* container_bytes / (2 * rows * cols) */
    double payload_ratio;        /* payload_bytes / (2 * rows * cols) = 0.75 */
    double exp_entropy_bits;     /* Shannon entropy of the exponent field */
    uint64_t exp_hist[256];      /* histogram of decoded exponent fields */
} oracle_stats_t;

int oracle_stats(const uint8_t *blob, uint64_t bytes, oracle_stats_t *out) {
    if (!out) return ORACLE_ERR_ARG;
    oracle_view V;
    int rc = open_view(blob, bytes, &V);
    if (rc != ORACLE_OK) return rc;
    memset(out, 0, sizeof *out);
    uint64_t nw = V.L.rows * V.L.cols;
    uint16_t tile[ORACLE_TILE];
    for (uint64_t t = 0; t < V.L.n_tiles; t++) {
        rc = decode_tile(&V, t, tile);
        if (rc != ORACLE_OK) return rc;
        for (uint32_t i = 0; i < ORACLE_TILE; i++) out->exp_hist[oracle_bf16_exponent(tile[i])]++;
    }
    out->rows = V.L.rows;
    out->cols = V.L.cols;
    out->n_tiles = V.L.n_tiles;
    out->n_esc = V.L.n_esc;
    out->container_bytes = V.L.total;
    out->payload_bytes = nw + nw / 2;
    out->header_bytes = V.L.n_tiles * 5;
    out->escape_bytes = 2 * V.L.n_esc;
    out->escape_rate = (double)V.L.n_esc / (double)nw;
    out->bits_per_weight = 8.0 * (double)V.L.total / (double)nw;
    out->ratio_vs_bf16 = (double)V.L.total / (2.0 * (double)nw);
    out->payload_ratio = (double)out->payload_bytes / (2.0 * (double)nw);
    double h = 0.0;
    for (int e = 0; e < 256; e++) {
        if (out->exp_hist[e] == 0) continue;
        double p = (double)out->exp_hist[e] / (double)nw;
        h -= p * log2(p);
    }
    out->exp_entropy_bits = h;
    return ORACLE_OK;
}
