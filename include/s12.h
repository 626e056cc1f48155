/*
 * s12.h -- C ABI of the Split12 library (libs12.so): lossless 12-bit BF16
 * weights decoded on the GPU and fused into the matrix-vector and skinny
 * matrix products of LLM decoding.  Built for NVIDIA B200 (sm_100a) only.
 *
 * Sources (web pages, cited by title and section):
 *   [W] "Lossless LLM Weight Compression vs 8-bit GGUF: What Is Ready for
 *       Production?" (wavect.io blog, with its Chinese and German editions).
 *   [M] "你的 bf16 模型,有 5 個 bit 是廢的" (meowlab blog, 2026-10-04).
 *   [T] "GPU 友善 12 位無損 BF16 壓縮格式" (setupai.cc digest of a Reddit post
 *       on a GPU-friendly 12-bit lossless BF16 format).
 *
 * FORMAT ("Split12 container").  A BF16 weight has 1 sign, 8 exponent and 7
 * mantissa bits ([M] section 1 table).  Trained weights use few exponents,
 * so common exponents get short fixed codes and rare ones go to an exact
 * escape stream ([W] "What did the GLM-5.2 experiment actually prove?").
 * Here each weight w becomes
 *     raw  = ((w >> 8) & 0x80) | (w & 0x7F)      one byte: sign + mantissa
 *     code = e - base  (0..14)  or 15 (escape)   one nibble, e = (w>>7)&0xFF
 * for a base shared by a tile of 128 weights along a row ([T] technical deep
 * dive: blocks of 128 weights share a base), chosen as the smallest base in
 * [0, 241] whose window [base, base+14] holds the most of the tile's
 * exponents.  Decoding is one integer ADD, exponent = base + code ([T] key
 * points).  Escaped weights are stored whole in a separate stream ([T]
 * technical deep dive), in row-major order, located through per-tile prefix
 * offsets.  That is 12 bits per weight plus 5 header bytes per tile and 2
 * bytes per escape ([T] key points: fixed 12-bit rate, 1.33x smaller).
 *
 * Container bytes (little-endian; every part starts at a multiple of 256
 * bytes from the start and is zero-padded to a multiple of 256 bytes):
 *     header  64 bytes used: "S12\0", u32 version=1, u64 rows, u64 cols,
 *             u32 tile=128, u32 flags=0, u64 n_esc, zeros
 *     raw     u8 [rows*cols]          row-major
 *     code    u8 [rows*cols/2]        even weight in the low nibble
 *     base    u8 [n_tiles]            tile t = r*(cols/128) + j covers
 *                                     w[r][128j .. 128j+127]
 *     esc_off u32[n_tiles+1]          escapes before tile t; last = n_esc
 *     esc     u16[n_esc]              escaped BF16 values
 *
 * CONVENTIONS
 *   - Every call returns an s12 status (0 = S12_OK).
 *   - Pointers marked "device" are CUDA device pointers on the current
 *     device; the caller allocates and owns all of them.  The library never
 *     allocates or frees device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernel calls are enqueued on it and return at once, except
 *     where a call says it synchronises.
 *   - Device pointers must be 16-byte aligned unless stated otherwise.
 *   - `err_flag` (device, u32, nullable): kernels that read a container
 *     OR into it S12_FLAG_* bits when they meet corrupt data.  They never
 *     trap or hang: the offending escape index is clamped and work goes on.
 *     The caller reads the word back (and clears it) when it wants to.
 *   - Global state: per-device caches filled once and then only read (the
 *     SM count, the tensor-map encoder's entry point, the static workspace's
 *     device address) and ONE mutable object, the static workspace of
 *     s12_gemv_noalloc (documented there).  Every other call keeps no
 *     state between calls, and all calls are thread-safe.
 *   - Citations: every entry point names the page and section it follows,
 *     in a "Follows:" line, or says that the pages have no counterpart.
 */
#ifndef S12_H
#define S12_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define S12_OK 0
#define S12_ERR_ARG 1      /* null pointer or negative / zero size           */
#define S12_ERR_SHAPE 2    /* cols % 128 != 0, batch out of range, too large */
#define S12_ERR_ALIGN 3    /* a device pointer is not 16-byte aligned        */
#define S12_ERR_CAPACITY 4 /* destination or workspace too small             */
#define S12_ERR_CORRUPT 5  /* container header or offsets inconsistent       */
#define S12_ERR_CUDA 6     /* a CUDA runtime call failed                     */
#define S12_ERR_DEVICE 7   /* current device is not compute capability 10.0  */

/* ---- err_flag bits set by kernels ---- */
#define S12_FLAG_ESC_COUNT 1u   /* a tile's code-15 count != its esc_off span */
#define S12_FLAG_ESC_RANGE 2u   /* esc_off points outside the escape stream   */
#define S12_FLAG_BASE 4u        /* a tile base above 241 (version 4: a code
                                   of an unused symbol-table entry)           */
#define S12_FLAG_TIMEOUT 8u     /* a bounded wait inside a kernel gave up     */

#define S12_TILE 128
#define S12_GEMV_MAX_BATCH 8
#define S12_GEMV_MAX_PROBLEMS 8 /* matrices in one s12_gemv_multi call */
#define S12_GEMM_MIN_M 16
#define S12_GEMM_MAX_M 256
#define S12_GEMM_MAX_PROBLEMS 16 /* matrices per s12_gemm_skinny_multi call */

/* Host-side description of an opened container.  All pointers are device
 * pointers into the caller's container buffer.  A version 1 container has
 * `base` and `esc_off` (and NULL tmeta/row_esc); a version 2 container (the
 * compact tile header of s12_to_v2_host) has `tmeta` and `row_esc` (and NULL
 * base/esc_off).  A version 3 container (packed 24-bit pairs, [T] technical
 * deep dive: weights 2i and 2i+1 stored as raw(2i), raw(2i+1),
 * code(2i) | code(2i+1) << 4 in one pair plane of rows*cols*3/2 bytes, then
 * version 1's base, esc_off and esc planes) has `raw` pointing at the pair
 * plane, NULL `code`, and `base`/`esc_off` as version 1.  A version 4
 * container (sign-and-exponent symbol codes, [W] "What did the GLM-5.2
 * experiment actually prove?": the tensor's 31 most frequent sign+exponent
 * symbols, w >> 7, in a table; code = the index or 31 for an escape;
 * raw = (code & 1) << 7 | mantissa; nibble = code >> 1) has `symtab`, `raw`,
 * `code` and `esc_off` (tile offsets as version 1) and NULL base.  Decode and
 * stats read all four versions; the fused GEMV and GEMM read versions 1 and
 * 2 (S12_ERR_ARG otherwise). */
typedef struct s12_view {
    uint64_t rows;            /* output features (N)                      */
    uint64_t cols;            /* input features (K), multiple of 128      */
    uint64_t n_tiles;         /* rows * cols / 128                        */
    uint64_t n_esc;           /* escaped weights                          */
    uint64_t container_bytes; /* total size, multiple of 256              */
    const void *container;    /* start of the container                   */
    const uint8_t *raw;       /* u8 [rows*cols] (v3: pairs, rows*cols*3/2) */
    const uint8_t *code;      /* u8 [rows*cols/2] (v3: NULL)              */
    const uint8_t *base;      /* version 1: u8 [n_tiles]                  */
    const uint32_t *esc_off;  /* version 1: u32[n_tiles+1]                */
    const uint16_t *esc;      /* u16[n_esc]                               */
    uint32_t version;         /* 1 .. 4                                   */
    uint32_t reserved;        /* 0                                        */
    const uint16_t *tmeta;    /* version 2: u16[n_tiles], base | count<<8 */
    const uint32_t *row_esc;  /* version 2: u32[rows+1], escapes before r */
    const uint16_t *symtab;   /* version 4: u16[32], the symbol table     */
} s12_view;

typedef struct s12_stats_t {
    uint64_t rows, cols, n_tiles, n_esc;
    uint64_t container_bytes; /* everything, padding included            */
    uint64_t payload_bytes;   /* raw + code = 1.5 bytes per weight       */
    uint64_t header_bytes;    /* v1, v3: 5 per tile; v2: 2 per tile + 4 per row; v4: 4 per tile + 68 */
    uint64_t escape_bytes;    /* 2 bytes per escape                      */
    double escape_rate;       /* n_esc / (rows*cols)                     */
    double bits_per_weight;   /* 8 * container_bytes / (rows*cols)       */
    double ratio_vs_bf16;     /* container_bytes / (2*rows*cols)         */
    double payload_ratio;     /* payload_bytes / (2*rows*cols) = 0.75    */
    double exp_entropy_bits;  /* Shannon entropy of the exponent field   */
    uint64_t exp_hist[256];   /* histogram of decoded exponent fields    */
} s12_stats_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *s12_error_string(int status);

/* S12_OK when the current device is a B200-class part (compute capability
 * 10.0, sm_100a code in this library), S12_ERR_DEVICE otherwise. */
int s12_device_check(void);

/* Container size in bytes for a shape and escape count (closed form of the
 * layout above); 0 when the shape is invalid (cols % 128 != 0 or zero).
 * Follows: [T] key points (a fixed 12-bit rate: 1.5 bytes per weight, plus
 * the tile headers and escapes of this container). */
uint64_t s12_container_bytes(int64_t rows, int64_t cols, uint64_t n_esc);

/* ---- encoder ([W] "What did the GLM-5.2 experiment actually prove?":
 * short codes for common exponents, rare ones to an exact escape stream;
 * [T] technical deep dive: 128-weight blocks with a shared base) ---- */

/* Workspace bytes s12_encode needs for this shape (device scratch, any
 * content, 16-byte aligned, owned by the caller). */
size_t s12_encode_ws_bytes(int64_t rows, int64_t cols);

/* Follows: [W] "What did the GLM-5.2 experiment actually prove?" (short
 * fixed codes, an exact escape stream); [T] technical deep dive (128-weight
 * blocks sharing a base).
 * Encode a row-major BF16 matrix `w` (device, rows x cols, cols % 128 == 0,
 * rows*cols < 2^32) into a Split12 container.
 *   dst == NULL: only computes *bytes_out (the exact container size).
 *   dst != NULL: writes the whole container (header, planes, zero padding)
 *                to dst (device, dst_cap bytes); S12_ERR_CAPACITY when
 *                dst_cap < the size, with *bytes_out set to the size.
 * Both forms run the per-tile histogram/window and escape-count kernels and
 * then SYNCHRONISE `stream` once to read the escape total; the packing
 * kernels of the second form are then enqueued asynchronously.  A caller
 * that sizes dst for an escape count it expects (s12_container_bytes) gets
 * the container from one call, reading W twice in all; the size query is
 * only needed when that guess fails.
 * The result is byte-for-byte the same container on every call. */
int s12_encode(const uint16_t *w, int64_t rows, int64_t cols, void *dst, size_t dst_cap,
               size_t *bytes_out, void *ws, size_t ws_bytes, void *stream);

/* Follows: the container layout above, which restates [M] section 1 (the
 * BF16 bit fields) and [T] key points (tile base, escape stream).
 * Validate the 64-byte header of a container (device, `bytes` long, version
 * 1 to 4) and fill *out with its shape, version and plane pointers.  Copies
 * the header to the host and so SYNCHRONISES (the legacy default stream).
 * S12_ERR_CORRUPT on a bad magic, version, tile size, flags, shape or a size
 * above `bytes`. */
int s12_open(const void *container, size_t bytes, s12_view *out);

/* ---- standalone decode ([T] key points: one integer ADD per weight,
 * code 15 read from the escape stream) ---- */

/* Follows: [T] key points (exponent = base + code, one integer ADD; code
 * 15 read from the separate escape stream); [W] "What does 'lossless' mean
 * for LLM weights?" (the exact round trip is the definition).
 * Decode the whole container to BF16 `out` (device, rows x cols, row-major).
 * Bit-exact: out equals the encoded matrix. */
int s12_decode(const s12_view *v, uint16_t *out, uint32_t *err_flag, void *stream);

/* ---- fused decode-GEMV ([W] "What does 'lossless' mean for LLM weights?":
 * decode the exact BF16 values into registers or shared memory and use them
 * at once in the matrix product) ---- */

/* Workspace bytes s12_gemv needs for this container (any 1 <= B <= 8; 0
 * for an invalid view or B).  The size depends on the row count and on the
 * SM count of the current device, not on B, so one workspace of the largest
 * size serves every matrix of a model on that device. */
size_t s12_gemv_ws_bytes(const s12_view *v, int B);

/* Follows: [W] "What does 'lossless' mean for LLM weights?" (decode into
 * registers and multiply at once); [T] key points (one-ADD decode).
 * y[b][n] = sum_k W[n][k] * x[b][k] for b < B, 1 <= B <= 8.
 *   x:  device BF16, B x cols row-major.
 *   y:  device FP32, B x rows row-major (4-byte alignment suffices),
 *       overwritten.
 *   ws: device workspace of at least s12_gemv_ws_bytes(v, B) bytes (else
 *       S12_ERR_CAPACITY), owned by the caller.  It must be ZERO-FILLED
 *       before its first use (for instance one cudaMemsetAsync after
 *       allocation); every call leaves it zero-filled again when it returns,
 *       a call whose bounded waits gave up (S12_FLAG_TIMEOUT) included.
 *       Two calls that may run at the same time (different streams) need
 *       different workspaces.
 * Each warp decodes 16 rows x 128 columns at a time into the registers of
 * the warp-level tensor-core product (BF16 operands, FP32 accumulation).
 * Rows are split across warps by contiguous ranges of such blocks; a row
 * group shared by several warps is summed by the last of them in a fixed
 * order, so repeated calls give identical y.
 * With err_flag given, every tile's code-15 count is checked against its
 * esc_off span and bases above 241 are flagged; without it only tiles whose
 * span is non-empty are checked (slightly faster; corrupt data then gives a
 * wrong y but never an out-of-range read). */
int s12_gemv(const s12_view *v, const uint16_t *x, int B, float *y, void *ws, size_t ws_bytes,
             uint32_t *err_flag, void *stream);

/* Workspace bytes s12_gemv_multi needs for these `count` containers (0 for
 * invalid arguments).  Like s12_gemv_ws_bytes it depends on the row counts
 * and the SM count, not on B. */
size_t s12_gemv_multi_ws_bytes(const s12_view *views, int count, int B);

/* Follows: as s12_gemv ([W] "What does 'lossless' mean for LLM weights?").
 * Up to S12_GEMV_MAX_PROBLEMS independent fused decode-GEMVs in ONE kernel
 * launch: for i < count, y[i][b][n] = sum_k W_i[n][k] * x[i][b][k], b < B.
 *   views: host array of `count` opened containers (shapes may differ).
 *   x, y:  host arrays of `count` device pointers, laid out as in s12_gemv.
 *   ws:    zero-filled device workspace of s12_gemv_multi_ws_bytes bytes,
 *          left zero-filled on return (same rules as s12_gemv).
 * The blocks of all matrices are dealt to the warps of one grid as a single
 * range, so the launch, ramp-up and tail are paid once for the group (for
 * instance the q, k and v projections of a decoder layer, or gate and up).
 * Results are identical to `count` separate s12_gemv calls up to the
 * summation order (each is within the same tolerance), and identical from
 * call to call.  Errors as for s12_gemv; a bad entry fails the whole call
 * before any launch. */
int s12_gemv_multi(const s12_view *views, int count, const uint16_t *const *x, int B, float *const *y,
                   void *ws, size_t ws_bytes, uint32_t *err_flag, void *stream);

/* Follows: [W] "What does 'lossless' mean for LLM weights?" (decoded
 * weights used at once by the decode kernel; the gated-MLP epilogue is this
 * library's own addition).
 * Fused decode-GEMV with a SwiGLU epilogue, for a gated MLP's gate and up
 * projections (F rows each): h[b][f] = silu(g[b][f]) * u[b][f], where
 * g = W_gate x_b, u = W_up x_b and silu(t) = t / (1 + exp(-t)), rounded to
 * BF16 (round to nearest even).
 *   v:  ONE container of 2F rows that interleaves the two matrices in
 *       blocks of 8 rows: rows 16i .. 16i+7 are gate rows 8i .. 8i+7 and
 *       rows 16i+8 .. 16i+15 are up rows 8i .. 8i+7 (so 2F must be a
 *       multiple of 16, else S12_ERR_SHAPE).  The Python binding's
 *       interleave_gate_up builds that matrix before encoding.
 *   x:  device BF16, B x cols; 1 <= B <= 8.
 *   h:  device BF16, B x F row-major (2-byte alignment), overwritten.  It is
 *       the input of the down projection, so the gate and up outputs never
 *       go to memory.
 *   ws: as for s12_gemv (size s12_gemv_ws_bytes(v, B)).
 * The warp-level product gives each lane rows r and r + 8 of a 16-row group,
 * which here are gate row f and up row f: the activation is applied where
 * the sums are stored ([W] "What does 'lossless' mean for LLM weights?":
 * decode and use the weights at once; the epilogue is this library's own). */
int s12_gemv_swiglu(const s12_view *v, const uint16_t *x, int B, uint16_t *h, void *ws, size_t ws_bytes,
                    uint32_t *err_flag, void *stream);

/* Follows: [W] "What does 'lossless' mean for LLM weights?" (decode into
 * registers and multiply at once); the BF16 result is this library's own
 * option for callers whose next step takes BF16.
 * s12_gemv with a BF16 output: y[b][n] = bf16_rne(sum_k W[n][k] x[b][k]),
 * the FP32 sum of s12_gemv rounded to nearest even.
 *   y:  device BF16, B x rows row-major (2-byte alignment), overwritten.
 * The rounding adds up to 2^-9 |y| to the error of the FP32 sum (within
 * 1e-3 sum_k |W[n][k] x[b][k]|), so the result is within that bound plus
 * 2^-9 |y|.  Other arguments, errors and the workspace as for s12_gemv. */
int s12_gemv_bf16(const s12_view *v, const uint16_t *x, int B, uint16_t *y, void *ws, size_t ws_bytes,
                  uint32_t *err_flag, void *stream);

/* The pages have no counterpart of this call: it exists for integration,
 * not for the method.
 * s12_gemv for callers that cannot allocate device memory.  Examples are
 * a plugin whose host engine owns all device memory through its own
 * allocator, code under a fixed memory budget, or a path where cudaMalloc's
 * implicit synchronisation is not allowed.  Same arguments and result as
 * s12_gemv, minus the workspace.  Instead, the call uses a 2.75 MiB workspace
 * that is a static array inside the library, reserved on every device that
 * loads the library and held until the process exits.
 *   - Limits: containers of at most 2^20 rows, devices of at most 160 SMs;
 *     beyond them S12_ERR_CAPACITY, before any device work.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call outside any
 *     stream capture.
 *   - Each call first clears its arrival counters with an asynchronous
 *     memset on `stream`, then runs the s12_gemv kernel.  It allocates and
 *     frees nothing.
 *   - All calls share one array, which keeps the last call's contents.
 *     Calls that can overlap on the GPU (different streams without ordering)
 *     race on it and give wrong results; serialise them or use s12_gemv. */
int s12_gemv_noalloc(const s12_view *v, const uint16_t *x, int B, float *y, uint32_t *err_flag,
                     void *stream);

/* ---- fused decode-skinny-GEMM on tcgen05 tensor cores ---- */

/* Workspace bytes s12_gemm_skinny needs for this container and M. */
size_t s12_gemm_ws_bytes(const s12_view *v, int M);

/* Follows: [W] "How does this compare with prior lossless systems?" (a
 * fused decompression-GEMM: the weights are decoded inside the matrix
 * product, not to a BF16 copy in memory); [T] key points (the one-ADD
 * decode feeding tensor-core kernels).
 * y[m][n] = sum_k W[n][k] * x[m][k] for 16 <= M <= 256.
 *   x: device BF16, M x cols row-major.  y: device FP32, M x rows row-major,
 *   overwritten.  ws: device scratch of s12_gemm_ws_bytes(v, M) bytes,
 *   ZERO-FILLED before its first use; every call leaves it zero-filled,
 *   a call whose bounded waits gave up (S12_FLAG_TIMEOUT) included.
 * Decoded BF16 tiles are written to shared memory and multiplied by the
 * tensor cores with FP32 accumulation.  Reads container version 1 or 2. */
int s12_gemm_skinny(const s12_view *v, const uint16_t *x, int M, float *y, void *ws,
                    size_t ws_bytes, uint32_t *err_flag, void *stream);

/* Follows: as s12_gemm_skinny ([W] "How does this compare with prior
 * lossless systems?": fused decompression-GEMM); the BF16 result is this
 * library's own option for callers whose next step takes BF16.
 * s12_gemm_skinny with a BF16 output: y[m][n] = bf16_rne(FP32 sum).
 *   y: device BF16, M x rows row-major (2-byte alignment), overwritten.
 * The rounding adds up to 2^-9 |y| to the error of the FP32 sum.  Other
 * arguments, errors and the workspace as for s12_gemm_skinny. */
int s12_gemm_skinny_bf16(const s12_view *v, const uint16_t *x, int M, uint16_t *y, void *ws,
                         size_t ws_bytes, uint32_t *err_flag, void *stream);

/* Workspace bytes s12_gemm_skinny_multi needs for these `count` containers
 * with token rows M[i] (0 for invalid arguments). */
size_t s12_gemm_multi_ws_bytes(const s12_view *views, int count, const int *M);

/* Follows: as s12_gemm_skinny ([W] "How does this compare with prior
 * lossless systems?": fused decompression-GEMM; [T] key points).
 * Up to S12_GEMM_MAX_PROBLEMS independent fused decode-skinny-GEMMs in ONE
 * kernel launch: for i < count, y[i][m][n] = sum_k W_i[n][k] * x[i][m][k]
 * for m < M[i], 1 <= M[i] <= 256 (below 16 too: every matrix is multiplied
 * at the call's shared padded M).  Built for a mixture-of-experts block,
 * where each expert's matrices see a different number of routed tokens.
 *   views: host array of `count` opened containers (shapes may differ).
 *   x, y:  host arrays of `count` device pointers, laid out as in
 *          s12_gemm_skinny (x[i]: M[i] x cols_i bf16, y[i]: M[i] x rows_i
 *          fp32, overwritten).
 *   M:     host array of the token rows of each matrix.
 *   ws:    device workspace of s12_gemm_multi_ws_bytes bytes, zero-filled
 *          before its first use and left zero-filled (as for
 *          s12_gemm_skinny).
 * The 128-row x 128-column units of all matrices are dealt to the SMs as one
 * range, so the launch, ramp-up and tail are paid once for the group.  All
 * matrices are multiplied at the largest M rounded up to 16 (rows of x past
 * a matrix's own M are read as zeros and never stored), so matrices of
 * similar M group best.  Each y[i] equals what s12_gemm_skinny gives for
 * that matrix up to the summation order, within the same tolerance.  A bad
 * entry fails the whole call before any launch; so does a call that mixes
 * container versions. */
int s12_gemm_skinny_multi(const s12_view *views, int count, const uint16_t *const *x, const int *M,
                          float *const *y, void *ws, size_t ws_bytes, uint32_t *err_flag, void *stream);

/* ---- statistics ([M] section 1: exponent entropy; [T] key points:
 * escape rate) ---- */

/* Workspace bytes s12_stats needs (device scratch). */
size_t s12_stats_ws_bytes(void);

/* Follows: [M] section 1 entropy table (exponent entropy in bits); [T] key
 * points (escape rate, size ratio).
 * Fill *out with sizes, rates and the exponent histogram/entropy of the
 * decoded weights.  Runs a histogram kernel and SYNCHRONISES `stream`. */
int s12_stats(const s12_view *v, s12_stats_t *out, void *ws, size_t ws_bytes, void *stream);

/* ---- host-side validation and plane hashes ([W] "A 14-day
 * production-readiness pilot": inject corruption and confirm that it is
 * detected, not decoded into wrong weights) ---- */

#define S12_BAD_HEADER 1u       /* magic, version, tile, flags, reserved bytes or shape */
#define S12_BAD_SIZE 2u         /* fewer bytes than the header's planes need          */
#define S12_BAD_OFFSETS 3u      /* esc_off[0] != 0 or esc_off[n_tiles] != n_esc       */
#define S12_BAD_TILE_OFFSETS 4u /* a tile's offsets decrease or pass n_esc            */
#define S12_BAD_BASE 5u         /* a tile base above 241                              */
#define S12_BAD_ESC_COUNT 6u    /* a tile's code-15 count != its offset span          */
#define S12_NOTE_PADDING 1u     /* a padding byte is not zero (nothing reads it)      */

typedef struct s12_report {
    uint32_t problem;       /* S12_BAD_* of the first problem found, 0 if valid */
    uint32_t notes;         /* S12_NOTE_* bits (do not make the container invalid) */
    uint64_t tile;          /* the tile of a per-tile problem                   */
    uint64_t n_esc_counted; /* code-15 nibbles in the tiles checked             */
} s12_report;

/* Follows: [W] "A 14-day production-readiness pilot" (verify what was
 * loaded; inject corruption and confirm that it is detected).
 * Check a whole container in HOST memory (for instance a file read before
 * it is copied to the device): S12_OK when it is valid, S12_ERR_CORRUPT with
 * *out describing the first problem otherwise (S12_ERR_ARG for NULLs).  A
 * valid container decodes without any err_flag bit.  Raw bytes and escape
 * values carry no redundancy, so a change there is only caught by
 * s12_plane_hashes_host. */
int s12_validate_host(const void *container, size_t bytes, s12_report *out);

/* Follows: [W] "A 14-day production-readiness pilot" (hash what was
 * stored and compare after loading).
 * 64-bit FNV-1a hashes of the exact bytes of the five planes, in the order
 * raw, code, base, esc_off, esc (padding excluded), of a container in HOST
 * memory with a valid header.  Any change of a single byte changes its
 * plane's hash.  Store them at encode time and compare after loading. */
int s12_plane_hashes_host(const void *container, size_t bytes, uint64_t out[5]);

/* Follows: [W] "A 14-day production-readiness pilot" (the hash behind
 * s12_plane_hashes_host).
 * FNV-1a 64-bit hash of `bytes` bytes (offset basis 0xcbf29ce484222325,
 * prime 0x100000001b3), the function s12_plane_hashes_host uses. */
uint64_t s12_fnv1a64(const void *data, size_t bytes);

/* Outcome of s12_load_bf16. */
#define S12_LOAD_DECODED 0  /* every check passed; out holds the decoded tensor    */
#define S12_LOAD_FALLBACK 1 /* a check failed; out holds the caller's BF16 copy    */
#define S12_LOAD_REJECTED 2 /* a check failed and no BF16 copy was given          */

typedef struct s12_load_result {
    uint32_t outcome;       /* S12_LOAD_*                                          */
    uint32_t problem;       /* S12_BAD_* of the host validation, 0 if it passed    */
    uint32_t hash_mismatch; /* bit i: plane i's hash differs from expected[i]      */
    uint32_t device_flags;  /* S12_FLAG_* bits of the device decode (0 if not run) */
} s12_load_result;

/* Follows: [W] "A 14-day production-readiness pilot" (operations and
 * reversibility: keep the original BF16 weights, check what was loaded, and
 * fall back to the original for a tensor that fails).
 * Load one tensor to the device as BF16, whole, with a fallback.  Steps:
 *   1. s12_validate_host(container) and, when expected_hashes (5 values of
 *      s12_plane_hashes_host taken at encode time) is given, the plane
 *      hashes; the header must also say rows x cols;
 *   2. if they pass: copy the container to dev_container, decode it into
 *      dev_out with the device err word dev_err (cleared first), read the
 *      word back;
 *   3. if any check failed: with `fallback` (host BF16, rows x cols) copy it
 *      to dev_out (outcome S12_LOAD_FALLBACK); without it leave the decision
 *      to the caller (outcome S12_LOAD_REJECTED, dev_out not valid; the
 *      caller may reload the tensor).
 *   container:      host, `bytes` long, version 1 (convert a version 2 one
 *                   with s12_from_v2_host first).
 *   dev_container:  device, 256-byte aligned, dev_cap >= bytes (else
 *                   S12_ERR_CAPACITY); receives the container.
 *   dev_out:        device BF16, rows x cols.   dev_err: device u32.
 *   res:            host, filled on S12_OK.
 * Returns S12_OK when an outcome was reached (see res->outcome); argument,
 * alignment and CUDA errors as usual.  SYNCHRONISES `stream`.  Steps 1 and
 * a rejection run on the host alone. */
int s12_load_bf16(const void *container, size_t bytes, const uint64_t *expected_hashes,
                  const uint16_t *fallback, uint64_t rows, uint64_t cols, void *dev_container,
                  size_t dev_cap, uint16_t *dev_out, uint32_t *dev_err, s12_load_result *res,
                  void *stream);

/* Follows: [W] English edition, opening summary (the 24.967 % payload
 * reduction leaves little room for per-tile metadata).
 * Container version 2, a compact tile header, as a storage format: the same
 * raw, code and escape planes, with per tile ONE u16 (base | escape count
 * << 8) and per row one u32 escape offset instead of a u8 base and a u32
 * offset per tile (2 bytes per tile + 4 per row instead of 5 per tile; [W]
 * English edition, opening summary: the 24.967 % payload reduction leaves
 * little room for metadata).  Header as version 1 with version = 2.  Every
 * kernel call (decode, stats, GEMV, GEMM) reads either version in device
 * memory; these calls convert between them in HOST memory, snprintf-style
 * (dst == NULL: only *bytes_out), S12_ERR_CAPACITY if dst_cap is too small,
 * S12_ERR_CORRUPT for an invalid source (a version 1 source must pass
 * s12_validate_host; a version 2 source must have row offsets and tile
 * counts that describe its escape stream).  Converting back gives the
 * original version 1 container byte for byte. */
int s12_to_v2_host(const void *v1, size_t v1_bytes, void *dst, size_t dst_cap, size_t *bytes_out);
int s12_from_v2_host(const void *v2, size_t v2_bytes, void *dst, size_t dst_cap, size_t *bytes_out);

/* Follows: [T] technical deep dive (the 12-bit representation packed into
 * 3-byte words, two weights per word).
 * Container version 3 (packed 24-bit pairs) as a storage format, converted
 * in HOST memory like version 2 (snprintf-style; S12_ERR_CAPACITY,
 * S12_ERR_CORRUPT as there): version 1's raw and code planes regrouped into
 * one pair plane, the base, esc_off and esc planes byte for byte.  A
 * version 1 source must pass s12_validate_host; converting back gives it
 * byte for byte, and the result must pass s12_validate_host. */
int s12_to_v3_host(const void *v1, size_t v1_bytes, void *dst, size_t dst_cap, size_t *bytes_out);
int s12_from_v3_host(const void *v3, size_t v3_bytes, void *dst, size_t dst_cap, size_t *bytes_out);

/* ---- uncompressed baseline ---- */

/* Follows: the plain matrix-vector product that [W] "What does 'lossless'
 * mean for LLM weights?" says the decoded weights must reproduce; it is the
 * uncompressed comparison point.
 * Plain BF16 GEMV, the comparison point for s12_gemv: y[b][n] =
 * sum_k w[n][k] * x[b][k], w device BF16 rows x cols (cols % 8 == 0),
 * 1 <= B <= 8, y FP32 B x rows. */
int s12_bf16_gemv(const uint16_t *w, int64_t rows, int64_t cols, const uint16_t *x, int B,
                  float *y, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* S12_H */
