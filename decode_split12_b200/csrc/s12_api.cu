// s12_api.cu -- the C ABI of libs12.so (declared in include/s12.h): argument
// checks, container parsing, and dispatch to the kernel launchers.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace

int check_view(const s12_view *v) {
    if (!v || !v->container || !v->raw || !v->esc) return S12_ERR_ARG;
    if (v->version == 1) {
        if (!v->code || !v->base || !v->esc_off) return S12_ERR_ARG;
    } else if (v->version == 2) {
        if (!v->code || !v->tmeta || !v->row_esc) return S12_ERR_ARG;
    } else if (v->version == 3) {
        if (!v->base || !v->esc_off) return S12_ERR_ARG;  // raw = the pair plane, no code plane
    } else if (v->version == 4) {
        if (!v->code || !v->esc_off || !v->symtab) return S12_ERR_ARG;
    } else {
        return S12_ERR_ARG;
    }
    if (v->rows == 0 || v->cols == 0 || v->cols % kTile) return S12_ERR_SHAPE;
    if (!aligned16(v->container)) return S12_ERR_ALIGN;
    return S12_OK;
}

namespace {

uint32_t get_u32(const uint8_t *p) {
    return uint32_t(p[0]) | uint32_t(p[1]) << 8 | uint32_t(p[2]) << 16 | uint32_t(p[3]) << 24;
}
uint64_t get_u64(const uint8_t *p) { return uint64_t(get_u32(p)) | uint64_t(get_u32(p + 4)) << 32; }
}  // namespace

cudaError_t device_sms(int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) {
        const int c = g_sms[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *sms = c;
            return cudaSuccess;
        }
    }
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) g_sms[dev].store(n, std::memory_order_relaxed);
    *sms = n;
    return cudaSuccess;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
std::once_flag g_encode_once;
}  // namespace

namespace {
int encode_2d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t rows,
              uint64_t row_stride, uint32_t box_inner, uint32_t box_rows, int swizzle);
}  // namespace

int make_tmap_bf16_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows, uint64_t row_stride,
                      uint32_t box_inner, uint32_t box_rows, int swizzle) {
    return encode_2d(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, rows, row_stride, box_inner, box_rows,
                     swizzle);
}

int make_tmap_u8_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows, uint64_t row_stride,
                    uint32_t box_inner, uint32_t box_rows, int swizzle) {
    return encode_2d(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, rows, row_stride, box_inner, box_rows,
                     swizzle);
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode_tiled;
}

CUtensorMapSwizzle swizzle_mode(int swizzle) {
    return swizzle == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
           : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                           : CU_TENSOR_MAP_SWIZZLE_NONE;
}

int encode_2d(CUtensorMap *out, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t rows,
              uint64_t row_stride, uint32_t box_inner, uint32_t box_rows, int swizzle) {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode_tiled) return S12_ERR_CUDA;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_stride};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode_tiled(out, dtype, 2, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                swizzle == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? S12_OK : S12_ERR_CUDA;
}
}  // namespace

int make_tmap_u8_3d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t d1, uint64_t d2, uint64_t stride1,
                    uint64_t stride2, uint32_t box_inner, uint32_t box1, uint32_t box2, int swizzle) {
    auto enc = encoder();
    if (!enc) return S12_ERR_CUDA;
    const cuuint64_t dims[3] = {inner, d1, d2};
    const cuuint64_t strides[2] = {stride1, stride2};
    const cuuint32_t box[3] = {box_inner, box1, box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_mode(swizzle), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? S12_OK : S12_ERR_CUDA;
}

}  // namespace s12

using namespace s12;

extern "C" {

const char *s12_error_string(int status) {
    switch (status) {
        case S12_OK: return "S12_OK";
        case S12_ERR_ARG: return "S12_ERR_ARG: null pointer or invalid size";
        case S12_ERR_SHAPE: return "S12_ERR_SHAPE: unsupported shape or batch";
        case S12_ERR_ALIGN: return "S12_ERR_ALIGN: device pointer not 16-byte aligned";
        case S12_ERR_CAPACITY: return "S12_ERR_CAPACITY: buffer or workspace too small";
        case S12_ERR_CORRUPT: return "S12_ERR_CORRUPT: container header or offsets inconsistent";
        case S12_ERR_CUDA: return "S12_ERR_CUDA: CUDA runtime call failed";
        case S12_ERR_DEVICE: return "S12_ERR_DEVICE: current device is not compute capability 10.0";
        default: return "S12: unknown status";
    }
}

int s12_device_check(void) {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return S12_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return S12_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return S12_ERR_CUDA;
    return (major == 10 && minor == 0) ? S12_OK : S12_ERR_DEVICE;
}

uint64_t s12_container_bytes(int64_t rows, int64_t cols, uint64_t n_esc) {
    if (rows <= 0 || cols <= 0 || cols % kTile) return 0;
    return geometry(static_cast<uint64_t>(rows), static_cast<uint64_t>(cols), n_esc).total;
}

size_t s12_encode_ws_bytes(int64_t rows, int64_t cols) { return encode_ws_bytes(rows, cols); }

int s12_encode(const uint16_t *w, int64_t rows, int64_t cols, void *dst, size_t dst_cap, size_t *bytes_out,
               void *ws, size_t ws_bytes, void *stream) {
    if (!w || !bytes_out || !ws) return S12_ERR_ARG;
    if (rows <= 0 || cols <= 0) return S12_ERR_ARG;
    if (cols % kTile) return S12_ERR_SHAPE;
    if (static_cast<uint64_t>(rows) * static_cast<uint64_t>(cols) >= (uint64_t(1) << 32)) return S12_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(ws) || (dst && !aligned16(dst))) return S12_ERR_ALIGN;
    return launch_encode(w, rows, cols, dst, dst_cap, bytes_out, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int s12_open(const void *container, size_t bytes, s12_view *out) {
    if (!container || !out) return S12_ERR_ARG;
    if (!aligned16(container)) return S12_ERR_ALIGN;
    if (bytes < kHeaderBytes) return S12_ERR_CORRUPT;
    uint8_t h[64];
    if (cudaMemcpy(h, container, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return S12_ERR_CUDA;
    if (std::memcmp(h, "S12\0", 4) != 0) return S12_ERR_CORRUPT;
    const uint32_t version = get_u32(h + 4);
    if (version < 1 || version > 4 || get_u32(h + 24) != static_cast<uint32_t>(kTile) || get_u32(h + 28) != 0)
        return S12_ERR_CORRUPT;
    for (int i = 40; i < 64; ++i)
        if (h[i]) return S12_ERR_CORRUPT;
    const uint64_t rows = get_u64(h + 8), cols = get_u64(h + 16), n_esc = get_u64(h + 32);
    if (rows == 0 || cols == 0 || cols % kTile) return S12_ERR_CORRUPT;
    if (rows >= (uint64_t(1) << 32) || cols >= (uint64_t(1) << 32) || rows * cols >= (uint64_t(1) << 32))
        return S12_ERR_CORRUPT;
    if (n_esc > rows * cols) return S12_ERR_CORRUPT;
    const uint8_t *c = static_cast<const uint8_t *>(container);
    std::memset(out, 0, sizeof *out);
    out->rows = rows;
    out->cols = cols;
    out->n_esc = n_esc;
    out->container = container;
    out->version = version;
    if (version == 1) {
        const Geometry g = geometry(rows, cols, n_esc);
        if (g.total > bytes) return S12_ERR_CORRUPT;
        out->n_tiles = g.n_tiles;
        out->container_bytes = g.total;
        out->raw = c + g.off_raw;
        out->code = c + g.off_code;
        out->base = c + g.off_base;
        out->esc_off = reinterpret_cast<const uint32_t *>(c + g.off_esc_off);
        out->esc = reinterpret_cast<const uint16_t *>(c + g.off_esc);
    } else if (version == 4) {
        const Geometry4 g = geometry4(rows, cols, n_esc);
        if (g.total > bytes) return S12_ERR_CORRUPT;
        out->n_tiles = g.n_tiles;
        out->container_bytes = g.total;
        out->symtab = reinterpret_cast<const uint16_t *>(c + g.off_table);
        out->raw = c + g.off_raw;
        out->code = c + g.off_code;
        out->esc_off = reinterpret_cast<const uint32_t *>(c + g.off_esc_off);
        out->esc = reinterpret_cast<const uint16_t *>(c + g.off_esc);
    } else if (version == 3) {
        const Geometry3 g = geometry3(rows, cols, n_esc);
        if (g.total > bytes) return S12_ERR_CORRUPT;
        out->n_tiles = g.n_tiles;
        out->container_bytes = g.total;
        out->raw = c + g.off_pair;  // the pair plane; code stays NULL
        out->base = c + g.off_base;
        out->esc_off = reinterpret_cast<const uint32_t *>(c + g.off_esc_off);
        out->esc = reinterpret_cast<const uint16_t *>(c + g.off_esc);
    } else {
        const Geometry2 g = geometry2(rows, cols, n_esc);
        if (g.total > bytes) return S12_ERR_CORRUPT;
        out->n_tiles = g.n_tiles;
        out->container_bytes = g.total;
        out->raw = c + g.off_raw;
        out->code = c + g.off_code;
        out->tmeta = reinterpret_cast<const uint16_t *>(c + g.off_tmeta);
        out->row_esc = reinterpret_cast<const uint32_t *>(c + g.off_row_esc);
        out->esc = reinterpret_cast<const uint16_t *>(c + g.off_esc);
    }
    return S12_OK;
}

int s12_decode(const s12_view *v, uint16_t *out, uint32_t *err_flag, void *stream) {
    int rc = check_view(v);
    if (rc != S12_OK) return rc;
    if (!out) return S12_ERR_ARG;
    if (!aligned16(out) || (err_flag && !aligned4(err_flag))) return S12_ERR_ALIGN;
    return launch_decode(v, out, err_flag, static_cast<cudaStream_t>(stream));
}

size_t s12_gemv_ws_bytes(const s12_view *v, int B) { return s12_gemv_multi_ws_bytes(v, 1, B); }

size_t s12_gemv_multi_ws_bytes(const s12_view *views, int count, int B) {
    if (!views || count < 1 || count > S12_GEMV_MAX_PROBLEMS || B < 1 || B > S12_GEMV_MAX_BATCH) return 0;
    for (int i = 0; i < count; ++i)
        if (check_view(views + i) != S12_OK) return 0;
    return gemv_ws_bytes(views, count);
}

}  // extern "C"

namespace s12 {

int gemv_check(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *out,
               uint32_t *err_flag) {
    if (!views || !x || !y) return S12_ERR_ARG;
    if (count < 1 || count > S12_GEMV_MAX_PROBLEMS || B < 1 || B > S12_GEMV_MAX_BATCH) return S12_ERR_SHAPE;
    for (int i = 0; i < count; ++i) {
        const int rc = check_view(views + i);
        if (rc != S12_OK) return rc;
        if (!x[i] || !y[i]) return S12_ERR_ARG;
        if (views[i].rows > 0x7FFFFFFFull || views[i].cols > 0x7FFFFFFFull) return S12_ERR_SHAPE;
        if (views[i].version != views[0].version || views[i].version > 2) return S12_ERR_ARG;
        const int o = out ? out[i] : kGemvOutF32;
        if (o != kGemvOutF32 && o != kGemvOutSwiglu && o != kGemvOutBf16) return S12_ERR_ARG;
        if (o == kGemvOutSwiglu && views[i].rows % 16 != 0) return S12_ERR_SHAPE;
        const bool y_ok = o == kGemvOutF32 ? aligned4(y[i]) : (reinterpret_cast<uintptr_t>(y[i]) & 1) == 0;
        if (!aligned16(x[i]) || !y_ok) return S12_ERR_ALIGN;
    }
    if (err_flag && !aligned4(err_flag)) return S12_ERR_ALIGN;
    return S12_OK;
}

}  // namespace s12

extern "C" {

namespace {
// Checks shared by the GEMV calls (every entry, before any launch), then the
// launch.  out[i] is the output kind of entry i (null: all FP32).
int gemv_group(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *out,
               void *ws, size_t ws_bytes, uint32_t *err_flag, void *stream) {
    const int rc = gemv_check(views, count, x, B, y, out, err_flag);
    if (rc != S12_OK) return rc;
    if (!ws) return S12_ERR_ARG;
    if (!aligned16(ws)) return S12_ERR_ALIGN;
    return launch_gemv(views, count, x, B, y, out, ws, ws_bytes, err_flag, static_cast<cudaStream_t>(stream));
}
}  // namespace

int s12_gemv_multi(const s12_view *views, int count, const uint16_t *const *x, int B, float *const *y, void *ws,
                   size_t ws_bytes, uint32_t *err_flag, void *stream) {
    void *out[S12_GEMV_MAX_PROBLEMS];
    if (!y || count < 1 || count > S12_GEMV_MAX_PROBLEMS) return y ? S12_ERR_SHAPE : S12_ERR_ARG;
    for (int i = 0; i < count; ++i) out[i] = y[i];
    return gemv_group(views, count, x, B, out, nullptr, ws, ws_bytes, err_flag, stream);
}

int s12_gemv_swiglu(const s12_view *v, const uint16_t *x, int B, uint16_t *h, void *ws, size_t ws_bytes,
                    uint32_t *err_flag, void *stream) {
    if (!v || !x || !h || !ws) return S12_ERR_ARG;
    void *out[1] = {h};
    const int kind[1] = {kGemvOutSwiglu};
    return gemv_group(v, 1, &x, B, out, kind, ws, ws_bytes, err_flag, stream);
}

int s12_gemv_bf16(const s12_view *v, const uint16_t *x, int B, uint16_t *y, void *ws, size_t ws_bytes,
                  uint32_t *err_flag, void *stream) {
    if (!v || !x || !y || !ws) return S12_ERR_ARG;
    void *out[1] = {y};
    const int kind[1] = {kGemvOutBf16};
    return gemv_group(v, 1, &x, B, out, kind, ws, ws_bytes, err_flag, stream);
}

int s12_gemv(const s12_view *v, const uint16_t *x, int B, float *y, void *ws, size_t ws_bytes, uint32_t *err_flag,
             void *stream) {
    if (!v || !x || !y || !ws) return S12_ERR_ARG;
    int rc = check_view(v);
    if (rc != S12_OK) return rc;
    return s12_gemv_multi(v, 1, &x, B, &y, ws, ws_bytes, err_flag, stream);
}

size_t s12_gemm_ws_bytes(const s12_view *v, int M) {
    if (check_view(v) != S12_OK || M < S12_GEMM_MIN_M || M > S12_GEMM_MAX_M) return 0;
    return gemm_ws_bytes(v, 1, &M);
}

namespace {
// Shared checks of the GEMM calls: every entry valid, before any launch.
// min_m: the smallest token count an entry may have (a grouped call pads
// every matrix to the shared multiple of 16, so it accepts any M >= 1).
// out: null (all FP32) or one output kind per entry (0 FP32, 1 BF16).
int check_gemm_group(const s12_view *views, int count, const uint16_t *const *x, const int *M, void *const *y,
                     const int *out, int min_m) {
    if (!views || !x || !M || !y || count < 1 || count > S12_GEMM_MAX_PROBLEMS) return S12_ERR_ARG;
    for (int i = 0; i < count; ++i) {
        const int rc = check_view(views + i);
        if (rc != S12_OK) return rc;
        if (!x[i] || !y[i]) return S12_ERR_ARG;
        if (M[i] < min_m || M[i] > S12_GEMM_MAX_M) return S12_ERR_SHAPE;
        if (views[i].rows > 0x7FFFFFFFull || views[i].cols > 0x7FFFFFFFull) return S12_ERR_SHAPE;
        const bool bf16 = out && out[i] == 1;
        const bool y_ok = bf16 ? (reinterpret_cast<uintptr_t>(y[i]) & 1) == 0 : aligned4(y[i]);
        if (!aligned16(x[i]) || !y_ok) return S12_ERR_ALIGN;
    }
    return S12_OK;
}

// One fused GEMM with output kind `kind` (0 FP32, 1 BF16).
int gemm_one(const s12_view *v, const uint16_t *x, int M, void *y, int kind, void *ws, size_t ws_bytes,
             uint32_t *err_flag, void *stream) {
    int rc = check_view(v);
    if (rc != S12_OK) return rc;
    if (!x || !y) return S12_ERR_ARG;
    void *yy[1] = {y};
    const int out[1] = {kind};
    rc = check_gemm_group(v, 1, &x, &M, yy, out, S12_GEMM_MIN_M);
    if (rc != S12_OK) return rc;
    if ((ws && !aligned16(ws)) || (err_flag && !aligned4(err_flag))) return S12_ERR_ALIGN;
    if (ws_bytes < gemm_ws_bytes(v, 1, &M)) return S12_ERR_CAPACITY;
    return launch_gemm(v, 1, &x, &M, yy, out, ws, ws_bytes, err_flag, static_cast<cudaStream_t>(stream));
}
}  // namespace

int s12_gemm_skinny(const s12_view *v, const uint16_t *x, int M, float *y, void *ws, size_t ws_bytes,
                    uint32_t *err_flag, void *stream) {
    return gemm_one(v, x, M, y, 0, ws, ws_bytes, err_flag, stream);
}

int s12_gemm_skinny_bf16(const s12_view *v, const uint16_t *x, int M, uint16_t *y, void *ws, size_t ws_bytes,
                         uint32_t *err_flag, void *stream) {
    return gemm_one(v, x, M, y, 1, ws, ws_bytes, err_flag, stream);
}

size_t s12_gemm_multi_ws_bytes(const s12_view *views, int count, const int *M) {
    if (!views || !M || count < 1 || count > S12_GEMM_MAX_PROBLEMS) return 0;
    for (int i = 0; i < count; ++i)
        if (check_view(views + i) != S12_OK || M[i] < 1 || M[i] > S12_GEMM_MAX_M) return 0;
    return gemm_ws_bytes(views, count, M);
}

int s12_gemm_skinny_multi(const s12_view *views, int count, const uint16_t *const *x, const int *M,
                          float *const *y, void *ws, size_t ws_bytes, uint32_t *err_flag, void *stream) {
    if (!y) return S12_ERR_ARG;
    void *yy[S12_GEMM_MAX_PROBLEMS];
    for (int i = 0; i < count && i < S12_GEMM_MAX_PROBLEMS; ++i) yy[i] = y[i];
    const int rc = check_gemm_group(views, count, x, M, yy, nullptr, 1);
    if (rc != S12_OK) return rc;
    if (!ws) return S12_ERR_ARG;
    if (!aligned16(ws) || (err_flag && !aligned4(err_flag))) return S12_ERR_ALIGN;
    if (ws_bytes < gemm_ws_bytes(views, count, M)) return S12_ERR_CAPACITY;
    return launch_gemm(views, count, x, M, yy, nullptr, ws, ws_bytes, err_flag, static_cast<cudaStream_t>(stream));
}

size_t s12_stats_ws_bytes(void) { return 256 * sizeof(unsigned long long); }

int s12_stats(const s12_view *v, s12_stats_t *out, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_view(v);
    if (rc != S12_OK) return rc;
    if (!out || !ws) return S12_ERR_ARG;
    if (!aligned16(ws)) return S12_ERR_ALIGN;
    if (ws_bytes < s12_stats_ws_bytes()) return S12_ERR_CAPACITY;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned long long *hist = static_cast<unsigned long long *>(ws);
    rc = launch_stats_hist(v, hist, st);
    if (rc != S12_OK) return rc;
    unsigned long long h[256];
    if (cudaMemcpyAsync(h, hist, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return S12_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return S12_ERR_CUDA;
    std::memset(out, 0, sizeof *out);
    const uint64_t nw = v->rows * v->cols;
    out->rows = v->rows;
    out->cols = v->cols;
    out->n_tiles = v->n_tiles;
    out->n_esc = v->n_esc;
    out->container_bytes = v->container_bytes;
    out->payload_bytes = nw + nw / 2;
    out->header_bytes = v->version == 2   ? v->n_tiles * 2 + 4 * (v->rows + 1)
                        : v->version == 4 ? 4 * (v->n_tiles + 1) + 64
                                          : v->n_tiles * 5;
    out->escape_bytes = 2 * v->n_esc;
    out->escape_rate = static_cast<double>(v->n_esc) / static_cast<double>(nw);
    out->bits_per_weight = 8.0 * static_cast<double>(v->container_bytes) / static_cast<double>(nw);
    out->ratio_vs_bf16 = static_cast<double>(v->container_bytes) / (2.0 * static_cast<double>(nw));
    out->payload_ratio = static_cast<double>(out->payload_bytes) / (2.0 * static_cast<double>(nw));
    double ent = 0.0;
    for (int e = 0; e < 256; ++e) {
        out->exp_hist[e] = h[e];
        if (h[e]) {
            const double p = static_cast<double>(h[e]) / static_cast<double>(nw);
            ent -= p * std::log2(p);
        }
    }
    out->exp_entropy_bits = ent;
    return S12_OK;
}

int s12_bf16_gemv(const uint16_t *w, int64_t rows, int64_t cols, const uint16_t *x, int B, float *y,
                  void *stream) {
    if (!w || !x || !y) return S12_ERR_ARG;
    if (rows <= 0 || cols <= 0) return S12_ERR_ARG;
    if (cols % 8 || B < 1 || B > S12_GEMV_MAX_BATCH) return S12_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(x) || !aligned4(y)) return S12_ERR_ALIGN;
    return launch_bf16_gemv(w, rows, cols, x, B, y, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
