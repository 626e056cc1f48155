// s12_launch.h -- internal host-side declarations of the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "s12.h"

namespace s12 {

// Fused GEMV launch geometry, shared by the kernel and by the static
// workspace of s12_gemv_noalloc (which sizes its array from them).
constexpr int kGemvWarps = 16;             // warps per CTA, one CTA per SM
constexpr uint32_t kGemvSlotBytes = 512;   // one stream-K partial: 32 lanes x 4 floats
// Stream-K partial sums: two slots per warp of the largest grid.
constexpr uint64_t gemv_part_bytes(int sms) {
    return (static_cast<uint64_t>(sms) * kGemvWarps * 2 * kGemvSlotBytes + 255) / 256 * 256;
}
// Arrival counters: one u32 per 16-row group.
constexpr uint64_t gemv_cnt_bytes(uint64_t row_groups) { return (row_groups * 4 + 255) / 256 * 256; }

// S12_OK when the view is usable by the kernels (pointers of its version
// present, cols a multiple of 128, container 16-byte aligned), else the
// status the entry points return for it.
int check_view(const s12_view *v);

// Output kinds of the fused GEMV: FP32 y, the SwiGLU epilogue (BF16 h of
// half the rows), or BF16 y.
enum : int { kGemvOutF32 = 0, kGemvOutSwiglu = 1, kGemvOutBf16 = 2 };

// The argument checks every GEMV entry point makes before any device work
// (views, batch, pointers, output kinds, alignment, one container version
// per call), with the status s12_gemv returns for each failure.
int gemv_check(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *out,
               uint32_t *err_flag);

// Number of SMs of the current device (cached per device).
cudaError_t device_sms(int *sms);

// Tiled TMA descriptor for a row-major 2-D array of bytes: `inner` bytes
// per row, `rows` rows, `row_stride` bytes between rows (multiple of 16),
// box of box_inner x box_rows bytes (box_inner a multiple of 16, and at most
// the swizzle width), out-of-bounds bytes read as 0.  swizzle: 0 (none), 64
// or 128 (the copy engine's 64- or 128-byte swizzle of 16-byte chunks).
int make_tmap_u8_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows, uint64_t row_stride,
                    uint32_t box_inner, uint32_t box_rows, int swizzle);
// The same for a row-major 2-D array of BF16 values (`inner` and the box's
// inner extent counted in elements, `row_stride` in bytes).
// Tiled TMA descriptor for a 3-D array of bytes: dims {inner, d1, d2} with
// byte strides {stride1, stride2} for the two outer dimensions (multiples
// of 16, in any order), box {box_inner, box1, box2}, out-of-bounds bytes
// read as 0; swizzle as above.
int make_tmap_u8_3d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t d1, uint64_t d2, uint64_t stride1,
                    uint64_t stride2, uint32_t box_inner, uint32_t box1, uint32_t box2, int swizzle);
int make_tmap_bf16_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows, uint64_t row_stride,
                      uint32_t box_inner, uint32_t box_rows, int swizzle);

int launch_decode(const s12_view *v, uint16_t *out, uint32_t *err, cudaStream_t stream);
size_t gemv_ws_bytes(const s12_view *views, int count);
// y[i]: float* (B x rows) for kGemvOutF32 (or a null `out`), uint16_t* BF16
// (B x rows) for kGemvOutBf16, uint16_t* BF16 (B x rows/2) for
// kGemvOutSwiglu (interleaved gate/up rows).
int launch_gemv(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *out,
                void *ws, size_t ws_bytes, uint32_t *err, cudaStream_t stream);
int launch_bf16_gemv(const uint16_t *w, int64_t rows, int64_t cols, const uint16_t *x, int B, float *y,
                     cudaStream_t stream);
size_t encode_ws_bytes(int64_t rows, int64_t cols);
int launch_encode(const uint16_t *w, int64_t rows, int64_t cols, void *dst, size_t dst_cap, size_t *bytes_out,
                  void *ws, size_t ws_bytes, cudaStream_t stream);
int launch_stats_hist(const s12_view *v, unsigned long long *hist_dev, cudaStream_t stream);
size_t gemm_ws_bytes(const s12_view *views, int count, const int *M);
// y[i]: float* (M[i] x rows) for out[i] == 0 (or a null `out`), uint16_t*
// BF16 for out[i] == 1.
int launch_gemm(const s12_view *views, int count, const uint16_t *const *x, const int *M, void *const *y,
                const int *out, void *ws, size_t ws_bytes, uint32_t *err, cudaStream_t stream);

}  // namespace s12
