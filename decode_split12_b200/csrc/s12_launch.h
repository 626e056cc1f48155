// s12_launch.h -- internal host-side declarations of the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "s12.h"

namespace s12 {

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
int make_tmap_bf16_2d(CUtensorMap *out, const void *base, uint64_t inner, uint64_t rows, uint64_t row_stride,
                      uint32_t box_inner, uint32_t box_rows, int swizzle);

int launch_decode(const s12_view *v, uint16_t *out, uint32_t *err, cudaStream_t stream);
size_t gemv_ws_bytes(const s12_view *views, int count);
// y[i]: float* (B x rows) when act is null or act[i] == 0; uint16_t* BF16
// (B x rows/2) when act[i] == 1 (SwiGLU of interleaved gate/up rows).
int launch_gemv(const s12_view *views, int count, const uint16_t *const *x, int B, void *const *y, const int *act,
                void *ws, size_t ws_bytes, uint32_t *err, cudaStream_t stream);
int launch_bf16_gemv(const uint16_t *w, int64_t rows, int64_t cols, const uint16_t *x, int B, float *y,
                     cudaStream_t stream);
size_t encode_ws_bytes(int64_t rows, int64_t cols);
int launch_encode(const uint16_t *w, int64_t rows, int64_t cols, void *dst, size_t dst_cap, size_t *bytes_out,
                  void *ws, size_t ws_bytes, cudaStream_t stream);
int launch_stats_hist(const s12_view *v, unsigned long long *hist_dev, cudaStream_t stream);
size_t gemm_ws_bytes(const s12_view *views, int count, const int *M);
int launch_gemm(const s12_view *views, int count, const uint16_t *const *x, const int *M, float *const *y, void *ws,
                size_t ws_bytes, uint32_t *err, cudaStream_t stream);

}  // namespace s12
