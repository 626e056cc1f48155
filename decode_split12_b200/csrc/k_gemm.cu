// k_gemm.cu -- fused decode-skinny-GEMM (tcgen05).  Placeholder until the
// tensor-core kernel lands: reports an unsupported shape.
#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

size_t gemm_ws_bytes(const s12_view *, int) { return 256; }

int launch_gemm(const s12_view *, const uint16_t *, int, float *, void *, size_t, uint32_t *, cudaStream_t) {
    return S12_ERR_SHAPE;
}

}  // namespace s12
