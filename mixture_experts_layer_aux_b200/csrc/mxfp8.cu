// mxfp8.cu -- MXFP8 expert GEMM path (E4M3 operands, UE8M0 1x32 block scales).
#include "common.cuh"
#include "layout.h"

namespace moe_impl {

size_t layer_ws_mxfp8(const moe_config*) { return 0; }

int layer_fwd_mxfp8(const moe_config*, const void*, const void*, const float*, const void*, const void*, const void*,
                    const uint8_t*, const uint8_t*, const uint8_t*, const void*, const void*, const void*,
                    const uint8_t*, const uint8_t*, const uint8_t*, void*, float*, int32_t*, float*, int32_t*,
                    int32_t*, void*, size_t, cudaStream_t) {
  return MOE_ERR_UNSUPPORTED;
}

int grouped_gemm_fwd(const moe_config*, int, const void*, const uint8_t*, const void*, const uint8_t*, const void*,
                     const uint8_t*, const int32_t*, const float*, void*, uint8_t*, void*, void*, size_t,
                     cudaStream_t) {
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe_impl
