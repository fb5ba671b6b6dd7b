// Tensor-core (tcgen05 / TMEM / TMA) GEMMs of the bf16 path.
#pragma once

#include "common.cuh"

namespace moe {
namespace tc {

inline bool router_supported(const moe_shape&) { return false; }
inline bool ffn_supported(const moe_shape&) { return false; }

inline moe_status launch_router_gemm(const moe_shape&, const void*, const void*, const float*,
                                     float*, int, cudaStream_t, char*, size_t) {
  return MOE_ERR_UNSUPPORTED;
}
inline moe_status launch_gate_up(const moe_shape&, const void*, const void*, const void*,
                                 const int32_t*, void*, uint32_t*, int, cudaStream_t, char*,
                                 size_t) {
  return MOE_ERR_UNSUPPORTED;
}
inline moe_status launch_down(const moe_shape&, const void*, const void*, const int32_t*, void*,
                              uint32_t*, int, cudaStream_t, char*, size_t) {
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace tc
}  // namespace moe
