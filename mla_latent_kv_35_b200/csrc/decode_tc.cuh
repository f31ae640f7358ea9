// decode_tc.cuh -- split-KV flash-decode on the latent cache with tcgen05
// (placeholder until the tensor-core kernel lands).
#pragma once
#include "common.cuh"

namespace mla {
constexpr bool kDecodeTcReady = false;
inline mla_status launch_decode_tc(const void*, const void*, int, const int32_t*, int,
                                   const int32_t*, int, int, int, float, int, const int32_t*,
                                   float*, float*, cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}
}  // namespace mla
