// attn_decode_tc.cuh -- tensor-core split-KV decode attention over the latent cache.
#pragma once
#include "ptx.cuh"
#include "mla.h"

namespace mla {

constexpr int kAttnTileTokens = 64;
constexpr bool kAttnTcReady = false;

inline mla_status launch_attn_decode_tc(const __nv_bfloat16*, const mla_cache*, const int32_t*, const int*, const int*,
                                        int, int, float*, float*, int*, cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}

}  // namespace mla
