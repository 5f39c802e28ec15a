// Stage 3 (tensor-core path): placeholder until the tcgen05 kernel lands.
#pragma once
#include "common.cuh"
#include "attn_simt.cuh"

namespace ddt {
inline bool tc_attn_supported(int group) { (void)group; return false; }
inline size_t tc_attn_ws_bytes(const AttnGeom&, int) { return 0; }
inline int tc_attn_launch(const void*, const void*, const void*, const int32_t*, const int32_t*,
                          const uint32_t*, const int32_t*, const AttnGeom&, void*, float*, void*, int,
                          cudaStream_t) {
  return DDTREE_ERR_UNSUPPORTED;
}
}  // namespace ddt
