// MoE gather_qmm -- placeholder until the grouped kernel lands.
#pragma once
#include <cstdio>
#include "common.cuh"
#include "nvfp4.h"

namespace nvfp4 {
inline size_t gather_workspace_bytes(int64_t T, int64_t topk, int64_t E) { return 256; }
inline nvfp4_status gather_qmm_launch(const void* x, const uint32_t* w_codes, const uint8_t* w_scales,
                                      const float* g, const int32_t* idx, int64_t T, int64_t topk, int64_t E,
                                      int64_t N, int64_t K, void* y, void* workspace, int sm_count,
                                      cudaStream_t stream, char* msg, size_t msg_len) {
  snprintf(msg, msg_len, "[gather_qmm] kernel not built yet");
  return NVFP4_ERR_UNSUPPORTED;
}
}  // namespace nvfp4
