// lora_small_m.cuh — forward path for few tokens (memory-bound: W read once).
#pragma once

#include "lora_linear.h"
#include "sm100.cuh"

namespace lora {

// Token counts up to this use the small-M path.  0 = path disabled.
constexpr int64_t kSmallMMax = 0;

inline lora_status_t small_m_forward(const lora_linear_desc*, const void*, const void*, const void*, const void*,
                                     void*, float*, float*, uint32_t*, int, cudaStream_t) {
  return LORA_ERR_UNSUPPORTED;
}

}  // namespace lora
