// bwd_bf16.cuh — backward pass (placeholder until the tensor-core kernel lands).
#pragma once
#include "common.cuh"

namespace fa {

inline fa_status bwd_launch(const void*, const void*, const void*, const void*, const float*, const void*, void*,
                            void*, void*, fa_dtype, int, int, int, int, int, int, float, int, void*, cudaStream_t,
                            uint64_t) {
  return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
