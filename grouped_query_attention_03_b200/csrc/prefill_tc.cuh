// prefill_tc.cuh -- tcgen05/TMEM causal-windowed prefill (bf16, sm_100a).
#pragma once

#include "common.cuh"

namespace gqa {
namespace pf {

inline bool supported(int) { return false; }

inline gqa_status launch(const void *, const void *, const void *, void *,
                         const int32_t *, int, int, int, int, int, int, float,
                         int32_t *, int, cudaStream_t) {
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace pf
}  // namespace gqa
