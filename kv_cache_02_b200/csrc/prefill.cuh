// Causal GQA prefill (tcgen05 / TMEM / TMA). Not built yet: reports
// GQA_ERR_UNSUPPORTED.
#pragma once

#include "common.cuh"

namespace gqa {

inline int launch_prefill(void*, const void*, const void*, const void*, void*, void*, int, int, int, int, int, int,
                          float, cudaStream_t, int) {
  return GQA_ERR_UNSUPPORTED;
}

}  // namespace gqa
