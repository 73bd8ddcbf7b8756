// paged.cuh -- history-only attention over a paged FP8 KV cache (sm_100a).
#pragma once

#include "ptx.cuh"

namespace attn {
namespace paged {

inline int launch(const uint16_t*, const uint8_t*, const uint8_t*, const int32_t*, int, int, int,
                  int, float, float, float, int, int, int, int, int, uint16_t*, cudaStream_t) {
    return -3;
}

}  // namespace paged
}  // namespace attn
