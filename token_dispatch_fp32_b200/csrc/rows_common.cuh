// rows_common.cuh -- launch shape and load helper shared by the row movers
// (gather.cuh, combine.cuh).
#pragma once

#include "mr_common.cuh"

namespace mr {


constexpr int kRowThreads = 128;
constexpr int kRowUnroll = 4;
constexpr int kRowMaxK = 32;

template <typename V>
__device__ __forceinline__ V ld_stream(const V* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ uint16_t ld_stream<uint16_t>(const uint16_t* p) {
  return *p;
}

}  // namespace mr
