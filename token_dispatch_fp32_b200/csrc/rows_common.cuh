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

// Store of an output row that is not read again by this kernel: streaming
// (evict-first) for the vector and word types.
template <typename V>
__device__ __forceinline__ void st_stream(V* p, const V& v) {
  __stcs(p, v);
}
template <>
__device__ __forceinline__ void st_stream<uint16_t>(uint16_t* p, const uint16_t& v) {
  *p = v;
}

}  // namespace mr
