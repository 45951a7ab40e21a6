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

// Where the row of slot (t, j) lives, for the row movers: each policy returns
// its address (nullptr for a slot that has none) and loads from it.

// One buffer of expert-sorted rows, through the inverse permutation
// (row inv[t*k + j]; -1 for a dropped slot).
template <typename P>
struct SlotRowsLocal {
  static constexpr bool kPeer = false;
  P* base;
  const int32_t* inv;
  __device__ __forceinline__ P* row(long t, int j, int k, long nvec) const {
    const long r = inv[t * k + j];
    return r < 0 ? nullptr : base + r * nvec;
  }
  template <typename V>
  __device__ __forceinline__ V load(const V* p) const {
    return ld_stream(p);
  }
};

// Expert parallelism over peer memory: one buffer per rank (device pointers,
// this GPU's own or another GPU's mapped into this process), the experts
// owned in contiguous blocks of E_loc; slot (t, j) has row dest[t*k + j] in
// the buffer of expert idx[t*k + j]'s owner.  A slot whose id or row lies
// outside [0, N_r) x [0, capacity) has none.
constexpr int kEpMaxRanks = 64;
struct EpPeers {
  void* p[kEpMaxRanks];
};

template <typename P>
struct SlotRowsPeer {
  static constexpr bool kPeer = true;
  EpPeers bufs;
  const int32_t* idx;
  const int32_t* dest;
  int E_loc, N_r;
  long capacity;
  __device__ __forceinline__ P* row(long t, int j, int k, long nvec) const {
    const int g = idx[t * k + j];
    const long r = dest[t * k + j];
    if (g < 0 || g >= N_r || r < 0 || r >= capacity) return nullptr;
    return static_cast<P*>(bufs.p[g / E_loc]) + r * nvec;
  }
  // rows of other GPUs: loads through L2 (ld.global.cg), not the
  // non-coherent path
  template <typename V>
  __device__ __forceinline__ V load(const V* p) const {
    return __ldcg(p);
  }
};

}  // namespace mr
