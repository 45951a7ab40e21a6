// rows_common.cuh -- launch shape and load helper shared by the row movers
// (gather.cuh, combine.cuh).
#pragma once

#include "mr_common.cuh"

namespace mr {


constexpr int kRowThreads = 128;
constexpr int kRowMaxK = 32;

// 32-byte vector: sm_100 moves it with one load or store instruction
// (ld/st .v8.b32), half the instructions of 16-byte vectors.  The local row
// movers use it when the row size and every row base are multiples of 32
// bytes: on the full DeepSeek-V3 batch the gather takes 334 us with it
// against 346 us with 16-byte vectors, and the combine 362.5 us against
// 368.6 us (same-box A/B).
struct alignas(32) Vec32 {
  uint32_t w[8];
};

__device__ __forceinline__ uint32_t word(const uint4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t word(const Vec32& v, int q) { return v.w[q]; }
__device__ __forceinline__ void set_word(uint4& v, int q, uint32_t x) {
  if (q == 0) v.x = x;
  else if (q == 1) v.y = x;
  else if (q == 2) v.z = x;
  else v.w = x;
}
__device__ __forceinline__ void set_word(Vec32& v, int q, uint32_t x) { v.w[q] = x; }

template <typename V>
__device__ __forceinline__ V ld_stream(const V* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ uint16_t ld_stream<uint16_t>(const uint16_t* p) {
  return *p;
}
template <>
__device__ __forceinline__ Vec32 ld_stream<Vec32>(const Vec32* p) {
  Vec32 r;
  asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]),
                 "=r"(r.w[5]), "=r"(r.w[6]), "=r"(r.w[7])
               : "l"(p));
  return r;
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
template <>
__device__ __forceinline__ void st_stream<Vec32>(Vec32* p, const Vec32& v) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
               "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
               "r"(v.w[6]), "r"(v.w[7])
               : "memory");
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
