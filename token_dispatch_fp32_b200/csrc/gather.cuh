// gather.cuh -- sorted_tokens = x[idxs // k] (Kimi K2 "Add shared output"
// page, moe_infer).  With the inverse permutation each token row is read once
// and written to its k expert-sorted positions (read d, write k*d elements);
// with only perm each sorted row fetches its token row.  One CTA per token
// (grid-stride); 32-byte vectors for local rows of a 32-byte multiple,
// 16-byte vectors when the row size allows, elements otherwise.
// (A copy-engine variant -- cp.async.bulk row loads into a shared-memory ring
// and k bulk stores per row -- measured no faster on the full DeepSeek-V3
// batch, so the plain vector copy stays.)
#pragma once

#include "rows_common.cuh"

namespace mr {

// 128 bytes in flight per thread (eight 16-byte or four 32-byte vectors) and
// streaming stores: 340 us on the full DeepSeek-V3 batch against 354 us with
// 64 bytes and plain stores (measured sweep, 16-byte vectors).
template <typename V>
__host__ __device__ constexpr int gather_unroll() {
  return sizeof(V) >= 16 ? (int)(128 / sizeof(V)) : 8;
}

// Each token row read once, stored to the k rows `dst` names for its slots
// (SlotRowsLocal: the expert-sorted buffer through inv; SlotRowsPeer: the
// receive buffers of the experts' owners, peer memory included).
template <typename V, typename Dst>
__global__ void __launch_bounds__(kRowThreads)
    gather_inv_kernel(const V* __restrict__ x, long T, long nvec, int k, Dst dst) {
  constexpr int U = gather_unroll<V>();
  __shared__ V* out_row[kRowMaxK];
  for (long t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) out_row[threadIdx.x] = dst.row(t, threadIdx.x, k, nvec);
    __syncthreads();
    const V* src = x + t * nvec;
    for (long v0 = threadIdx.x; v0 < nvec; v0 += U * kRowThreads) {
      V val[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const long v = v0 + (long)u * kRowThreads;
        if (v < nvec) val[u] = ld_stream(src + v);
      }
      for (int j = 0; j < k; ++j) {
        V* out = out_row[j];
        if (!out) continue;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const long v = v0 + (long)u * kRowThreads;
          if (v < nvec) st_stream(out + v, val[u]);
        }
      }
    }
    __syncthreads();
  }
  // stores into other GPUs' memory: ordered before whatever this GPU does
  // next (the collective that tells the owners their rows are in)
  if (Dst::kPeer) __threadfence_system();
}

template <typename V>
__global__ void __launch_bounds__(kRowThreads)
    gather_perm_kernel(const V* __restrict__ x, long rows, long nvec, int k,
                       const int32_t* __restrict__ perm, V* __restrict__ xs) {
  for (long i = blockIdx.x; i < rows; i += gridDim.x) {
    const long p = perm[i];
    if (p < 0) continue;
    const V* src = x + (p / k) * nvec;
    V* out = xs + i * nvec;
    for (long v = threadIdx.x; v < nvec; v += kRowThreads) out[v] = ld_stream(src + v);
  }
}

}  // namespace mr
