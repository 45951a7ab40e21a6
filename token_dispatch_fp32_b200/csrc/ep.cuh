// ep.cuh -- receive-side bookkeeping of the expert-parallel exchange (Kimi K2
// "Add shared output" page, moe_infer, the ep_size > 1 branch).
//
// With ep ranks, rank r owns the experts [r*E_loc, (r+1)*E_loc).  After the
// row all-to-all, rank r holds the rows it was sent source by source, and
// within a source in the source's expert-sorted order: the (source s, local
// expert e) segments in s-major order, segment (s, e) holding recv[s][e]
// rows.  The page labels each received row with e and argsorts the labels
// (taken stable).  The stable order has a closed form, so no sort runs here:
// row i of segment (s, e), at offset j within it, goes to
//     local_offsets[e] + sum_{s' < s} recv[s'][e] + j,
// local_offsets being the exclusive prefix of the column sums of recv
// (tokens_per_expert_post_gather).  One kernel: every CTA rebuilds those
// prefixes in shared memory (N_r = ep * E_loc <= 1024 segments, one per
// thread), then places its rows.
#pragma once

#include "mr_common.cuh"

namespace mr {

constexpr int kEpThreads = 1024;   // one thread per (source, expert) segment
constexpr int kEpMaxSegments = 1024;
constexpr int kEpRowsPerCta = 4096;

// Exclusive prefix of v over the CTA's 1024 threads (warp shuffles, then the
// 32 warp totals); also returns the total.  Every thread calls it.
__device__ __forceinline__ int ep_block_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = wsum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t += y;
    }
    wsum[lane] = t;  // inclusive over warps
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? wsum[warp - 1] : 0);
  *total = wsum[31];
  __syncthreads();
  return excl;
}

// recv [ep][E_loc] counts (device), R their expected sum.  Writes
// order[dest] = i and inv[i] = dest for every received row i (inv nullable),
// and (CTA 0) local_counts [E_loc], local_offsets [E_loc + 1].  A count
// below zero, or a sum other than R, raises the device flag and writes
// nothing.
__global__ void __launch_bounds__(kEpThreads)
    ep_recv_order_kernel(const int32_t* __restrict__ recv, int ep, int E_loc, long R,
                         int32_t* __restrict__ order, int32_t* __restrict__ inv,
                         int32_t* __restrict__ local_counts, int32_t* __restrict__ local_offsets) {
  __shared__ int seg_start[kEpMaxSegments + 1];
  __shared__ int dest_start[kEpMaxSegments];
  __shared__ int col_off[kEpMaxSegments];
  __shared__ int wsum[32];
  __shared__ int bad_s;
  const int tid = threadIdx.x;
  const int nseg = ep * E_loc;
  if (tid == 0) bad_s = 0;
  __syncthreads();
  const int c = tid < nseg ? recv[tid] : 0;
  if (c < 0) atomicOr(&bad_s, 1);
  // arrival order: segments (s, e) in s-major order
  int total = 0;
  const int start = ep_block_scan(c, wsum, &total);
  if (tid < nseg) seg_start[tid] = start;
  if (tid == 0) seg_start[nseg] = total;
  // column sums (tokens_per_expert_post_gather) and their exclusive prefix
  int colsum = 0;
  if (tid < E_loc)
    for (int s = 0; s < ep; ++s) colsum += recv[s * E_loc + tid];
  int ctot = 0;
  const int coff = ep_block_scan(tid < E_loc ? colsum : 0, wsum, &ctot);
  if (tid < E_loc) col_off[tid] = coff;
  __syncthreads();
  if (tid < nseg) {
    const int s = tid / E_loc, e = tid % E_loc;
    int before = 0;
    for (int sp = 0; sp < s; ++sp) before += recv[sp * E_loc + e];
    dest_start[tid] = col_off[e] + before;
  }
  if (total != R && tid == 0) bad_s = 1;
  __syncthreads();
  if (bad_s) {
    if (blockIdx.x == 0 && tid == 0) mr_raise(MR_FLAG_BAD_INDEX);
    return;
  }
  if (blockIdx.x == 0) {
    if (tid < E_loc) {
      local_counts[tid] = colsum;
      local_offsets[tid] = coff;
    }
    if (tid == 0) local_offsets[E_loc] = ctot;
  }
  const long r0 = (long)blockIdx.x * kEpRowsPerCta;
  const long r1 = r0 + kEpRowsPerCta < R ? r0 + kEpRowsPerCta : R;
  for (long i = r0 + tid; i < r1; i += kEpThreads) {
    // last segment whose start is <= i (empty segments share the next start)
    int lo = 0, hi = nseg;  // seg_start[lo] <= i < seg_start[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (seg_start[mid] <= i) lo = mid; else hi = mid;
    }
    const int dest = dest_start[lo] + (int)(i - seg_start[lo]);
    order[dest] = (int32_t)i;
    if (inv) inv[i] = dest;
  }
}

}  // namespace mr
