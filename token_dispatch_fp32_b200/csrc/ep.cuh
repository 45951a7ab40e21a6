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

// ---- exchange over peer memory ---------------------------------------------
//
// Instead of two all-to-alls and a receive-side sort, every source writes
// each of its rows straight into the owner's receive buffer at the row's final
// place in the owner's local-expert-sorted order.  That place follows from
// all ranks' tokens_per_expert (C[s][g], the all-gathered counts) alone:
// owner o's buffer holds its experts in order, each expert's rows source by
// source, each source's rows in the source's stable order, so slot (t, j) of
// source s with expert g = o*E_loc + e, at position p of s's own sorted order,
// goes to row
//     sum_{e' < e} sum_{s'} C[s'][o*E_loc + e']     (the earlier local experts)
//   + sum_{s' < s} C[s'][g]                          (earlier sources, same expert)
//   + p - offsets[g]                                 (its place within s's segment)
// One CTA of 1024 threads rebuilds the per-expert part (base[g], one thread per
// expert) from C in shared memory, then maps its 4096 slots.

// idx/inv/offsets: this rank's top-k ids and mr_dispatch's inverse
// permutation and offsets; C [ep][N_r]; n = T*k.  Writes dest [n] (the row in
// the owner's buffer, -1 for a slot without one) and, from CTA 0, this rank's
// local_counts [E_loc] and local_offsets [E_loc + 1] as an owner, clamped to
// the capacity.  Counts below zero, or a row of C for this rank that
// disagrees with offsets, raise MR_FLAG_BAD_INDEX and leave every dest at -1
// and the local counts at 0; a row past the capacity is dropped (dest -1)
// and raises MR_FLAG_OVERFLOW.
__global__ void __launch_bounds__(kEpThreads)
    ep_dest_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ inv,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ C, long n,
                   int ep, int rank, int N_r, long capacity, int32_t* __restrict__ dest,
                   int32_t* __restrict__ local_counts, int32_t* __restrict__ local_offsets) {
  __shared__ int pre[kEpMaxSegments + 1];  // exclusive prefix of the column sums
  __shared__ int base[kEpMaxSegments];
  __shared__ int wsum[32];
  __shared__ int bad_s, over_s;
  const int tid = threadIdx.x;
  const int E_loc = N_r / ep;
  if (tid == 0) {
    bad_s = 0;
    over_s = 0;
  }
  __syncthreads();
  int colsum = 0, before = 0;
  if (tid < N_r) {
    for (int s = 0; s < ep; ++s) {
      const int c = C[(long)s * N_r + tid];
      if (c < 0) bad_s = 1;
      colsum += c;
      if (s < rank) before += c;
    }
    if (C[(long)rank * N_r + tid] != offsets[tid + 1] - offsets[tid]) bad_s = 1;
  }
  int total = 0;
  const int excl = ep_block_scan(tid < N_r ? colsum : 0, wsum, &total);
  if (tid < N_r) pre[tid] = excl;
  if (tid == 0) pre[N_r] = total;
  __syncthreads();
  const bool bad = bad_s != 0;
  if (tid < N_r) base[tid] = pre[tid] - pre[(tid / E_loc) * E_loc] + before;
  if (blockIdx.x == 0 && tid < E_loc) {
    const int g0 = rank * E_loc;
    const long lo = pre[g0 + tid] - pre[g0], hi = pre[g0 + tid + 1] - pre[g0];
    const long clo = bad ? 0 : (lo < capacity ? lo : capacity);
    const long chi = bad ? 0 : (hi < capacity ? hi : capacity);
    local_counts[tid] = (int32_t)(chi - clo);
    local_offsets[tid] = (int32_t)clo;
    if (tid == E_loc - 1) local_offsets[E_loc] = (int32_t)chi;
  }
  __syncthreads();
  const long i0 = (long)blockIdx.x * kEpRowsPerCta;
  const long i1 = i0 + kEpRowsPerCta < n ? i0 + kEpRowsPerCta : n;
  for (long i = i0 + tid; i < i1; i += kEpThreads) {
    long r = -1;
    const int g = idx[i];
    const int p = inv[i];
    if (!bad && g >= 0 && g < N_r && p >= 0) {
      r = (long)base[g] + (p - offsets[g]);
      if (r >= capacity) {
        over_s = 1;
        r = -1;
      } else if (r < 0 || p >= offsets[g + 1]) {
        bad_s = 1;  // inv and offsets disagree
        r = -1;
      }
    }
    dest[i] = (int32_t)r;
  }
  __syncthreads();
  if (tid == 0) {
    if (bad_s) mr_raise(MR_FLAG_BAD_INDEX);
    if (over_s) mr_raise(MR_FLAG_OVERFLOW);
  }
}

}  // namespace mr
