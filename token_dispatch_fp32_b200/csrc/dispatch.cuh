// dispatch.cuh -- moe_infer dispatch bookkeeping (Kimi K2 "Add shared output"
// page, moe_infer): tokens_per_expert, the running expert offsets and the
// stable expert-sorted permutation idxs = argsort(topk_ids.view(-1)), plus its
// inverse.  A counting sort in three launches:
//   1. count:   each CTA histograms a fixed chunk of the flat ids in shared
//               memory with warp-aggregated atomics (__match_any_sync).
//   2. scan:    one CTA turns the per-chunk histograms into counts, offsets
//               and each chunk's starting position per expert.
//   3. scatter: each CTA re-reads its chunk; each warp owns a contiguous
//               sub-chunk, so (chunk base + warp prefix + in-warp rank) gives
//               a stable position without any global atomics.
#pragma once

#include "mr_common.cuh"

namespace mr {

constexpr int kDispThreads = 256;
constexpr int kDispWarps = kDispThreads / 32;
constexpr int kDispChunk = 1024;                     // flat entries per CTA
constexpr int kDispSub = kDispChunk / kDispWarps;    // entries per warp
constexpr int kDispMaxExperts = 1024;

__host__ __device__ inline long disp_num_chunks(long n) { return (n + kDispChunk - 1) / kDispChunk; }

// Valid expert id, or -1 for one that is out of range (raises the flag once
// per warp that sees it).
__device__ __forceinline__ int disp_load(const int32_t* __restrict__ idx, long i, long n, int N_r,
                                         bool* bad) {
  if (i >= n) return -1;
  const int e = idx[i];
  if (e < 0 || e >= N_r) {
    *bad = true;
    return -1;
  }
  return e;
}

__global__ void __launch_bounds__(kDispThreads)
    dispatch_count_kernel(const int32_t* __restrict__ idx, long n, int N_r,
                          int32_t* __restrict__ chunk_hist) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < N_r; e += kDispThreads) hist[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long base = (long)blockIdx.x * kDispChunk + (long)warp * kDispSub;
  bool bad = false;
  for (int r = 0; r < kDispSub; r += 32) {
    const int e = disp_load(idx, base + r + lane, n, N_r, &bad);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[e], __popc(peers));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) mr_raise(MR_FLAG_BAD_INDEX);
  __syncthreads();
  for (int e = threadIdx.x; e < N_r; e += kDispThreads)
    chunk_hist[(long)blockIdx.x * N_r + e] = hist[e];  // chunk-major [chunk][expert]
}

// One CTA of 1024 threads; chunk_hist is [nchunks][N_r].  Q = 1024 / N_r
// (rounded down to a power of two) threads share an expert, each owning a
// contiguous range of chunks, so all loads of a phase are independent and
// coalesced across experts.  Produces counts and offsets (block scan over the
// expert totals) and replaces chunk_hist[c][e] by the position in perm where
// chunk c's first entry of expert e goes.
__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(int32_t* __restrict__ chunk_hist, long nchunks, int N_r, long n,
                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                         int32_t* __restrict__ perm) {
  __shared__ int part[1024];  // [q][e] partial sums
  __shared__ int start_e[kDispMaxExperts];
  __shared__ int warp_tot[32];
  __shared__ int total_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int Q = 1;
  while (Q * 2 * N_r <= 1024) Q *= 2;
  const int e = tid % N_r, q = tid / N_r;
  const bool active = q < Q;
  const long span = (nchunks + Q - 1) / Q;
  const long c_lo = active ? q * span : 0;
  const long c_hi = active ? (c_lo + span < nchunks ? c_lo + span : nchunks) : 0;
  // 1. partial sums over this thread's chunk range
  int sum = 0;
#pragma unroll 8
  for (long c = c_lo; c < c_hi; ++c) sum += chunk_hist[c * N_r + e];
  if (active) part[q * N_r + e] = sum;
  __syncthreads();
  // 2. expert totals and their exclusive scan (thread t = expert t)
  int cnt = 0;
  if (tid < N_r)
    for (int qq = 0; qq < Q; ++qq) cnt += part[qq * N_r + tid];
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = warp_tot[lane];
    int ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += v;
    }
    warp_tot[lane] = ti - t;
    if (lane == 31) total_s = ti;
  }
  __syncthreads();
  if (tid < N_r) {
    const int excl = warp_tot[warp] + incl - cnt;
    counts[tid] = cnt;
    offsets[tid] = excl;
    start_e[tid] = excl;
  }
  __syncthreads();
  // 3. starting position of each chunk: expert start + earlier ranges + running sum
  if (active) {
    int run = start_e[e];
    for (int qq = 0; qq < q; ++qq) run += part[qq * N_r + e];
#pragma unroll 8
    for (long c = c_lo; c < c_hi; ++c) {
      const int h = chunk_hist[c * N_r + e];
      chunk_hist[c * N_r + e] = run;
      run += h;
    }
  }
  const int total = total_s;
  if (tid == 0) offsets[N_r] = total;
  // slots of dropped (out-of-range) entries
  for (long i = total + tid; i < n; i += 1024) perm[i] = -1;
}

__global__ void __launch_bounds__(kDispThreads)
    dispatch_scatter_kernel(const int32_t* __restrict__ idx, long n, int N_r,
                            const int32_t* __restrict__ chunk_base, int32_t* __restrict__ perm,
                            int32_t* __restrict__ inv) {
  extern __shared__ int wbase[];  // [kDispWarps][N_r]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kDispWarps * N_r; i += kDispThreads) wbase[i] = 0;
  __syncthreads();
  const long base = (long)blockIdx.x * kDispChunk + (long)warp * kDispSub;
  int* mine = wbase + warp * N_r;
  bool bad = false;
  // per-warp histogram of this warp's sub-chunk
  for (int r = 0; r < kDispSub; r += 32) {
    const int e = disp_load(idx, base + r + lane, n, N_r, &bad);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) mine[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // warp-exclusive prefix per expert, offset by this chunk's base
  for (int e = threadIdx.x; e < N_r; e += kDispThreads) {
    int run = chunk_base[(long)blockIdx.x * N_r + e];
#pragma unroll
    for (int w = 0; w < kDispWarps; ++w) {
      const int h = wbase[w * N_r + e];
      wbase[w * N_r + e] = run;
      run += h;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kDispSub; r += 32) {
    const long i = base + r + lane;
    const int e = disp_load(idx, i, n, N_r, &bad);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int pos = mine[e] + __popc(peers & lt);
      perm[pos] = (int32_t)i;
      if (inv) inv[i] = pos;
    } else if (i < n && inv) {
      inv[i] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) mine[e] += __popc(peers);
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// The same counting sort in ONE cooperative launch (every CTA resident):
//   phase 1  CTA c histograms chunk c (as dispatch_count_kernel);
//   barrier
//   phase 2  CTA j owns experts [j*E, (j+1)*E): their totals, and each chunk's
//            exclusive prefix within the expert's column (in place);
//   barrier
//   phase 3  every CTA scans the expert totals (offsets), CTA 0 writes counts,
//            offsets and the dropped slots' -1, and CTA c scatters chunk c (as
//            dispatch_scatter_kernel) from base offsets[e] + prefix[c][e].
// The barrier counter lives in the workspace and is zeroed before the launch;
// each wait is bounded (MR_WAIT_LIMIT_NS): a CTA that gives up raises
// MR_FLAG_TIMEOUT and skips the remaining phases.
struct DispFusedWs {
  int* barrier;      // 1 int (zeroed by the host before the launch)
  int32_t* hist;     // [nchunks][N_r]
  int32_t* totals;   // [N_r]
};

__device__ __forceinline__ bool disp_grid_barrier(int* counter, int target) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(counter, 1);
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      int v;
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
      if (v >= target) break;
      if (it == 0) t0 = mr_globaltimer_ns();
      if ((it & 63u) == 63u && mr_globaltimer_ns() - t0 > MR_WAIT_LIMIT_NS) {
        mr_raise(MR_FLAG_TIMEOUT);
        ok = 0;
        break;
      }
      // the barrier usually opens within a few microseconds: poll without
      // sleeping first, then back off
      if (it >= 2048u) __nanosleep(64);
    }
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

__global__ void __launch_bounds__(kDispThreads)
    dispatch_fused_kernel(const int32_t* __restrict__ idx, long n, int N_r, DispFusedWs ws,
                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                          int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ int sm[];  // max(kDispThreads, kDispWarps * N_r) ints, reused by the phases
  __shared__ int start_s[kDispMaxExperts];
  __shared__ int warp_tot[kDispWarps];
  __shared__ int ids_s[kDispChunk];  // this chunk's ids from phase 1 (-1: none)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int nchunks = gridDim.x, c = blockIdx.x;
  const long base = (long)c * kDispChunk + (long)warp * kDispSub;
  bool bad = false;

  // ---- phase 1: chunk histogram
  for (int e = tid; e < N_r; e += kDispThreads) sm[e] = 0;
  __syncthreads();
  for (int r = 0; r < kDispSub; r += 32) {
    const int e = disp_load(idx, base + r + lane, n, N_r, &bad);
    ids_s[warp * kDispSub + r + lane] = e;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sm[e], __popc(peers));
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) mr_raise(MR_FLAG_BAD_INDEX);
  __syncthreads();
  for (int e = tid; e < N_r; e += kDispThreads) ws.hist[(long)c * N_r + e] = sm[e];
  if (!disp_grid_barrier(ws.barrier, nchunks)) return;

  // ---- phase 2: this CTA's experts: totals and per-chunk exclusive prefix
  {
    const int E = (N_r + nchunks - 1) / nchunks;  // experts per CTA
    const int e0 = c * E, e_end = e0 + E < N_r ? e0 + E : N_r;
    if (E > kDispThreads / 2) {
      // few chunks: one thread per expert, serial over the chunks
      for (int e = e0 + tid; e < e_end; e += kDispThreads) {
        int run = 0;
        for (long cc = 0; cc < nchunks; ++cc) {
          const int h = __ldcg(&ws.hist[cc * N_r + e]);
          ws.hist[cc * N_r + e] = run;
          run += h;
        }
        ws.totals[e] = run;
      }
    } else {
      // Q >= 2 threads per expert, each a contiguous range of chunks
      int Q = 1;
      while (Q * 2 * E <= kDispThreads) Q *= 2;
      const int el = tid % E, q = tid / E;
      const int e = e0 + el;
      const bool active = q < Q && e < e_end;
      const long span = ((long)nchunks + Q - 1) / Q;
      const long c_lo = active ? q * span : 0;
      const long c_hi = active ? (c_lo + span < nchunks ? c_lo + span : nchunks) : 0;
      int sum = 0;
      for (long cc = c_lo; cc < c_hi; ++cc) sum += __ldcg(&ws.hist[cc * N_r + e]);
      if (q < Q) sm[q * E + el] = sum;
      __syncthreads();
      if (active) {
        int run = 0;
        for (int qq = 0; qq < q; ++qq) run += sm[qq * E + el];
        if (q == Q - 1) ws.totals[e] = run + sum;
        for (long cc = c_lo; cc < c_hi; ++cc) {
          const int h = __ldcg(&ws.hist[cc * N_r + e]);
          ws.hist[cc * N_r + e] = run;
          run += h;
        }
      }
    }
  }
  if (!disp_grid_barrier(ws.barrier, 2 * nchunks)) return;

  // ---- phase 3a: expert offsets (every CTA; exclusive scan of the totals)
  {
    constexpr int kPer = kDispMaxExperts / kDispThreads;  // 4
    int v[kPer], loc = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid * kPer + j;
      v[j] = e < N_r ? __ldcg(&ws.totals[e]) : 0;
      loc += v[j];
    }
    int incl = loc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int wex = 0;
    for (int w = 0; w < warp; ++w) wex += warp_tot[w];
    int run = wex + incl - loc;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = tid * kPer + j;
      if (e < N_r) {
        start_s[e] = run;
        if (c == 0) {
          counts[e] = v[j];
          offsets[e] = run;
        }
      }
      run += v[j];
    }
    __syncthreads();
    if (c == 0) {
      int total = 0;
      for (int w = 0; w < kDispWarps; ++w) total += warp_tot[w];
      if (tid == 0) offsets[N_r] = total;
      for (long i = total + tid; i < n; i += kDispThreads) perm[i] = -1;  // dropped slots
    }
  }

  // ---- phase 3b: stable scatter of this chunk
  int* wbase = sm;  // [kDispWarps][N_r]
  for (int i = tid; i < kDispWarps * N_r; i += kDispThreads) wbase[i] = 0;
  __syncthreads();
  int* mine = wbase + warp * N_r;
  for (int r = 0; r < kDispSub; r += 32) {
    const int e = ids_s[warp * kDispSub + r + lane];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(peers) - 1) mine[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < N_r; e += kDispThreads) {
    int run = start_s[e] + __ldcg(&ws.hist[(long)c * N_r + e]);
#pragma unroll
    for (int w = 0; w < kDispWarps; ++w) {
      const int h = wbase[w * N_r + e];
      wbase[w * N_r + e] = run;
      run += h;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int r = 0; r < kDispSub; r += 32) {
    const long i = base + r + lane;
    const int e = ids_s[warp * kDispSub + r + lane];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int pos = mine[e] + __popc(peers & lt);
      perm[pos] = (int32_t)i;
      if (inv) inv[i] = pos;
    } else if (i < n && inv) {
      inv[i] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) mine[e] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace mr
