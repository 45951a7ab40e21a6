// combine.cuh -- scatter-back, weighted combine and shared add (Kimi K2 "Add
// shared output" page: new_x[idxs] = outs, weighted sum over k, cast back to
// the row dtype, plus the shared expert's output).  Each token gathers its k
// expert rows through the inverse permutation -- the scatter-back is fused
// into the read -- accumulates in fp32 (FMA, slot order), rounds to the row
// dtype, adds the shared row and rounds again (bf16, nearest-even).  One CTA
// per token (grid-stride), 16-byte vectors when the row size allows.
#pragma once

#include <type_traits>

#include "rows_common.cuh"

namespace mr {

__device__ __forceinline__ void bf16x2_unpack(uint32_t u, float& lo, float& hi) {
  lo = __uint_as_float(u << 16);
  hi = __uint_as_float(u & 0xffff0000u);
}

__device__ __forceinline__ uint32_t bf16x2_pack_rn(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// bf16 rows, 8 elements (one uint4) per vector.  `src` locates the expert
// rows of each slot (SlotRowsLocal: one expert-sorted buffer through inv;
// SlotRowsPeer: the owners' output buffers, peer memory included).
template <typename Src>
__global__ void __launch_bounds__(kRowThreads)
    combine_bf16_vec_kernel(Src src, const float* __restrict__ w,
                            const uint4* __restrict__ shared, uint4* __restrict__ y, long T,
                            long nvec, int k) {
  __shared__ const uint4* row[kRowMaxK];
  __shared__ float wt[kRowMaxK];
  for (long t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      row[threadIdx.x] = src.row(t, threadIdx.x, k, nvec);
      wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (long v = threadIdx.x; v < nvec; v += kRowThreads) {
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll 8
      for (int j = 0; j < k; ++j) {
        const uint4* r = row[j];
        if (!r) continue;
        const uint4 e = src.load(r + v);
        const float wj = wt[j];
        float lo, hi;
        bf16x2_unpack(e.x, lo, hi); acc[0] = fmaf(wj, lo, acc[0]); acc[1] = fmaf(wj, hi, acc[1]);
        bf16x2_unpack(e.y, lo, hi); acc[2] = fmaf(wj, lo, acc[2]); acc[3] = fmaf(wj, hi, acc[3]);
        bf16x2_unpack(e.z, lo, hi); acc[4] = fmaf(wj, lo, acc[4]); acc[5] = fmaf(wj, hi, acc[5]);
        bf16x2_unpack(e.w, lo, hi); acc[6] = fmaf(wj, lo, acc[6]); acc[7] = fmaf(wj, hi, acc[7]);
      }
      uint4 o;
      if (shared) {
        const uint4 sv = __ldg(shared + t * nvec + v);
        const uint32_t s4[4] = {sv.x, sv.y, sv.z, sv.w};
        uint32_t r4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float slo, shi;
          bf16x2_unpack(s4[q], slo, shi);
          r4[q] = bf16x2_pack_rn(bf16_round(acc[2 * q]) + slo, bf16_round(acc[2 * q + 1]) + shi);
        }
        o = make_uint4(r4[0], r4[1], r4[2], r4[3]);
      } else {
        o = make_uint4(bf16x2_pack_rn(acc[0], acc[1]), bf16x2_pack_rn(acc[2], acc[3]),
                       bf16x2_pack_rn(acc[4], acc[5]), bf16x2_pack_rn(acc[6], acc[7]));
      }
      st_stream(y + t * nvec + v, o);
    }
    __syncthreads();
  }
}

// fp32 rows, 4 elements (one float4) per vector.
template <typename Src>
__global__ void __launch_bounds__(kRowThreads)
    combine_f32_vec_kernel(Src src, const float* __restrict__ w,
                           const float4* __restrict__ shared, float4* __restrict__ y, long T,
                           long nvec, int k) {
  __shared__ const float4* row[kRowMaxK];
  __shared__ float wt[kRowMaxK];
  for (long t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      row[threadIdx.x] = src.row(t, threadIdx.x, k, nvec);
      wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (long v = threadIdx.x; v < nvec; v += kRowThreads) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < k; ++j) {
        const float4* r = row[j];
        if (!r) continue;
        const float4 e = src.load(r + v);
        const float wj = wt[j];
        acc.x = fmaf(wj, e.x, acc.x);
        acc.y = fmaf(wj, e.y, acc.y);
        acc.z = fmaf(wj, e.z, acc.z);
        acc.w = fmaf(wj, e.w, acc.w);
      }
      if (shared) {
        const float4 s = __ldg(shared + t * nvec + v);
        acc.x += s.x;
        acc.y += s.y;
        acc.z += s.z;
        acc.w += s.w;
      }
      st_stream(y + t * nvec + v, acc);
    }
    __syncthreads();
  }
}

// Any row size, element by element (Src over uint16_t for bf16 rows, float
// for fp32).
template <bool BF16, typename Src>
__global__ void __launch_bounds__(kRowThreads)
    combine_scalar_kernel(Src src, const float* __restrict__ w,
                          const void* __restrict__ sharedv, void* __restrict__ yv, long T,
                          long d, int k) {
  using E = typename std::conditional<BF16, uint16_t, float>::type;
  __shared__ const E* row[kRowMaxK];
  __shared__ float wt[kRowMaxK];
  for (long t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      row[threadIdx.x] = src.row(t, threadIdx.x, k, d);
      wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (long c = threadIdx.x; c < d; c += kRowThreads) {
      float acc = 0.0f;
      for (int j = 0; j < k; ++j) {
        const E* r = row[j];
        if (!r) continue;
        const E raw = src.load(r + c);
        float e;
        if constexpr (BF16) e = mr_bf16_to_f32(raw); else e = raw;
        acc = fmaf(wt[j], e, acc);
      }
      if (BF16) {
        float out = bf16_round(acc);
        if (sharedv) out = out + mr_bf16_to_f32(static_cast<const uint16_t*>(sharedv)[t * d + c]);
        __nv_bfloat16 b = __float2bfloat16_rn(out);
        static_cast<uint16_t*>(yv)[t * d + c] = *reinterpret_cast<uint16_t*>(&b);
      } else {
        if (sharedv) acc += static_cast<const float*>(sharedv)[t * d + c];
        static_cast<float*>(yv)[t * d + c] = acc;
      }
    }
    __syncthreads();
  }
}

}  // namespace mr
