// combine.cuh -- scatter-back, weighted combine and shared add (Kimi K2 "Add
// shared output" page: new_x[idxs] = outs, weighted sum over k, cast back to
// the row dtype, plus the shared expert's output).  Each token gathers its k
// expert rows through the inverse permutation -- the scatter-back is fused
// into the read -- accumulates in fp32 (FMA, slot order), rounds to the row
// dtype, adds the shared row and rounds again (bf16, nearest-even).  One CTA
// per token (grid-stride); bf16 rows move in 32-byte vectors when they are
// local and 32-byte multiples, 16-byte vectors when the row size allows.
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

// bf16 rows, two elements per 32-bit word of a vector V (uint4: 8 elements;
// Vec32: 16).  `src` locates the expert rows of each slot (SlotRowsLocal: one
// expert-sorted buffer through inv; SlotRowsPeer: the owners' output buffers,
// peer memory included).  The loads of up to kCombineGroup rows and of the
// shared row are issued before the group's FMAs, so a thread keeps that many
// vectors in flight; the FMAs still run in slot order.
constexpr int kCombineGroup = 8;

template <typename V, typename Src>
__global__ void __launch_bounds__(kRowThreads)
    combine_bf16_vec_kernel(Src src, const float* __restrict__ w,
                            const V* __restrict__ shared, V* __restrict__ y, long T, long nvec,
                            int k) {
  constexpr int W = (int)(sizeof(V) / 4);  // bf16 pairs per vector
  __shared__ const V* row[kRowMaxK];
  __shared__ float wt[kRowMaxK];
  for (long t = blockIdx.x; t < T; t += gridDim.x) {
    if (threadIdx.x < k) {
      row[threadIdx.x] = src.row(t, threadIdx.x, k, nvec);
      wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (long v = threadIdx.x; v < nvec; v += kRowThreads) {
      float acc[2 * W];
#pragma unroll
      for (int q = 0; q < 2 * W; ++q) acc[q] = 0.0f;
      V sv{};
      if (shared) sv = ld_stream(shared + t * nvec + v);
      for (int j0 = 0; j0 < k; j0 += kCombineGroup) {
        V e[kCombineGroup];
#pragma unroll
        for (int u = 0; u < kCombineGroup; ++u) {
          const V* r = j0 + u < k ? row[j0 + u] : nullptr;
          e[u] = r ? src.load(r + v) : V{};
        }
#pragma unroll
        for (int u = 0; u < kCombineGroup; ++u) {
          if (j0 + u >= k || !row[j0 + u]) continue;
          const float wj = wt[j0 + u];
#pragma unroll
          for (int q = 0; q < W; ++q) {
            float lo, hi;
            bf16x2_unpack(word(e[u], q), lo, hi);
            acc[2 * q] = fmaf(wj, lo, acc[2 * q]);
            acc[2 * q + 1] = fmaf(wj, hi, acc[2 * q + 1]);
          }
        }
      }
      V o;
#pragma unroll
      for (int q = 0; q < W; ++q) {
        if (shared) {
          float slo, shi;
          bf16x2_unpack(word(sv, q), slo, shi);
          set_word(o, q,
                   bf16x2_pack_rn(bf16_round(acc[2 * q]) + slo, bf16_round(acc[2 * q + 1]) + shi));
        } else {
          set_word(o, q, bf16x2_pack_rn(acc[2 * q], acc[2 * q + 1]));
        }
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
