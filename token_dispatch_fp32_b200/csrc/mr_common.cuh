// mr_common.cuh -- device helpers shared by the libmr kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mr.h"

// Sticky per-device error flag (bit set; read and cleared by mr_get_error).
// The library is one translation unit, so the flag is defined here.
#define MR_FLAG_BAD_INDEX 1u
#define MR_FLAG_TIMEOUT 2u
__device__ unsigned int g_mr_error_flag = 0;

__device__ __forceinline__ void mr_raise(unsigned int f) { atomicOr(&g_mr_error_flag, f); }

__device__ __forceinline__ uint64_t mr_globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded waits give up after this long (then raise MR_FLAG_TIMEOUT).
#define MR_WAIT_LIMIT_NS 1000000000ull

// s = sigmoid(L) = 1 / (1 + e^-L) in fp32 (Kimi K2 "Normalize weights" page:
// logits.sigmoid()), with CUDA's fast exponential and division intrinsics: a
// few ulp for the O(1) logits of a router, and L -> -inf gives 0, L -> +inf 1.
__device__ __forceinline__ float mr_sigmoid(float L) {
  return __fdividef(1.0f, 1.0f + __expf(-L));
}

// Total order used by every top-k: larger value first, lower index on ties.
__device__ __forceinline__ bool mr_better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ float mr_bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------------------
// Warp-cooperative routing of one token from its N_r logits.
//
// Lane `l` owns experts e = l + 32*j, j < NJ (N_r <= 32*NJ).  Steps, in the
// pages' order (Kimi K2 "Normalize weights" page, MoEGate.forward;
// DeepSeek-V3.2-Exp "Normalize weights" page, Gate.forward):
//   s = sigmoid(L); c = s + b; if n_group > 1: group score = top-2 sum of c,
//   keep topk_group groups (warp argmax, lower group on ties), masked c =
//   -inf or 0.0; token top-k by repeated warp argmax (lower expert on ties);
//   w_j = (s_j / (sum s + 1e-20)) * route_scale.
// Lane j < k writes slot j.  L may live in shared or global memory.
// ---------------------------------------------------------------------------
template <int NJ>
__device__ __forceinline__ void mr_route_token_warp(const float* __restrict__ L,
                                                    const float* __restrict__ bias, int N_r,
                                                    int n_group, int topk_group, int k,
                                                    float route_scale, int mask_mode,
                                                    int32_t* __restrict__ idx_out,
                                                    float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int S = N_r / n_group;
  float s[NJ], m[NJ];
  int grp[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    if (e < N_r) {
      s[j] = mr_sigmoid(L[e]);
      m[j] = s[j] + (bias ? bias[e] : 0.0f);
      grp[j] = e / S;
    } else {
      s[j] = 0.0f;
      m[j] = -INFINITY;
      grp[j] = -1;
    }
  }

  if (n_group > 1) {
    // group scores: lane g ends up holding gs[g]
    float gs_mine = -INFINITY;
    for (int g = 0; g < n_group; ++g) {
      float a1 = -INFINITY, a2 = -INFINITY;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (grp[j] == g) {
          const float v = m[j];
          if (v > a1) {
            a2 = a1;
            a1 = v;
          } else if (v > a2) {
            a2 = v;
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float b1 = __shfl_xor_sync(0xffffffffu, a1, off);
        const float b2 = __shfl_xor_sync(0xffffffffu, a2, off);
        if (a1 >= b1) {
          a2 = fmaxf(a2, b1);
        } else {
          a2 = fmaxf(a1, b2);
          a1 = b1;
        }
      }
      if (lane == g) gs_mine = a1 + a2;
    }
    uint32_t kept = 0;
    for (int r = 0; r < topk_group; ++r) {
      const bool cand = lane < n_group && !((kept >> lane) & 1u);
      float v = cand ? gs_mine : -INFINITY;
      int id = cand ? lane : 0x7fffffff;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, id, off);
        if (mr_better(ov, oi, v, id)) {
          v = ov;
          id = oi;
        }
      }
      kept |= 1u << id;
    }
    const float fill = (mask_mode == MR_MASK_NEG_INF) ? -INFINITY : 0.0f;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (grp[j] >= 0 && !((kept >> grp[j]) & 1u)) m[j] = fill;
  }

  uint32_t taken = 0;
  int my_idx = 0;
  float my_s = 0.0f, den = 0.0f;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY, bs = 0.0f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      if (grp[j] >= 0 && !((taken >> j) & 1u) && mr_better(m[j], e, bv, bi)) {
        bv = m[j];
        bi = e;
        bs = s[j];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      const float os = __shfl_xor_sync(0xffffffffu, bs, off);
      if (mr_better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
        bs = os;
      }
    }
    if (lane == (bi & 31)) taken |= 1u << (bi >> 5);
    if (lane == r) {
      my_idx = bi;
      my_s = bs;
    }
    den += bs;
  }
  den += 1e-20f;
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = (my_s / den) * route_scale;
  }
}
