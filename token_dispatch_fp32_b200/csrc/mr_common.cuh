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
#define MR_FLAG_OVERFLOW 4u
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
// Scores and weights, with the scoring variants of the DeepSeek-V3.2-Exp
// "Normalize weights" page (Gate.forward): MR_SCORE_SOFTMAX takes
// s = softmax(L) over all experts and uses the scaled scores as weights
// without renormalisation; otherwise s = sigmoid(L) and the weights are
// renormalised by the sum of the k scores, + 1e-20 unless MR_NORM_NO_EPS.

// Scores of the lane's experts e = lane + 32*j (0 past N_r).
template <int NJ>
__device__ __forceinline__ void mr_scores_warp(const float* __restrict__ L, int N_r, int flags,
                                               float (&s)[NJ]) {
  const int lane = threadIdx.x & 31;
  if (flags & MR_SCORE_SOFTMAX) {
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (lane + 32 * j < N_r) mx = fmaxf(mx, L[lane + 32 * j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      s[j] = lane + 32 * j < N_r ? __expf(L[lane + 32 * j] - mx) : 0.0f;
      sum += s[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
#pragma unroll
    for (int j = 0; j < NJ; ++j) s[j] = s[j] / sum;
  } else {
#pragma unroll
    for (int j = 0; j < NJ; ++j) s[j] = lane + 32 * j < N_r ? mr_sigmoid(L[lane + 32 * j]) : 0.0f;
  }
}

// Weight of a chosen expert with score s_j; den = the sum of the k scores.
__device__ __forceinline__ float mr_weight(float s_j, float den, float route_scale, int flags) {
  if (flags & MR_SCORE_SOFTMAX) return s_j * route_scale;
  if (!(flags & MR_NORM_NO_EPS)) den += 1e-20f;
  return (s_j / den) * route_scale;
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
                                                    float* __restrict__ w_out, int flags = 0) {
  const int lane = threadIdx.x & 31;
  const int S = N_r / n_group;
  float s[NJ], m[NJ];
  int grp[NJ];
  mr_scores_warp<NJ>(L, N_r, flags, s);
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    if (e < N_r) {
      m[j] = s[j] + (bias ? bias[e] : 0.0f);
      grp[j] = e / S;
    } else {
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
      if (lane == g) gs_mine = (flags & MR_GROUP_MAX) ? a1 : a1 + a2;
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
  if (lane < k) {
    idx_out[lane] = my_idx;
    w_out[lane] = mr_weight(my_s, den, route_scale, flags);
  }
}

// The same routing with short dependency chains, for groups that are whole
// 32-expert columns of the lane layout (N_r / n_group a multiple of 32) or no
// groups, and k <= 32:
//   * every group's top-2 pair is reduced across the warp in one butterfly
//     (the groups' chains interleave) and the kept groups are found by
//     counting, for each group, the groups that beat it;
//   * tau = the k-th best of the 32 lane maxima of the masked scores: those
//     are k distinct experts, so the token's k-th best is >= tau;
//   * the scores >= tau (at least k, usually little more) are compacted into
//     `scratch` (warp-private shared memory, 96 words) and each one's place is
//     the number of candidates that beat it (value desc, index asc).
// More than 32 candidates (ties at the 0.0 fill, or tau = -inf) or other group
// shapes take mr_route_token_warp.  Results are those of mr_route_token_warp
// except for the order in which the k unbiased scores are summed.
template <int NJ>
__device__ __forceinline__ void mr_route_token_warp_fast(const float* __restrict__ L,
                                                         const float* __restrict__ bias, int N_r,
                                                         int n_group, int topk_group, int k,
                                                         float route_scale, int mask_mode,
                                                         int32_t* __restrict__ idx_out,
                                                         float* __restrict__ w_out,
                                                         float* scratch, int flags = 0) {
  const int lane = threadIdx.x & 31;
  const int S = N_r / n_group;
  if (k > 32 || (n_group > 1 && (S % 32 != 0 || n_group > NJ))) {
    mr_route_token_warp<NJ>(L, bias, N_r, n_group, topk_group, k, route_scale, mask_mode,
                            idx_out, w_out, flags);
    return;
  }
  float s[NJ], m[NJ];
  mr_scores_warp<NJ>(L, N_r, flags, s);
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    m[j] = e < N_r ? s[j] + (bias ? bias[e] : 0.0f) : -INFINITY;
  }
  if (n_group > 1) {
    const int jpg = S / 32;  // lane slots j per group: group of slot j is j / jpg
    int gj[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) gj[j] = jpg == 1 ? j : j / jpg;
    float a1[NJ], a2[NJ];
#pragma unroll
    for (int g = 0; g < NJ; ++g) {
      a1[g] = -INFINITY;
      a2[g] = -INFINITY;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (gj[j] == g) {
          a2[g] = fmaxf(a2[g], fminf(a1[g], m[j]));
          a1[g] = fmaxf(a1[g], m[j]);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int g = 0; g < NJ; ++g) {
        const float b1 = __shfl_xor_sync(0xffffffffu, a1[g], off);
        const float b2 = __shfl_xor_sync(0xffffffffu, a2[g], off);
        const float hi = fmaxf(a1[g], b1);
        a2[g] = fmaxf(fminf(a1[g], b1), fmaxf(a2[g], b2));
        a1[g] = hi;
      }
    }
    uint32_t kept = 0;
    const bool gmax = (flags & MR_GROUP_MAX) != 0;
#pragma unroll
    for (int g = 0; g < NJ; ++g) {
      if (g < n_group) {
        const float sg = gmax ? a1[g] : a1[g] + a2[g];
        int rank = 0;
#pragma unroll
        for (int o = 0; o < NJ; ++o) {
          const float so = gmax ? a1[o] : a1[o] + a2[o];
          if (o < n_group && o != g) rank += (so > sg || (so == sg && o < g)) ? 1 : 0;
        }
        if (rank < topk_group) kept |= 1u << g;
      }
    }
    const float fill = (mask_mode == MR_MASK_NEG_INF) ? -INFINITY : 0.0f;
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (lane + 32 * j < N_r && !((kept >> gj[j]) & 1u)) m[j] = fill;
  }
  // tau: the k-th best lane maximum (ties: lower lane first)
  float lm = -INFINITY;
#pragma unroll
  for (int j = 0; j < NJ; ++j) lm = fmaxf(lm, m[j]);
  int lr = 0;
#pragma unroll
  for (int o = 0; o < 32; ++o) {
    const float v = __shfl_sync(0xffffffffu, lm, o);
    lr += (v > lm || (v == lm && o < lane)) ? 1 : 0;
  }
  const uint32_t at = __ballot_sync(0xffffffffu, lr == k - 1);
  const float tau = __shfl_sync(0xffffffffu, lm, __ffs(at) - 1);
  // candidates: valid experts with masked score >= tau, compacted in slot order
  uint32_t bal[NJ];
  int n = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    bal[j] = __ballot_sync(0xffffffffu, lane + 32 * j < N_r && m[j] >= tau);
    n += __popc(bal[j]);
  }
  if (n > 32) {
    mr_route_token_warp<NJ>(L, bias, N_r, n_group, topk_group, k, route_scale, mask_mode,
                            idx_out, w_out, flags);
    return;
  }
  int base = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    if ((bal[j] >> lane) & 1u) {
      const int slot = base + __popc(bal[j] & ((1u << lane) - 1u));
      scratch[slot] = m[j];
      scratch[32 + slot] = s[j];
      scratch[64 + slot] = __int_as_float(lane + 32 * j);
    }
    base += __popc(bal[j]);
  }
  __syncwarp();
  float cv = -INFINITY, cs = 0.0f;
  int ci = 0x7fffffff, rank = 32;
  if (lane < n) {
    cv = scratch[lane];
    cs = scratch[32 + lane];
    ci = __float_as_int(scratch[64 + lane]);
    rank = 0;
    for (int o = 0; o < n; ++o)
      rank += mr_better(scratch[o], __float_as_int(scratch[64 + o]), cv, ci) ? 1 : 0;
  }
  float den = rank < k ? cs : 0.0f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  if (rank < k) {
    idx_out[rank] = ci;
    w_out[rank] = mr_weight(cs, den, route_scale, flags);
  }
  __syncwarp();  // scratch may be reused by the caller's next token
}
