// route.cuh -- routing of tokens whose logits are in memory (Kimi K2
// "Normalize weights" page, MoEGate.forward after the linear map; DeepSeek-
// V3.2-Exp "Normalize weights" page, Gate.forward), for the tensor-core
// router when the caller's workspace holds its logits and for the split-K
// router of small batches: part[s][t][e] fp32, the slices s < KS added in
// slice order.
//
// P lanes route one token (P = 8, 16 or 32 consecutive lanes of a warp), lane
// j owning the contiguous experts [j*EL, (j+1)*EL), N = P*EL, so the work of
// a batch is spread over T*P threads -- thousands of warps, where a routing
// epilogue inside the GEMM has eight per SM.  Per token:
//   * L = sum of the slices; s = sigmoid(L) (or the softmax over the token's
//     N logits: the row maximum and the sum of exponentials meet by shuffles);
//   * groups: each group spans S/EL whole lanes; every lane's top-2 of
//     c = s + b (a tree of pair merges) meets its group's other lanes by
//     shuffles; every lane gathers the G group scores (the top-2 sum, or the
//     best score), keeps topk_group groups by counting the groups that beat
//     each one (lower group first on ties);
//   * top-k: the candidates >= tau (a lower bound on the k-th best: the
//     smallest of the kept groups' top-2 values, or with one group the k-th
//     largest of the lanes' maxima) are ranked by counting, each rank its
//     slot;
//   * else (a token with more candidates than lanes, or 2*topk_group < k)
//     k rounds: every lane offers the best of its experts not yet taken
//     (value desc, index asc); the token's best is found with two warp
//     reductions when a token has the whole warp (the largest value as an
//     order-preserving integer, then the smallest index among the lanes that
//     hold it), else by a shuffle tree, and its lane marks it taken.  A
//     masked score of -inf is never taken (the slot keeps index INT_MAX, as
//     in the GEMM's epilogue);
//   * weights = route_scale * s / (sum of the chosen s + 1e-20).
// Shapes outside this layout (a group inside a lane, groups not a power-of-
// two number of lanes) are routed by the GEMM's own epilogue instead.
#pragma once

#include "mr_common.cuh"

namespace mr {
namespace rt {

constexpr int kThreads = 256;
constexpr int kMaxN = 512;
constexpr int kTop = 8;
constexpr int kMaxSlices = 4;  // slices added with all their loads in flight at once

struct Params {
  const float* part;  // [KS][T][N]
  int KS, T, N, P;    // P lanes per token, N = P * EL
  int n_group, topk_group, k, mask_mode, flags;
  float route_scale;
  const float* bias;
  int32_t* idx_out;
  float* w_out;
  float* logits_out;
};

// Top-2 of the union of two top-2 pairs (a1 >= a2, b1 >= b2).
__device__ __forceinline__ void merge2(float& a1, float& a2, float b1, float b2) {
  const float hi = fmaxf(a1, b1);
  a2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
  a1 = hi;
}

template <int EL>
__global__ void __launch_bounds__(kThreads)
    route_kernel(const Params p) {
  __shared__ float bs[kMaxN];
  // the bias does not come from the GEMM: fetch it while the GEMM runs
  for (int e = threadIdx.x; e < p.N; e += kThreads) bs[e] = p.bias ? p.bias[e] : 0.0f;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  const int P = p.P, N = p.N, k = p.k;
  const int j = threadIdx.x % P;                                 // lane within the token
  const long t = (long)blockIdx.x * (kThreads / P) + threadIdx.x / P;
  const bool live = t < p.T;
  const int e0 = j * EL;
  const int lane = threadIdx.x & 31;
  const int seg0 = lane - j;  // first lane of this token's segment
  const unsigned full = 0xffffffffu;

  // ---- logits: the slices added in order (all loads issued first) ----
  float L[EL];
  const long stride = (long)p.T * N;
  const float4* src = reinterpret_cast<const float4*>(p.part + (live ? t : 0) * N + e0);
  if (p.KS > kMaxSlices) {
    // more slices (the split-K GEMM of small batches): slice by slice, each
    // slice's loads issued together, the sums still in slice order
    constexpr int kSlUnroll = EL <= 8 ? 4 : (EL <= 16 ? 2 : 1);  // ~8 float4 loads in flight
    float4 a[EL / 4];
#pragma unroll
    for (int m = 0; m < EL / 4; ++m) a[m] = live ? src[m] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll kSlUnroll
    for (int sl = 1; sl < p.KS; ++sl) {
      float4 b[EL / 4];
#pragma unroll
      for (int m = 0; m < EL / 4; ++m)
        b[m] = live ? src[sl * stride / 4 + m] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int m = 0; m < EL / 4; ++m) {
        a[m].x += b[m].x;
        a[m].y += b[m].y;
        a[m].z += b[m].z;
        a[m].w += b[m].w;
      }
    }
#pragma unroll
    for (int m = 0; m < EL / 4; ++m) {
      L[4 * m] = a[m].x;
      L[4 * m + 1] = a[m].y;
      L[4 * m + 2] = a[m].z;
      L[4 * m + 3] = a[m].w;
    }
  } else {
#pragma unroll
    for (int m = 0; m < EL / 4; ++m) {
      float4 v[kMaxSlices];
#pragma unroll
      for (int sl = 0; sl < kMaxSlices; ++sl)
        v[sl] = (live && sl < p.KS) ? src[sl * stride / 4 + m] : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 a = v[0];
#pragma unroll
      for (int sl = 1; sl < kMaxSlices; ++sl)
        if (sl < p.KS) {
          a.x += v[sl].x;
          a.y += v[sl].y;
          a.z += v[sl].z;
          a.w += v[sl].w;
        }
      L[4 * m] = a.x;
      L[4 * m + 1] = a.y;
      L[4 * m + 2] = a.z;
      L[4 * m + 3] = a.w;
    }
  }
  if (p.logits_out && live)
#pragma unroll
    for (int i = 0; i < EL; ++i) p.logits_out[t * N + e0 + i] = L[i];

  // ---- scores ----
  float s[EL];
  if (p.flags & MR_SCORE_SOFTMAX) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EL; ++i) mx = fmaxf(mx, L[i]);
    for (int off = 1; off < P; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < EL; ++i) {
      s[i] = __expf(L[i] - mx);
      z += s[i];
    }
    for (int off = 1; off < P; off <<= 1) z += __shfl_xor_sync(full, z, off);
    const float inv = 1.0f / z;
#pragma unroll
    for (int i = 0; i < EL; ++i) s[i] *= inv;
  } else {
#pragma unroll
    for (int i = 0; i < EL; ++i) s[i] = mr_sigmoid(L[i]);
  }

  // ---- this lane's top-2 of c = s + b ----
  float c[EL];
#pragma unroll
  for (int i = 0; i < EL; ++i) c[i] = s[i] + bs[e0 + i];
  float a1 = -INFINITY, a2 = -INFINITY;
  {
    float p1[EL / 2], p2[EL / 2];
#pragma unroll
    for (int i = 0; i < EL / 2; ++i) {
      p1[i] = fmaxf(c[2 * i], c[2 * i + 1]);
      p2[i] = fminf(c[2 * i], c[2 * i + 1]);
    }
#pragma unroll
    for (int i = 0; i < EL / 2; ++i) merge2(a1, a2, p1[i], p2[i]);
  }

  // ---- groups ----
  const int G = p.n_group;
  bool keep = true;
  if (G > 1) {
    const int S = N / G, LG = S / EL;  // lanes per group
    for (int off = 1; off < LG; off <<= 1) {
      const float b1 = __shfl_xor_sync(full, a1, off), b2 = __shfl_xor_sync(full, a2, off);
      merge2(a1, a2, b1, b2);
    }
    const bool gmax = (p.flags & MR_GROUP_MAX) != 0;
    const float my_sc = gmax ? a1 : a1 + a2;  // the score of this lane's group
    // lane j < G of the segment ranks group j: the groups that beat it
    // (lower group first on ties), read from each group's first lane
    const int gj = j < G ? j : 0;
    const float gj_sc = __shfl_sync(full, my_sc, seg0 + gj * LG);
    int rank = 0;
    for (int o = 0; o < G; ++o) {
      const float so = __shfl_sync(full, my_sc, seg0 + o * LG);
      rank += (so > gj_sc || (so == gj_sc && o < gj)) ? 1 : 0;
    }
    const bool kept_j = j < G && rank < p.topk_group;
    const uint32_t kept = __ballot_sync(full, kept_j) >> seg0;
    keep = ((kept >> (e0 / S)) & 1u) != 0;
  }

  // ---- masked scores ----
  const float fill = (G > 1 && p.mask_mode == MR_MASK_ZERO) ? 0.0f : -INFINITY;
#pragma unroll
  for (int i = 0; i < EL; ++i) c[i] = keep ? c[i] : fill;

  // ---- candidates: the scores >= tau, a lower bound on the k-th best ----
  // With groups, the kept groups' top-2 values are 2*topk_group distinct
  // experts, so when that is >= k the k-th best is >= the smallest of them;
  // with one group, the k largest of the lanes' maxima are k distinct
  // experts, so the k-th best is >= the k-th of them (a bitonic sort of the
  // lanes' maxima).  Every expert of the top-k is then a candidate and its
  // rank among the candidates (value desc, index asc) is its slot, found by
  // counting; the candidates go through shared memory, one slot per lane of
  // the token.  A warp with a token of more candidates than lanes (ties at
  // the 0.0 fill, say) takes the k rounds below instead -- the same result.
  // Measured (same-box A/Bs, outputs bit-identical): DeepSeek-V3 prefill
  // router 60.4 -> 56.3 us, Kimi K2 prefill router 142.4 -> 138.2 us (a
  // looser one-group bound, the smallest second-best of the ceil(k/2) lanes
  // with the largest maxima, left too many candidates: 140.3 -> 144.4 us).
  const bool grouped = G > 1 && 2 * p.topk_group >= k;  // the same for the whole grid
  if (grouped || (G == 1 && k <= P)) {
    float tau;
    if (grouped) {
      tau = keep ? a2 : INFINITY;  // a2: the group's second best
      for (int off = 1; off < P; off <<= 1) tau = fminf(tau, __shfl_xor_sync(full, tau, off));
    } else {
      // one group: the k-th largest of the lanes' maxima (k distinct experts
      // are >= it), by a bitonic sort of the token's P lanes, descending
      float v = a1;
      for (int size = 2; size <= P; size <<= 1)
        for (int st = size >> 1; st > 0; st >>= 1) {
          const float o = __shfl_xor_sync(full, v, st);
          v = (((j & st) == 0) == ((j & size) == 0)) ? fmaxf(v, o) : fminf(v, o);
        }
      tau = __shfl_sync(full, v, seg0 + k - 1);
    }
    int nl = 0;
#pragma unroll
    for (int i = 0; i < EL; ++i) nl += (c[i] >= tau && c[i] > -INFINITY) ? 1 : 0;
    int incl = nl;  // inclusive prefix of the counts over the token's lanes
    for (int off = 1; off < P; off <<= 1) {
      const int o = __shfl_up_sync(full, incl, off);
      if (j >= off) incl += o;
    }
    const int ntot = __shfl_sync(full, incl, seg0 + P - 1);
    if (__all_sync(full, tau != INFINITY && ntot <= P)) {
      __shared__ float cv_s[kThreads], cs_s[kThreads];
      __shared__ int ci_s[kThreads];
      const int sb = (threadIdx.x & ~31) + seg0;  // this token's slots: [sb, sb + P)
      int slot = sb + incl - nl;
#pragma unroll
      for (int i = 0; i < EL; ++i)
        if (c[i] >= tau && c[i] > -INFINITY) {
          cv_s[slot] = c[i];
          cs_s[slot] = s[i];
          ci_s[slot] = e0 + i;
          ++slot;
        }
      __syncwarp();
      float v = -INFINITY, sc = 0.0f;
      int ix = 0x7fffffff, rank = P;
      if (j < ntot) {
        v = cv_s[sb + j];
        sc = cs_s[sb + j];
        ix = ci_s[sb + j];
        rank = 0;
        for (int o = 0; o < ntot; ++o)
          rank += mr_better(cv_s[sb + o], ci_s[sb + o], v, ix) ? 1 : 0;
      }
      __syncwarp();
      if (rank < k) cs_s[sb + rank] = sc;  // the winners' scores in slot order
      __syncwarp();
      const int nwin = ntot < k ? ntot : k;
      float den = 0.0f;
#pragma unroll
      for (int r = 0; r < kTop; ++r)
        if (r < nwin) den += cs_s[sb + r];
      if (!live) return;
      if (rank < k) {
        p.idx_out[t * k + rank] = ix;
        p.w_out[t * k + rank] = mr_weight(sc, den, p.route_scale, p.flags);
      } else if (j >= nwin && j < k) {  // fewer than k finite scores: empty slots
        p.idx_out[t * k + j] = 0x7fffffff;
        p.w_out[t * k + j] = mr_weight(0.0f, den, p.route_scale, p.flags);
      }
      return;
    }
  }

  // ---- k rounds of the best not yet taken ----
  uint32_t taken = 0;  // bit i: expert e0 + i already chosen (EL <= 32)
  float win_s[kTop];
  int win_i[kTop];
#pragma unroll
  for (int r = 0; r < kTop; ++r) {
    win_s[r] = 0.0f;
    win_i[r] = 0x7fffffff;
    if (r >= k) continue;
    // this lane's best remaining expert (ascending scan: lower index first)
    float bv = -INFINITY, bsc = 0.0f;
    int bl = -1;
#pragma unroll
    for (int i = 0; i < EL; ++i) {
      const bool better = !((taken >> i) & 1u) && c[i] > bv;
      bv = better ? c[i] : bv;
      bsc = better ? s[i] : bsc;
      bl = better ? i : bl;
    }
    int bi = bl >= 0 ? e0 + bl : 0x7fffffff;  // -inf is never taken
    if (P == 32) {
      // the largest value as an order-preserving integer, then the smallest
      // index among the lanes holding it
      const uint32_t u = __float_as_uint(bv);
      const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
      const uint32_t mx = __reduce_max_sync(full, key);
      bi = (int)__reduce_min_sync(full, key == mx ? (uint32_t)bi : 0xffffffffu);
    } else {
      for (int off = 1; off < P; off <<= 1) {
        const float ov = __shfl_xor_sync(full, bv, off);
        const int oi = __shfl_xor_sync(full, bi, off);
        if (mr_better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
    }
    // the winner's lane holds its score; it marks the expert taken
    const int wl = bi == 0x7fffffff ? j : bi / EL;
    const float wsc = __shfl_sync(full, bsc, seg0 + wl);
    if (bi != 0x7fffffff) {
      win_s[r] = wsc;
      win_i[r] = bi;
      if (wl == j) taken |= 1u << (bi - e0);
    }
  }
  if (!live) return;
  float den = 0.0f;
#pragma unroll
  for (int r = 0; r < kTop; ++r)
    if (r < k) den += win_s[r];
#pragma unroll
  for (int r = 0; r < kTop; ++r) {
    if (r < k && r == j) {
      p.idx_out[t * k + r] = win_i[r];
      p.w_out[t * k + r] = mr_weight(win_s[r], den, p.route_scale, p.flags);
    }
  }
}

// Lanes per token for a batch of T tokens and N experts in groups of N/G:
// the most lanes whose layout fits (32, else 16, else 8 -- measured fastest
// on the DeepSeek-V3 and Kimi K2 prefill batches), 0 when none does (the
// GEMM's epilogue routes instead); pin > 0 asks for that many lanes (0 when
// they do not fit).
inline int lanes_per_token(long T, int N, int G, int k, int sms, int pin = 0) {
  (void)T;
  (void)sms;
  if (N > kMaxN || k > kTop) return 0;
  const int cand[3] = {32, 16, 8};
  for (int ci = 0; ci < 3; ++ci) {
    const int P = cand[ci];
    if (pin > 0 && P != pin) continue;
    if (N % P) continue;
    const int EL = N / P;
    if (EL != 8 && EL != 12 && EL != 16 && EL != 24 && EL != 32) continue;
    if (G > 1) {
      const int S = N / G;
      if (S % EL) continue;
      const int LG = S / EL;
      if (LG & (LG - 1)) continue;  // a power of two: groups align with shuffle trees
    }
    return P;
  }
  return 0;
}

}  // namespace rt
}  // namespace mr
