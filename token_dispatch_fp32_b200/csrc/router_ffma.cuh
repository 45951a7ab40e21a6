// router_ffma.cuh -- CUDA-core (fp32 FMA) router: one CTA computes the logits
// of 32 tokens against all N_r experts into shared memory, then each warp
// routes 4 of those tokens.  Works for any d and N_r <= 512; it is the
// general-shape path and the independent cross-check of the tensor-core path.
#pragma once

#include "mr_common.cuh"

namespace mr {

constexpr int kFfmaTokens = 32;   // tokens per CTA
constexpr int kFfmaThreads = 256; // 8 warps x 4 tokens
constexpr int kFfmaBK = 16;       // K slice staged per iteration

__host__ __device__ constexpr size_t ffma_smem_bytes(int nj) {
  return sizeof(float) * (size_t)(kFfmaBK * (kFfmaTokens + 1) + kFfmaBK * (32 * nj + 1) +
                                  kFfmaTokens * (32 * nj + 1));
}

// XBF16: x rows stored in bf16; WBF16: W stored in bf16 (both widened exactly).
template <int NJ, bool XBF16, bool WBF16 = false>
__global__ void __launch_bounds__(kFfmaThreads)
    router_ffma_kernel(const void* __restrict__ xv, const void* __restrict__ Wv,
                       const float* __restrict__ bias, int T, int d, int N_r, int n_group,
                       int topk_group, int k, float route_scale, int mask_mode, int flags,
                       int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                       float* __restrict__ logits_out) {
  constexpr int NP = 32 * NJ;       // padded expert count
  constexpr int XLD = kFfmaTokens + 1;
  constexpr int WLD = NP + 1;
  constexpr int LLD = NP + 1;
  extern __shared__ float smem[];
  float* xs = smem;                      // [BK][XLD]  x slice, K-major
  float* ws = xs + kFfmaBK * XLD;        // [BK][WLD]  W slice, K-major
  float* Ls = ws + kFfmaBK * WLD;        // [32][LLD]  logits

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long t0 = (long)blockIdx.x * kFfmaTokens;
  float acc[4][NJ];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[a][j] = 0.0f;

  for (int k0 = 0; k0 < d; k0 += kFfmaBK) {
    for (int i = threadIdx.x; i < kFfmaTokens * kFfmaBK; i += kFfmaThreads) {
      const int tok = i / kFfmaBK, kk = i % kFfmaBK;
      const long gt = t0 + tok;
      const int gk = k0 + kk;
      float v = 0.0f;
      if (gt < T && gk < d) {
        if (XBF16)
          v = mr_bf16_to_f32(static_cast<const uint16_t*>(xv)[gt * d + gk]);
        else
          v = static_cast<const float*>(xv)[gt * d + gk];
      }
      xs[kk * XLD + tok] = v;
    }
    for (int i = threadIdx.x; i < NP * kFfmaBK; i += kFfmaThreads) {
      const int e = i / kFfmaBK, kk = i % kFfmaBK;
      const int gk = k0 + kk;
      float v = 0.0f;
      if (e < N_r && gk < d) {
        if (WBF16)
          v = mr_bf16_to_f32(static_cast<const uint16_t*>(Wv)[(long)e * d + gk]);
        else
          v = static_cast<const float*>(Wv)[(long)e * d + gk];
      }
      ws[kk * WLD + e] = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kFfmaBK; ++kk) {
      float xr[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) xr[a] = xs[kk * XLD + 4 * warp + a];
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const float wv = ws[kk * WLD + lane + 32 * j];
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a][j] = fmaf(xr[a], wv, acc[a][j]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int tok = 4 * warp + a;
#pragma unroll
    for (int j = 0; j < NJ; ++j) Ls[tok * LLD + lane + 32 * j] = acc[a][j];
    const long gt = t0 + tok;
    if (logits_out && gt < T) {
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        if (e < N_r) logits_out[gt * N_r + e] = acc[a][j];
      }
    }
  }
  __syncwarp();
#pragma unroll 1
  for (int a = 0; a < 4; ++a) {
    const int tok = 4 * warp + a;
    const long gt = t0 + tok;
    if (gt < T)
      mr_route_token_warp<NJ>(Ls + tok * LLD, bias, N_r, n_group, topk_group, k, route_scale,
                              mask_mode, idx_out + gt * k, w_out + gt * k, flags);
  }
}

}  // namespace mr
