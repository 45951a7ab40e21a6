// router_splitk.cuh -- gate GEMM for small batches (decode): split-K over all
// SMs on the tensor cores, then a reduce-and-route kernel.
//
// With T of order 64 the fused kernel would give the weight read to one or two
// SMs.  Here the roles of the operands are swapped so the 128-row MMA tile
// runs over experts: A = W rows [128 experts x K], B = x rows [NT tokens x K],
// D = logits^T [128 experts (TMEM lanes) x NT tokens (columns)], and the K
// loop is split into KS slices, one CTA per (slice, expert tile, token tile),
// so every SM streams a share of W.  Operands get the same 3xTF32 split as the
// fused kernel; a slice spans only a few K chunks, so its accumulator stays
// small and the tensor core's round-toward-zero accumulation costs nothing
// measurable (partials are summed in fp32 with round-to-nearest afterwards).
// Each CTA writes its fp32 partial logits to the workspace
// part[slice][token][expert]; router_reduce_route_kernel sums the slices in
// slice order (deterministic) and routes every token with one warp
// (mr_route_token_warp).
#pragma once

#include "router_tc.cuh"

namespace mr {
namespace sk {

using namespace mr::tc;

constexpr int kThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2..5 split + epilogue
constexpr int kMaxNT = 256;     // tokens per CTA (MMA N)

struct Params {
  int T, d, N, NT, KS, num_kc, use3x;
  float* part;  // [KS][T][N]
};

struct Plan {
  int stages;
  uint32_t a_bytes, b_bytes, hi_bytes, stage_bytes, bar_off, misc_off, total;
};

__host__ __device__ inline Plan make_plan(int NT, int max_chunks) {
  Plan p;
  p.a_bytes = BM * BK * 4;                 // 128 experts
  p.b_bytes = NT * BK * 4;                 // NT tokens
  p.hi_bytes = p.a_bytes + p.b_bytes;
  p.stage_bytes = align_up(2 * p.hi_bytes, 1024);
  int s = (int)((kSmemBudget - 1024 - 512 - 64) / p.stage_bytes);
  if (s > kMaxStages) s = kMaxStages;
  if (s > max_chunks) s = max_chunks < 1 ? 1 : max_chunks;
  p.stages = s;
  p.bar_off = p.stages * p.stage_bytes;
  p.misc_off = p.bar_off + 512;
  p.total = p.misc_off + 64;
  return p;
}

__host__ __device__ inline int slice_begin(int ks, int KS, int KC) {
  return (int)(((long)ks * KC) / KS);
}

__global__ void __launch_bounds__(kThreads, 1)
    router_splitk_gemm_kernel(const __grid_constant__ CUtensorMap map_w,
                              const __grid_constant__ CUtensorMap map_x, const Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int ks = blockIdx.x, mt = blockIdx.y, tt = blockIdx.z;
  const int c_beg = slice_begin(ks, P.KS, P.num_kc), c_end = slice_begin(ks + 1, P.KS, P.num_kc);
  const int NC = c_end - c_beg;
  const int NT = P.NT;
  const Plan plan = make_plan(NT, (P.num_kc + P.KS - 1) / P.KS);
  const int STAGES = plan.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + plan.misc_off);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + plan.misc_off + 8);
  const uint32_t smem0 = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int B_FULL = 0, B_CONV = STAGES, B_EMPTY = 2 * STAGES, B_ACC = 3 * STAGES;
  const uint32_t tmem_cols = NT <= 32 ? 32 : NT <= 64 ? 64 : NT <= 128 ? 128 : 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_CONV + s), 128);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_ACC), 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t tx = (uint32_t)(BM + NT) * BK * 4;
      int issued = 0;
      for (int i = 0; i < NC; ++i) {
        const int s = i % STAGES, kc = c_beg + i;
        if (i >= STAGES && !mbar_wait(bar(B_EMPTY + s), ((i / STAGES) - 1) & 1, abort)) break;
        ++issued;
        const uint32_t base = smem0 + s * plan.stage_bytes;
        mbar_arrive_expect_tx(bar(B_FULL + s), tx);
        tma_load_2d(base, &map_w, bar(B_FULL + s), kc * BK, mt * BM);
        tma_load_2d(base + plan.a_bytes, &map_x, bar(B_FULL + s), kc * BK, tt * NT);
      }
      for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; ++i)
        mbar_wait(bar(B_FULL + i % STAGES), (i / STAGES) & 1, abort, true);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(NT);
      for (int i = 0; i < NC; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(P.use3x ? bar(B_CONV + s) : bar(B_FULL + s), (i / STAGES) & 1, abort))
          break;
        tc_fence_after();
        const uint32_t a_hi = smem0 + s * plan.stage_bytes;
        const uint32_t b_hi = a_hi + plan.a_bytes;
        const uint32_t a_lo = a_hi + plan.hi_bytes;
        const uint32_t b_lo = b_hi + plan.hi_bytes;
#pragma unroll
        for (int kk = 0; kk < BK / 8; ++kk) {
          const uint32_t ko = kk * 32;
          const uint32_t acc0 = (i > 0 || kk > 0) ? 1u : 0u;
          const uint64_t dah = make_desc(a_hi + ko), dbh = make_desc(b_hi + ko);
          mma_tf32(tmem_base, dah, dbh, idesc, acc0);
          if (P.use3x) {
            mma_tf32(tmem_base, dah, make_desc(b_lo + ko), idesc, 1u);
            mma_tf32(tmem_base, make_desc(a_lo + ko), dbh, idesc, 1u);
          }
        }
        mma_commit(bar(B_EMPTY + s));
      }
      mma_commit(bar(B_ACC));
    }
  } else {
    const int ct = threadIdx.x - 64;  // 0..127
    if (P.use3x) {
      const int n4 = (int)(plan.hi_bytes / 16);
      for (int i = 0; i < NC; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(bar(B_FULL + s), (i / STAGES) & 1, abort)) break;
        // staged fp32 = hi (the tensor core truncates tf32 operands); write lo
        const float4* hi = reinterpret_cast<const float4*>(smem + s * plan.stage_bytes);
        float4* lo = reinterpret_cast<float4*>(smem + s * plan.stage_bytes + plan.hi_bytes);
        for (int j = ct; j < n4; j += 128) {
          const float4 v = hi[j];
          float4 l;
          l.x = v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
          l.y = v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
          l.z = v.z - __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
          l.w = v.w - __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
          lo[j] = l;
        }
        fence_proxy_async();
        mbar_arrive(bar(B_CONV + s));
      }
    }
    // The accumulator barrier is always committed (also after an abort), so
    // this wait drains every MMA before TMEM is released.
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar(B_ACC), 0, abort, true)) && !*abort;
    tc_fence_after();
    const int q = warp & 3;
    const int e = mt * BM + q * 32 + lane;  // expert of this TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float v[16];
    for (int c = 0; c < NT / 16; ++c) {
      tmem_ld16(tmem_base + lane_off + (uint32_t)(c * 16), v);  // whole warp
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = tt * NT + c * 16 + j;
        if (ok && t < P.T && e < P.N) P.part[((long)ks * P.T + t) * P.N + e] = v[j];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(tmem_cols)
                 : "memory");
  }
}

// One CTA per token: sum the KS partial logits of each expert in slice order,
// then route the token with one warp.
template <int NJ>
__global__ void __launch_bounds__(256)
    router_reduce_route_kernel(const float* __restrict__ part, int KS, int T, int N_r,
                               const float* __restrict__ bias, int n_group, int topk_group, int k,
                               float route_scale, int mask_mode, int32_t* __restrict__ idx_out,
                               float* __restrict__ w_out, float* __restrict__ logits_out) {
  __shared__ float L[32 * NJ];
  const int t = blockIdx.x;
  for (int e = threadIdx.x; e < N_r; e += blockDim.x) {
    float acc = 0.0f;
    const float* p = part + (long)t * N_r + e;
    const long stride = (long)T * N_r;
#pragma unroll 8
    for (int s = 0; s < KS; ++s) acc += p[s * stride];
    L[e] = acc;
    if (logits_out) logits_out[(long)t * N_r + e] = acc;
  }
  __syncthreads();
  if (threadIdx.x < 32)
    mr_route_token_warp<NJ>(L, bias, N_r, n_group, topk_group, k, route_scale, mask_mode,
                            idx_out + (long)t * k, w_out + (long)t * k);
}

}  // namespace sk
}  // namespace mr
