// router_splitk.cuh -- gate GEMM for small batches (decode): split-K over all
// SMs on the tensor cores, a cluster reduction through distributed shared
// memory, then a reduce-and-route kernel.
//
// With T of order 64 the fused kernel would give the weight read to one or two
// SMs.  Here the roles of the operands are swapped so the 128-row MMA tile
// runs over experts: A = W rows [128 experts x K], B = x rows [NT tokens x K],
// D = logits^T [128 experts (TMEM lanes) x NT tokens (columns)], and the K
// loop is split into KS slices, one CTA per (slice, expert tile, token tile),
// so every SM streams a share of W once.
//
// Arithmetic: 3xTF32 on the staged fp32 values (the tensor core reads a tf32
// operand with its 13 low mantissa bits ignored, so a staged tile serves as hi
// and only lo = v - trunc(v) is written): W_hi*x_hi + W_lo*x_hi + W_hi*x_lo.
// bf16 activations are staged by TMA as bf16 and widened into the fp32 B tile
// by the workers; a bf16 value is exact in tf32, so x_lo = 0 and its MMA is
// skipped.  With W stored in bf16 and bf16 rows (bf16_mma), both tiles are
// staged by TMA with the 64-byte swizzle and feed kind::f16 MMAs directly:
// W*x is exact in fp32, no conversion, one product per multiply-add.  A slice
// spans only a few K chunks, so the tensor core's round-toward-zero
// accumulation stays within a few ulp.
//
// Reduction: the CL CTAs of a cluster hold consecutive K slices of the same
// (expert tile, token tile).  Each copies its partial tile from TMEM to shared
// memory; after a cluster barrier CTA r sums rows [r*NT/CL, (r+1)*NT/CL) of
// the CL partials in rank order (deterministic) through distributed shared
// memory and writes them to part[ks / CL][token][expert].  A second cluster
// barrier keeps every CTA's shared memory alive until its peers have read it.
// The KS / CL slices are then summed in order and routed by a programmatic
// dependent of the GEMM: the routing kernel of route.cuh (one warp per token)
// where its lane layout fits, else router_reduce_route_kernel below, which
// routes each token with the whole CTA (route_token_cta), or with one warp for
// the shapes that does not cover.
#pragma once

#include "router_tc.cuh"

namespace mr {
namespace sk {

using namespace mr::tc;

constexpr int kWorkersSk = 8;   // worker warps 2..9
constexpr int kThreads = 64 + 32 * kWorkersSk;  // warp 0 TMA, warp 1 MMA, then workers
constexpr int kMaxNT = 256;     // tokens per CTA (MMA N)
constexpr int kCluster = 8;     // CTAs per cluster reduction (when KS allows)

struct Params {
  int T, d, N, NT, KS, CL, num_kc, use3x, x_bf16;
  int bf16_mma;  // W and x both bf16: kind::f16 on the staged tiles
  float* part;  // [KS / CL][T][N]
};

struct Plan {
  int stages;
  uint32_t a_bytes, b_bytes, hi_bytes, xs_bytes, stage_bytes, bar_off, misc_off, total;
};

// Stage: [A hi (W) | B hi (x fp32)] [A lo | B lo] [x bf16 staging]; with
// bf16_mma: [A (W bf16) | B (x bf16)], 64-byte rows.
__host__ __device__ inline Plan make_plan(int NT, int max_chunks, bool x_bf16,
                                          bool bf16_mma = false) {
  Plan p;
  const uint32_t esz = bf16_mma ? 2 : 4;
  p.a_bytes = BM * BK * esz;               // 128 experts
  p.b_bytes = NT * BK * esz;               // NT tokens
  p.hi_bytes = p.a_bytes + p.b_bytes;
  p.xs_bytes = (x_bf16 && !bf16_mma) ? NT * BK * 2 : 0;
  p.stage_bytes = align_up((bf16_mma ? 1 : 2) * p.hi_bytes + p.xs_bytes, 1024);
  int s = (int)((kSmemBudget - 1024 - 512 - 64) / p.stage_bytes);
  if (s > kMaxStages) s = kMaxStages;
  if (s > max_chunks) s = max_chunks < 1 ? 1 : max_chunks;
  // the reduction buffer [NT][128] fp32 aliases the ring after the K loop
  while (s * p.stage_bytes < (uint32_t)NT * BM * 4) ++s;
  p.stages = s;
  p.bar_off = p.stages * p.stage_bytes;
  p.misc_off = p.bar_off + 512;
  p.total = p.misc_off + 64;
  return p;
}

__host__ __device__ inline int slice_begin(int ks, int KS, int KC) {
  return (int)(((long)ks * KC) / KS);
}

// Byte offset of fp32 element (row, k) of a K-major tile with 128-byte rows
// and the 128-byte swizzle (16-byte chunk c of row r sits at chunk c ^ (r % 8)).
__device__ __forceinline__ uint32_t sw128_f32(int row, int k) {
  return (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u +
         ((uint32_t)((k >> 2) ^ (row & 7)) << 4) + (uint32_t)(k & 3) * 4u;
}

__global__ void __launch_bounds__(kThreads, 1)
    router_splitk_gemm_kernel(const __grid_constant__ CUtensorMap map_w,
                              const __grid_constant__ CUtensorMap map_x, const Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned start by pointer arithmetic on the shared array, so the
  // compiler keeps the shared address space for every access through it (an
  // integer round trip would turn them into generic loads and stores)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int ks = blockIdx.x, mt = blockIdx.y, tt = blockIdx.z;
  const int c_beg = slice_begin(ks, P.KS, P.num_kc), c_end = slice_begin(ks + 1, P.KS, P.num_kc);
  const int NC = c_end - c_beg;
  const int NT = P.NT;
  const bool xb = P.x_bf16 != 0;
  const bool bm = P.bf16_mma != 0;
  const bool conv = !bm && (P.use3x || xb);  // the workers touch every stage
  const Plan plan = make_plan(NT, (P.num_kc + P.KS - 1) / P.KS, xb, bm);
  const int STAGES = plan.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CL = P.CL;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + plan.misc_off);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + plan.misc_off + 8);
  const uint32_t smem0 = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int B_FULL = 0, B_CONV = STAGES, B_EMPTY = 2 * STAGES, B_ACC = 3 * STAGES;
  const uint32_t tmem_cols = NT <= 32 ? 32 : NT <= 64 ? 64 : NT <= 128 ? 128 : 256;

  // the reduce-and-route grid may be scheduled now: it waits for this grid's
  // completion (griddepcontrol.wait) before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_CONV + s), kWorkersSk);  // one elected arrival per worker warp
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_ACC), 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  // The producer (thread 0) fills the whole ring before the block-wide
  // barrier: the first loads are in flight while TMEM is being allocated.
  const uint32_t tx = plan.a_bytes + ((xb && !bm) ? plan.xs_bytes : plan.b_bytes);
  const int pre = NC < STAGES ? NC : STAGES;
  auto issue = [&](int i) {
    const int s = i % STAGES, kc = c_beg + i;
    const uint32_t base = smem0 + s * plan.stage_bytes;
    mbar_arrive_expect_tx(bar(B_FULL + s), tx);
    tma_load_2d(base, &map_w, bar(B_FULL + s), kc * BK, mt * BM);
    tma_load_2d((xb && !bm) ? base + 2 * plan.hi_bytes : base + plan.a_bytes, &map_x,
                bar(B_FULL + s), kc * BK, tt * NT);
  };
  if (threadIdx.x == 0)
    for (int i = 0; i < pre; ++i) issue(i);
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
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      int issued = pre;
      for (int i = pre; i < NC; ++i) {
        if (!mbar_wait(bar(B_EMPTY + i % STAGES), ((i / STAGES) - 1) & 1, abort)) break;
        ++issued;
        issue(i);
      }
      for (int i = issued - STAGES < 0 ? 0 : issued - STAGES; i < issued; ++i)
        mbar_wait(bar(B_FULL + i % STAGES), (i / STAGES) & 1, abort, true);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = bm ? make_idesc_bf16(NT, BM) : make_idesc(NT);
      for (int i = 0; i < NC; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(conv ? bar(B_CONV + s) : bar(B_FULL + s), (i / STAGES) & 1, abort))
          break;
        tc_fence_after();
        if (bm) {
          const uint32_t a = smem0 + s * plan.stage_bytes, b = a + plan.a_bytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t ko = kk * 32;  // 16 bf16 = 32 bytes along K
            mma_bf16(tmem_base, make_desc_sw64(a + ko), make_desc_sw64(b + ko), idesc,
                     (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(B_EMPTY + s));
          continue;
        }
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
            mma_tf32(tmem_base, make_desc(a_lo + ko), dbh, idesc, 1u);   // W_lo * x
            if (!xb) mma_tf32(tmem_base, dah, make_desc(b_lo + ko), idesc, 1u);  // W * x_lo
          }
        }
        mma_commit(bar(B_EMPTY + s));
      }
      mma_commit(bar(B_ACC));
    }
  } else {
    const int ct = threadIdx.x - 64;  // 0 .. 32 * kWorkersSk - 1
    constexpr int kW = 32 * kWorkersSk;
    if (conv) {
      for (int i = 0; i < NC; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(bar(B_FULL + s), (i / STAGES) & 1, abort)) break;
        uint8_t* st = smem + s * plan.stage_bytes;
        if (xb) {
          // widen the bf16 x tile [NT][32] into the swizzled fp32 B tile
          const uint16_t* xs = reinterpret_cast<const uint16_t*>(st + 2 * plan.hi_bytes);
          uint8_t* bh = st + plan.a_bytes;
          for (int j = ct; j < NT * BK; j += kW) {
            const int r = j / BK, kk = j % BK;
            *reinterpret_cast<float*>(bh + sw128_f32(r, kk)) = mr_bf16_to_f32(xs[j]);
          }
        }
        if (P.use3x) {
          // lo = v - trunc_tf32(v) of W (and of fp32 x), same layout
          const int n4 = (int)((xb ? plan.a_bytes : plan.hi_bytes) / 16);
          const float4* hi = reinterpret_cast<const float4*>(st);
          float4* lo = reinterpret_cast<float4*>(st + plan.hi_bytes);
          for (int j = ct; j < n4; j += kW) {
            const float4 v = hi[j];
            float4 l;
            l.x = v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
            l.y = v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
            l.z = v.z - __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
            l.w = v.w - __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
            lo[j] = l;
          }
        }
        // each thread's generic-proxy writes are made visible to the tensor
        // core's async proxy, then one lane per warp releases the stage
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_CONV + s));
      }
    }
    // The accumulator barrier is always committed (also after an abort), so
    // this wait drains every MMA before TMEM is released.
    ok = __all_sync(0xffffffffu, mbar_wait(bar(B_ACC), 0, abort, true)) && !*abort;
    tc_fence_after();
    const int q = warp & 3;
    const int hf = (warp - 2) >> 2;  // warps w and w+4 share lanes, split the columns
    const int el = q * 32 + lane;  // expert (within the tile) of this TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float* red = reinterpret_cast<float*>(smem);  // [NT][128], aliases the idle ring
    float v[16];
    const int nc = NT / 16, ch = (nc + 1) / 2;
    for (int c = hf * ch; c < nc && c < (hf + 1) * ch; ++c) {
      tmem_ld16(tmem_base + lane_off + (uint32_t)(c * 16), v);  // whole warp
      if (CL > 1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) red[(c * 16 + j) * BM + el] = v[j];
      } else {
        const int e = mt * BM + el;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = tt * NT + c * 16 + j;
          if (ok && t < P.T && e < P.N) P.part[((long)ks * P.T + t) * P.N + e] = v[j];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (CL > 1) {
    // every thread of the cluster takes both barriers, whatever happened above
    cluster_sync_all();
    const uint32_t rank = cluster_rank();
    const int rows = NT / CL;  // tokens reduced by this CTA
    const float* red = reinterpret_cast<const float*>(smem);
    // a CTA that gave up on a wait (abort flag) leaves no valid partial; the
    // CL flags are loaded together (independent remote loads), then combined
    int fl[kCluster];
#pragma unroll
    for (int src = 0; src < kCluster; ++src)
      fl[src] = src < CL ? __float_as_int(ld_peer_f32(
                               reinterpret_cast<const float*>(const_cast<const int*>(abort)),
                               (uint32_t)src))
                         : 0;
    int bad = 0;
#pragma unroll
    for (int src = 0; src < kCluster; ++src) bad |= fl[src];
    ok = ok && bad == 0;
    for (int j = threadIdx.x; j < rows * (BM / 4); j += kThreads) {
      const int tl = (int)rank * rows + j / (BM / 4), el = (j % (BM / 4)) * 4;
      // CL == kCluster here: all loads in flight before the first add
      float4 o[kCluster];
#pragma unroll
      for (int src = 0; src < kCluster; ++src)
        o[src] = ld_peer_f32x4(&red[tl * BM + el], (uint32_t)src);
      float4 acc = o[0];
#pragma unroll
      for (int src = 1; src < kCluster; ++src) {
        acc.x += o[src].x;
        acc.y += o[src].y;
        acc.z += o[src].z;
        acc.w += o[src].w;
      }
      const int t = tt * NT + tl, e = mt * BM + el;
      if (ok && t < P.T && e < P.N) {
        float* dst = P.part + ((long)(ks / CL) * P.T + t) * P.N + e;
        if (e + 3 < P.N) {
          *reinterpret_cast<float4*>(dst) = acc;
        } else {
          dst[0] = acc.x;
          if (e + 1 < P.N) dst[1] = acc.y;
          if (e + 2 < P.N) dst[2] = acc.z;
        }
      }
    }
    cluster_sync_all();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(tmem_cols)
                 : "memory");
  }
}

// Shared state of route_token_cta.
struct CtaRouteSmem {
  float a1[8], a2[8];  // per-warp top-2 of the biased scores (distinct experts)
  float tau;           // lower bound on the token's k-th best masked score
  uint32_t kept;       // bit g: group g kept
  int cnt[8];          // candidates per warp
  float cm[32], cs[32];
  int ci[32];
};

// Routing of one token by a CTA of 256 threads, thread e owning expert e
// (N_r <= 256, sigmoid scores; groups that are whole warps, or no groups).
// The steps and their order are those of mr_route_token_warp_fast, with the
// per-lane loops of one warp spread over eight warps:
//   * each warp reduces the top-2 pair of its 32 biased scores;
//   * warp 0 merges the pairs of each group into its score (top-2 sum, or
//     the best), keeps topk_group groups by counting the groups that beat
//     each one (lower group on ties), and takes tau = the k-th best of the
//     kept warps' pairs -- k distinct experts, so the token's k-th best
//     masked score is >= tau;
//   * the experts with masked score >= tau are compacted in expert order and
//     each one's place is the number of candidates that beat it (value desc,
//     index asc); the k best write their slots.
// Returns false, having written nothing, when there are more than 32
// candidates (ties at the 0.0 fill, or fewer than k finite pair values); the
// caller then routes with the one-warp routine.  Every thread of the CTA
// calls it (it synchronises the CTA).
__device__ __forceinline__ bool route_token_cta(float Lv, const float* __restrict__ bs, int N_r,
                                                int n_group, int topk_group, int k,
                                                float route_scale, int mask_mode, int flags,
                                                int32_t* __restrict__ idx_out,
                                                float* __restrict__ w_out, CtaRouteSmem& sm) {
  const int e = threadIdx.x, warp = e >> 5, lane = e & 31;
  const bool valid = e < N_r;
  const float s = valid ? mr_sigmoid(Lv) : 0.0f;
  const float c = valid ? s + bs[e] : -INFINITY;
  float a1 = c, a2 = -INFINITY;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float b1 = __shfl_xor_sync(0xffffffffu, a1, off);
    const float b2 = __shfl_xor_sync(0xffffffffu, a2, off);
    const float hi = fmaxf(a1, b1);
    a2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
    a1 = hi;
  }
  if (lane == 0) {
    sm.a1[warp] = a1;
    sm.a2[warp] = a2;
  }
  __syncthreads();
  const int nw = (N_r + 31) / 32;                           // warps that hold experts
  const int q = n_group > 1 ? (N_r / n_group) / 32 : nw;    // warps per group
  if (warp == 0) {
    uint32_t kept = 1u;
    if (n_group > 1) {
      float g1 = -INFINITY, g2 = -INFINITY;
      if (lane < n_group) {
        for (int i = 0; i < q; ++i) {
          const float b1 = sm.a1[lane * q + i], b2 = sm.a2[lane * q + i];
          const float hi = fmaxf(g1, b1);
          g2 = fmaxf(fminf(g1, b1), fmaxf(g2, b2));
          g1 = hi;
        }
      }
      const float gsc = (flags & MR_GROUP_MAX) ? g1 : g1 + g2;
      int rank = 0;
      for (int o = 0; o < n_group; ++o) {
        const float so = __shfl_sync(0xffffffffu, gsc, o);
        rank += (so > gsc || (so == gsc && o < lane)) ? 1 : 0;
      }
      kept = __ballot_sync(0xffffffffu, lane < n_group && rank < topk_group);
    }
    const int w = lane >> 1;
    float v = -INFINITY;
    if (lane < 2 * nw && ((kept >> (w / q)) & 1u)) v = (lane & 1) ? sm.a2[w] : sm.a1[w];
    int r = 0;
    for (int o = 0; o < 2 * nw; ++o) {
      const float vo = __shfl_sync(0xffffffffu, v, o);
      r += (vo > v || (vo == v && o < lane)) ? 1 : 0;
    }
    const uint32_t at = __ballot_sync(0xffffffffu, lane < 2 * nw && r == k - 1);
    const float tau = at ? __shfl_sync(0xffffffffu, v, __ffs(at) - 1) : -INFINITY;
    if (lane == 0) {
      sm.kept = kept;
      sm.tau = tau;
    }
  }
  __syncthreads();
  // fewer than k finite pair values: no bound, every expert is a candidate
  if (sm.tau == -INFINITY && N_r > 32) return false;
  const float fill = (mask_mode == MR_MASK_NEG_INF) ? -INFINITY : 0.0f;
  const float m = !valid ? -INFINITY : ((sm.kept >> (warp / q)) & 1u) ? c : fill;
  const bool cand = valid && m >= sm.tau;
  const uint32_t bal = __ballot_sync(0xffffffffu, cand);
  if (lane == 0) sm.cnt[warp] = __popc(bal);
  __syncthreads();
  int base = 0, n = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int ni = sm.cnt[i];
    base += i < warp ? ni : 0;
    n += ni;
  }
  if (n > 32) return false;  // the same n in every thread
  if (cand) {
    const int slot = base + __popc(bal & ((1u << lane) - 1u));
    sm.cm[slot] = m;
    sm.cs[slot] = s;
    sm.ci[slot] = e;
  }
  __syncthreads();
  if (warp == 0) {
    float cv = -INFINITY, cs = 0.0f;
    int ci = 0x7fffffff, rank = 32;
    if (lane < n) {
      cv = sm.cm[lane];
      cs = sm.cs[lane];
      ci = sm.ci[lane];
      rank = 0;
      for (int o = 0; o < n; ++o) rank += mr_better(sm.cm[o], sm.ci[o], cv, ci) ? 1 : 0;
    }
    float den = rank < k ? cs : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (rank < k) {
      idx_out[rank] = ci;
      w_out[rank] = mr_weight(cs, den, route_scale, flags);
    }
  }
  return true;
}

// One CTA per token: sum the KS partial logits of each expert in slice order,
// then route the token (route_token_cta where its shape allows, else one
// warp).  Launched as a programmatic dependent of the GEMM: it waits for that
// grid's results before reading them.
template <int NJ>
__global__ void __launch_bounds__(256, 1)
    router_reduce_route_kernel(const float* __restrict__ part, int KS, int T, int N_r,
                               const float* __restrict__ bias, int n_group, int topk_group, int k,
                               float route_scale, int mask_mode, int flags,
                               int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                               float* __restrict__ logits_out) {
  __shared__ float L[32 * NJ];
  __shared__ float bs[32 * NJ];
  __shared__ float scratch[96];
  __shared__ CtaRouteSmem rs;
  // the bias does not come from the GEMM: fetch it while the GEMM runs
  for (int e = threadIdx.x; e < N_r; e += blockDim.x) bs[e] = bias ? bias[e] : 0.0f;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int t = blockIdx.x;
  float mine = 0.0f;  // the logit of expert threadIdx.x
  for (int e = threadIdx.x; e < N_r; e += blockDim.x) {
    float acc = 0.0f;
    const float* p = part + (long)t * N_r + e;
    const long stride = (long)T * N_r;
#pragma unroll 8
    for (int s = 0; s < KS; ++s) acc += p[s * stride];
    L[e] = acc;
    if (e == (int)threadIdx.x) mine = acc;
    if (logits_out) logits_out[(long)t * N_r + e] = acc;
  }
  __syncthreads();
  const bool cta = blockDim.x == 256 && N_r <= 256 && !(flags & MR_SCORE_SOFTMAX) &&
                   (n_group == 1 || (N_r % n_group == 0 && (N_r / n_group) % 32 == 0));
  if (cta && route_token_cta(mine, bs, N_r, n_group, topk_group, k, route_scale, mask_mode, flags,
                             idx_out + (long)t * k, w_out + (long)t * k, rs))
    return;
  if (threadIdx.x < 32)
    mr_route_token_warp_fast<NJ>(L, bs, N_r, n_group, topk_group, k, route_scale, mask_mode,
                                 idx_out + (long)t * k, w_out + (long)t * k, scratch, flags);
}

}  // namespace sk
}  // namespace mr
