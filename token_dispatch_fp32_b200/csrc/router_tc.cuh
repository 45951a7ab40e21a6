// router_tc.cuh -- fused gate GEMM + routing on the 5th-generation tensor cores.
//
// One CTA owns a tile of 128 tokens and ALL N_r experts, so a token's logits
// never leave the chip: the accumulator lives in tensor memory (TMEM lane =
// token, column = expert) and the routing epilogue reads it back directly.
//
//   warp 0       TMA producer: x tile [128 x BK] and W tile [N_r x BK] per
//                stage (fp32, hardware swizzle), completion on an mbarrier.
//   warp 1       TMEM owner and MMA issuer (one thread): tcgen05.mma
//                kind::tf32, M=128, N=N_r (two MMAs when N_r > 256).
//   warps 2..5   3xTF32 split while the main loop runs: each staged fp32 value
//                v becomes hi = v with the low 13 mantissa bits cleared (exact
//                in tf32) and lo = v - hi (exact in fp32), so
//                x.w ~= hi.hi + hi.lo + lo.hi with fp32 accumulation.
//                Afterwards the same warps are the epilogue: warp w reads TMEM
//                lanes 32*(w%4).. with tcgen05.ld and routes its token in
//                registers (sigmoid, bias, group top-2, group top-k, top-8
//                insertion with lower-index tie-break, renormalise, scale).
//
// Arithmetic follows the pages (Kimi K2 "Normalize weights" page,
// MoEGate.forward; DeepSeek-V3.2-Exp "Normalize weights" page, Gate.forward).
// Every mbarrier wait is bounded (MR_WAIT_LIMIT_NS); on expiry the CTA raises
// MR_FLAG_TIMEOUT, stops issuing work, drains its MMAs and frees its TMEM.
#pragma once

#include <cuda.h>

#include "mr_common.cuh"

namespace mr {
namespace tc {

constexpr int BM = 128;
constexpr int kThreads = 192;
constexpr int kMaxN = 512;
constexpr int kMaxGroups = 32;
constexpr int kTopMax = 8;
constexpr size_t kSmemBudget = 232448;  // 227 KB opt-in per CTA

struct Params {
  int T, d, N, n_group, topk_group, k, mask_mode, num_kc, use3x;
  float route_scale;
  const float* bias;
  int32_t* idx_out;
  float* w_out;
  float* logits_out;
};

// Shared-memory plan, identical on host and device.
struct Plan {
  int BK, stages;
  uint32_t a_bytes, b_bytes, hi_bytes, stage_bytes;
  uint32_t bar_off, misc_off, bias_off, gs_off, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline Plan make_plan(int N, int stages_cap) {
  Plan p;
  p.BK = (N <= 256) ? 32 : 16;
  p.a_bytes = BM * p.BK * 4;
  p.b_bytes = N * p.BK * 4;
  p.hi_bytes = p.a_bytes + p.b_bytes;          // [A | B] of one kind (hi or lo)
  p.stage_bytes = align_up(2 * p.hi_bytes, 1024);
  const uint32_t extras = 1024 /*align slack*/ + 256 /*barriers*/ + 64 + 4 * kMaxN +
                          4 * kMaxGroups * BM;
  int s = (int)((kSmemBudget - extras) / p.stage_bytes);
  if (s > stages_cap) s = stages_cap;
  p.stages = s;
  p.bar_off = p.stages * p.stage_bytes;
  p.misc_off = p.bar_off + 256;
  p.bias_off = p.misc_off + 64;
  p.gs_off = p.bias_off + 4 * kMaxN;
  p.total = p.gs_off + 4 * kMaxGroups * BM;
  return p;
}

// ---- PTX wrappers ----------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Returns false if it gave up, or (unless `drain`) as soon as
// the CTA is aborting because some other wait timed out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = mr_globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (!drain && *abort) return false;
      if (mr_globaltimer_ns() - t0 > MR_WAIT_LIMIT_NS) {
        *abort = 1;
        mr_raise(MR_FLAG_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// UMMA shared-memory descriptor, K-major operand, swizzled rows of BK fp32.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, int BK) {
  const uint64_t sbo = (BK == 32) ? 1024u : 512u;      // 8 rows x row bytes
  const uint64_t layout = (BK == 32) ? 2u : 4u;        // SWIZZLE_128B / SWIZZLE_64B
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                              // LBO (unused when swizzled)
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;                              // descriptor version (sm_100)
  d |= layout << 61;
  return d;
}

// Instruction descriptor: D fp32, A/B tf32, both K-major, M=128, N=n.
__device__ __forceinline__ uint32_t make_idesc(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t dtmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(dtmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Keep the best 8 (value desc, index asc).  Candidates arrive in increasing
// index order, so an equal value never displaces an earlier one.
struct Top8 {
  float v[kTopMax];
  float s[kTopMax];
  int i[kTopMax];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < kTopMax; ++j) {
      v[j] = -INFINITY;
      s[j] = 0.0f;
      i[j] = 0x7fffffff;
    }
  }
  __device__ __forceinline__ void push(float cv, int ci, float cs) {
    v[kTopMax - 1] = cv;
    i[kTopMax - 1] = ci;
    s[kTopMax - 1] = cs;
#pragma unroll
    for (int j = kTopMax - 1; j > 0; --j) {
      if (v[j] > v[j - 1]) {
        const float tv = v[j]; v[j] = v[j - 1]; v[j - 1] = tv;
        const float ts = s[j]; s[j] = s[j - 1]; s[j - 1] = ts;
        const int ti = i[j]; i[j] = i[j - 1]; i[j - 1] = ti;
      }
    }
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_w0,
                     const __grid_constant__ CUtensorMap map_w1, const Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan plan = make_plan(P.N, 4);
  const int BK = plan.BK, STAGES = plan.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  // bars[0..S) full, [S..2S) converted, [2S..3S) empty, [3S] accumulator ready
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + plan.misc_off);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + plan.misc_off + 8);
  float* bias_s = reinterpret_cast<float*>(smem + plan.bias_off);
  float* gs_s = reinterpret_cast<float*>(smem + plan.gs_off);

  const uint32_t smem0 = smem_u32(smem);
  auto bar_full = [&](int s) { return smem_u32(&bars[s]); };
  auto bar_conv = [&](int s) { return smem_u32(&bars[STAGES + s]); };
  auto bar_empty = [&](int s) { return smem_u32(&bars[2 * STAGES + s]); };
  const uint32_t bar_acc = smem_u32(&bars[3 * STAGES]);

  const int N = P.N;
  const int n0 = N < 256 ? N : 256;
  const int n1 = N - n0;
  const uint32_t tmem_cols = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : N <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_conv(s), 128);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_acc, 1);
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
  for (int e = threadIdx.x; e < N; e += kThreads) bias_s[e] = P.bias ? P.bias[e] : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m0 = blockIdx.x * BM;
  const int KC = P.num_kc;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint32_t tx = (uint32_t)(BM + N) * BK * 4;
      int issued = 0;
      for (int kc = 0; kc < KC; ++kc) {
        const int s = kc % STAGES;
        if (kc >= STAGES && !mbar_wait(bar_empty(s), ((kc / STAGES) - 1) & 1, abort)) break;
        ++issued;
        const uint32_t base = smem0 + s * plan.stage_bytes;
        mbar_arrive_expect_tx(bar_full(s), tx);
        tma_load_2d(base, &map_x, bar_full(s), kc * BK, m0);
        tma_load_2d(base + plan.a_bytes, &map_w0, bar_full(s), kc * BK, 0);
        if (n1 > 0)
          tma_load_2d(base + plan.a_bytes + (uint32_t)n0 * BK * 4, &map_w1, bar_full(s), kc * BK,
                      n0);
      }
      // Before the CTA may exit, every copy it issued must have landed (on the
      // normal path these waits succeed at once).
      for (int kc = issued - STAGES < 0 ? 0 : issued - STAGES; kc < issued; ++kc)
        mbar_wait(bar_full(kc % STAGES), (kc / STAGES) & 1, abort, true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t id0 = make_idesc(n0);
      const uint32_t id1 = n1 > 0 ? make_idesc(n1) : 0u;
      const uint32_t b1_off = (uint32_t)n0 * BK * 4;
      for (int kc = 0; kc < KC; ++kc) {
        const int s = kc % STAGES;
        const uint32_t ph = (kc / STAGES) & 1;
        if (!mbar_wait(P.use3x ? bar_conv(s) : bar_full(s), ph, abort)) break;
        tc_fence_after();
        const uint32_t a_hi = smem0 + s * plan.stage_bytes;
        const uint32_t b_hi = a_hi + plan.a_bytes;
        const uint32_t a_lo = a_hi + plan.hi_bytes;
        const uint32_t b_lo = b_hi + plan.hi_bytes;
        for (int kk = 0; kk < BK / 8; ++kk) {
          const uint32_t ko = kk * 32;  // 8 tf32 = 32 bytes along K
          const uint32_t acc0 = (kc > 0 || kk > 0) ? 1u : 0u;
          const uint64_t dah = make_desc(a_hi + ko, BK), dbh = make_desc(b_hi + ko, BK);
          mma_tf32(tmem_base, dah, dbh, id0, acc0);
          if (n1 > 0) mma_tf32(tmem_base + n0, dah, make_desc(b_hi + b1_off + ko, BK), id1, acc0);
          if (P.use3x) {
            const uint64_t dal = make_desc(a_lo + ko, BK), dbl = make_desc(b_lo + ko, BK);
            mma_tf32(tmem_base, dah, dbl, id0, 1u);
            mma_tf32(tmem_base, dal, dbh, id0, 1u);
            if (n1 > 0) {
              mma_tf32(tmem_base + n0, dah, make_desc(b_lo + b1_off + ko, BK), id1, 1u);
              mma_tf32(tmem_base + n0, dal, make_desc(b_hi + b1_off + ko, BK), id1, 1u);
            }
          }
        }
        mma_commit(bar_empty(s));
      }
      // Always commit the accumulator barrier, also after an abort, so the
      // epilogue can wait for every issued MMA to finish before TMEM is freed.
      mma_commit(bar_acc);
    }
  } else {
    // ---------------- 3xTF32 split, then epilogue ----------------
    const int ct = threadIdx.x - 64;  // 0..127
    if (P.use3x) {
      const int n4 = (int)(plan.hi_bytes / 16);
      for (int kc = 0; kc < KC; ++kc) {
        const int s = kc % STAGES;
        if (!mbar_wait(bar_full(s), (kc / STAGES) & 1, abort)) break;
        float4* hi = reinterpret_cast<float4*>(smem + s * plan.stage_bytes);
        float4* lo = reinterpret_cast<float4*>(smem + s * plan.stage_bytes + plan.hi_bytes);
        for (int i = ct; i < n4; i += 128) {
          float4 v = hi[i], h, l;
          h.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u); l.x = v.x - h.x;
          h.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u); l.y = v.y - h.y;
          h.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u); l.z = v.z - h.z;
          h.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u); l.w = v.w - h.w;
          hi[i] = h;
          lo[i] = l;
        }
        fence_proxy_async();
        mbar_arrive(bar_conv(s));
      }
    }

    // ---------------- epilogue: one thread = one token ----------------
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_acc, 0, abort));
    tc_fence_after();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const long tok = (long)m0 + row;
    const uint32_t trow = tmem_base + ((uint32_t)(q * 32) << 16);
    const int G = P.n_group, S = N / G;
    float v[32];

    if (ok && P.logits_out) {
      for (int c0 = 0; c0 < N; c0 += 32) {
        tmem_ld32(trow + c0, v);
        if (tok < P.T)
#pragma unroll
          for (int i = 0; i < 32; ++i) P.logits_out[tok * N + c0 + i] = v[i];
      }
    }

    uint32_t kept = 0xffffffffu;
    if (ok && G > 1) {
      // pass 1: group scores = sum of the two largest biased scores
      float a1 = -INFINITY, a2 = -INFINITY;
      int g = 0, next_b = S;
      for (int c0 = 0; c0 < N; c0 += 32) {
        tmem_ld32(trow + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = c0 + i;
          if (e == next_b) {
            gs_s[g * BM + row] = a1 + a2;
            ++g;
            next_b += S;
            a1 = -INFINITY;
            a2 = -INFINITY;
          }
          const float c = mr_sigmoid(v[i]) + bias_s[e];
          if (c > a1) {
            a2 = a1;
            a1 = c;
          } else if (c > a2) {
            a2 = c;
          }
        }
      }
      gs_s[g * BM + row] = a1 + a2;
      // keep topk_group groups (lower group index on ties)
      kept = 0;
      for (int r = 0; r < P.topk_group; ++r) {
        float bv = -INFINITY;
        int bg = -1;
        for (int gg = 0; gg < G; ++gg) {
          const float gv = gs_s[gg * BM + row];
          if (!((kept >> gg) & 1u) && (bg < 0 || gv > bv)) {
            bv = gv;
            bg = gg;
          }
        }
        kept |= 1u << bg;
      }
    }

    if (ok) {
      // pass 2: token top-k over the masked scores
      Top8 top;
      top.init();
      const bool zero_fill = (G > 1) && (P.mask_mode == MR_MASK_ZERO);
      int g = 0, next_b = S;
      for (int c0 = 0; c0 < N; c0 += 32) {
        tmem_ld32(trow + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = c0 + i;
          if (e == next_b) {
            ++g;
            next_b += S;
          }
          const bool keep = (kept >> g) & 1u;
          if (keep) {
            const float s = mr_sigmoid(v[i]);
            const float c = s + bias_s[e];
            if (c > top.v[kTopMax - 1]) top.push(c, e, s);
          } else if (zero_fill && 0.0f > top.v[kTopMax - 1]) {
            top.push(0.0f, e, mr_sigmoid(v[i]));
          }
        }
      }
      if (tok < P.T) {
        float den = 0.0f;
#pragma unroll
        for (int j = 0; j < kTopMax; ++j)
          if (j < P.k) den += top.s[j];
        den += 1e-20f;
#pragma unroll
        for (int j = 0; j < kTopMax; ++j) {
          if (j < P.k) {
            P.idx_out[tok * P.k + j] = top.i[j];
            P.w_out[tok * P.k + j] = (top.s[j] / den) * P.route_scale;
          }
        }
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

}  // namespace tc
}  // namespace mr
