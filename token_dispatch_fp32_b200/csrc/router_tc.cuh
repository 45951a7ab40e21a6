// router_tc.cuh -- fused gate GEMM + routing on the 5th-generation tensor cores.
//
// A cluster of CS CTAs (CS = 1, or 2 when the experts are split) owns a tile
// of 128 tokens; CTA r of the cluster owns experts [r*NL, (r+1)*NL), NL <= 256.
// A token's logits never go to HBM: they accumulate in tensor memory (TMEM
// lane = token, column = expert) and the routing epilogue reads them back.
//
//   warp 0      TMA producer: x tile [128 x BK] and W tile [NL x BK] per
//               stage (hardware swizzle), completion on an mbarrier.
//   warp 1      TMEM owner and MMA issuer (one elected thread), M = 128 (or
//               M = 256 over a CTA pair, cta_group::2), N = NL.
//   warps 2..9  "workers".
//
// Two ways to get fp32-accurate logits from the tensor cores:
//   3xTF32 (fp32 x): every staged fp32 value v splits into hi = v with the
//     low 13 mantissa bits cleared (exact in tf32) and lo = v - hi (exact in
//     fp32); kind::tf32 MMAs issue hi*hi + hi*lo + lo*hi.  The tensor core
//     ignores those 13 bits of a tf32 operand, so the staged tile serves as hi
//     unchanged and the workers only write lo; W's residuals may instead come
//     precomputed (TMA); lo(x)*hi(W) is skipped when a stage's x residuals are
//     all zero.
//   bf16x3 (bf16 x): W is stored once as three bf16 planes W1 + W2 + W3 that
//     sum to W exactly (24 significant bits); kind::f16 MMAs issue x*W1 +
//     x*W2 + x*W3, each product exact in fp32 -- the fp32 dot product of the
//     stored bf16 activations with the fp32 weights, up to accumulation order.
//   bf16 weights (bf16 x, W stored in bf16): the same kernel with one plane,
//     W itself; x*W is exact in fp32, one kind::f16 MMA per multiply-add.
//
// Promotion: the tensor core adds each product into its fp32 accumulator
// rounding toward zero, so one accumulator over all d would drift by ~1 ulp per
// MMA.  The K loop is cut into intervals of 128 K that alternate between two
// TMEM buffers; the workers add each finished interval into fp32 registers
// (round to nearest) while the tensor core fills the other buffer.
//
// Routing epilogue (all 8 workers; the sums go back to TMEM first): warps w
// and w+4 read the same 32 TMEM lanes (tokens), each half of the expert
// columns.  Pass 1 turns logits into s = sigmoid(L) in place and keeps the
// per-group top-2 of c = s + b (branch-free); the halves' pairs (and, with
// CS = 2, the peer CTA's through distributed shared memory) meet in shared
// memory and the topk_group best groups are kept.  Pass 2 forms each chunk's
// 16 masked candidates and inserts only those above the current 8th into a
// sorted top-8 list (lower index first on ties); the halves' lists (and the
// peer's) are merged bitonically; then renormalise and scale.
//
// Arithmetic follows the pages (Kimi K2 "Normalize weights" page,
// MoEGate.forward; DeepSeek-V3.2-Exp "Normalize weights" page, Gate.forward).
// Every mbarrier wait is bounded (MR_WAIT_LIMIT_NS); on expiry the CTA raises
// MR_FLAG_TIMEOUT, stops issuing work, drains its own copies and MMAs, still
// takes part in every cluster barrier, and frees its TMEM.
#pragma once

#include <cuda.h>

#include "mr_common.cuh"

namespace mr {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 32;                        // K elements per stage (fp32: 128-byte rows)
constexpr int kWorkers = 8;                   // worker warps 2..9
constexpr int kThreads = 64 + 32 * kWorkers;  // 320
constexpr int kPromote = 128 / BK;            // K chunks per accumulation interval (128 K)
constexpr int kMaxNL = 256;
constexpr int kMaxGroups = 32;
constexpr int kTopMax = 8;
constexpr int kMaxStages = 8;
constexpr uint32_t kSmemBudget = 232448;      // 227 KB opt-in per CTA

struct Params {
  int T, d, N, NL, CS, n_group, topk_group, k, mask_mode, num_kc, use3x;
  int wlo;  // W residuals W - trunc_tf32(W) arrive by TMA (map_wlo) instead of being split here
  // bf16x3: x is bf16 and W arrives as three bf16 planes W1 + W2 + W3 (map_w
  // over [3*N, d]); every product x*Wi is exact in fp32 (kind::f16 MMA).
  int bf16x3;
  // pair (bf16x3, N <= 256): the cluster's two CTAs own consecutive 128-token
  // tiles and run one M = 256 MMA (cta_group::2) issued by CTA 0; each CTA
  // stages its own x tile and half of W's rows, and keeps its own 128 tokens
  // x all N experts in its TMEM.
  int pair;
  // ksplit (CS = 1, not pair): a cluster of ksplit CTAs shares one 128-token
  // tile, CTA r taking K chunks [r*num_kc/ksplit, (r+1)*num_kc/ksplit); their
  // fp32 partial sums meet through distributed shared memory, summed in rank
  // order by the CTA that owns each lane quarter (quarter q % ksplit == r),
  // and only that CTA writes the quarter's tokens.
  int ksplit;
  int flags;  // MR_SCORE_SOFTMAX | MR_GROUP_MAX | MR_NORM_NO_EPS
  // part (the KS instantiation only): each CTA's fp32 sums over its K chunks
  // and expert columns go to part[slice][token][col0 + column], slice = its
  // K-split rank (0 without a K split), and the routing kernel that follows
  // adds the slices in order and routes the tokens; no exchange and no
  // epilogue run here
  float* part;
  float route_scale;
  const float* bias;
  int32_t* idx_out;
  float* w_out;
  float* logits_out;
};

// Shared-memory plan, identical on host and device.
struct Plan {
  int stages;
  uint32_t a_bytes, b_bytes, hi_bytes, stage_bytes;
  uint32_t bar_off, misc_off, bias_off, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Bytes of epilogue exchange space (aliases the stage ring after the K loop):
// per column half, group top-2 pairs and top-8 lists of 128 tokens, row
// maxima and sums of exponentials.
__host__ __device__ inline uint32_t exchange_bytes(int G) {
  return 4u * 2u * (2u * G * BM + 3u * kTopMax * BM + 2u * BM);
}
// Then, with one group, each worker thread's chunk top-2 pairs (16 slots);
// then the scores pass 1 leaves for pass 2, row by row ([BM][NL + 4] fp32).
constexpr uint32_t kChunkPairBytes = 4u * 16u * 32u * kWorkers;
__host__ __device__ inline uint32_t score_rows_offset(int G) {
  return exchange_bytes(G) + (G == 1 ? kChunkPairBytes : 0u);
}
__host__ __device__ inline uint32_t epilogue_smem_bytes(int G, int NL) {
  return score_rows_offset(G) + 4u * BM * (uint32_t)(NL + 4);
}

// Stage layout.  tf32: [x | W] fp32 tiles (hi) followed by their residuals
// (lo), 128-byte rows.  bf16: [x | W1 | W2 | W3] bf16 tiles (nplanes = 3) or
// [x | W] (nplanes = 1, W stored in bf16), 64-byte rows.  The ring and, after
// the K loop, the epilogue's space (G groups) share the front of shared
// memory; the barriers, flags and bias slice follow the larger of the two.
__host__ __device__ inline Plan make_plan(int NL, bool bf16x3 = false, bool pair = false,
                                          int nplanes = 3, int G = 1) {
  Plan p;
  const int esz = bf16x3 ? 2 : 4;
  p.a_bytes = BM * BK * esz;
  p.b_bytes = (pair ? NL / 2 : NL) * BK * esz;
  p.hi_bytes = p.a_bytes + (bf16x3 ? nplanes : 1) * p.b_bytes;
  p.stage_bytes = align_up((bf16x3 ? 1 : 2) * p.hi_bytes, 1024);
  // after the front: 256 B of mbarriers, 256 B of flags, the CTA's bias
  // slice; the launch adds 1 KB so the ring can start on a 1024-byte boundary
  const uint32_t extras = 1024 + 256 + 256 + 4 * kMaxNL;
  const uint32_t epi = align_up(epilogue_smem_bytes(G, NL), 16);
  int s = (int)((kSmemBudget - extras) / p.stage_bytes);
  p.stages = s > kMaxStages ? kMaxStages : s;
  auto front = [&](int st) {
    const uint32_t ring = (uint32_t)st * p.stage_bytes;
    return ring > epi ? ring : epi;
  };
  while (p.stages > 0 && front(p.stages) + extras > kSmemBudget) --p.stages;
  p.bar_off = front(p.stages);
  p.misc_off = p.bar_off + 256;
  p.bias_off = p.misc_off + 256;
  p.total = p.bias_off + 4 * kMaxNL;
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

// The same copy for a 2-SM pair: completes on an mbarrier given by its
// shared::cluster address, which may be the peer CTA's.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

// shared::cluster address of `local` in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local), "r"(rank));
  return ra;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from this CTA's shared memory to global memory, in the thread's bulk group.
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc),
               "r"(bytes)
               : "memory");
}
// Commit the thread's bulk stores and wait until they have completed (their
// writes performed, not only their shared-memory reads), so the grid's end
// orders them before a dependent grid's reads.
__device__ __forceinline__ void bulk_store_commit_and_wait() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void workers_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(32 * kWorkers) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Whole-cluster barrier; every thread of every CTA in the cluster calls it
// the same number of times, with its warp converged (.aligned).
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// 16 bytes from the same offset in CTA `peer`'s shared memory (16-byte aligned).
__device__ __forceinline__ float4 ld_peer_f32x4(const float* local, uint32_t peer) {
  uint32_t ra;
  float4 v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(peer));
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(ra)
               : "memory");
  return v;
}

__device__ __forceinline__ float ld_peer_f32(const float* local, uint32_t peer) {
  uint32_t ra, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(peer));
  asm volatile("ld.shared::cluster.b32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
  return __uint_as_float(v);
}

// UMMA shared-memory descriptor: K-major operand, rows of BK fp32 (128 bytes),
// 128-byte swizzle, 8-row groups 8 * 128 bytes apart.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr) {
  static_assert(BK == 32, "descriptor written for 128-byte rows");
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                      // LBO (unused when swizzled)
  d |= (uint64_t)(1024u >> 4) << 32;            // SBO
  d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                      // SWIZZLE_128B
  return d;
}

// Same for bf16 operands: rows of BK bf16 (64 bytes), 64-byte swizzle, 8-row
// groups 8 * 64 bytes apart.
__device__ __forceinline__ uint64_t make_desc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                      // LBO (unused when swizzled)
  d |= (uint64_t)(512u >> 4) << 32;             // SBO
  d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
  d |= (uint64_t)4u << 61;                      // SWIZZLE_64B
  return d;
}

// Instruction descriptor: D fp32, A/B tf32, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t make_idesc(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

// Instruction descriptor: D fp32, A/B bf16, both K-major, M = m, N = n.
__device__ __forceinline__ uint32_t make_idesc_bf16(int n, int m = BM) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t dtmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(dtmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
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

__device__ __forceinline__ void mma_bf16_pair(uint32_t dtmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(dtmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once every
// pair MMA issued so far has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 16-column loads (columns at ta and tb) and their wait in one asm
// statement, so one TMEM round trip serves 32 columns and no output register
// is visible to the compiler before the data has arrived.
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, float (&va)[16],
                                            float (&vb)[16]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(r[16 + i]);
  }
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
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
  // Keep the better (value desc, index asc) of slots a and b in a.
  __device__ __forceinline__ void order(int a, int b) {
    if (mr_better(v[b], i[b], v[a], i[a])) {
      const float tv = v[a]; v[a] = v[b]; v[b] = tv;
      const float ts = s[a]; s[a] = s[b]; s[b] = ts;
      const int ti = i[a]; i[a] = i[b]; i[b] = ti;
    }
  }
  // Merge another sorted list into this one, keeping the best 8: taking the
  // better of (this[j], other[7-j]) leaves the 8 best as a bitonic sequence,
  // which three half-cleaner rounds sort (all indices static, no branches
  // beyond the selects).
  __device__ __forceinline__ void merge(const float (&ov)[kTopMax], const float (&os)[kTopMax],
                                        const int (&oi)[kTopMax]) {
#pragma unroll
    for (int j = 0; j < kTopMax; ++j) {
      const int r = kTopMax - 1 - j;
      if (mr_better(ov[r], oi[r], v[j], i[j])) {
        v[j] = ov[r];
        s[j] = os[r];
        i[j] = oi[r];
      }
    }
#pragma unroll
    for (int d = kTopMax / 2; d > 0; d >>= 1)
#pragma unroll
      for (int j = 0; j < kTopMax; ++j)
        if ((j & d) == 0) order(j, j + d);
  }
  // Insert a candidate that beats the 8th entry.  Candidates arrive in index
  // order, so an equal value already listed keeps its place ahead of it
  // (lower index first): its slot is the count of listed values >= cv, and
  // every slot below it shifts down by one -- all slots at once, no chain of
  // compare-and-swap steps.
  __device__ __forceinline__ void push(float cv, int ci, float cs) {
    int pos = 0;
#pragma unroll
    for (int j = 0; j < kTopMax; ++j) pos += v[j] >= cv ? 1 : 0;
#pragma unroll
    for (int j = kTopMax - 1; j > 0; --j) {
      const bool sh = j > pos, put = j == pos;
      v[j] = sh ? v[j - 1] : (put ? cv : v[j]);
      s[j] = sh ? s[j - 1] : (put ? cs : s[j]);
      i[j] = sh ? i[j - 1] : (put ? ci : i[j]);
    }
    if (pos == 0) {
      v[0] = cv;
      s[0] = cs;
      i[0] = ci;
    }
  }
};

// Group choice of one token (one thread): the group score is the sum of the
// two best biased scores of the group, over the top-2 pairs that this CTA's
// two column halves (and, with CS = 2, the peer CTA's) left in exA1/exA2
// [half][group][row]; the topk_group best groups are kept (lower index first
// on ties), by counting for each group how many groups beat it.  tau: the
// smallest second-best score of the kept groups when 2*topk_group >= k.
template <int MAXG>
__device__ __forceinline__ void select_groups(int G, int topk_group, int k, int cs, uint32_t crank,
                                              const float* exA1, const float* exA2, int row,
                                              bool gmax, uint32_t& kept, float& tau) {
  float ga1[MAXG], ga2[MAXG];
#pragma unroll
  for (int g = 0; g < MAXG; ++g) {
    float a1 = -INFINITY, a2 = -INFINITY;
    if (g < G) {
#pragma unroll
      for (int src = 0; src < 4; ++src) {
        if (src >= 2 && cs == 1) break;
        const int hh = src & 1;
        float b1, b2;
        if (src < 2) {
          b1 = exA1[(hh * G + g) * BM + row];
          b2 = exA2[(hh * G + g) * BM + row];
        } else {
          b1 = ld_peer_f32(&exA1[(hh * G + g) * BM + row], crank ^ 1u);
          b2 = ld_peer_f32(&exA2[(hh * G + g) * BM + row], crank ^ 1u);
        }
        // top-2 of the union of two top-2 pairs
        const float hi = fmaxf(a1, b1);
        a2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
        a1 = hi;
      }
    }
    ga1[g] = a1;
    ga2[g] = a2;
  }
  kept = 0;
  float t = INFINITY;
#pragma unroll
  for (int g = 0; g < MAXG; ++g) {
    if (g < G) {
      const float sg = gmax ? ga1[g] : ga1[g] + ga2[g];
      int rank = 0;
#pragma unroll
      for (int o = 0; o < MAXG; ++o) {
        if (o < G && o != g) {
          const float so = gmax ? ga1[o] : ga1[o] + ga2[o];
          rank += (so > sg || (so == sg && o < g)) ? 1 : 0;
        }
      }
      if (rank < topk_group) {
        kept |= 1u << g;
        t = fminf(t, ga2[g]);
      }
    }
  }
  tau = (2 * topk_group >= k) ? t : -INFINITY;
}

// SOFTMAX: the MR_SCORE_SOFTMAX instantiation (its two statistics passes and
// cluster barriers are compiled out of the sigmoid kernel).
// NPL: bf16 planes of W (3: bf16x3; 1: W stored in bf16; the tf32 paths
// ignore it).  A compile-time count keeps the MMA issue loop fully unrolled.
// KS: the K-split instantiation (P.ksplit > 1); without it the K-split code
// is compiled out of the one-CTA-per-tile kernel.
template <bool PAIR, bool SOFTMAX, int NPL = 3, bool KS = false>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_wlo, const Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned start by pointer arithmetic on the shared array, so the
  // compiler keeps the shared address space for every access through it (an
  // integer round trip would turn them into generic loads and stores)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int NL = P.NL;
  const bool bf16x3 = P.bf16x3 != 0;
  // The 2-SM instructions exist only in the PAIR instantiation: a kernel that
  // contains them must be launched in clusters of two.
  constexpr bool pair = PAIR;
  constexpr int NP = NPL;
  const Plan plan = make_plan(NL, bf16x3, pair, NP, P.n_group);
  const int STAGES = plan.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KSP = KS ? P.ksplit : 1;
  const uint32_t crank = (P.CS > 1 || pair || KSP > 1) ? cluster_rank() : 0u;
  const int tile = pair ? (int)blockIdx.x : (int)blockIdx.x / (P.CS * KSP);
  const int col0 = (pair || KSP > 1) ? 0 : (int)crank * NL;  // first expert of the accumulator
  const bool leader = !pair || crank == 0;       // issues the MMAs
  const int wrow0 = pair ? (int)crank * (NL / 2) : col0;  // first W row this CTA stages

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  // [0,S) full  [S,2S) converted  [2S,3S) empty  3S+{0,1} acc full
  // 3S+{2,3} acc free  3S+4 MMA drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + plan.misc_off);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + plan.misc_off + 8);
  // xnz[s][w]: worker warp w saw a nonzero x residual in stage s on this pass of the ring
  volatile uint32_t* xnz = reinterpret_cast<volatile uint32_t*>(smem + plan.misc_off + 32);
  float* bias_s = reinterpret_cast<float*>(smem + plan.bias_off);

  const uint32_t smem0 = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int B_FULL = 0, B_CONV = STAGES, B_EMPTY = 2 * STAGES, B_ACCF = 3 * STAGES,
            B_ACCE = 3 * STAGES + 2, B_DRAIN = 3 * STAGES + 4;
  const uint32_t tmem_cols = 2 * NL <= 32 ? 32 : 2 * NL <= 64 ? 64 : 2 * NL <= 128 ? 128
                           : 2 * NL <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    // the descriptors live in the kernel parameters: fetch them during set-up
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    if (P.wlo)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_wlo))
                   : "memory");
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_CONV + s), kWorkers);  // one elected arrival per worker warp
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_ACCF + 0), 1);
    mbar_init(bar(B_ACCF + 1), 1);
    // one arrival per worker warp (of both CTAs in a pair)
    mbar_init(bar(B_ACCE + 0), (pair ? 2 : 1) * kWorkers);
    mbar_init(bar(B_ACCE + 1), (pair ? 2 : 1) * kWorkers);
    mbar_init(bar(B_DRAIN), 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(tmem_cols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(tmem_cols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  // pair: barriers must be initialised in both CTAs before any remote use
  if (pair) cluster_sync_all();
  // Launched as a programmatic dependent: the set-up above overlaps the
  // preceding kernel (W's planes or residuals); no global input is read
  // before that grid has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // with part, the routing kernel is this grid's programmatic dependent: it
  // may be scheduled now and waits for this grid's completion itself
  if (KS && P.part) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int e = threadIdx.x; e < NL; e += kThreads)
    bias_s[e] = P.bias ? P.bias[col0 + e] : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int m0 = tile * BM;
  // this CTA's K chunks: all of them, or its share of a K-split cluster
  const int kc0 = KSP > 1 ? (int)(((long)crank * P.num_kc) / KSP) : 0;
  const int KC = KSP > 1 ? (int)(((long)(crank + 1) * P.num_kc) / KSP) - kc0 : P.num_kc;
  const int J = (KC + kPromote - 1) / kPromote;  // accumulation intervals

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint32_t tx = bf16x3 ? plan.hi_bytes
                                 : (uint32_t)(BM + (P.wlo ? 2 : 1) * NL) * BK * 4;
      int issued = 0;
      // stage s of the ring and the parity ph of its current round, kept
      // incrementally (no division by the run-time stage count per chunk)
      int s = 0;
      uint32_t ph = 0;
      for (int kc = 0; kc < KC; ++kc, (++s == STAGES ? (s = 0, ph ^= 1u) : 0u)) {
        if (kc >= STAGES && !mbar_wait(bar(B_EMPTY + s), ph ^ 1u, abort)) break;
        ++issued;
        const uint32_t base = smem0 + s * plan.stage_bytes;
        if constexpr (PAIR) {
          // both CTAs' copies complete on CTA 0's full barrier
          const uint32_t fb = cluster_addr(bar(B_FULL + s), 0);
          if (leader) mbar_arrive_expect_tx(bar(B_FULL + s), 2 * tx);
          tma_load_2d_pair(base, &map_x, fb, (kc0 + kc) * BK, m0);
#pragma unroll
          for (int pl = 0; pl < NP; ++pl)
            tma_load_2d_pair(base + plan.a_bytes + pl * plan.b_bytes, &map_w, fb, (kc0 + kc) * BK,
                             pl * P.N + wrow0);
          continue;
        }
        mbar_arrive_expect_tx(bar(B_FULL + s), tx);
        tma_load_2d(base, &map_x, bar(B_FULL + s), (kc0 + kc) * BK, m0);
        if (bf16x3) {
#pragma unroll
          for (int pl = 0; pl < NP; ++pl)
            tma_load_2d(base + plan.a_bytes + pl * plan.b_bytes, &map_w, bar(B_FULL + s),
                        (kc0 + kc) * BK, pl * P.N + col0);
        } else {
          tma_load_2d(base + plan.a_bytes, &map_w, bar(B_FULL + s), (kc0 + kc) * BK, col0);
          if (P.wlo)
            tma_load_2d(base + plan.hi_bytes + plan.a_bytes, &map_wlo, bar(B_FULL + s), (kc0 + kc) * BK,
                        col0);
        }
      }
      // Every copy this CTA issued must land before the CTA may exit (on the
      // normal path these waits succeed at once).  A pair's copies complete
      // on CTA 0's barriers: CTA 0 drains them, CTA 1 is held by the final
      // cluster barrier until then.
      if (leader)
        for (int kc = issued - STAGES < 0 ? 0 : issued - STAGES; kc < issued; ++kc)
          mbar_wait(bar(B_FULL + kc % STAGES), (kc / STAGES) & 1, abort, true);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && !leader) {
      // CTA 1 of a pair: CTA 0's MMAs write this CTA's TMEM; wait for them
      mbar_wait(bar(B_DRAIN), 0, abort, true);
    } else if (lane == 0) {
      const uint32_t idesc = bf16x3 ? make_idesc_bf16(NL, pair ? 2 * BM : BM) : make_idesc(NL);
      int s = 0;
      uint32_t ph = 0;  // stage and round parity, kept incrementally
      for (int kc = 0; kc < KC; ++kc, (++s == STAGES ? (s = 0, ph ^= 1u) : 0u)) {
        const int j = kc / kPromote, b = j & 1;
        const bool first = (kc % kPromote) == 0;
        if (first && j >= 2 && !mbar_wait(bar(B_ACCE + b), ((j >> 1) - 1) & 1, abort)) break;
        if (!mbar_wait((P.use3x && !bf16x3) ? bar(B_CONV + s) : bar(B_FULL + s), ph, abort))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(b * NL);
        if (bf16x3) {
          const uint32_t a = smem0 + s * plan.stage_bytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t ko = kk * 32;  // 16 bf16 = 32 bytes along K
            const uint64_t da = make_desc_sw64(a + ko);
#pragma unroll
            for (int pl = 0; pl < NP; ++pl) {
              const uint64_t db = make_desc_sw64(a + plan.a_bytes + pl * plan.b_bytes + ko);
              const uint32_t acc = (!first || kk > 0 || pl > 0) ? 1u : 0u;
              if constexpr (PAIR)
                mma_bf16_pair(d_tmem, da, db, idesc, acc);
              else
                mma_bf16(d_tmem, da, db, idesc, acc);
            }
          }
          const bool iv_end = (kc % kPromote) == kPromote - 1 || kc == KC - 1;
          if constexpr (PAIR) {
            mma_commit_pair(bar(B_EMPTY + s));
            if (iv_end) mma_commit_pair(bar(B_ACCF + b));
          } else {
            mma_commit(bar(B_EMPTY + s));
            if (iv_end) mma_commit(bar(B_ACCF + b));
          }
          continue;
        }
        const uint32_t a_hi = smem0 + s * plan.stage_bytes;
        const uint32_t b_hi = a_hi + plan.a_bytes;
        const uint32_t a_lo = a_hi + plan.hi_bytes;
        const uint32_t b_lo = b_hi + plan.hi_bytes;
        // lo(x) * hi(W) adds exact zeros when every x residual of the stage
        // is 0 (x already tf32-exact, e.g. bf16 activations): skip it.
        bool x_lo = false;
        if (P.use3x)
#pragma unroll
          for (int w = 0; w < kWorkers; ++w) x_lo |= xnz[s * kWorkers + w] != 0u;
#pragma unroll
        for (int kk = 0; kk < BK / 8; ++kk) {
          const uint32_t ko = kk * 32;  // 8 tf32 = 32 bytes along K
          const uint32_t acc0 = (!first || kk > 0) ? 1u : 0u;
          const uint64_t dah = make_desc(a_hi + ko), dbh = make_desc(b_hi + ko);
          mma_tf32(d_tmem, dah, dbh, idesc, acc0);
          if (P.use3x) {
            mma_tf32(d_tmem, dah, make_desc(b_lo + ko), idesc, 1u);
            if (x_lo) mma_tf32(d_tmem, make_desc(a_lo + ko), dbh, idesc, 1u);
          }
        }
        mma_commit(bar(B_EMPTY + s));
        if ((kc % kPromote) == kPromote - 1 || kc == KC - 1) mma_commit(bar(B_ACCF + b));
      }
      // Track every MMA issued so far; waited on before TMEM is released.
      if constexpr (PAIR)
        mma_commit_pair(bar(B_DRAIN));
      else
        mma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, abort, true);
    }
  } else {
    // ---------------- workers: split, promotion ----------------
    const int wt = threadIdx.x - 64;  // 0..255
    const int q = warp & 3;           // TMEM lane quarter
    const int h = (warp - 2) >> 2;    // column half
    const int n16 = NL / 16;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float acc[8][16];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[i][c] = 0.0f;
    int promoted = 0;
    bool ok = true;

    auto promote = [&](int j) {
      const int b = j & 1;
      if (!mbar_wait(bar(B_ACCF + b), (j >> 1) & 1, abort)) {
        ok = false;
        return;
      }
      tc_fence_after();
      // chunks h, h+2, ..., two per TMEM round trip
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const int c = h + 2 * i;
        if (c + 2 < n16) {
          float v0[16], v1[16];
          tmem_ld16x2(tmem_base + lane_off + (uint32_t)(b * NL + c * 16),
                      tmem_base + lane_off + (uint32_t)(b * NL + (c + 2) * 16), v0, v1);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            acc[i][e] += v0[e];
            acc[i + 1][e] += v1[e];
          }
        } else if (c < n16) {
          float v0[16];
          tmem_ld16(tmem_base + lane_off + (uint32_t)(b * NL + c * 16), v0);
#pragma unroll
          for (int e = 0; e < 16; ++e) acc[i][e] += v0[e];
        }
      }
      // Every lane's loads have completed (tcgen05.wait::ld); one elected
      // arrival per warp releases the buffer to the MMA issuer (a pair's
      // CTA 1 arrives on CTA 0's barrier, a cluster-scope release).
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && !leader)
          mbar_arrive_cluster(cluster_addr(bar(B_ACCE + b), 0));
        else
          mbar_arrive(bar(B_ACCE + b));
      }
      ++promoted;
    };

    const int n4a = (int)(plan.a_bytes / 16);  // the x part of [A | B]
    const int n4 = P.wlo ? n4a : (int)(plan.hi_bytes / 16);
    int s = 0;
    uint32_t ph = 0;
    for (int kc = 0; kc < KC && ok; ++kc, (++s == STAGES ? (s = 0, ph ^= 1u) : 0u)) {
      if (P.use3x && !bf16x3) {
        if (!mbar_wait(bar(B_FULL + s), ph, abort)) {
          ok = false;
          break;
        }
        // The tensor core reads a kind::tf32 operand with its 13 low mantissa
        // bits ignored (truncation), so the staged fp32 tile already is the
        // hi part; only the residual lo = v - trunc(v) is written.
        const float4* hi = reinterpret_cast<const float4*>(smem + s * plan.stage_bytes);
        float4* lo = reinterpret_cast<float4*>(smem + s * plan.stage_bytes + plan.hi_bytes);
        uint32_t nz = 0;
        for (int i = wt; i < n4; i += 32 * kWorkers) {
          const float4 v = hi[i];
          float4 l;
          l.x = v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
          l.y = v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
          l.z = v.z - __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
          l.w = v.w - __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
          lo[i] = l;
          if (i < n4a)
            nz |= __float_as_uint(l.x) | __float_as_uint(l.y) | __float_as_uint(l.z) |
                  __float_as_uint(l.w);
        }
        const bool any_nz = __any_sync(0xffffffffu, (nz << 1) != 0u);  // ignore -0.0
        if (lane == 0) xnz[s * kWorkers + (warp - 2)] = any_nz ? 1u : 0u;
        // each thread's residual writes become visible to the async proxy;
        // then one lane per warp releases the stage
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_CONV + s));
      }
      // promote the interval before the one the tensor core is working on
      if ((kc % kPromote) == kPromote - 1 && kc / kPromote >= 1) promote(kc / kPromote - 1);
    }
    while (ok && promoted < J) promote(promoted);
    ok = __all_sync(0xffffffffu, ok);

    if (KS && P.part) {
      // the fp32 sums of this CTA's rows over its K chunks to
      // part[rank][token][expert]: staged row by row in the idle ring
      // ([BM][NL + 4], the pad keeps a warp's rows on distinct banks), then
      // one bulk copy per row (a thread's own row stores would scatter every
      // warp store over 32 rows)
      const int row = q * 32 + lane;
      const int NLp = NL + 4;
      float* xrow = reinterpret_cast<float*>(smem) + row * NLp;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = h + 2 * i;
        if (c < n16) {
          float4* d4 = reinterpret_cast<float4*>(xrow + c * 16);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            d4[jj] = make_float4(acc[i][4 * jj], acc[i][4 * jj + 1], acc[i][4 * jj + 2],
                                 acc[i][4 * jj + 3]);
        }
      }
      fence_proxy_async();  // the generic writes, visible to the bulk copies
      workers_sync();
      if (ok && wt < BM && (long)m0 + wt < P.T) {
        const long slice = KSP > 1 ? (long)crank : 0;
        bulk_store(P.part + (slice * P.T + m0 + wt) * P.N + col0,
                   smem_u32(reinterpret_cast<float*>(smem) + wt * NLp), (uint32_t)NL * 4);
        bulk_store_commit_and_wait();
      }
    } else {

    // K-split: the ksplit CTAs of the cluster hold partial sums over their K
    // chunks.  Each writes its partials to its (now idle) ring, [BM][NL + 4]
    // fp32 (the pad keeps a warp's rows on distinct banks); after a cluster
    // barrier the owner of each lane quarter (q % ksplit == rank) sums the
    // ksplit partials of its rows in rank order (the same order whichever CTA
    // owns them), and a second barrier keeps every ring alive until its
    // readers are done.  The other quarters' rows keep their partials; their
    // routing below runs but writes nothing.
    const bool own_q = KSP == 1 || (q % KSP) == (int)crank;
    if (KSP > 1) {
      const int row = q * 32 + lane;
      const int NLp = NL + 4;
      float* xpart = reinterpret_cast<float*>(smem);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = h + 2 * i;
        if (c < n16) {
          float4* d4 = reinterpret_cast<float4*>(&xpart[row * NLp + c * 16]);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_float4(acc[i][4 * j], acc[i][4 * j + 1], acc[i][4 * j + 2],
                                acc[i][4 * j + 3]);
        }
      }
      if (!ok && lane == 0) *abort = 1;
      cluster_sync_all();  // K-split #1: partials and abort flags visible
      int bad = 0;
      for (int r = 0; r < KSP; ++r)
        bad |= __float_as_int(
            ld_peer_f32(reinterpret_cast<const float*>(const_cast<const int*>(abort)), (uint32_t)r));
      ok = ok && bad == 0;
      if (own_q && ok) {
        // per 8 columns, every peer's two float4 loads are issued before the
        // first add (one remote round trip per 8 columns, not one per load),
        // then summed in rank order
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c = h + 2 * i;
          if (c < n16) {
#pragma unroll
            for (int jj = 0; jj < 4; jj += 2) {
              float4 v[4][2];  // [peer][float4]
#pragma unroll
              for (int r = 0; r < 4; ++r)
                if (r < KSP)
#pragma unroll
                  for (int j = 0; j < 2; ++j)
                    v[r][j] = ld_peer_f32x4(&xpart[row * NLp + c * 16 + 4 * (jj + j)],
                                            (uint32_t)r);
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                float4 sum = v[0][j];
#pragma unroll
                for (int r = 1; r < 4; ++r)
                  if (r < KSP) {
                    sum.x += v[r][j].x;
                    sum.y += v[r][j].y;
                    sum.z += v[r][j].z;
                    sum.w += v[r][j].w;
                  }
                acc[i][4 * (jj + j)] = sum.x;
                acc[i][4 * (jj + j) + 1] = sum.y;
                acc[i][4 * (jj + j) + 2] = sum.z;
                acc[i][4 * (jj + j) + 3] = sum.w;
              }
            }
          }
        }
      }
      cluster_sync_all();  // K-split #2: every peer has read this CTA's partials
    }

    // final sums back to TMEM buffer 0 for the routing epilogue
    if (ok) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = h + 2 * i;
        if (c < n16) tmem_st16(tmem_base + lane_off + (uint32_t)(c * 16), acc[i]);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    workers_sync();
    tc_fence_after();
    if (*abort) ok = false;
    ok = __all_sync(0xffffffffu, ok);

    // ---------------- routing epilogue: all 8 workers ----------------
    // Warps w and w+4 read the same 32 TMEM lanes (tokens); half h of the
    // pair takes chunks [h*nh, (h+1)*nh) of this CTA's expert columns.  Group
    // top-2 pairs and top-8 lists of the halves (and, with CS = 2, of the peer
    // CTA's halves) meet in shared memory, so every routing step runs on two
    // warps per SM sub-partition.
    {
      const int row = q * 32 + lane;
      const long tok = (long)m0 + row;
      const int G = P.n_group, S = P.N / G;
      const int cs = P.CS;
      const int nh = (n16 + 1) / 2;
      const int c_beg = h * nh, c_end = (c_beg + nh < n16) ? c_beg + nh : n16;
      // exchange space aliases the (now idle) stage ring
      float* exA1 = reinterpret_cast<float*>(smem);             // [2][G][BM]
      float* exA2 = exA1 + 2 * G * BM;                           // [2][G][BM]
      float* exV = exA2 + 2 * G * BM;                            // [2][8][BM]
      float* exS = exV + 2 * kTopMax * BM;                       // [2][8][BM]
      int* exI = reinterpret_cast<int*>(exS + 2 * kTopMax * BM); // [2][8][BM]
      float* exM = reinterpret_cast<float*>(exI + 2 * kTopMax * BM);  // [2][BM] row max
      float* exZ = exM + 2 * BM;                                 // [2][BM] sum of exp
      constexpr bool softmax = SOFTMAX;
      float v[16], v2[16], bv[16];
      auto load_bias = [&](int c) {
        const float4* b4 = reinterpret_cast<const float4*>(bias_s + c * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 t = b4[i];
          bv[4 * i] = t.x;
          bv[4 * i + 1] = t.y;
          bv[4 * i + 2] = t.z;
          bv[4 * i + 3] = t.w;
        }
      };

      if (ok && P.logits_out) {
        for (int c = c_beg; c < c_end; ++c) {
          __syncwarp();
          tmem_ld16(tmem_base + lane_off + (uint32_t)(c * 16), v);  // whole warp
          if (tok < P.T && own_q)
#pragma unroll
            for (int e = 0; e < 16; ++e) P.logits_out[tok * P.N + col0 + c * 16 + e] = v[e];
        }
      }

      // softmax scores need the row's largest logit and its sum of
      // exponentials over all experts (both halves; with CS = 2 the peer's)
      float smx = 0.0f, sinv = 1.0f;
      if constexpr (softmax) {
        float mx = -INFINITY;
        if (ok)
          for (int c = c_beg; c < c_end; c += 2) {
            const int c2 = c + 1 < c_end ? c + 1 : c;
            tmem_ld16x2(tmem_base + lane_off + (uint32_t)(c * 16),
                        tmem_base + lane_off + (uint32_t)(c2 * 16), v, v2);
#pragma unroll
            for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fmaxf(v[i], v2[i]));
          }
        exM[h * BM + row] = mx;
        workers_sync();
        if (cs > 1) cluster_sync_all();  // softmax #a: row maxima visible
        smx = fmaxf(exM[row], exM[BM + row]);
        if (cs > 1) smx = fmaxf(smx, fmaxf(ld_peer_f32(&exM[row], crank ^ 1u),
                                           ld_peer_f32(&exM[BM + row], crank ^ 1u)));
        float z = 0.0f;
        if (ok)
          for (int c = c_beg; c < c_end; c += 2) {
            const int c2 = c + 1 < c_end ? c + 1 : c;
            tmem_ld16x2(tmem_base + lane_off + (uint32_t)(c * 16),
                        tmem_base + lane_off + (uint32_t)(c2 * 16), v, v2);
#pragma unroll
            for (int i = 0; i < 16; ++i) z += __expf(v[i] - smx);
            if (c2 != c)
#pragma unroll
              for (int i = 0; i < 16; ++i) z += __expf(v2[i] - smx);
          }
        exZ[h * BM + row] = z;
        workers_sync();
        if (cs > 1) cluster_sync_all();  // softmax #b: partial sums visible
        // the CTA that owns experts [0, NL) adds first: both CTAs of a
        // cluster form the same sum
        float zsum = exZ[row] + exZ[BM + row];
        if (cs > 1) {
          const float zp = ld_peer_f32(&exZ[row], crank ^ 1u) + ld_peer_f32(&exZ[BM + row], crank ^ 1u);
          zsum = crank == 0 ? zsum + zp : zp + zsum;
        }
        sinv = 1.0f / zsum;
      }

      // pass 1: s = sigmoid(L) (or softmax) into this row of shared memory;
      // per-group top-2 of c = s + b
      uint32_t kept = 0xffffffffu;
      // with one group, each chunk's top-2 goes to slots 2j, 2j + 1 (chunk
      // c_beg + j) of this thread's pairs, for the bound tau below
      float* chunk_pairs = reinterpret_cast<float*>(smem + exchange_bytes(G));
      // the scores, [BM][NL + 4] (the pad keeps a warp's rows on distinct banks)
      float* srow = reinterpret_cast<float*>(smem + score_rows_offset(G)) + row * (NL + 4);
      {
        if (G > 1)
          for (int g = 0; g < G; ++g) {
            exA1[(h * G + g) * BM + row] = -INFINITY;
            exA2[(h * G + g) * BM + row] = -INFINITY;
          }
        if (ok && c_beg < c_end) {
          float a1 = -INFINITY, a2 = -INFINITY;
          int g = (col0 + c_beg * 16) / S, next_b = (g + 1) * S;
          // S a multiple of 16: every 16-column chunk lies inside one group
          const bool chunk_groups = (S % 16) == 0;
          // one chunk per iteration (one copy of the body in the code: the
          // routing runs once per CTA, so its instructions are fetched cold)
#pragma unroll 1
          for (int c = c_beg; c < c_end; ++c) {
            __syncwarp();
            tmem_ld16(tmem_base + lane_off + (uint32_t)(c * 16), v);
            load_bias(c);
            if constexpr (softmax) {
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = __expf(v[i] - smx) * sinv;
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = mr_sigmoid(v[i]);
            }
            {
              float4* d4 = reinterpret_cast<float4*>(srow + c * 16);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                d4[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            }
            if (G == 1 || chunk_groups) {
              const int gc = (col0 + c * 16) / S;
              if (G > 1 && gc != g) {
                exA1[(h * G + g) * BM + row] = a1;
                exA2[(h * G + g) * BM + row] = a2;
                g = gc;
                a1 = -INFINITY;
                a2 = -INFINITY;
              }
              // the chunk's top-2 of c = s + b as a tree of pair merges
              float p1[8], p2[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float x0 = v[2 * j] + bv[2 * j], x1 = v[2 * j + 1] + bv[2 * j + 1];
                p1[j] = fmaxf(x0, x1);
                p2[j] = fminf(x0, x1);
              }
#pragma unroll
              for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) {
                  const float hi = fmaxf(p1[j], p1[j + w]);
                  p2[j] = fmaxf(fminf(p1[j], p1[j + w]), fmaxf(p2[j], p2[j + w]));
                  p1[j] = hi;
                }
              if (G == 1) {
                chunk_pairs[(2 * (c - c_beg)) * 32 * kWorkers + wt] = p1[0];
                chunk_pairs[(2 * (c - c_beg) + 1) * 32 * kWorkers + wt] = p2[0];
                continue;
              }
              const float hi = fmaxf(a1, p1[0]);
              a2 = fmaxf(fminf(a1, p1[0]), fmaxf(a2, p2[0]));
              a1 = hi;
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int e = col0 + c * 16 + i;
                if (e == next_b) {
                  exA1[(h * G + g) * BM + row] = a1;
                  exA2[(h * G + g) * BM + row] = a2;
                  ++g;
                  next_b += S;
                  a1 = -INFINITY;
                  a2 = -INFINITY;
                }
                const float cval = v[i] + bv[i];
                a2 = fmaxf(a2, fminf(a1, cval));  // top-2 of the values seen
                a1 = fmaxf(a1, cval);
              }
            }
          }
          if (G > 1) {
            exA1[(h * G + g) * BM + row] = a1;
            exA2[(h * G + g) * BM + row] = a2;
          }
        }
      }
      workers_sync();
      if (cs > 1) cluster_sync_all();  // #1: group pairs visible to the peer
      // Group choice from the merged per-group top-2 pairs, and a lower
      // bound tau on the k-th best masked score: the kept groups' top-2
      // values are 2*topk_group distinct candidates, so when that is >= k
      // the k-th best of all candidates is >= the smallest of them.
      float tau = -INFINITY;
      if (G == 1 && ok && c_beg < c_end) {
        // One group: the ceil(k/2) chunks of this half with the largest
        // maxima hold at least k distinct scores >= the smallest of their
        // second-best values, so the half's -- and the token's -- k-th best
        // is >= that value.
        const int nc = c_end - c_beg, need = (P.k + 1) / 2;
        if (nc >= need) {
          float u1[8], u2[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            u1[j] = j < nc ? chunk_pairs[(2 * j) * 32 * kWorkers + wt] : -INFINITY;
            u2[j] = j < nc ? chunk_pairs[(2 * j + 1) * 32 * kWorkers + wt] : -INFINITY;
          }
          float t = INFINITY;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            int rank = 0;
#pragma unroll
            for (int l = 0; l < 8; ++l) rank += (u1[l] > u1[j] || (u1[l] == u1[j] && l < j)) ? 1 : 0;
            if (j < nc && rank < need) t = fminf(t, u2[j]);
          }
          tau = t;
        }
      }
      if (G > 1) {
        const bool gmax = (P.flags & MR_GROUP_MAX) != 0;
        if (G <= 8)
          select_groups<8>(G, P.topk_group, P.k, cs, crank, exA1, exA2, row, gmax, kept, tau);
        else
          select_groups<kMaxGroups>(G, P.topk_group, P.k, cs, crank, exA1, exA2, row, gmax, kept,
                                    tau);
      }

      // pass 2: top-8 of this half's masked scores.  Each chunk's candidates
      // (scores >= tau) are marked in a 16-bit mask from the scores pass 1
      // left in shared memory; only the marked ones are read back and
      // inserted, in index order, when they beat the list's current 8th.
      Top8 top;
      top.init();
      if (ok && c_beg < c_end) {
        const float fill = (G > 1 && P.mask_mode == MR_MASK_ZERO) ? 0.0f : -INFINITY;
        // bit i: expert col0 + 16c + i lies in a kept group
        auto keep_mask = [&](int c) -> uint32_t {
          if (G == 1) return 0xffffu;
          const int e0 = col0 + c * 16;
          if ((S % 16) == 0) return ((kept >> (e0 / S)) & 1u) ? 0xffffu : 0u;
          uint32_t km = 0;
#pragma unroll
          for (int i = 0; i < 16; ++i) km |= ((kept >> ((e0 + i) / S)) & 1u) << i;
          return km;
        };
#pragma unroll 1
        for (int c = c_beg; c < c_end; ++c) {
          load_bias(c);
          const uint32_t km = keep_mask(c);
          const float4* s4 = reinterpret_cast<const float4*>(srow + c * 16);
          uint32_t mlo = 0, mhi = 0;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const float4 sv = s4[q4];
            const float e4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int i = 4 * q4 + u;
              const float cval = ((km >> i) & 1u) ? e4[u] + bv[i] : fill;
              const uint32_t bit = (cval >= tau ? 1u : 0u) << i;
              if (i < 8) mlo |= bit; else mhi |= bit;
            }
          }
          for (uint32_t m = mlo | mhi; m != 0u; m &= m - 1u) {
            const int i = __ffs(m) - 1;
            const float sv = srow[c * 16 + i];
            const float cval = ((km >> i) & 1u) ? sv + bias_s[c * 16 + i] : fill;
            if (cval > top.v[kTopMax - 1]) top.push(cval, col0 + c * 16 + i, sv);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kTopMax; ++j) {
        exV[(h * kTopMax + j) * BM + row] = top.v[j];
        exS[(h * kTopMax + j) * BM + row] = top.s[j];
        exI[(h * kTopMax + j) * BM + row] = top.i[j];
      }
      workers_sync();
      if (cs > 1) cluster_sync_all();  // #2: top-8 lists visible to the peer
      if (h == 0 && (PAIR || cs == 1 || crank == 0)) {
        // merge the other half's list, then (experts split over the cluster)
        // the peer CTA's two lists; a pair's CTAs each own their tokens, and
        // so do a K-split cluster's (by lane quarter, own_q)
#pragma unroll 1
        for (int src = 1; src < 4; ++src) {
          if (src >= 2 && cs == 1) break;
          const int hh = src & 1;
          float pv[kTopMax], ps[kTopMax];
          int pi[kTopMax];
#pragma unroll
          for (int j = 0; j < kTopMax; ++j) {
            const int o = (hh * kTopMax + j) * BM + row;
            if (src < 2) {
              pv[j] = exV[o];
              ps[j] = exS[o];
              pi[j] = exI[o];
            } else {
              pv[j] = ld_peer_f32(&exV[o], 1u);
              ps[j] = ld_peer_f32(&exS[o], 1u);
              pi[j] = __float_as_int(ld_peer_f32(reinterpret_cast<float*>(&exI[o]), 1u));
            }
          }
          top.merge(pv, ps, pi);
        }
        if (ok && tok < P.T && own_q) {
          float den = 0.0f;
#pragma unroll
          for (int j = 0; j < kTopMax; ++j)
            if (j < P.k) den += top.s[j];
#pragma unroll
          for (int j = 0; j < kTopMax; ++j) {
            if (j < P.k) {
              P.idx_out[tok * P.k + j] = top.i[j];
              P.w_out[tok * P.k + j] = mr_weight(top.s[j], den, P.route_scale, P.flags);
            }
          }
        }
      }
      if (cs > 1) cluster_sync_all();  // #3: the peer's lists have been read
    }
    }  // !P.part
  }

  // Threads that take no part in the routing epilogue still join its cluster
  // barriers (three; five with softmax scores), so a cluster always completes
  // them.
  if (P.CS > 1 && !(KS && P.part) && warp < 2) {
    const int n_sync = SOFTMAX ? 5 : 3;
    for (int i = 0; i < n_sync; ++i) cluster_sync_all();
  }
  // ... and the two barriers of the K-split exchange
  if (KSP > 1 && !(KS && P.part) && warp < 2) {
    cluster_sync_all();
    cluster_sync_all();
  }
  tc_fence_before();
  __syncthreads();
  // pair: neither CTA leaves while the other may still read its shared memory
  // (CTA 0's MMAs read CTA 1's tiles), arrive on its barriers or copy into it
  if (pair) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(tmem_cols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(tmem_cols)
                   : "memory");
  }
}

// W_lo = W - trunc_tf32(W), once per call, so the router's CTAs stream the
// residuals by TMA instead of each re-deriving them in shared memory.
__global__ void __launch_bounds__(256) split_residual_kernel(const float4* __restrict__ W,
                                                             float4* __restrict__ Wlo, long n4) {
  // the router grid (a programmatic dependent) may be scheduled now; it
  // waits for this grid's completion before it reads anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (long i = blockIdx.x * 256L + threadIdx.x; i < n4; i += (long)gridDim.x * 256) {
    const float4 v = __ldg(W + i);
    float4 l;
    l.x = v.x - __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
    l.y = v.y - __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
    l.z = v.z - __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
    l.w = v.w - __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
    Wlo[i] = l;
  }
}

// W -> three bf16 planes with W1 + W2 + W3 = W to within 2^-24 relative:
// W1 = bf16(W), W2 = bf16(W - W1), W3 = bf16(W - W1 - W2) (round to nearest
// even; each difference is exact in fp32).  Planes stacked as [3][N_r*d].
__device__ __forceinline__ void split3(float w, __nv_bfloat16& p1, __nv_bfloat16& p2,
                                       __nv_bfloat16& p3) {
  p1 = __float2bfloat16_rn(w);
  const float r1 = w - __bfloat162float(p1);
  p2 = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(p2);
  p3 = __float2bfloat16_rn(r2);
}

// Eight weights per thread (two 16-byte loads, one 16-byte store per plane)
// when n % 8 == 0 and the pointers are 16-byte aligned; one otherwise.
__global__ void __launch_bounds__(256) split_planes_kernel(const float* __restrict__ W,
                                                           __nv_bfloat16* __restrict__ planes,
                                                           long n) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool vec = (n % 8) == 0 && (reinterpret_cast<uintptr_t>(W) % 16) == 0 &&
                   (reinterpret_cast<uintptr_t>(planes) % 16) == 0;
  if (vec) {
    const long n8 = n / 8;
    for (long i = blockIdx.x * 256L + threadIdx.x; i < n8; i += (long)gridDim.x * 256) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(W) + 2 * i);
      const float4 b = __ldg(reinterpret_cast<const float4*>(W) + 2 * i + 1);
      const float w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      __align__(16) __nv_bfloat16 p[3][8];
#pragma unroll
      for (int e = 0; e < 8; ++e) split3(w[e], p[0][e], p[1][e], p[2][e]);
#pragma unroll
      for (int pl = 0; pl < 3; ++pl)
        reinterpret_cast<uint4*>(planes + pl * n)[i] = *reinterpret_cast<const uint4*>(p[pl]);
    }
    return;
  }
  for (long i = blockIdx.x * 256L + threadIdx.x; i < n; i += (long)gridDim.x * 256) {
    __nv_bfloat16 p1, p2, p3;
    split3(__ldg(W + i), p1, p2, p3);
    planes[i] = p1;
    planes[n + i] = p2;
    planes[2 * n + i] = p3;
  }
}

}  // namespace tc
}  // namespace mr
