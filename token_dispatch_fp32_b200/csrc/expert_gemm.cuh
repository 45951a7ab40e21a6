// expert_gemm.cuh -- one expert layer over the expert-sorted rows with the
// row gather fused into the GEMM (Kimi K2 "Add shared output" page, moe_infer:
// sorted_tokens = x[idxs // k], then expert(sorted_tokens[start_idx:end_idx])
// for each expert).
//
// The expert is one linear map per expert (synthetic weights W[e] [n_out, d],
// bf16, nn.Linear layout): out[j] = x[perm[j] / k] . W[e(j)]^T for the sorted
// row j, e(j) the expert whose segment [offsets[e], offsets[e+1]) holds j.
// The gathered rows are never written to memory: the A tile of a 128-row
// block of an expert's segment is loaded straight from the token rows x by
// TMA tile::gather4 (four rows per copy, their indices taken from the
// permutation), and the B tile from W[e].  tcgen05 kind::f16, M = 128,
// N = 256, fp32 accumulation in TMEM, rounded to bf16 on the way out.  K is
// staged in chunks of 32 or 64 bf16 (BKE: 64- or 128-byte rows).
//
//   warp 0      producer: all 32 lanes issue the gather4 copies of a stage
//               (lane l: rows 4l..4l+3), lane 0 also the W tile.
//   warp 1      TMEM owner and MMA issuer (one elected thread).
//   warps 2..5  epilogue: TMEM lanes -> bf16 -> global (one row per thread).
//
// Grid: x = 128-row blocks over all experts (an upper bound from the host;
// each CTA finds its expert and block from the offsets, surplus CTAs exit),
// y = 256-column blocks of n_out.  Every mbarrier wait is bounded.
//
// With the combine fused in (COMBINE; the same page: new_x[idxs] = outs,
// weighted sum over k, cast back, plus the shared expert's output) the
// expert outputs are never written either: the epilogue rounds each row to
// bf16, multiplies it by its slot's router weight (fp32), stages it in the
// idle ring and adds it into the token's fp32 row of a [T, n_out] accumulator
// with one bulk reduction per row (cp.reduce.async.bulk .add.f32, resolved in
// L2).  Rows of one expert segment belong to distinct tokens, so the k
// additions into a token row come from k different CTAs in no fixed order.  combine_acc_finalize_kernel then rounds
// the accumulator to bf16, adds the shared row and rounds again.
#pragma once

#include "router_tc.cuh"

namespace mr {
namespace eg {

using namespace mr::tc;

constexpr int kBN = 256;                    // output columns per CTA (MMA N)
constexpr int kThreads = 192;               // producer, MMA, 4 epilogue warps

// Shared-memory plan for K chunks of BKE bf16 (32: 64-byte rows, 64-byte
// swizzle; 64: 128-byte rows, 128-byte swizzle).
template <int BKE>
struct EgPlan {
  static constexpr int kStages = BKE == 32 ? 8 : 4;
  static constexpr uint32_t kABytes = BM * BKE * 2;   // 128 gathered rows
  static constexpr uint32_t kBBytes = kBN * BKE * 2;  // 256 weight rows
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kBarOff = kStages * kStageBytes;
  static constexpr uint32_t kSmemBytes = kBarOff + 256 + 4 * BM + 64 + 1024;
};

struct Params {
  int T, d, k, N_r, n_out;
  const void* x;  // token rows (the copy warps read them directly)
  const int32_t* perm;
  const int32_t* offsets;
  const __nv_bfloat16* w_packed;  // packed weights (PACKED only)
  __nv_bfloat16* out;  // [offsets[N_r], n_out] (not COMBINE)
  const float* wts;    // [T*k] router weights by slot (COMBINE)
  float* acc;          // [T, n_out] fp32, zeroed before the launch (COMBINE)
};

// Adds `bytes` of fp32 from shared memory into global memory element by
// element (a bulk reduction by the copy engine, resolved in L2; both
// addresses 16-byte aligned, bytes a multiple of 16); committed and waited
// for with bulk_store_commit_and_wait.
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                   gdst),
               "r"(ssrc), "r"(bytes)
               : "memory");
}

// One contiguous global -> shared copy completing on an mbarrier (16-byte
// aligned addresses, a multiple of 16 bytes).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int col, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(col), "r"(r0), "r"(r1), "r"(r2),
      "r"(r3)
      : "memory");
}

// Packed weight layout (PACKED): W[e] cut into tiles of 256 output rows x 64
// K columns, tile (e, nt, kc) stored as one contiguous 32 KB block at block
// index (e * NT + nt) * KC + kc (NT = ceil(n_out / 256), KC = ceil(d / 64);
// rows past n_out and columns past d are zero), its bytes already in the
// order the tensor core reads a 128-byte-swizzled K-major tile (16-byte
// chunk c of row r at chunk c ^ (r % 8) of that row).  A stage's weight tile
// is then one bulk copy of 32 contiguous KB instead of 256 row requests of
// 128 bytes.
// How a stage's A tile (128 sorted rows x BKE) reaches shared memory:
//   kRowsSorted  the rows are already in expert-sorted order (x is [T*k, d],
//                row j = sorted row j): one tiled copy of 128 consecutive
//                rows -- the plain grouped GEMM without the fused gather;
//   kGatherTma   TMA tile::gather4 copies, four token rows each (warp 0);
//   kGatherLsu   the four epilogue warps, idle during the K loop, copy the
//                token rows 16 bytes per thread (cp.async) straight into the
//                128-byte-swizzled layout, three stages ahead; each warp
//                waits for its copies, fences them to the async proxy and
//                arrives on the stage's barrier (its arrival count is 5:
//                warp 0's expect-tx arrival and the four copy warps).
constexpr int kRowsSorted = 0, kGatherTma = 1, kGatherLsu = 2;

// COMBINE: the epilogue does not write the expert outputs; it scales each
// row (rounded to bf16, the expert's output dtype) by its slot's router weight
// and adds it into the token's fp32 row of P.acc.
template <int BKE, bool PACKED = false, int AMODE = kGatherTma, bool COMBINE = false>
__global__ void __launch_bounds__(kThreads, 1)
    expert_gemm_gather_kernel(const __grid_constant__ CUtensorMap map_x,
                              const __grid_constant__ CUtensorMap map_w, const Params P) {
  constexpr bool GATHER = AMODE != kRowsSorted;
  static_assert(!COMBINE || GATHER, "the combine needs each row's slot (perm)");
  static_assert(AMODE != kGatherLsu || BKE == 64, "the copy warps fill 128-byte rows");
  static_assert(!PACKED || BKE == 64, "the packed layout has 64-column tiles");
  using PL = EgPlan<BKE>;
  constexpr int kStages = PL::kStages;
  constexpr uint32_t kABytes = PL::kABytes, kStageBytes = PL::kStageBytes,
                     kBarOff = PL::kBarOff;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned start by pointer arithmetic on the shared array, so the
  // compiler keeps the shared address space for every access through it (an
  // integer round trip would turn them into generic loads and stores)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  int* tok_s = reinterpret_cast<int*>(smem + kBarOff + 256);      // [128] token of each row
  int* misc = reinterpret_cast<int*>(smem + kBarOff + 256 + 4 * BM);
  volatile int* abort = reinterpret_cast<volatile int*>(misc + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 6);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t smem0 = smem_u32(smem);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int B_FULL = 0, B_EMPTY = kStages, B_ACC = 2 * kStages;

  // ---- which expert and which 128-row block of its segment -----------------
  // blocks of expert e: ceil(count_e / 128); a CTA-wide exclusive scan of
  // them over the experts (thread i owns experts [i*c, (i+1)*c))
  {
    const int c = (P.N_r + kThreads - 1) / kThreads;
    const int e0 = tid * c, e1 = e0 + c < P.N_r ? e0 + c : P.N_r;
    int mine = 0;
    for (int e = e0; e < e1; ++e) mine += (P.offsets[e + 1] - P.offsets[e] + BM - 1) / BM;
    int x = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    __shared__ int wsum[kThreads / 32];
    if (lane == 31) wsum[warp] = x;
    if (tid == 0) misc[0] = -1;
    __syncthreads();
    int before = x - mine;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    const int t = blockIdx.x;
    if (t >= before && t < before + mine) {
      int acc = before;
      for (int e = e0; e < e1; ++e) {
        const int nb = (P.offsets[e + 1] - P.offsets[e] + BM - 1) / BM;
        if (t < acc + nb) {
          misc[0] = e;
          misc[1] = t - acc;
          break;
        }
        acc += nb;
      }
    }
    __syncthreads();
  }
  const int e = misc[0];
  if (e < 0) return;  // past the last block: every thread leaves together
  const int row0 = P.offsets[e] + misc[1] * BM;
  const int row_end = P.offsets[e + 1];
  const int n0 = blockIdx.y * kBN;
  const int KC = (P.d + BKE - 1) / BKE;

  if (GATHER && tid < BM) {
    const int j = row0 + tid;
    // rows past the segment load some valid token row; their results are dropped
    tok_s[tid] = j < row_end ? P.perm[j] / P.k : P.perm[row0] / P.k;
  }
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), AMODE == kGatherLsu ? 5 : 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_ACC), 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---- producer: 32 gather4 copies (one per lane) + the W tile ----------
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    if (GATHER) {
      r0 = tok_s[4 * lane];
      r1 = tok_s[4 * lane + 1];
      r2 = tok_s[4 * lane + 2];
      r3 = tok_s[4 * lane + 3];
    }
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;
    for (int kc = 0; kc < KC; ++kc, (++s == kStages ? (s = 0, ph ^= 1u) : 0u)) {
      bool go = true;
      if (lane == 0 && kc >= kStages) go = mbar_wait(bar(B_EMPTY + s), ph ^ 1u, abort);
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) break;
      const uint32_t base = smem0 + s * kStageBytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_FULL + s),
                              AMODE == kGatherLsu ? PL::kBBytes : kStageBytes);
        if constexpr (PACKED)
          bulk_load(base + kABytes,
                    P.w_packed + ((long)(e * (int)gridDim.y + (int)blockIdx.y) * KC + kc) *
                                     (kBN * 64),
                    PL::kBBytes, bar(B_FULL + s));
        else
          tma_load_2d(base + kABytes, &map_w, bar(B_FULL + s), kc * BKE, e * P.n_out + n0);
      }
      __syncwarp();
      if constexpr (AMODE == kGatherTma)
        tma_gather4(base + (uint32_t)lane * 4u * (BKE * 2), &map_x, bar(B_FULL + s), kc * BKE,
                    r0, r1, r2, r3);
      else if (AMODE == kRowsSorted && lane == 0)  // 128 consecutive sorted rows
        tma_load_2d(base, &map_x, bar(B_FULL + s), kc * BKE, row0);
      ++issued;
    }
    // every copy this CTA issued lands before the CTA may exit
    if (lane == 0)
      for (int kc = issued - kStages < 0 ? 0 : issued - kStages; kc < issued; ++kc)
        mbar_wait(bar(B_FULL + kc % kStages), (kc / kStages) & 1, abort, true);
  } else if (warp == 1) {
    // ---- MMA issuer -------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(kBN, BM);
      int s = 0;
      uint32_t ph = 0;
      for (int kc = 0; kc < KC; ++kc, (++s == kStages ? (s = 0, ph ^= 1u) : 0u)) {
        if (!mbar_wait(bar(B_FULL + s), ph, abort)) break;
        tc_fence_after();
        const uint32_t a = smem0 + s * kStageBytes, b = a + kABytes;
#pragma unroll
        for (int kk = 0; kk < BKE / 16; ++kk) {
          // 16 bf16 = 32 bytes along K; 64- or 128-byte swizzled rows
          const uint64_t da = BKE == 32 ? make_desc_sw64(a + kk * 32) : make_desc(a + kk * 32);
          const uint64_t db = BKE == 32 ? make_desc_sw64(b + kk * 32) : make_desc(b + kk * 32);
          mma_bf16(tmem_base, da, db, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(B_EMPTY + s));
      }
      // always committed (also after an abort): drains every MMA before the
      // epilogue reads TMEM and before TMEM is released
      mma_commit(bar(B_ACC));
    }
    __syncwarp();
  } else {
    if constexpr (AMODE == kGatherLsu) {
      // ---- A tiles: 128 token rows x 64 bf16 per stage, 16 bytes a copy ----
      // copy i of a stage (i = ct + 128 * u): row i / 8, 16-byte chunk i % 8,
      // stored at chunk (i % 8) ^ (row % 8) of the row (128-byte swizzle)
      const int ct = tid - 64;  // 0..127
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(P.x);
      constexpr int kLag = kStages - 1;  // stages in flight per thread
      // hand over the stage issued kLag iterations ago: its copies have landed
      // once at most kLag - 1 newer groups are pending
      auto hand_over = [&](int st) {
        asm volatile("cp.async.wait_group %0;" ::"n"(kLag - 1) : "memory");
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_FULL + st));
      };
      int s = 0;
      uint32_t ph = 0;
      bool go = true;
      for (int kc = 0; kc < KC; ++kc, (++s == kStages ? (s = 0, ph ^= 1u) : 0u)) {
        // first the hand-over, so the MMA never waits on this warp's wait for
        // a free stage below
        if (kc >= kLag) hand_over((kc - kLag) % kStages);
        if (kc >= kStages) {
          bool g = true;
          if (lane == 0) g = mbar_wait(bar(B_EMPTY + s), ph ^ 1u, abort);
          go = __shfl_sync(0xffffffffu, g, 0);
          if (!go) break;
        }
        const uint32_t base = smem0 + s * kStageBytes;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = ct + 128 * u, rr = i >> 3, c = i & 7;
          const int col = kc * 64 + c * 8;
          const uint32_t dst = base + (uint32_t)rr * 128u + ((uint32_t)(c ^ (rr & 7)) << 4);
          const __nv_bfloat16* src = xb + (long)tok_s[rr] * P.d + (col < P.d ? col : 0);
          const uint32_t nbytes = col < P.d ? 16u : 0u;  // K tail: zero fill
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                       "r"(nbytes)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      // the last stages (and, after a give-up, every issued copy) land
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      fence_proxy_async();
      __syncwarp();
      if (go && lane == 0)
        for (int kc = KC - kLag < 0 ? 0 : KC - kLag; kc < KC; ++kc)
          mbar_arrive(bar(B_FULL + kc % kStages));
    }
    // ---- epilogue: warp w reads TMEM lanes 32*(w % 4).., one row per lane --
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar(B_ACC), 0, abort, true)) && !*abort;
    tc_fence_after();
    const int j = row0 + r;
    const bool store = ok && j < row_end;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    if constexpr (COMBINE) {
      // slot perm[j] = t * k + slot: weight w[perm[j]], token row t of acc.
      // The row, scaled, goes to the idle ring (every MMA that read it has
      // completed: B_ACC), one [kBN] fp32 row per thread, rows kRedRow
      // bytes apart so a quarter-warp's 16-byte stores fall on distinct
      // banks; then one bulk reduction adds the whole row into acc (one
      // coalesced kBN * 4-byte transfer, not 16-byte pieces of 32 rows).
      constexpr uint32_t kRedRow = kBN * 4 + 16;
      static_assert(BM * kRedRow <= kBarOff, "the scaled rows fit in the ring");
      const int slot = store ? P.perm[j] : 0;
      const float wj = store ? P.wts[slot] : 0.0f;
      float* srow = reinterpret_cast<float*>(smem + (uint32_t)r * kRedRow);
      const int ncols = P.n_out - n0 < kBN ? P.n_out - n0 : kBN;
      for (int c = 0; c < kBN / 16; ++c) {
        float v[16];
        tmem_ld16(tmem_base + lane_off + (uint32_t)(c * 16), v);  // whole warp
        if (store && c * 16 < ncols) {
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(srow + c * 16 + i) =
                make_float4(wj * __bfloat162float(__float2bfloat16_rn(v[i])),
                            wj * __bfloat162float(__float2bfloat16_rn(v[i + 1])),
                            wj * __bfloat162float(__float2bfloat16_rn(v[i + 2])),
                            wj * __bfloat162float(__float2bfloat16_rn(v[i + 3])));
        }
      }
      if (store) {
        fence_proxy_async();  // this thread's row, visible to the bulk copy
        bulk_reduce_add_f32(P.acc + (long)(slot / P.k) * P.n_out + n0, smem_u32(srow),
                            (uint32_t)ncols * 4u);
        bulk_store_commit_and_wait();
      }
    }
    __nv_bfloat16* dst = COMBINE ? nullptr : P.out + (long)j * P.n_out + n0;
    for (int c = 0; c < (COMBINE ? 0 : kBN / 16); ++c) {
      float v[16];
      tmem_ld16(tmem_base + lane_off + (uint32_t)(c * 16), v);  // whole warp
      if (store && n0 + c * 16 < P.n_out) {
        uint4 pk[2];
        uint32_t* w = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
          w[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        uint4* o = reinterpret_cast<uint4*>(dst + c * 16);
        o[0] = pk[0];
        o[1] = pk[1];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kBN)
                 : "memory");
  }
}

// y = bf16(bf16(acc) + shared) (or bf16(acc) without a shared row), eight
// elements (two float4 of acc, one 16-byte vector of bf16) per thread and step.
__global__ void __launch_bounds__(256)
    combine_acc_finalize_kernel(const float4* __restrict__ acc, const uint4* __restrict__ shared,
                                uint4* __restrict__ y, long n8) {
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n8;
       i += (long)gridDim.x * blockDim.x) {
    const float4 a0 = __ldcs(acc + 2 * i), a1 = __ldcs(acc + 2 * i + 1);
    float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    uint32_t o[4];
    if (shared) {
      const uint4 sv = __ldcs(shared + i);
      const uint32_t s4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float slo = __uint_as_float(s4[q] << 16), shi = __uint_as_float(s4[q] & 0xffff0000u);
        const __nv_bfloat162 h = __floats2bfloat162_rn(
            __bfloat162float(__float2bfloat16_rn(v[2 * q])) + slo,
            __bfloat162float(__float2bfloat16_rn(v[2 * q + 1])) + shi);
        o[q] = *reinterpret_cast<const uint32_t*>(&h);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
        o[q] = *reinterpret_cast<const uint32_t*>(&h);
      }
    }
    __stcs(y + i, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// W [N_r][n_out][d] -> the packed layout above (swizzled within each row),
// eight bf16 (16 bytes) per thread and step; d % 8 == 0.
__global__ void __launch_bounds__(256)
    expert_pack_kernel(const uint4* __restrict__ W, uint4* __restrict__ Wp, int n_out, int d,
                       int NT, int KC, long n_vec) {
  const int cv = 64 / 8;  // 16-byte vectors per packed row
  for (long o = (long)blockIdx.x * blockDim.x + threadIdx.x; o < n_vec;
       o += (long)gridDim.x * blockDim.x) {
    const int c8o = (int)(o % cv);  // 16-byte chunk position in the packed row
    const int r = (int)((o / cv) % kBN);
    const int c8 = c8o ^ (r & 7);   // the K chunk stored there (128-byte swizzle)
    const long blk = o / ((long)cv * kBN);
    const int kc = (int)(blk % KC);
    const int nt = (int)((blk / KC) % NT);
    const long e = blk / ((long)KC * NT);
    const int n = nt * kBN + r, col = kc * 64 + c8 * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < n_out && col < d) v = W[((e * n_out + n) * (long)d + col) / 8];
    Wp[o] = v;
  }
}

}  // namespace eg
}  // namespace mr
