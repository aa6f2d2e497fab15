// kernels_model.cuh -- batch-invariant dense layers of the policy model: the bf16 GEMM
// Y = X W^T on CTA pairs, and RMSNorm.
//
// Sources: "Zero Mismatch, Simple Async RL", section "Only one probability gap comes from old
// weights" (kernel selection by batch shape, reduction order and prefill/decode arithmetic change
// logprobs at fixed parameters) and section "Large-model validation exposes concrete failure
// mechanisms" (shape-selected library kernels are a source of batch variance); "REINFORCE Zero:
// 为什么内核对齐后...", the paragraph before Fig. 2 (batch-invariant kernels and a matched forward
// computation remove the kernel-mismatch term).
//
// GEMM.  One tile shape for every M: 256 x 256 output tiles, K in 64-column chunks taken in
// increasing order, fp32 accumulation in tensor memory, no split-K, no atomics.  A row of Y is
// therefore computed by the same instruction sequence whatever M is and wherever the row sits.
// A cluster is one CTA pair; the even CTA ("leader") issues M = 256 pair MMAs whose A rows come
// from each CTA's own shared memory (its 128 rows of X) and whose B is split along N (each CTA
// loads 128 rows of W).  The follower's copies complete on the leader's stage barrier (pair form
// of the tiled TMA load; no multicast), so one wait covers both halves.  Two accumulator buffers
// of 256 TMEM columns let the epilogue of one tile overlap the MMAs of the next.
//
// RMSNorm.  One warp per row: the row's sum of squares in a fixed per-lane order, a fixed shuffle
// tree, lane 0's total broadcast to the warp, then y = bf16((x * r) * g), r = rsqrt(ss / H + eps).
#pragma once

#include "kernels_lm.cuh"

namespace bi {

// ---------------------------------------------------------------------------------------------
// GEMM on CTA pairs
// ---------------------------------------------------------------------------------------------
constexpr int kGemmTileM = 256;
constexpr int kGemmTileN = 256;
constexpr int kGemmStageBytes = 2 * kAUnitBytes;  // this CTA's X rows [128 x 64] + W rows [128 x 64]
constexpr int kGemmMaxStages = 8;
constexpr int kGemmThreads = 192;  // warp 0 TMA, warp 1 MMA (leader), warps 2-5 epilogue

struct GemmShared {
  uint64_t full[kGemmMaxStages];   // leader: both halves of the stage have landed
  uint64_t empty[kGemmMaxStages];  // the pair's MMAs have read the stage (multicast commit)
  uint64_t acc_full[2];            // the accumulator buffer holds a finished tile (multicast commit)
  uint64_t acc_empty[2];           // leader: both halves' epilogues have read the buffer
  uint64_t ep_bar;                 // rendezvous of this CTA's 128 epilogue threads
  uint64_t mma_done;               // every MMA of the pair has completed (multicast commit)
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};
constexpr int kGemmSharedBytes = static_cast<int>((sizeof(GemmShared) + 127) / 128 * 128);
constexpr int kGemmFit = (kLmSmemLimit - kGemmSharedBytes) / kGemmStageBytes;
constexpr int kGemmStages = kGemmFit < kGemmMaxStages ? kGemmFit : kGemmMaxStages;
constexpr int kGemmSmem = kGemmStages * kGemmStageBytes + kGemmSharedBytes;
static_assert(kGemmStages >= 4, "GEMM pipeline needs at least four stages");

struct GemmArgs {
  uint16_t* y;        // [M, N] bf16
  int64_t M;
  int32_t N, K;
  int32_t* status;
  uint64_t limit_ns;
};

// Bounded wait; on a timeout or an abort the other CTA of the pair is told to stop too.
template <bool kClusterAcq>
__device__ __forceinline__ bool gm_wait(GemmShared& sh, const GemmArgs& a, uint64_t* bar, uint32_t parity) {
  const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
  const bool ok = mbar_wait<kClusterAcq>(bar, parity, wc);
  if (!ok) {
    const uint32_t la = smem_u32(const_cast<uint32_t*>(&sh.abort_flag));
    st_cluster_u32(mapa_shared(la, 0u), 1u);
    st_cluster_u32(mapa_shared(la, 1u), 1u);
  }
  return ok;
}

struct GemmCtx {
  uint32_t half, cl, ncl;
  int64_t ntiles, tiles_n;
  int KB;
  uint32_t ring;
};

// ---- TMA producer (one thread per CTA) ----
__device__ __forceinline__ void gemm_load_role(GemmShared& sh, const GemmArgs& a, const GemmCtx& x,
                                               const CUtensorMap* mx, const CUtensorMap* mw) {
  tma_prefetch_desc(mx);
  tma_prefetch_desc(mw);
  const bool lead = x.half == 0;
  const uint32_t lead_full = mapa_shared(smem_u32(&sh.full[0]), 0u);
  uint32_t stage = 0, phase = 0;
  bool ok = true;
  for (int64_t t = x.cl; ok && t < x.ntiles; t += x.ncl) {
    const int64_t mt = t / x.tiles_n;
    const int64_t nt = t - mt * x.tiles_n;
    const int32_t row = static_cast<int32_t>(mt * kGemmTileM + x.half * 128);
    const int32_t col = static_cast<int32_t>(nt * kGemmTileN + x.half * 128);
#pragma unroll 1
    for (int kb = 0; kb < x.KB; ++kb) {
      if (!gm_wait<false>(sh, a, &sh.empty[stage], phase ^ 1u)) { ok = false; break; }
      const uint32_t dst = x.ring + stage * kGemmStageBytes;
      if (lead) {
        mbar_arrive_expect_tx(&sh.full[stage], 2u * kGemmStageBytes);
        tma_load_2d(dst, mx, &sh.full[stage], kb * 64, row);
        tma_load_2d(dst + kAUnitBytes, mw, &sh.full[stage], kb * 64, col);
      } else {
        tma_load_2d_pair(dst, mx, lead_full + stage * 8u, kb * 64, row);
        tma_load_2d_pair(dst + kAUnitBytes, mw, lead_full + stage * 8u, kb * 64, col);
      }
      ring_advance(stage, phase, kGemmStages);
    }
  }
}

// ---- MMA issuer (the leader's one thread) ----
__device__ __forceinline__ void gemm_mma_role(GemmShared& sh, const GemmArgs& a, const GemmCtx& x, uint32_t tmem) {
  constexpr uint32_t idesc = idesc_bf16(kGemmTileM, kGemmTileN, false, false);
  constexpr uint64_t sb = static_cast<uint64_t>(kGemmStageBytes >> 4);
  constexpr uint16_t pair_mask = 3u;
  const uint64_t da0 = sdesc_k_sw128(x.ring);
  const uint64_t db0 = sdesc_k_sw128(x.ring + kAUnitBytes);
  uint32_t stage = 0, phase = 0, tc = 0;
  bool ok = true;
  for (int64_t t = x.cl; ok && t < x.ntiles; t += x.ncl, ++tc) {
    const uint32_t b = tc & 1u;
    if (!gm_wait<true>(sh, a, &sh.acc_empty[b], ((tc >> 1) & 1u) ^ 1u)) break;
    tc_fence_after();
    const uint32_t acc = tmem + b * static_cast<uint32_t>(kGemmTileN);
#pragma unroll 1
    for (int kb = 0; kb < x.KB; ++kb) {
      if (!gm_wait<false>(sh, a, &sh.full[stage], phase)) { ok = false; break; }
      tc_fence_after();
      const uint64_t da = da0 + stage * sb;
      const uint64_t db = db0 + stage * sb;
#pragma unroll
      for (int k = 0; k < 4; ++k) umma_bf16_pair(acc, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
      umma_commit_pair(&sh.empty[stage], pair_mask);
      ring_advance(stage, phase, kGemmStages);
    }
    if (!ok) break;
    umma_commit_pair(&sh.acc_full[b], pair_mask);
  }
  umma_commit_pair(&sh.mma_done, pair_mask);
}

// ---- epilogue (128 threads per CTA): this CTA's 128 rows of the tile, fp32 -> bf16 ----
__device__ __forceinline__ void gemm_epilogue_role(GemmShared& sh, const GemmArgs& a, const GemmCtx& x,
                                                   uint32_t tmem) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;  // tensor-memory lanes this warp may read
  const int row = quarter * 32 + lane;
  const int et = threadIdx.x - 64;
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const uint32_t lead_empty = mapa_shared(smem_u32(&sh.acc_empty[0]), 0u);
  const bool wide = (a.N % 16 == 0) && ((reinterpret_cast<uintptr_t>(a.y) & 31u) == 0);
  uint32_t tc = 0, epc = 0;
  for (int64_t t = x.cl; t < x.ntiles; t += x.ncl, ++tc) {
    const int64_t mt = t / x.tiles_n;
    const int64_t nt = t - mt * x.tiles_n;
    const uint32_t b = tc & 1u;
    if (!__all_sync(0xffffffffu, gm_wait<false>(sh, a, &sh.acc_full[b], (tc >> 1) & 1u))) break;
    tc_fence_after();
    const int64_t grow = mt * kGemmTileM + x.half * 128 + row;
    const int32_t col0 = static_cast<int32_t>(nt * kGemmTileN);
    const bool rvalid = grow < a.M;
    uint16_t* dst = a.y + (rvalid ? grow : 0) * static_cast<int64_t>(a.N) + col0;
#pragma unroll 1
    for (int c = 0; c < kGemmTileN / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(tl + b * static_cast<uint32_t>(kGemmTileN) + c * 32, v);
      tmem_ld_wait();
      const int cb = col0 + c * 32;
      if (rvalid) {
        uint32_t p[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) p[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        if (wide) {
          // N a multiple of 16 and y 32-byte aligned: whole 32-byte sectors, 16 columns a store
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (cb + 16 * h < a.N) st_global_v8(dst + c * 32 + 16 * h, p + 8 * h);
        } else {
#pragma unroll
          for (int g = 0; g < 4; ++g)
            if (cb + 8 * g < a.N)  // N is a multiple of 8: an 8-column group is all in or all out
              *reinterpret_cast<uint4*>(dst + c * 32 + 8 * g) = make_uint4(p[4 * g], p[4 * g + 1], p[4 * g + 2], p[4 * g + 3]);
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&sh.ep_bar);
    if (!__all_sync(0xffffffffu, gm_wait<false>(sh, a, &sh.ep_bar, (epc++) & 1u))) break;
    if (et == 0) {
      if (x.half == 0)
        mbar_arrive(&sh.acc_empty[b]);
      else
        mbar_arrive_cluster(lead_empty + b * 8u);
    }
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, GemmArgs a) {
  // tm_x: X [M][K], box {64, 128}; tm_w: W [N][K], box {64, 128}; both 128-byte swizzled
  extern __shared__ __align__(1024) uint8_t dsmem[];
  GemmShared& sh = *reinterpret_cast<GemmShared*>(dsmem + kGemmStages * kGemmStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  GemmCtx x;
  x.half = cluster_ctarank() & 1u;
  x.cl = cluster_id_x();
  x.ncl = ncluster_x();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmMaxStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.acc_full[i], 1);
      mbar_init(&sh.acc_empty[i], 2);
    }
    mbar_init(&sh.ep_bar, 128);
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sh.tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrive or copy
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  x.ring = smem_u32(dsmem);
  const bool misaligned = (x.ring & 1023u) != 0;
  if (misaligned && threadIdx.x == 0) raise_status(a.status, 4 /* BI_ERR_CUDA */);
  x.tiles_n = (a.N + kGemmTileN - 1) / kGemmTileN;
  x.ntiles = misaligned ? 0 : ((a.M + kGemmTileM - 1) / kGemmTileM) * x.tiles_n;
  x.KB = (a.K + 63) / 64;

  if (warp == 0) {
    if (lane == 0) gemm_load_role(sh, a, x, &tm_x, &tm_w);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      if (x.half == 0) gemm_mma_role(sh, a, x, tmem);
      // both CTAs wait for the pair's last MMAs (and their commits) before tearing down
      const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
      mbar_wait<false>(&sh.mma_done, 0u, wc);
    }
    __syncwarp();
  } else {
    gemm_epilogue_role(sh, a, x, tmem);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no peer touches this CTA's shared memory after this point
  if (sh.abort_flag != 0u) {
    // on the error path a copy or a commit of the pair may still be in flight towards this CTA
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 50000u) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// RMSNorm: one warp per row
// ---------------------------------------------------------------------------------------------
constexpr int kNormThreads = 256;

__device__ __forceinline__ uint4 ldg_nc_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Rows of at most 256 kVec elements: the row stays in registers (one read of x), and the next
// row's vectors are requested before the current row is reduced.  Same per-lane order and shuffle
// tree as the general kernel below.
constexpr int kNormRegMaxVec = 12;  // rows of up to 3072 elements stay in registers
constexpr int kNormRegBlocks(int vec) { return vec <= 8 ? 2 : 1; }  // resident blocks per SM
template <int kVec>
__global__ void __launch_bounds__(kNormThreads, kNormRegBlocks(kVec))
    k_rmsnorm_reg(const uint16_t* __restrict__ x, const uint16_t* __restrict__ g, float eps,
                  uint16_t* __restrict__ y, int64_t M, int32_t H) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * kNormThreads) >> 5;
  const int nvec = H / 8;
  const float inv_h = 1.0f / static_cast<float>(H);
  uint4 cur[kVec];
  auto load_row = [&](int64_t r, uint4 (&q)[kVec]) {
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const int v = lane + 32 * i;
      q[i] = (r < M && v < nvec) ? ldg_nc_u4(x + r * H + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  load_row(w0, cur);
  for (int64_t r = w0; r < M; r += nw) {
    uint4 nxt[kVec];
    load_row(r + nw, nxt);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const uint32_t u[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(u[e] << 16);
        const float hi = __uint_as_float(u[e] & 0xffff0000u);
        ss = fmaf(lo, lo, ss);
        ss = fmaf(hi, hi, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    ss = __shfl_sync(0xffffffffu, ss, 0);
    const float rs = rsqrtf(ss * inv_h + eps);
    uint16_t* yr = y + r * H;
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) {
        const uint4 gq = ldg_nc_u4(g + 8 * v);
        const uint32_t u[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
        const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = (__uint_as_float(u[e] << 16) * rs) * __uint_as_float(gw[e] << 16);
          const float hi = (__uint_as_float(u[e] & 0xffff0000u) * rs) * __uint_as_float(gw[e] & 0xffff0000u);
          o[e] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4*>(yr + 8 * v) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
#pragma unroll
    for (int i = 0; i < kVec; ++i) cur[i] = nxt[i];
  }
}

// Any H (a multiple of 8): two passes over the row, the second from L1/L2.
__global__ void __launch_bounds__(kNormThreads)
    k_rmsnorm(const uint16_t* __restrict__ x, const uint16_t* __restrict__ g, float eps, uint16_t* __restrict__ y,
              int64_t M, int32_t H) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * kNormThreads + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * kNormThreads) >> 5;
  const int nvec = H / 8;  // 16-byte vectors of 8 bf16
  const float inv_h = 1.0f / static_cast<float>(H);
  for (int64_t r = w0; r < M; r += nw) {
    const uint16_t* xr = x + r * H;
    float ss = 0.f;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) {
      const uint4 q = ldg_nc_u4(xr + 8 * v);
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(u[e] << 16);
        const float hi = __uint_as_float(u[e] & 0xffff0000u);
        ss = fmaf(lo, lo, ss);
        ss = fmaf(hi, hi, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    ss = __shfl_sync(0xffffffffu, ss, 0);  // every lane scales by the same value
    const float rs = rsqrtf(ss * inv_h + eps);
    uint16_t* yr = y + r * H;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) {
      const uint4 q = ldg_nc_u4(xr + 8 * v);
      const uint4 gq = ldg_nc_u4(g + 8 * v);
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
      const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = (__uint_as_float(u[e] << 16) * rs) * __uint_as_float(gw[e] << 16);
        const float hi = (__uint_as_float(u[e] & 0xffff0000u) * rs) * __uint_as_float(gw[e] & 0xffff0000u);
        o[e] = pack_bf16x2(lo, hi);
      }
      *reinterpret_cast<uint4*>(yr + 8 * v) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace bi
