// kernels_decode.cuh -- log pi for a few rows (decode-style scoring, T <= 128) on every SM, with
// the same bits as the cluster kernel (kernels_lm.cuh, kModeFwd).
//
// "Zero Mismatch, Simple Async RL", section "Alignment permits a simpler learning path": rollout
// and learner logprobs bit-identical for the same weights and tokens, whether a row is scored
// alone or packed.  The cluster kernel gives a one-row call the same bits as a packed one, but it
// sweeps the whole vocabulary on one cluster.  Here the same arithmetic is spread over the GPU:
//
// Phase 1 (k_lm_ztiles): one CTA per vocabulary tile j at a time computes z_j = H W_j^T for the
//   128-row tile with the cluster kernel's instruction sequence (tcgen05 M = 128, N = NZ, K = H in
//   64-column chunks of four K = 16 instructions, first without accumulate), and writes z (fp32)
//   and the tile's row maximum M_j over the valid columns for the T real rows.
// Phase 2 (k_lm_zscan, one block per row): the lazy reference chain m_j = (M_j > m_{j-1} + tau) ?
//   M_j : m_{j-1}; every 32-column chunk sum cs = sum_q e^{z - m_j} (target column and columns
//   past V excluded, q in order); per class k (steps j = k mod C) the partial sum with its rescale
//   at each change of reference and the chunk sums added in order; the combine of the C classes
//   in class order.  Each of these is the cluster kernel's epilogue expression for expression;
//   only the chunk sums run in parallel, and they are independent there too.
#pragma once

#include "kernels_lm.cuh"

namespace bi {

constexpr int kDecodeRows = 128;  // rows one tile holds: the largest T this path serves
constexpr int kZtThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

template <int kNZ>
struct ZtTile {
  static constexpr int stage_bytes = kAUnitBytes + kNZ * 128;  // hidden [128 x 64] + W rows [NZ x 64]
  static constexpr int nstages = 4;
  static constexpr int smem = nstages * stage_bytes + 1024;
  static_assert(smem <= kLmSmemLimit, "stages do not fit");
};

struct ZtShared {
  uint64_t full[4], empty[4];
  uint64_t z_full[2], z_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

struct ZtArgs {
  int64_t T;        // real rows (<= 128)
  int32_t V, nvz, KB;
  float* z;         // [T][z_ld] fp32 logits, z_ld = nvz * NZ
  int64_t z_ld;
  float* tmax;      // [T][nvz] row maximum of each tile over its valid columns
  int32_t* status;
  uint64_t limit_ns;
};

template <int kNZ>
__global__ void __launch_bounds__(kZtThreads, 1)
    k_lm_ztiles(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w, ZtArgs a) {
  // tm_h: hidden [T][H], box {64, 128}; tm_w: W [V][H], box {64, NZ}; both 128-byte swizzled
  using ZT = ZtTile<kNZ>;
  extern __shared__ __align__(1024) uint8_t dsmem[];
  ZtShared& sh = *reinterpret_cast<ZtShared*>(dsmem + ZT::nstages * ZT::stage_bytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.z_full[i], 1);
      mbar_init(&sh.z_empty[i], 128);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t ring = smem_u32(dsmem);
  const bool misaligned = (ring & 1023u) != 0;
  if (misaligned && threadIdx.x == 0) raise_status(a.status, 4 /* BI_ERR_CUDA */);
  const int ntiles = misaligned ? 0 : a.nvz;
  const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
  constexpr uint32_t nst = static_cast<uint32_t>(ZT::nstages);

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_h);
      tma_prefetch_desc(&tm_w);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int j = blockIdx.x; ok && j < ntiles; j += gridDim.x) {
#pragma unroll 1
        for (int kb = 0; kb < a.KB; ++kb) {
          if (!mbar_wait<false>(&sh.empty[stage], phase ^ 1u, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&sh.full[stage], static_cast<uint32_t>(ZT::stage_bytes));
          const uint32_t dst = ring + stage * ZT::stage_bytes;
          tma_load_2d(dst, &tm_h, &sh.full[stage], kb * 64, 0);
          tma_load_2d(dst + kAUnitBytes, &tm_w, &sh.full[stage], kb * 64, j * kNZ);
          ring_advance(stage, phase, nst);
        }
      }
      // copies still in flight land before the CTA may exit
      for (uint32_t i = 0; i < nst; ++i) {
        const uint32_t ph = (i < stage) ? phase : (phase ^ 1u);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_test(&sh.full[i], ph))
          if (globaltimer_ns() - t0 > a.limit_ns) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // the logit tile of kernels_lm.cuh: the same descriptors and the same instruction sequence
      constexpr uint32_t idesc_z = idesc_bf16(128, kNZ, false, false);
      constexpr uint64_t sb = static_cast<uint64_t>(ZT::stage_bytes >> 4);
      const uint64_t dk0 = sdesc_k_sw128(ring);
      const uint64_t dkb0 = sdesc_k_sw128(ring + kAUnitBytes);
      uint32_t stage = 0, phase = 0, tc = 0;
      bool ok = true;
      for (int j = blockIdx.x; ok && j < ntiles; j += gridDim.x, ++tc) {
        const uint32_t b = tc & 1u;
        if (!mbar_wait<false>(&sh.z_empty[b], ((tc >> 1) & 1u) ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t zt = tmem + b * 256u;
#pragma unroll 1
        for (int kb = 0; kb < a.KB; ++kb) {
          if (!mbar_wait<false>(&sh.full[stage], phase, wc)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = dk0 + stage * sb;
          const uint64_t db = dkb0 + stage * sb;
          umma_bf16(zt, da, db, idesc_z, kb != 0 ? 1u : 0u);
          umma_bf16(zt, da + 2, db + 2, idesc_z, 1u);
          umma_bf16(zt, da + 4, db + 4, idesc_z, 1u);
          umma_bf16(zt, da + 6, db + 6, idesc_z, 1u);
          umma_commit(&sh.empty[stage]);
          ring_advance(stage, phase, nst);
        }
        if (!ok) break;
        umma_commit(&sh.z_full[b]);
      }
      // every MMA (and its commits) completes before the CTA may release its memory
      umma_commit(&sh.mma_done);
      mbar_wait<false>(&sh.mma_done, 0u, wc);
    }
    __syncwarp();
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w mod 4) ..; one row per thread
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool warp_rows = static_cast<int64_t>(quarter * 32) < a.T;  // warp-uniform
    uint32_t tc = 0;
    for (int j = blockIdx.x; j < ntiles; j += gridDim.x, ++tc) {
      const uint32_t b = tc & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait<false>(&sh.z_full[b], (tc >> 1) & 1u, wc))) break;
      tc_fence_after();
      if (warp_rows) {
        const bool real = row < a.T;
        float* zr = a.z + (real ? row : 0) * a.z_ld + static_cast<int64_t>(j) * kNZ;
        float M = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kNZ / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tl + b * 256u + c * 32, v);
          tmem_ld_wait();
          const int vb = j * kNZ + c * 32;
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (vb + q < a.V) M = fmaxf(M, __uint_as_float(v[q]));
          if (real) {
            uint4* d4 = reinterpret_cast<uint4*>(zr + c * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) d4[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
        if (real) a.tmax[static_cast<int64_t>(row) * a.nvz + j] = M;
      }
      tc_fence_before();
      mbar_arrive(&sh.z_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (sh.abort_flag != 0u) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 50000u) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr int kZsThreads = 1024;

// Dynamic shared memory of k_lm_zscan: the references and the chunk sums of one row.
__host__ __device__ constexpr size_t zscan_smem(int nvz, int nz) {
  return static_cast<size_t>(nvz) * 4 + static_cast<size_t>(nvz) * (nz / 32) * 4 + 2 * 8 * 4;
}

template <int kNZ>
__global__ void __launch_bounds__(kZsThreads)
    k_lm_zscan(const float* __restrict__ z, int64_t z_ld, const float* __restrict__ tmax, const int32_t* __restrict__ y,
               int64_t T, int V, int nvz, int C, float* __restrict__ logprob, float* __restrict__ lse_out,
               int32_t* status) {
  constexpr int kChunks = kNZ / 32;
  extern __shared__ float zs[];
  float* mref = zs;                                     // [nvz] reference after each step
  float* csum = zs + nvz;                               // [nvz][kChunks] chunk sums
  float* cls = csum + static_cast<int64_t>(nvz) * kChunks;  // [8] class reference, [8] class sum
  const int64_t t = blockIdx.x;
  if (t >= T) return;
  const float* zrow = z + t * z_ld;
  const int32_t yt = y[t];
  // the chain (as the producers of consecutive steps pass it on), from the tile maxima staged in
  // shared memory
  for (int j = threadIdx.x; j < nvz; j += kZsThreads) mref[j] = tmax[t * nvz + j];
  __syncthreads();
  if (threadIdx.x == 0) {
    float mprev = -INFINITY;
#pragma unroll 8
    for (int j = 0; j < nvz; ++j) {
      const float M = mref[j];
      const float mnew = (M > mprev + kTau) ? M : mprev;
      mref[j] = mnew;
      mprev = mnew;
    }
  }
  __syncthreads();
  // every 32-column chunk: e^{z - m_j} summed in column order, the target column excluded
  for (int idx = threadIdx.x; idx < nvz * kChunks; idx += kZsThreads) {
    const int j = idx / kChunks;
    const int c = idx - j * kChunks;
    const float mn2 = mref[j] * kLog2e;
    const int vb = j * kNZ + c * 32;
    float zv[32];
    const float4* z4 = reinterpret_cast<const float4*>(zrow + vb);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 f = __ldg(z4 + q);
      zv[4 * q] = f.x;
      zv[4 * q + 1] = f.y;
      zv[4 * q + 2] = f.z;
      zv[4 * q + 3] = f.w;
    }
    float cs = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const bool tgt = (vb + q == yt);
      const bool in = (vb + q < V) && !tgt;
      const float pr = in ? ex2_approx(fmaf(zv[q], kLog2e, -mn2)) : 0.f;
      cs += pr;
    }
    csum[idx] = cs;
  }
  __syncthreads();
  // class k: its steps in order, rescaled at each change of reference
  if (threadIdx.x < C) {
    const int k = threadIdx.x;
    float mp = -INFINITY, sp = 0.f;
#pragma unroll 4
    for (int j = k; j < nvz; j += C) {
      const float mnew = mref[j];
      if (mnew != mp) {
        sp = (mp == -INFINITY) ? 0.f : sp * ex2_approx((mp - mnew) * kLog2e);
        mp = mnew;
      }
#pragma unroll
      for (int c = 0; c < kChunks; ++c) sp += csum[j * kChunks + c];
    }
    cls[k] = mp;
    cls[8 + k] = sp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float mstar = -INFINITY;
    for (int k = 0; k < C; ++k) mstar = fmaxf(mstar, cls[k]);
    float s_ex = 0.f;
    for (int k = 0; k < C; ++k) {
      const float mq = cls[k];
      if (mq != -INFINITY) s_ex = fmaf(cls[8 + k], ex2_approx((mq - mstar) * kLog2e), s_ex);
    }
    const bool ybad = yt < 0 || yt >= V;
    float lp = __int_as_float(0x7fc00000), lse = __int_as_float(0x7fc00000);
    if (!ybad) {
      const float zy = zrow[yt];
      const float s = s_ex + ex2_approx(fmaf(zy, kLog2e, -mstar * kLog2e));
      lse = mstar + logf(s);
      lp = zy - lse;
    } else {
      raise_status(status, 6 /* BI_ERR_BAD_TARGET */);
    }
    logprob[t] = lp;
    if (lse_out) lse_out[t] = lse;
  }
}

}  // namespace bi
