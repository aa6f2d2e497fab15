// kernels_decode.cuh -- log pi for a few rows (decode-style scoring, T <= 128) on every SM, with
// the same bits as the cluster kernel (kernels_lm.cuh, kModeFwd), and nothing of size T x V in
// memory.
//
// "Zero Mismatch, Simple Async RL", section "Alignment permits a simpler learning path": rollout
// and learner logprobs bit-identical for the same weights and tokens, whether a row is scored
// alone or packed.  The cluster kernel gives a one-row call the same bits as a packed one, but it
// sweeps the whole vocabulary on one cluster.  Here the same arithmetic is spread over the GPU in
// two passes over W; between them only per-tile maxima, references and 32-column partial sums
// (1/32 of the logits) are kept:
//
// Pass 1 (k_lm_ztiles<NZ, false>): one CTA per vocabulary tile j at a time computes z_j = H W_j^T
//   for the 128-row tile with the cluster kernel's instruction sequence (tcgen05 M = 128, N = NZ,
//   K = H in 64-column chunks of four K = 16 instructions, first without accumulate) and writes
//   the tile's row maximum M_j over the valid columns for the T real rows.
// Chain (k_lm_zchain, one thread per row): the lazy reference chain m_j = (M_j > m_{j-1} + tau) ?
//   M_j : m_{j-1}, as the producers of consecutive steps pass it on.
// Pass 2 (k_lm_ztiles<NZ, true>): the same tiles again; every 32-column chunk sum
//   cs = sum_q e^{z - m_j} (target column and columns past V excluded, q in order) and the target
//   logit, exactly as the cluster kernel's producer epilogue forms them.
// Combine (k_lm_zscan, one block per row): per class k (steps j = k mod C) the partial sum with its
//   rescale at each change of reference and the chunk sums added in order; then the combine of
//   the C classes in class order.  Each of these is the cluster kernel's epilogue expression for
//   expression.
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
  float* tmax;      // [nvz][T] row maximum of each tile over its valid columns (pass 1 writes)
  const float* mref;  // [nvz][T] reference of each row at each step (pass 2 reads)
  float* csum;      // [T][nvz][NZ / 32] 32-column chunk sums of e^{z - m_j} (pass 2 writes)
  float* zy;        // [T] target logit (pass 2 writes, from the tile holding the target)
  const int32_t* y; // [T] targets
  int32_t* status;
  uint64_t limit_ns;
};

template <int kNZ, bool kSums>
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
    const bool real = row < a.T;
    const int32_t yt = real ? a.y[row] : -1;
    for (int j = blockIdx.x; j < ntiles; j += gridDim.x, ++tc) {
      const uint32_t b = tc & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait<false>(&sh.z_full[b], (tc >> 1) & 1u, wc))) break;
      tc_fence_after();
      if (warp_rows) {
        if (!kSums) {
          // pass 1: the tile's row maximum over the valid columns (the producer's first pass)
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
          }
          if (real) a.tmax[static_cast<int64_t>(j) * a.T + row] = M;
        } else {
          // pass 2: chunk sums against the step's reference, and the target logit (the
          // producer's second pass)
          const float mn2 = (real ? a.mref[static_cast<int64_t>(j) * a.T + row] : 0.f) * kLog2e;
          float* cs_out = a.csum + (static_cast<int64_t>(real ? row : 0) * a.nvz + j) * (kNZ / 32);
#pragma unroll 1
          for (int c = 0; c < kNZ / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tl + b * 256u + c * 32, v);
            tmem_ld_wait();
            const int vb = j * kNZ + c * 32;
            float cs = 0.f;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float z = __uint_as_float(v[q]);
              const bool tgt = (vb + q == yt);
              const bool in = (vb + q < a.V) && !tgt;
              const float pr = in ? ex2_approx(fmaf(z, kLog2e, -mn2)) : 0.f;
              cs += pr;
              if (tgt && real) a.zy[row] = z;
            }
            if (real) cs_out[c] = cs;
          }
        }
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

// One thread per row: the reference chain from the tile maxima, in step order.
__global__ void k_lm_zchain(const float* __restrict__ tmax, int64_t T, int nvz, float* __restrict__ mref) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float mprev = -INFINITY;
#pragma unroll 4
  for (int j = 0; j < nvz; ++j) {
    const float M = tmax[static_cast<int64_t>(j) * T + t];
    const float mnew = (M > mprev + kTau) ? M : mprev;
    mref[static_cast<int64_t>(j) * T + t] = mnew;
    mprev = mnew;
  }
}

constexpr int kZsThreads = 32;

// One block (one warp) per row: the class partial sums and their combine.
template <int kNZ>
__global__ void __launch_bounds__(kZsThreads)
    k_lm_zscan(const float* __restrict__ csum, const float* __restrict__ mref, const float* __restrict__ zyb,
               const int32_t* __restrict__ y, int64_t T, int V, int nvz, int C, float* __restrict__ logprob,
               float* __restrict__ lse_out, int32_t* status) {
  constexpr int kChunks = kNZ / 32;
  __shared__ float cls[2 * 8];  // [8] class reference, [8] class sum
  const int64_t t = blockIdx.x;
  if (t >= T) return;
  const float* crow = csum + t * static_cast<int64_t>(nvz) * kChunks;
  // class k: its steps in order, rescaled at each change of reference
  if (static_cast<int>(threadIdx.x) < C) {
    const int k = threadIdx.x;
    float mp = -INFINITY, sp = 0.f;
#pragma unroll 2
    for (int j = k; j < nvz; j += C) {
      const float mnew = mref[static_cast<int64_t>(j) * T + t];
      if (mnew != mp) {
        sp = (mp == -INFINITY) ? 0.f : sp * ex2_approx((mp - mnew) * kLog2e);
        mp = mnew;
      }
      float cv[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) cv[c] = crow[j * kChunks + c];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) sp += cv[c];
    }
    cls[k] = mp;
    cls[8 + k] = sp;
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    float mstar = -INFINITY;
    for (int k = 0; k < C; ++k) mstar = fmaxf(mstar, cls[k]);
    float s_ex = 0.f;
    for (int k = 0; k < C; ++k) {
      const float mq = cls[k];
      if (mq != -INFINITY) s_ex = fmaf(cls[8 + k], ex2_approx((mq - mstar) * kLog2e), s_ex);
    }
    const int32_t yt = y[t];
    const bool ybad = yt < 0 || yt >= V;
    float lp = __int_as_float(0x7fc00000), lse = __int_as_float(0x7fc00000);
    if (!ybad) {
      const float zy = zyb[t];
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
