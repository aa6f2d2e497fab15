// kernels_fwd.cuh -- forward pass of the token log-probability: a persistent tcgen05 GEMM over
// (128-row tile) x (256-wide vocabulary tile) with a fused online log-sum-exp epilogue.
//
// "Zero Mismatch, Simple Async RL", section "Only one probability gap comes from old weights":
// batch shape, reduction order and prefill/decode arithmetic must not change a row's logprob.
// Hence: one tile shape for every T, the hidden dimension reduced in one fixed K order inside
// the tensor core, and the vocabulary split into a fixed number of chunks that depends only
// on V; every row's statistics come from its own TMEM lane and are combined in a fixed order.
// The T x V logits exist only in TMEM.
#pragma once

#include "sm100.cuh"

namespace bi {

constexpr int kFwdBM = 128;
constexpr int kFwdBN = 256;
constexpr int kBK = 64;
constexpr int kFwdStages = 4;
constexpr int kFwdABytes = kFwdBM * kBK * 2;   // 16 KB
constexpr int kFwdBBytes = kFwdBN * kBK * 2;   // 32 KB
constexpr int kFwdStageBytes = kFwdABytes + kFwdBBytes;
constexpr int kFwdSmemBytes = kFwdStages * kFwdStageBytes + 1024;
constexpr int kFwdThreads = 192;
constexpr int kMaxVChunks = 16;  // vocabulary chunks: min(16, number of 256-wide tiles)

struct FwdArgs {
  int64_t T;               // rows covered by the tensor map (upper bound)
  const int64_t* d_rows;   // nullable: number of valid rows, read on the device
  int32_t H, V;
  int32_t nvt;             // number of 256-wide vocabulary tiles
  int32_t nchunks;         // vocabulary chunks
  const int32_t* targets;  // [rows]
  float* part_m;           // [nchunks][T] running max per row and chunk
  float* part_s;           // [nchunks][T] sum of exp(z - m)
  float* part_zy;          // [nchunks][T] target logit when the target lies in the chunk
  int32_t* status;
  uint64_t limit_ns;
  uint64_t force_timeout_ns;  // test hook: > 0 makes the epilogue wait on a barrier nobody signals
};

__host__ __device__ inline int vchunk_begin(int c, int nvt, int nchunks) {
  return static_cast<int>((static_cast<int64_t>(c) * nvt) / nchunks);
}

// Wait with a time limit that ignores the abort flag: used at teardown for work already in flight.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__global__ void __launch_bounds__(kFwdThreads, 1)
    k_fwd_logits(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w, FwdArgs a) {
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[kFwdStages];
  __shared__ __align__(8) uint64_t bar_empty[kFwdStages];
  __shared__ __align__(8) uint64_t bar_tfull[2];
  __shared__ __align__(8) uint64_t bar_tempty[2];
  __shared__ __align__(8) uint64_t bar_mma_done;
  __shared__ __align__(8) uint64_t bar_never;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile uint32_t abort_sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kFwdStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_tfull[i], 1);
      mbar_init(&bar_tempty[i], 128);
    }
    mbar_init(&bar_mma_done, 1);
    mbar_init(&bar_never, 1);
    abort_sh = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const WaitCtl wc{&abort_sh, a.status, a.limit_ns};

  const int64_t rows = a.d_rows ? *a.d_rows : a.T;
  const int mtiles = static_cast<int>((rows + kFwdBM - 1) / kFwdBM);
  const int nunits = mtiles * a.nchunks;
  const int KB = a.H / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tm_h);
      tma_prefetch_desc(&tm_w);
      uint32_t q = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const int chunk = u / mtiles, mt = u % mtiles;
        const int vt1 = vchunk_begin(chunk + 1, a.nvt, a.nchunks);
        for (int vt = vchunk_begin(chunk, a.nvt, a.nchunks); ok && vt < vt1; ++vt) {
          for (int kb = 0; kb < KB; ++kb, ++q) {
            const uint32_t st = q % kFwdStages, ph = (q / kFwdStages) & 1u;
            if (!mbar_wait<false>(&bar_empty[st], ph ^ 1u, wc)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bar_full[st], kFwdStageBytes);
            const uint32_t sa = smem_u32(smem + st * kFwdStageBytes);
            tma_load_2d(sa, &tm_h, &bar_full[st], kb * kBK, mt * kFwdBM);
            tma_load_2d(sa + kFwdABytes, &tm_w, &bar_full[st], kb * kBK, vt * kFwdBN);
          }
        }
      }
      // loads still in flight must land before the CTA may exit
      for (uint32_t i = (q > kFwdStages ? q - kFwdStages : 0u); i < q; ++i)
        mbar_wait_drain(&bar_full[i % kFwdStages], (i / kFwdStages) & 1u, a.limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_bf16(kFwdBM, kFwdBN, false, false);
      uint32_t q = 0, tc = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        const int chunk = u / mtiles;
        const int vt1 = vchunk_begin(chunk + 1, a.nvt, a.nchunks);
        for (int vt = vchunk_begin(chunk, a.nvt, a.nchunks); ok && vt < vt1; ++vt, ++tc) {
          const uint32_t acc = tc & 1u, tph = (tc >> 1) & 1u;
          if (!mbar_wait<false>(&bar_tempty[acc], tph ^ 1u, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem + acc * kFwdBN;
          for (int kb = 0; kb < KB; ++kb, ++q) {
            const uint32_t st = q % kFwdStages, ph = (q / kFwdStages) & 1u;
            if (!mbar_wait<false>(&bar_full[st], ph, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + st * kFwdStageBytes);
            const uint32_t sb = sa + kFwdABytes;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_bf16(dt, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), idesc, (kb | k) != 0);
            umma_commit(&bar_empty[st]);
          }
          if (ok) umma_commit(&bar_tfull[acc]);
        }
      }
      umma_commit(&bar_mma_done);
      mbar_wait_drain(&bar_mma_done, 0, a.limit_ns);
    }
  } else {
    // ---------------- epilogue: 4 warps, one row per thread ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    bool ok = true;
    if (a.force_timeout_ns != 0) {
      const WaitCtl w2{&abort_sh, a.status, a.force_timeout_ns};
      ok = __all_sync(0xffffffffu, mbar_wait<false>(&bar_never, 0, w2));
    }
    uint32_t tc = 0;
    for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
      const int chunk = u / mtiles, mt = u % mtiles;
      const int64_t r = static_cast<int64_t>(mt) * kFwdBM + row;
      const bool valid = r < rows;
      const int32_t y = valid ? a.targets[r] : -1;
      float m = -INFINITY, s = 0.f, zy = 0.f;
      const int vt1 = vchunk_begin(chunk + 1, a.nvt, a.nchunks);
      for (int vt = vchunk_begin(chunk, a.nvt, a.nchunks); vt < vt1; ++vt, ++tc) {
        const uint32_t acc = tc & 1u, tph = (tc >> 1) & 1u;
        // warp-uniform outcome: tcgen05.ld below is .sync.aligned
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&bar_tfull[acc], tph, wc))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kFwdBN / 32; ++c) {
          const int vbase = vt * kFwdBN + c * 32;
          uint32_t v[32];
          tmem_ld32(tl + acc * kFwdBN + c * 32, v);
          tmem_ld_wait();
          if (vbase < a.V) {
            float z[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) z[j] = __uint_as_float(v[j]);
            if (vbase + 32 > a.V) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (vbase + j >= a.V) z[j] = -INFINITY;
            }
            float cm = z[0];
#pragma unroll
            for (int j = 1; j < 32; ++j) cm = fmaxf(cm, z[j]);
            const float mn = fmaxf(m, cm);
            const float mn2 = mn * kLog2e;
            const float sc = (mn == m) ? 1.f : ex2_approx(m * kLog2e - mn2);
            float cs = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) cs += ex2_approx(fmaf(z[j], kLog2e, -mn2));
            s = fmaf(s, sc, cs);
            m = mn;
            const uint32_t yy = static_cast<uint32_t>(y - vbase);
            if (yy < 32u) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (static_cast<uint32_t>(j) == yy) zy = z[j];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bar_tempty[acc]);
      }
      if (ok && valid) {
        const int64_t o = static_cast<int64_t>(chunk) * a.T + r;
        a.part_m[o] = m;
        a.part_s[o] = s;
        a.part_zy[o] = zy;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Per-row combine of the chunk partials, in chunk order.  Shared by the logprob-only and the
// fused loss paths so that both produce identical bits.
__device__ __forceinline__ void combine_row(const float* __restrict__ pm, const float* __restrict__ ps,
                                            const float* __restrict__ pzy, int64_t stride, int64_t r,
                                            int nchunks, int nvt, int32_t y, float& lse, float& zy) {
  float m = -INFINITY;
  for (int c = 0; c < nchunks; ++c) m = fmaxf(m, pm[c * stride + r]);
  float s = 0.f;
  for (int c = 0; c < nchunks; ++c) {
    const float mc = pm[c * stride + r];
    const float sc = ps[c * stride + r];
    s += (mc == -INFINITY) ? 0.f : sc * ex2_approx((mc - m) * kLog2e);
  }
  lse = m + logf(s);
  const int vt = y / kFwdBN;
  int cy = 0;
  for (int c = 1; c < nchunks; ++c)
    if (vt >= vchunk_begin(c, nvt, nchunks)) cy = c;
  zy = pzy[cy * stride + r];
}

}  // namespace bi
