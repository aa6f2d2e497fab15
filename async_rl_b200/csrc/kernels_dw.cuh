// kernels_dw.cuh -- dW from the stored probability tiles: a persistent GEMM over the P store.
//
// The fused forward (kernels_lm.cuh, kModeFwdDH with a P store) leaves, for every scored row t
// and vocabulary column v, P[t][v] = bf16(e^{z_tv - m_tj}) (0 at the target column), the reference
// m_tj of the vocabulary step j that holds v, lse_t, g_t = -c_i w_t and s'_t / s_t.  With
// m_t = the row's last reference (lse_t = m_t + log s_t),
//     dZ_tv = -g_t e^{m_tj - lse_t} P[t][v] = sigma_t c_tj P[t][v]          (v != y_t)
//     dZ_{t,y_t} = g_t (1 - p_{t,y_t}) = g_t s'_t / s_t
// with sigma_t = -g_t e^{m_t - lse_t} and c_tj = e^{m_tj - m_t} (exactly 1 unless the row's
// reference moved after step j).  k_dw_rows folds sigma_t into a scaled copy of the hidden states,
// H'_t = bf16(sigma_t h_t), and writes the target entry into the P store in the units of the last
// reference, P[t][y_t] = -(s'_t / s_t) e^{lse_t - m_t} = -s'_t (finite whatever the row's
// history), so that sigma_t P[t][y_t] = dZ_{t,y_t}.  Then
//     dW_v = sum_t (c_tj P[t][v]) H'_t     (c taken as 1 at the target entry),
// a plain GEMM whose A operand needs a rewrite only in the (rare) chunks with c_tj != 1.
// ("Zero Mismatch, Simple Async RL", section "Alignment permits a simpler learning path": the
// gradient of the token-level IS loss through the LM head.)
//
// Work item = (two 128-row vocabulary tiles 2w, 2w+1, Hs-column slice q of H); a CTA owns one
// item at a time (grid = one CTA per SM, items strided by the grid) and sweeps the tokens in
// chunks of 64:
//   TMA warp     P^T chunk [256 v x 64 t] (four MN-major 64-column blocks) + H' chunk [64 t x Hs]
//                + the chunk's references (each block's and the last)
//   fix-up       8 warps rescale, in shared memory, the P rows of tokens whose reference moved
//   MMA lane     O_0, O_1 [128 x Hs] += P^T halves * H' chunk (A and B MN-major)
//   drain        4 warps write the finished O_0, O_1 of an item to dW
// A stage of two 128-row tiles and one H' chunk carries 8.4 MFLOP per 64 KB; the slices of one
// vocabulary pair run on neighbouring CTAs at the same time, so a P chunk is read from HBM once
// and from L2 by the others.
#pragma once

#include "kernels_lm.cuh"

namespace bi {

constexpr int kDwThreads = 448;  // TMA warp, MMA warp, 8 transform warps, 4 drain warps
constexpr int kDwXfThreads = 256;
constexpr int kDwAUnit = 8192;   // [64 tokens][64 vocabulary] bf16, 128B-swizzled
constexpr int kDwABytes = 4 * kDwAUnit;   // two 128-row vocabulary tiles
constexpr int kDwTokBytes = 6 * 256;      // per chunk: m of each 64-column block, last m, target, x 64 tokens

#define BI_DW_CONFIGS(X) X(64) X(128) X(192) X(256)

struct DwArgs {
  int32_t H, V;
  int32_t Hs;               // columns per item (multiple of 64, <= 256)
  int32_t nsl;              // H / Hs
  int32_t NZf;              // vocabulary step width of the forward (granularity of the references)
  int32_t nvz;              // steps of the forward (rows of the reference history)
  int64_t Tpad;             // leading dimension of the reference history (rows of the P store)
  const int64_t* d_rows;    // number of scored rows on the device
  int32_t nv128;            // ceil(V / 128)
  int32_t nitems;           // ceil(nv128 / 2) * nsl
  const float* mhist;       // [nvz][Tpad] reference of each row at each vocabulary step
  const int32_t* y_c;       // [Tpad] target of each row
  float* grad_w;            // [V, H] fp32
  int32_t* status;
  uint64_t limit_ns;
};

struct DwShared {
  uint64_t full[kMaxStages];    // TMA -> transform (transaction bytes)
  uint64_t tready[kMaxStages];  // fix-up (256 threads) -> MMA
  uint64_t empty[kMaxStages];   // MMA commit -> TMA
  uint64_t o_full, o_empty;
  uint64_t mma_done;
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

constexpr int kDwSharedBytes = static_cast<int>((sizeof(DwShared) + 127) / 128 * 128);

template <int kHS>
struct DwTile {
  static constexpr int tok_off = kDwABytes + kHS * 128;  // per-token values after the two tiles
  static constexpr int stage_bytes = (tok_off + kDwTokBytes + 1023) / 1024 * 1024;
  static constexpr int fit = (kLmSmemLimit - kDwSharedBytes) / stage_bytes;
  static constexpr int nstages = fit < kMaxStages ? fit : kMaxStages;
  static constexpr int smem = nstages * stage_bytes + kDwSharedBytes;
  static_assert(kHS % 64 == 0 && kHS <= 256, "two accumulators of Hs columns fill at most 512 TMEM columns");
  static_assert(kDwABytes % 1024 == 0 && (kHS * 128) % 1024 == 0, "operand blocks stay 1024-byte aligned");
  static_assert(nstages >= 2, "pipeline needs at least two stages");
};

__device__ __forceinline__ bool dw_wait(DwShared& sh, const DwArgs& a, uint64_t* bar, uint32_t parity) {
  const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
  return mbar_wait<false>(bar, parity, wc);
}

// generic-proxy writes to shared memory -> visible to the tensor cores' (async proxy) reads
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int kHS>
__global__ void __launch_bounds__(kDwThreads, 1)
    k_dw_stream(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_h, DwArgs a) {
  // tm_p: the P store as [p_ld / 64][Tpad][64], box {64, 64, 4}; tm_h: the scaled hidden states
  // H' as [H / 64][Tpad][64], box {64, 64, Hs / 64}
  extern __shared__ __align__(1024) uint8_t dsmem[];
  constexpr int nst = DwTile<kHS>::nstages;
  constexpr uint32_t sbytes = DwTile<kHS>::stage_bytes;
  DwShared& sh = *reinterpret_cast<DwShared*>(dsmem + nst * sbytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.tready[i], kDwXfThreads);
      mbar_init(&sh.empty[i], 1);
    }
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.o_empty, 128);
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
  const int64_t rows = misaligned ? 0 : *a.d_rows;
  const int nk = static_cast<int>((rows + 63) / 64);  // token chunks per item
  const int nitems = misaligned ? 0 : a.nitems;

  if (warp == 0) {
    // ---------------- TMA ----------------
    if (lane == 0 && nk > 0) {
      tma_prefetch_desc(&tm_p);
      tma_prefetch_desc(&tm_h);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < nitems; it += gridDim.x) {
        const int w = it / a.nsl, q = it - (it / a.nsl) * a.nsl;
#pragma unroll 1
        for (int k = 0; k < nk; ++k) {
          if (!dw_wait(sh, a, &sh.empty[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&sh.full[stage], DwTile<kHS>::tok_off + kDwTokBytes);
          const uint32_t dst = ring + stage * sbytes;
          // the four 64-column blocks of the P chunk, then the Hs / 64 column blocks of the H
          // chunk, one instruction each (block-major tensor maps)
          tma_load_3d(dst, &tm_p, &sh.full[stage], 0, k * 64, w * 4);
          tma_load_3d(dst + kDwABytes, &tm_h, &sh.full[stage], 0, k * 64, q * (kHS / 64));
          // the chunk's references: each block's forward step, then the last step (64 x 4 bytes
          // each; the history holds Tpad >= 64 nk rows)
          const uint32_t tok = dst + DwTile<kHS>::tok_off;
          const int64_t t0 = static_cast<int64_t>(k) * 64;
#pragma unroll
          for (int h = 0; h < 4; ++h) {  // a block past V reads a valid, unused row
            const int jm = min((w * 256 + h * 64) / a.NZf, a.nvz - 1);
            bulk_load(tok + h * 256, a.mhist + static_cast<int64_t>(jm) * a.Tpad + t0, 256, &sh.full[stage]);
          }
          bulk_load(tok + 1024, a.mhist + static_cast<int64_t>(a.nvz - 1) * a.Tpad + t0, 256, &sh.full[stage]);
          bulk_load(tok + 1280, a.y_c + t0, 256, &sh.full[stage]);
          ring_advance(stage, phase, nst);
        }
      }
      for (uint32_t i = 0; i < static_cast<uint32_t>(nst); ++i) {
        const uint32_t ph = (i < stage) ? phase : (phase ^ 1u);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_test(&sh.full[i], ph))
          if (globaltimer_ns() - t0 > a.limit_ns) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA ----------------
    if (lane == 0 && nk > 0) {
      constexpr uint32_t idesc = idesc_bf16(128, kHS, true, true);
      const uint64_t da0 = sdesc_mn_sw128(ring, kDwAUnit);
      const uint64_t db0 = sdesc_mn_sw128(ring + kDwABytes, kDwAUnit);
      constexpr uint64_t sb = sbytes >> 4;
      uint32_t stage = 0, phase = 0, n_it = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < nitems; it += gridDim.x, ++n_it) {
        if (!dw_wait(sh, a, &sh.o_empty, (n_it & 1u) ^ 1u)) break;
        tc_fence_after();
#pragma unroll 1
        for (int k = 0; k < nk; ++k) {
          if (!dw_wait(sh, a, &sh.tready[stage], phase)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 16 tokens = 16 MN-major rows of 128 B = 2 KB
            const uint32_t accum = (k > 0 || kk > 0) ? 1u : 0u;
            const uint64_t db = db0 + stage * sb + kk * (2048 >> 4);
            umma_bf16(tmem, da0 + stage * sb + kk * (2048 >> 4), db, idesc, accum);
            umma_bf16(tmem + kHS, da0 + stage * sb + ((2 * kDwAUnit) >> 4) + kk * (2048 >> 4), db, idesc, accum);
          }
          umma_commit(&sh.empty[stage]);
          ring_advance(stage, phase, nst);
        }
        if (!ok) break;
        umma_commit(&sh.o_full);
      }
      umma_commit(&sh.mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_test(&sh.mma_done, 0))
        if (globaltimer_ns() - t0 > a.limit_ns) break;
    }
    __syncwarp();
  } else if (warp < 10) {
    // ---------------- fix-up: rows whose reference moved after this block's step ----------------
    // P of step j is relative to the reference m_tj; H' carries e^{m_t - lse_t} for the last
    // reference m_t.  Where they differ (a later tile raised the reference) the P row of that block
    // is multiplied by c = e^{m_tj - m_t} < 1 here, except the target entry, which k_dw_rows wrote
    // in the units of m_t already; elsewhere nothing is rewritten.
    const int tt = threadIdx.x - 64;  // 0..255
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && nk > 0 && it < nitems; it += gridDim.x) {
      const int w = it / a.nsl;
#pragma unroll 1
      for (int k = 0; k < nk; ++k) {
        if (!dw_wait(sh, a, &sh.full[stage], phase)) { ok = false; break; }
        const uint32_t base = ring + stage * sbytes;
        const float* tok = reinterpret_cast<const float*>(dsmem + stage * sbytes + DwTile<kHS>::tok_off);
        bool wrote = false;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          // 16-byte chunk c = tt + 256 i of each 8 KB block: token row tl, logical chunk cq
          const int c = tt + 256 * i;
          const int tl = c >> 3, cq = c & 7;
          if (static_cast<int64_t>(k) * 64 + tl >= rows) continue;  // padding rows: H' is zero there
          const float mlast = tok[256 + tl];
          const int32_t yy = reinterpret_cast<const int32_t*>(tok)[320 + tl];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float mj = tok[64 * h + tl];
            if (mj == mlast) continue;
            const float cf = ex2_approx((mj - mlast) * kLog2e);
            const uint32_t cf2 = pack_bf16x2(cf, cf);
            const uint32_t addr = base + h * kDwAUnit + static_cast<uint32_t>(tl * 128 + ((cq ^ (tl & 7)) << 4));
            uint32_t pv[4];
            asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(pv[0]), "=r"(pv[1]), "=r"(pv[2]), "=r"(pv[3])
                         : "r"(addr));
            const uint32_t dv = static_cast<uint32_t>(yy - (w * 256 + h * 64 + cq * 8));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint32_t q = pv[e];
              asm("mul.rn.bf16x2 %0, %0, %1;" : "+r"(q) : "r"(cf2));
              // keep the target entry as loaded (dv >= 8 when the target is not in this chunk)
              const uint32_t keep = ((dv == 2u * e) ? 0x0000ffffu : 0u) | ((dv == 2u * e + 1u) ? 0xffff0000u : 0u);
              pv[e] = (q & ~keep) | (pv[e] & keep);
            }
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(pv[0]), "r"(pv[1]), "r"(pv[2]),
                         "r"(pv[3])
                         : "memory");
            wrote = true;
          }
        }
        if (wrote) fence_proxy_async_shared();
        mbar_arrive(&sh.tready[stage]);
        ring_advance(stage, phase, nst);
      }
    }
  } else {
    // ---------------- drain: O_0, O_1 -> dW rows ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    // row chunks are 128-byte multiples from the base: whole sectors when the base allows
    const bool sectors = (reinterpret_cast<uintptr_t>(a.grad_w) & 31u) == 0;
    uint32_t n_it = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++n_it) {
      const int w = it / a.nsl, q = it - (it / a.nsl) * a.nsl;
      if (nk > 0) {
        const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&sh.o_full, n_it & 1u, wc))) break;
        tc_fence_after();
      }
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int64_t v = static_cast<int64_t>(w) * 256 + half * 128 + row;
        float* dst = (v < a.V) ? a.grad_w + v * a.H + q * kHS : nullptr;
        if (nk == 0) {  // no scored rows: the gradient is zero
          if (dst)
            for (int c = 0; c < kHS / 4; ++c) reinterpret_cast<float4*>(dst)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          continue;
        }
#pragma unroll 1
        for (int c = 0; c < kHS / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tl + half * kHS + c * 32, r);
          tmem_ld_wait();
          if (dst) {
            if (sectors) {
#pragma unroll
              for (int e = 0; e < 4; ++e) st_global_v8(dst + c * 32 + 8 * e, r + 8 * e);
            } else {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e) d4[e] = make_uint4(r[4 * e], r[4 * e + 1], r[4 * e + 2], r[4 * e + 3]);
            }
          }
        }
      }
      if (nk > 0) {
        tc_fence_before();
        mbar_arrive(&sh.o_empty);
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

// One warp per row of the P store (Tpad rows).  Scored rows: H'_t = bf16(sigma_t h_t) with
// sigma_t = -g_t e^{m_t - lse_t} (m_t the row's last reference), and the target entry of the P
// store P[t][y_t] = -(s'_t / s_t) e^{lse_t - m_t} so that sigma_t P[t][y_t] = g_t s'_t / s_t.
// Other rows: H'_t = 0.  Runs after the forward (and the sequence
// gate, whose rejected rows have g_t = 0) and before k_dw_stream.
__global__ void k_dw_rows(const uint16_t* __restrict__ hc, int H, const int64_t* __restrict__ d_rows, int64_t Tpad,
                          const float* __restrict__ lse_c, const float* __restrict__ g_c,
                          const float* __restrict__ sxr_c, const int32_t* __restrict__ y_c,
                          const float* __restrict__ mhist, int nvz, int V, uint16_t* __restrict__ hs,
                          uint16_t* __restrict__ pbuf, int64_t p_ld) {
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= Tpad) return;
  const int64_t rows = *d_rows;
  uint4* dst = reinterpret_cast<uint4*>(hs + t * H);
  if (t >= rows) {
    for (int q = lane; q < H / 8; q += 32) dst[q] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const float lse = lse_c[t];
  const float mlast = mhist[static_cast<int64_t>(nvz - 1) * Tpad + t];
  const float sig = -g_c[t] * ex2_approx((mlast - lse) * kLog2e);
  const uint4* src = reinterpret_cast<const uint4*>(hc + t * H);
  for (int q = lane; q < H / 8; q += 32) {
    const uint4 v = src[q];
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2(sig * __uint_as_float(in[e] << 16), sig * __uint_as_float(in[e] & 0xffff0000u));
    dst[q] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  const int32_t y = y_c[t];
  if (lane == 0 && y >= 0 && y < V) {
    const float val = -sxr_c[t] * ex2_approx((lse - mlast) * kLog2e);
    pbuf[t * p_ld + y] = static_cast<uint16_t>(pack_bf16x2(val, val) & 0xffffu);
  }
}

}  // namespace bi
