// kernels_bwd.cuh -- backward of the IS loss through the LM head, with the logits recomputed on
// chip and never stored:
//     dZ_tv = g_t (1[v = y_t] - exp(z_tv - lse_t)),   g_t = -c_i w_t
//     dH = dZ W          (mode kModeDH: a cluster owns a 128-row tile of hidden states and
//                         sweeps the vocabulary; reduction over v in ascending tile order)
//     dW = dZ^T H        (mode kModeDW: a cluster owns a 128-row tile of the vocabulary and
//                         sweeps the rows; reduction over t in ascending tile order)
//
// The [128 x H] fp32 accumulator does not fit one SM's tensor memory, so the H columns are split
// over a cluster of C CTAs (H / C <= 384 columns each).  The 128x128 logit tile of each step is
// computed once, by one CTA of the cluster in rotation (full K = H), turned into a bf16 dZ tile
// by its epilogue and published through a small L2-resident scratch slot; every CTA of the
// cluster then TMA-loads it as the A operand of its own slice update.  Cross-CTA hand-off uses
// mbarriers in each CTA's shared memory, signalled through the cluster's shared-memory window.
// Tile shape, K order and the order of the reduction are fixed and independent of T, so each
// row of dH has the same bits in any batch (the "Zero Mismatch" post, "Alignment permits a
// simpler learning path": bit-identical rows for the same weights and tokens).
#pragma once

#include "sm100.cuh"

namespace bi {

constexpr int kUnitBytes = 16384;  // one [128 rows][64 bf16] 128B-swizzled tile
constexpr int kRing = 13;          // shared-memory ring of units
constexpr int kBwdSmemBytes = kRing * kUnitBytes + 1024;
constexpr int kBwdThreads = 192;
constexpr int kZCol = 384;          // TMEM column of the 128-column logit accumulator
constexpr int kSlotsPerCta = 2;     // dZ scratch slots per producer CTA
constexpr int kMaxCluster = 8;
constexpr int kMaxSlots = kMaxCluster * kSlotsPerCta;

enum BwdMode : int { kModeDH = 0, kModeDW = 1 };

struct BwdArgs {
  int32_t H, V;
  int32_t C;              // CTAs per cluster
  int32_t Hs;             // H / C: columns owned by each CTA
  int32_t nchunk;         // MMA column chunks of the slice update (1 or 2)
  int32_t chunk_units[2]; // 64-column units per chunk
  int64_t T;              // rows of the compact hidden-state tensor map (upper bound)
  const int64_t* d_rows;  // number of valid compact rows (device)
  int32_t nvt128;         // ceil(V / 128)
  const float* lse;       // [rows] compact
  const float* g;         // [rows] compact: -c_i w_t (0 for rows without gradient)
  const int32_t* y;       // [rows] compact targets
  const int32_t* rowmap;  // [rows] compact row -> output row of grad_hidden
  uint16_t* grad_hidden;  // [*, H] bf16 (kModeDH)
  float* grad_w;          // [V, H] fp32 (kModeDW)
  uint16_t* dz_scratch;   // [clusters * C * kSlotsPerCta * 128][128] bf16
  int32_t* status;
  uint64_t limit_ns;
};

struct BwdShared {
  uint64_t full[kRing];
  uint64_t empty[kRing];
  uint64_t z_full, z_empty, o_full, o_empty, mma_done;
  uint64_t ep_bar;       // rendezvous of the 128 epilogue threads (bounded, unlike bar.sync)
  uint64_t dz_ready[kMaxSlots];
  uint64_t dz_free[kMaxSlots];
  float col_lse2[128];   // kModeDW: per-column lse * log2(e)
  float col_g[128];      // kModeDW: per-column g
  int32_t col_y[128];    // kModeDW: per-column target (INT32_MIN: column not valid)
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

template <int kMode>
__global__ void __launch_bounds__(kBwdThreads, 1)
    k_bwd_cluster(const __grid_constant__ CUtensorMap tm_stat, const __grid_constant__ CUtensorMap tm_stream,
                  const __grid_constant__ CUtensorMap tm_dz, BwdArgs a) {
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ BwdShared sh;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t C = static_cast<uint32_t>(a.C);
  const uint32_t rank = cluster_ctarank();
  const uint32_t cl = cluster_id_x();
  const uint32_t ncl = ncluster_x();
  const uint32_t nslot = C * kSlotsPerCta;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    mbar_init(&sh.z_full, 1);
    mbar_init(&sh.z_empty, 128);
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.o_empty, 128);
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.ep_bar, 128);
    for (uint32_t i = 0; i < nslot; ++i) {
      mbar_init(&sh.dz_ready[i], 1);
      mbar_init(&sh.dz_free[i], C);
    }
    sh.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // peers' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  // On a timeout, stop this CTA and its peers (their own waits would run out later anyway).
  auto wait = [&](uint64_t* bar, uint32_t parity, bool cluster_acq) -> bool {
    const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
    const bool ok = cluster_acq ? mbar_wait<true>(bar, parity, wc) : mbar_wait<false>(bar, parity, wc);
    if (!ok) {
      const uint32_t la = smem_u32(const_cast<uint32_t*>(&sh.abort_flag));
      for (uint32_t q = 0; q < C; ++q) st_cluster_u32(mapa_shared(la, q), 1u);
    }
    return ok;
  };

  const int64_t rows = *a.d_rows;
  const int mtiles = static_cast<int>((rows + 127) / 128);
  const int nunits = (kMode == kModeDH) ? mtiles : a.nvt128;
  const int steps = (kMode == kModeDH) ? a.nvt128 : mtiles;
  const int my_units = (static_cast<int>(cl) < nunits) ? (nunits - static_cast<int>(cl) + static_cast<int>(ncl) - 1) / static_cast<int>(ncl) : 0;
  const int64_t total = static_cast<int64_t>(my_units) * steps;
  const int KB = a.H / 64;
  const int slice0 = static_cast<int>(rank) * a.Hs;
  auto own = [&](int64_t s) { return static_cast<uint32_t>(s % C) == rank; };
  auto unit_of = [&](int64_t s) { return static_cast<int>(cl) + static_cast<int>(s / steps) * static_cast<int>(ncl); };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tm_stat);
      tma_prefetch_desc(&tm_stream);
      tma_prefetch_desc(&tm_dz);
      uint32_t pos = 0;
      bool ok = true;
      auto load_unit = [&](const CUtensorMap* m, int x, int y) {
        const uint32_t st = pos % kRing, ph = (pos / kRing) & 1u;
        if (!wait(&sh.empty[st], ph ^ 1u, false)) return false;
        mbar_arrive_expect_tx(&sh.full[st], kUnitBytes);
        tma_load_2d(smem_u32(ring + st * kUnitBytes), m, &sh.full[st], x, y);
        ++pos;
        return true;
      };
      auto pad_unit = [&]() {
        const uint32_t st = pos % kRing, ph = (pos / kRing) & 1u;
        if (!wait(&sh.empty[st], ph ^ 1u, false)) return false;
        mbar_arrive(&sh.full[st]);
        ++pos;
        return true;
      };
      auto ztile = [&](int64_t s) {
        const int u = unit_of(s), j = static_cast<int>(s % steps);
        for (int kb = 0; kb < KB; ++kb) {
          if (!load_unit(&tm_stat, kb * 64, u * 128)) return false;
          if (!load_unit(&tm_stream, kb * 64, j * 128)) return false;
        }
        return true;
      };
      auto ostep = [&](int64_t s) {
        const int j = static_cast<int>(s % steps);
        const uint32_t slot = static_cast<uint32_t>(s % nslot);
        if (!wait(&sh.dz_ready[slot], static_cast<uint32_t>((s / nslot) & 1), true)) return false;
        fence_proxy_async_global();
        const int dz_row = static_cast<int>((cl * nslot + slot) * 128);
        if (!load_unit(&tm_dz, 0, dz_row)) return false;
        if (!load_unit(&tm_dz, 64, dz_row)) return false;
        int su = 0;
        for (int ch = 0; ch < a.nchunk; ++ch) {
          const int g = a.chunk_units[ch];
          while ((pos % kRing) + g > kRing)
            if (!pad_unit()) return false;
          for (int i = 0; i < g; ++i)
            if (!load_unit(&tm_stream, slice0 + (su + i) * 64, j * 128)) return false;
          su += g;
        }
        return true;
      };
      for (int64_t s = 0; ok && s < total && s < C; ++s)
        if (own(s)) ok = ztile(s);
      for (int64_t s = 0; ok && s < total; ++s) {
        if (own(s) && s + C < total) ok = ztile(s + C);
        if (ok) ok = ostep(s);
      }
      for (uint32_t i = (pos > kRing ? pos - kRing : 0u); i < pos; ++i) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_test(&sh.full[i % kRing], (i / kRing) & 1u))
          if (globaltimer_ns() - t0 > a.limit_ns) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_z = idesc_bf16(128, 128, false, false);
      uint32_t pos = 0, zc = 0, oc = 0;
      bool ok = true;
      auto take = [&](uint32_t& st) {
        st = pos % kRing;
        const uint32_t ph = (pos / kRing) & 1u;
        ++pos;
        return wait(&sh.full[st], ph, false);
      };
      auto ztile = [&]() {
        if (!wait(&sh.z_empty, (zc & 1u) ^ 1u, false)) return false;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          uint32_t sa, sb;
          if (!take(sa) || !take(sb)) return false;
          tc_fence_after();
          const uint32_t aa = smem_u32(ring + sa * kUnitBytes), ab = smem_u32(ring + sb * kUnitBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + kZCol, sdesc_k_sw128(aa + k * 32), sdesc_k_sw128(ab + k * 32), idesc_z, (kb | k) != 0);
          umma_commit(&sh.empty[sa]);
          umma_commit(&sh.empty[sb]);
        }
        umma_commit(&sh.z_full);
        ++zc;
        return true;
      };
      auto ostep = [&](int64_t s) {
        const int j = static_cast<int>(s % steps);
        if (j == 0) {
          if (!wait(&sh.o_empty, (oc & 1u) ^ 1u, false)) return false;
          tc_fence_after();
        }
        uint32_t d0, d1;
        if (!take(d0) || !take(d1)) return false;
        tc_fence_after();
        // the tile is in shared memory now: its scratch slot may be refilled by the producer
        const uint32_t slot = static_cast<uint32_t>(s % nslot);
        mbar_arrive_cluster(mapa_shared(smem_u32(&sh.dz_free[slot]), static_cast<uint32_t>(s % C)));
        const uint32_t a0 = smem_u32(ring + d0 * kUnitBytes), a1 = smem_u32(ring + d1 * kUnitBytes);
        uint32_t col = 0;
        for (int ch = 0; ch < a.nchunk; ++ch) {
          const int g = a.chunk_units[ch];
          while ((pos % kRing) + g > kRing) {
            uint32_t sp;
            if (!take(sp)) return false;
            mbar_arrive(&sh.empty[sp]);
          }
          uint32_t first = 0;
          for (int i = 0; i < g; ++i) {
            uint32_t st;
            if (!take(st)) return false;
            if (i == 0) first = st;
          }
          tc_fence_after();
          const uint32_t bb = smem_u32(ring + first * kUnitBytes);
          const uint32_t idesc_o = idesc_bf16(128, 64 * g, false, true);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aa = ((kk < 4) ? a0 : a1) + (kk & 3) * 32;
            umma_bf16(tmem + col, sdesc_k_sw128(aa), sdesc_mn_sw128(bb + kk * 2048, kUnitBytes), idesc_o,
                      (j > 0 || kk > 0) ? 1u : 0u);
          }
          for (int i = 0; i < g; ++i) umma_commit(&sh.empty[first + i]);
          col += 64 * g;
        }
        umma_commit(&sh.empty[d0]);
        umma_commit(&sh.empty[d1]);
        if (j == steps - 1) {
          umma_commit(&sh.o_full);
          ++oc;
        }
        return true;
      };
      for (int64_t s = 0; ok && s < total && s < C; ++s)
        if (own(s)) ok = ztile();
      for (int64_t s = 0; ok && s < total; ++s) {
        if (own(s) && s + C < total) ok = ztile();
        if (ok) ok = ostep(s);
      }
      umma_commit(&sh.mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_test(&sh.mma_done, 0))
        if (globaltimer_ns() - t0 > a.limit_ns) break;
    }
  } else {
    // ---------------- epilogue: 4 warps, one accumulator lane (row) per thread ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..127
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t zc = 0, oc = 0, epc = 0;
    bool ok = true;
    // warp-uniform outcome of a wait: the tcgen05.ld that follows is .sync.aligned
    auto ewait = [&](uint64_t* bar, uint32_t parity, bool cluster_acq) {
      return __all_sync(0xffffffffu, wait(bar, parity, cluster_acq)) != 0;
    };
    auto ep_sync = [&]() {
      mbar_arrive(&sh.ep_bar);
      return ewait(&sh.ep_bar, (epc++) & 1u, false);
    };
    float r_lse2 = 0.f, r_g = 0.f;
    int32_t r_y = -1;
    bool r_valid = false;
    int64_t r_out = 0;

    auto drain = [&](int u, bool have_acc) {
      if (have_acc) {
        if (!ewait(&sh.o_full, oc & 1u, false)) return false;
        tc_fence_after();
      }
      if (kMode == kModeDH) {
        const int64_t t = static_cast<int64_t>(u) * 128 + row;
        const bool v_ok = t < rows;
        uint16_t* dst = v_ok ? a.grad_hidden + static_cast<int64_t>(a.rowmap[t]) * a.H + slice0 : nullptr;
        for (int c = 0; c < a.Hs / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tl + c * 32, v);
          tmem_ld_wait();
          if (v_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
              w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
              w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
              w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
              d4[q] = w;
            }
          }
        }
      } else {
        const int64_t vr = static_cast<int64_t>(u) * 128 + row;
        const bool v_ok = vr < a.V;
        float* dst = v_ok ? a.grad_w + vr * a.H + slice0 : nullptr;
        for (int c = 0; c < a.Hs / 32; ++c) {
          uint32_t v[32];
          if (have_acc) {
            tmem_ld32(tl + c * 32, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] = 0u;
          }
          if (v_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) d4[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
      if (have_acc) {
        tc_fence_before();
        mbar_arrive(&sh.o_empty);
        ++oc;
      }
      return true;
    };

    if (kMode == kModeDW && steps == 0) {
      // no rows: every owned vocabulary tile gets a zero gradient
      for (int u = static_cast<int>(cl); u < nunits; u += static_cast<int>(ncl)) drain(u, false);
    }
    for (int64_t s = 0; ok && s < total; ++s) {
      const int u = unit_of(s);
      const int j = static_cast<int>(s % steps);
      if (kMode == kModeDH && j == 0) {
        const int64_t t = static_cast<int64_t>(u) * 128 + row;
        r_valid = t < rows;
        r_lse2 = r_valid ? a.lse[t] * kLog2e : 0.f;
        r_g = r_valid ? a.g[t] : 0.f;
        r_y = r_valid ? a.y[t] : -1;
        r_out = t;
      }
      if (own(s)) {
        const uint32_t slot = static_cast<uint32_t>(s % nslot);
        if (kMode == kModeDW) {
          if (!ep_sync()) { ok = false; break; }  // previous step's column parameters are no longer read
          const int64_t t = static_cast<int64_t>(j) * 128 + et;
          const bool tv = t < rows;
          sh.col_lse2[et] = tv ? a.lse[t] * kLog2e : 0.f;
          sh.col_g[et] = tv ? a.g[t] : 0.f;
          sh.col_y[et] = tv ? a.y[t] : INT32_MIN;
          if (!ep_sync()) { ok = false; break; }
        }
        if (!ewait(&sh.z_full, zc & 1u, false)) { ok = false; break; }
        tc_fence_after();
        if (s >= nslot) {
          if (!ewait(&sh.dz_free[slot], static_cast<uint32_t>(((s / nslot) - 1) & 1), true)) { ok = false; break; }
        }
        uint16_t* dzrow = a.dz_scratch + (static_cast<int64_t>(cl * nslot + slot) * 128 + row) * 128;
        const int64_t vrow = static_cast<int64_t>(u) * 128 + row;  // kModeDW: this lane's vocabulary row
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tl + kZCol + c * 32, v);
          tmem_ld_wait();
          float d[32];
          if (kMode == kModeDH) {
            const int vbase = j * 128 + c * 32;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float p = ex2_approx(fmaf(__uint_as_float(v[q]), kLog2e, -r_lse2));
              const float oh = (vbase + q == r_y) ? 1.f : 0.f;
              d[q] = (r_valid && vbase + q < a.V) ? r_g * (oh - p) : 0.f;
            }
          } else {
            const bool v_ok = vrow < a.V;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int tc = c * 32 + q;
              const float p = ex2_approx(fmaf(__uint_as_float(v[q]), kLog2e, -sh.col_lse2[tc]));
              const int32_t yc = sh.col_y[tc];
              const float oh = (static_cast<int64_t>(yc) == vrow) ? 1.f : 0.f;
              d[q] = (v_ok && yc != INT32_MIN) ? sh.col_g[tc] * (oh - p) : 0.f;
            }
          }
          uint4* d4 = reinterpret_cast<uint4*>(dzrow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_uint4(pack_bf16x2(d[8 * q + 0], d[8 * q + 1]), pack_bf16x2(d[8 * q + 2], d[8 * q + 3]),
                               pack_bf16x2(d[8 * q + 4], d[8 * q + 5]), pack_bf16x2(d[8 * q + 6], d[8 * q + 7]));
        }
        tc_fence_before();
        mbar_arrive(&sh.z_empty);
        ++zc;
        __threadfence();
        fence_proxy_async_global();
        if (!ep_sync()) { ok = false; break; }
        if (et == 0) {
          const uint32_t la = smem_u32(&sh.dz_ready[slot]);
          for (uint32_t q = 0; q < C; ++q) mbar_arrive_cluster(mapa_shared(la, q));
        }
      }
      if (j == steps - 1) {
        if (!drain(u, true)) { ok = false; break; }
      }
    }
    (void)r_out;
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no peer touches this CTA's shared memory after this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bi
