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
//
// Issue-loop design: the single issuing lane is the critical resource (a tcgen05.mma takes 64-96
// tensor cycles here), so the MMA and TMA warps run converged loops with position counters (no
// integer division), precomputed descriptors, and one commit per 32 KB shared-memory slot.
#pragma once

#include "sm100.cuh"

namespace bi {

constexpr int kUnitBytes = 16384;             // one [128 rows][64 bf16] 128B-swizzled tile
constexpr int kSlotBytes = 2 * kUnitBytes;    // ring slot: two units, one barrier pair
constexpr int kSlots = 7;
constexpr int kBwdThreads = 192;
constexpr int kZCol = 384;                    // TMEM column of the 128-column logit accumulator
constexpr int kSlotsPerCta = 2;               // dZ scratch slots per producer CTA
constexpr int kMaxCluster = 8;
constexpr int kMaxSlots = kMaxCluster * kSlotsPerCta;
constexpr int kMaxChunks = 3;                 // slice update chunks of <= 128 columns (H / C <= 384)

enum BwdMode : int { kModeDH = 0, kModeDW = 1 };

struct BwdArgs {
  int32_t H, V;
  int32_t C;                      // CTAs per cluster
  int32_t Hs;                     // H / C: columns owned by each CTA
  int32_t nchunk;                 // slice-update chunks (<= 3)
  int32_t chunk_units[kMaxChunks];// 64-column units per chunk (1 or 2)
  int64_t T;                      // rows of the compact hidden-state tensor map (upper bound)
  const int64_t* d_rows;          // number of valid compact rows (device)
  int32_t nvt128;                 // ceil(V / 128)
  const float* lse;               // [rows] compact
  const float* g;                 // [rows] compact: -c_i w_t (0 for rows without gradient)
  const int32_t* y;               // [rows] compact targets
  const int32_t* rowmap;          // [rows] compact row -> output row of grad_hidden
  uint16_t* grad_hidden;          // [*, H] bf16 (kModeDH)
  float* grad_w;                  // [V, H] fp32 (kModeDW)
  uint16_t* dz_scratch;           // [clusters * C * kSlotsPerCta * 128][128] bf16
  int32_t* status;
  uint64_t limit_ns;
};

struct BwdShared {
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t z_full, z_empty, o_full, o_empty, mma_done;
  uint64_t ep_bar;                // rendezvous of the 128 epilogue threads (bounded, unlike bar.sync)
  uint64_t dz_ready[kMaxSlots];
  uint64_t dz_free[kMaxSlots];
  float col_lse2[128];            // kModeDW: per-column lse * log2(e)
  float col_g[128];               // kModeDW: per-column g
  int32_t col_y[128];             // kModeDW: per-column target (INT32_MIN: column not valid)
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

constexpr int kBwdSmemBytes = kSlots * kSlotBytes + static_cast<int>((sizeof(BwdShared) + 127) / 128 * 128);

__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile(
      "{\n\t.reg .pred q;\n\t.reg .b32 r;\n\t"
      "elect.sync r|q, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(p));
  return p != 0;
}

// Position in a cluster's step stream, advanced without division.
struct StreamPos {
  int64_t s;        // stream index
  int u_idx;        // index of the unit among this cluster's units
  int j;            // step inside the unit
  uint32_t modc;    // s mod C  (the producer CTA of step s)
  uint32_t slot;    // s mod (C * kSlotsPerCta)  (dZ scratch slot)
  uint32_t round;   // s div (C * kSlotsPerCta)
  __device__ __forceinline__ void zero() { s = 0; u_idx = 0; j = 0; modc = 0; slot = 0; round = 0; }
  __device__ __forceinline__ void next(int steps, uint32_t C, uint32_t nslot) {
    ++s;
    if (++j == steps) { j = 0; ++u_idx; }
    if (++modc == C) modc = 0;
    if (++slot == nslot) { slot = 0; ++round; }
  }
};

template <int kMode>
__global__ void __launch_bounds__(kBwdThreads, 1)
    k_bwd_cluster(const __grid_constant__ CUtensorMap tm_stat, const __grid_constant__ CUtensorMap tm_stream,
                  const __grid_constant__ CUtensorMap tm_dz, BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  uint8_t* ring = dsmem;
  BwdShared& sh = *reinterpret_cast<BwdShared*>(dsmem + kSlots * kSlotBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t C = static_cast<uint32_t>(a.C);
  const uint32_t rank = cluster_ctarank();
  const uint32_t cl = cluster_id_x();
  const uint32_t ncl = ncluster_x();
  const uint32_t nslot = C * kSlotsPerCta;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
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

  // Bounded wait with a warp-uniform outcome.  On a timeout, stop this CTA and its peers.
  auto wait = [&](uint64_t* bar, uint32_t parity, bool cluster_acq) -> bool {
    const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
    const bool ok = cluster_acq ? mbar_wait<true>(bar, parity, wc) : mbar_wait<false>(bar, parity, wc);
    if (!ok) {
      const uint32_t la = smem_u32(const_cast<uint32_t*>(&sh.abort_flag));
      for (uint32_t q = 0; q < C; ++q) st_cluster_u32(mapa_shared(la, q), 1u);
    }
    return __all_sync(0xffffffffu, ok) != 0;
  };

  const uint32_t ring_base = smem_u32(ring);
  // the 128B-swizzled tiles need 1024-byte aligned slots; refuse to run otherwise
  const bool misaligned = (ring_base & 1023u) != 0;
  if (misaligned && threadIdx.x == 0) raise_status(a.status, 4 /* BI_ERR_CUDA */);
  const int64_t rows = misaligned ? 0 : *a.d_rows;
  const int mtiles = static_cast<int>((rows + 127) / 128);
  const int nunits = misaligned ? 0 : ((kMode == kModeDH) ? mtiles : a.nvt128);
  const int steps = (kMode == kModeDH) ? a.nvt128 : mtiles;
  const int my_units =
      (static_cast<int>(cl) < nunits) ? (nunits - static_cast<int>(cl) + static_cast<int>(ncl) - 1) / static_cast<int>(ncl) : 0;
  const int64_t total = static_cast<int64_t>(my_units) * steps;
  const int KB = a.H / 64;
  const int slice0 = static_cast<int>(rank) * a.Hs;

  if (warp == 0) {
    // ---------------- TMA producer (whole warp; one elected lane issues) ----------------
    if (elect_one()) {
      tma_prefetch_desc(&tm_stat);
      tma_prefetch_desc(&tm_stream);
      tma_prefetch_desc(&tm_dz);
    }
    uint32_t slot = 0, phase = 0;
    auto acquire = [&](uint32_t bytes) -> bool {
      if (!wait(&sh.empty[slot], phase ^ 1u, false)) return false;
      if (elect_one()) mbar_arrive_expect_tx(&sh.full[slot], bytes);
      return true;
    };
    auto advance = [&]() {
      if (++slot == kSlots) { slot = 0; phase ^= 1u; }
    };
    auto ztile = [&](const StreamPos& p) -> bool {
      const int ustat = (static_cast<int>(cl) + p.u_idx * static_cast<int>(ncl)) * 128;
      const int ystr = p.j * 128;
      for (int kb = 0; kb < KB; ++kb) {
        if (!acquire(kSlotBytes)) return false;
        if (elect_one()) {
          const uint32_t dst = ring_base + slot * kSlotBytes;
          tma_load_2d(dst, &tm_stat, &sh.full[slot], kb * 64, ustat);
          tma_load_2d(dst + kUnitBytes, &tm_stream, &sh.full[slot], kb * 64, ystr);
        }
        advance();
      }
      return true;
    };
    auto ostep = [&](const StreamPos& p) -> bool {
      if (!wait(&sh.dz_ready[p.slot], p.round & 1u, true)) return false;
      if (!acquire(kSlotBytes)) return false;
      if (elect_one()) {
        const int dz_row = static_cast<int>((cl * nslot + p.slot) * 128);
        const uint32_t dst = ring_base + slot * kSlotBytes;
        tma_load_2d(dst, &tm_dz, &sh.full[slot], 0, dz_row);
        tma_load_2d(dst + kUnitBytes, &tm_dz, &sh.full[slot], 64, dz_row);
      }
      advance();
      int col = slice0;
      for (int ch = 0; ch < a.nchunk; ++ch) {
        const int nu = a.chunk_units[ch];
        if (!acquire(nu * kUnitBytes)) return false;
        if (elect_one()) {
          const uint32_t dst = ring_base + slot * kSlotBytes;
          tma_load_2d(dst, &tm_stream, &sh.full[slot], col, p.j * 128);
          if (nu == 2) tma_load_2d(dst + kUnitBytes, &tm_stream, &sh.full[slot], col + 64, p.j * 128);
        }
        advance();
        col += 64 * nu;
      }
      return true;
    };
    StreamPos p, pz;  // p: step whose slice update is loaded; pz: step whose logit tile is loaded (p + C)
    p.zero();
    pz.zero();
    bool ok = true;
    for (uint32_t i = 0; ok && i < C && pz.s < total; ++i) {
      if (pz.modc == rank) ok = ztile(pz);
      pz.next(steps, C, nslot);
    }
    for (; ok && p.s < total; p.next(steps, C, nslot)) {
      if (pz.s < total) {
        if (pz.modc == rank) ok = ztile(pz);
        pz.next(steps, C, nslot);
      }
      if (ok) ok = ostep(p);
    }
    // loads still in flight must land before the CTA may exit: the last fill of each slot
    if (elect_one()) {
      for (uint32_t i = 0; i < static_cast<uint32_t>(kSlots); ++i) {
        const uint32_t ph = (i < slot) ? phase : (phase ^ 1u);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_test(&sh.full[i], ph))
          if (globaltimer_ns() - t0 > a.limit_ns) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    constexpr uint32_t idesc_z = idesc_bf16(128, 128, false, false);
    constexpr uint32_t idesc_o2 = idesc_bf16(128, 128, false, true);
    constexpr uint32_t idesc_o1 = idesc_bf16(128, 64, false, true);
    // descriptors of slot 0 (K-major and MN-major forms); slot i adds i * kSlotBytes >> 4
    const uint64_t dk0 = sdesc_k_sw128(ring_base);
    const uint64_t dm0 = sdesc_mn_sw128(ring_base, kUnitBytes);
    uint32_t slot = 0, phase = 0, zc = 0, oc = 0;
    auto take = [&]() -> bool {
      if (!wait(&sh.full[slot], phase, false)) return false;
      tc_fence_after();
      return true;
    };
    auto advance = [&]() {
      if (++slot == kSlots) { slot = 0; phase ^= 1u; }
    };
    auto ztile = [&]() -> bool {
      if (!wait(&sh.z_empty, (zc & 1u) ^ 1u, false)) return false;
      tc_fence_after();
      for (int kb = 0; kb < KB; ++kb) {
        if (!take()) return false;
        if (elect_one()) {
          const uint64_t da = dk0 + static_cast<uint64_t>(slot * (kSlotBytes >> 4));
          const uint64_t db = da + (kUnitBytes >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_bf16(tmem + kZCol, da + 2 * k, db + 2 * k, idesc_z, (kb | k) != 0);
          umma_commit(&sh.empty[slot]);
        }
        advance();
      }
      if (elect_one()) umma_commit(&sh.z_full);
      ++zc;
      return true;
    };
    auto ostep = [&](const StreamPos& p) -> bool {
      if (p.j == 0) {
        if (!wait(&sh.o_empty, (oc & 1u) ^ 1u, false)) return false;
        tc_fence_after();
      }
      if (!take()) return false;
      const uint32_t dslot = slot;
      if (elect_one())  // the tile is in shared memory now: its scratch slot may be refilled
        mbar_arrive_cluster(mapa_shared(smem_u32(&sh.dz_free[p.slot]), p.modc));
      advance();
      const uint64_t da = dk0 + static_cast<uint64_t>(dslot * (kSlotBytes >> 4));
      uint32_t col = 0;
      for (int ch = 0; ch < a.nchunk; ++ch) {
        const int nu = a.chunk_units[ch];
        if (!take()) return false;
        if (elect_one()) {
          const uint64_t db = dm0 + static_cast<uint64_t>(slot * (kSlotBytes >> 4));
          const uint32_t idesc = (nu == 2) ? idesc_o2 : idesc_o1;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // A: dZ tile, K = 128 in two 64-wide units; B: slice tile, MN-major, 16 K-rows = 2 KB per step
            const uint64_t ak = da + ((kk < 4) ? 0 : (kUnitBytes >> 4)) + 2 * (kk & 3);
            umma_bf16(tmem + col, ak, db + (2048 >> 4) * kk, idesc, (p.j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&sh.empty[slot]);
        }
        advance();
        col += 64 * nu;
      }
      if (elect_one()) {
        umma_commit(&sh.empty[dslot]);
        if (p.j == steps - 1) umma_commit(&sh.o_full);
      }
      if (p.j == steps - 1) ++oc;
      return true;
    };
    StreamPos p, pz;
    p.zero();
    pz.zero();
    bool ok = true;
    for (uint32_t i = 0; ok && i < C && pz.s < total; ++i) {
      if (pz.modc == rank) ok = ztile();
      pz.next(steps, C, nslot);
    }
    for (; ok && p.s < total; p.next(steps, C, nslot)) {
      if (pz.s < total) {
        if (pz.modc == rank) ok = ztile();
        pz.next(steps, C, nslot);
      }
      if (ok) ok = ostep(p);
    }
    if (elect_one()) {
      umma_commit(&sh.mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_test(&sh.mma_done, 0))
        if (globaltimer_ns() - t0 > a.limit_ns) break;
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: 4 warps, one accumulator lane (row) per thread ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..127
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t zc = 0, oc = 0, epc = 0;
    bool ok = true;
    auto ep_sync = [&]() {
      mbar_arrive(&sh.ep_bar);
      return wait(&sh.ep_bar, (epc++) & 1u, false);
    };
    float r_lse2 = 0.f, r_g = 0.f;
    int32_t r_y = -1;
    bool r_valid = false;

    auto drain = [&](int u, bool have_acc) {
      if (have_acc) {
        if (!wait(&sh.o_full, oc & 1u, false)) return false;
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
    StreamPos p;
    p.zero();
    for (; ok && p.s < total; p.next(steps, C, nslot)) {
      const int u = static_cast<int>(cl) + p.u_idx * static_cast<int>(ncl);
      if (kMode == kModeDH && p.j == 0) {
        const int64_t t = static_cast<int64_t>(u) * 128 + row;
        r_valid = t < rows;
        r_lse2 = r_valid ? a.lse[t] * kLog2e : 0.f;
        r_g = r_valid ? a.g[t] : 0.f;
        r_y = r_valid ? a.y[t] : -1;
      }
      if (p.modc == rank) {
        if (kMode == kModeDW) {
          if (!ep_sync()) { ok = false; break; }  // previous step's column parameters are no longer read
          const int64_t t = static_cast<int64_t>(p.j) * 128 + et;
          const bool tv = t < rows;
          sh.col_lse2[et] = tv ? a.lse[t] * kLog2e : 0.f;
          sh.col_g[et] = tv ? a.g[t] : 0.f;
          sh.col_y[et] = tv ? a.y[t] : INT32_MIN;
          if (!ep_sync()) { ok = false; break; }
        }
        if (!wait(&sh.z_full, zc & 1u, false)) { ok = false; break; }
        tc_fence_after();
        if (p.round > 0) {
          if (!wait(&sh.dz_free[p.slot], (p.round - 1) & 1u, true)) { ok = false; break; }
        }
        uint16_t* dzrow = a.dz_scratch + (static_cast<int64_t>(cl * nslot + p.slot) * 128 + row) * 128;
        const int64_t vrow = static_cast<int64_t>(u) * 128 + row;  // kModeDW: this lane's vocabulary row
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(tl + kZCol + c * 32, v);
          tmem_ld_wait();
          float d[32];
          if (kMode == kModeDH) {
            const int vbase = p.j * 128 + c * 32;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float pr = ex2_approx(fmaf(__uint_as_float(v[q]), kLog2e, -r_lse2));
              const float oh = (vbase + q == r_y) ? 1.f : 0.f;
              d[q] = (r_valid && vbase + q < a.V) ? r_g * (oh - pr) : 0.f;
            }
          } else {
            const bool v_ok = vrow < a.V;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int tc = c * 32 + q;
              const float pr = ex2_approx(fmaf(__uint_as_float(v[q]), kLog2e, -sh.col_lse2[tc]));
              const int32_t yc = sh.col_y[tc];
              const float oh = (static_cast<int64_t>(yc) == vrow) ? 1.f : 0.f;
              d[q] = (v_ok && yc != INT32_MIN) ? sh.col_g[tc] * (oh - pr) : 0.f;
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
          const uint32_t la = smem_u32(&sh.dz_ready[p.slot]);
          for (uint32_t q = 0; q < C; ++q) mbar_arrive_cluster(mapa_shared(la, q));
        }
      }
      if (p.j == steps - 1) {
        if (!drain(u, true)) { ok = false; break; }
      }
    }
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
