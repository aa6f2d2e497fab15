// kernels_bwd.cuh -- backward of the IS loss through the LM head, with the logits recomputed on
// chip and never stored:
//     dZ_tv = g_t (1[v = y_t] - exp(z_tv - lse_t)),   g_t = -c_i w_t
//     dH = dZ W          (mode kModeDH: a cluster owns a 128-row tile of hidden states and
//                         sweeps the vocabulary; reduction over v in ascending tile order)
//     dW = dZ^T H        (mode kModeDW: a cluster owns a 128-row tile of the vocabulary and
//                         sweeps the rows; reduction over t in ascending tile order)
//
// The [128 x H] fp32 accumulator does not fit one SM's tensor memory, so the H columns are split
// over a cluster of C CTAs (Hs = H / C columns each).  Each step streams NZ rows of the other
// operand (NZ = 256 when Hs <= 256).  The 128 x NZ logit tile of a step is computed once, by one
// CTA of the cluster in rotation (full K = H), turned into a bf16 dZ tile by its epilogue and
// published through a small L2-resident scratch slot; every CTA of the cluster then TMA-loads it
// as the A operand of its own slice update O[:, Hs] += dZ[128 x NZ] * S[NZ x Hs].  Cross-CTA
// hand-off uses mbarriers in each CTA's shared memory, signalled through the cluster's
// shared-memory window.  Tile shape, K order and the order of the reduction are fixed and do not
// depend on T, so each row of dH has the same bits in any batch (the "Zero Mismatch" post,
// "Alignment permits a simpler learning path": bit-identical rows for the same weights and
// tokens).
//
// Issue rate: one lane issues every tcgen05.mma, and a barrier wait costs it ~80 cycles, so each
// pipeline stage carries 4 MMAs of N = 256 (512 tensor cycles) per wait: the logit phase and the
// slice-update phase use the same stage shape (A: 128 x 64, B: 64 x 256), one commit per stage.
#pragma once

#include "sm100.cuh"

namespace bi {

constexpr int kAUnitBytes = 16384;  // [128 rows][64 bf16], 128B-swizzled
constexpr int kSlUnitBytes = 8192;  // [64 rows][64 bf16] MN-major slice unit
constexpr int kMaxStages = 4;
constexpr int kBwdThreads = 192;
constexpr int kSlotsPerCta = 2;     // dZ scratch slots per producer CTA
constexpr int kMaxCluster = 8;
constexpr int kMaxSlots = kMaxCluster * kSlotsPerCta;
constexpr int kMaxNZ = 256;

enum BwdMode : int { kModeDH = 0, kModeDW = 1 };

// Column splits compiled in (Hs = columns per CTA, NZ = logit-tile width): the tiling of every
// H that has a split with Hs a multiple of 64, Hs <= 384 and C <= 8.
#define BI_BWD_CONFIGS(X) X(256, 64) X(256, 128) X(256, 192) X(256, 256) X(192, 320) X(128, 384)

struct BwdArgs {
  int32_t H, V;
  int32_t C;             // CTAs per cluster
  int32_t Hs;            // H / C: columns owned by each CTA (multiple of 64, <= 384)
  int32_t NZ;            // streamed rows per step (multiple of 64, <= 256, Hs + NZ <= 512)
  int64_t T;             // rows of the compact hidden-state tensor maps (upper bound)
  const int64_t* d_rows; // number of valid compact rows (device)
  int32_t nvz;           // ceil(V / NZ): vocabulary steps (kModeDH)
  int32_t nv128;         // ceil(V / 128): vocabulary units (kModeDW)
  const float* lse;      // [rows] compact
  const float* g;        // [rows] compact: -c_i w_t (0 for rows without gradient)
  const int32_t* y;      // [rows] compact targets
  const int32_t* rowmap; // [rows] compact row -> output row of grad_hidden
  uint16_t* grad_hidden; // [*, H] bf16 (kModeDH)
  float* grad_w;         // [V, H] fp32 (kModeDW)
  uint16_t* dz_scratch;  // [clusters * C * kSlotsPerCta * 128][NZ] bf16
  int32_t* status;
  uint64_t limit_ns;
};

struct BwdShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t z_full, z_empty, o_full, o_empty, mma_done;
  uint64_t ep_bar;                 // rendezvous of the 128 epilogue threads (bounded, unlike bar.sync)
  uint64_t dz_ready[kMaxSlots];
  uint64_t dz_free[kMaxSlots];
  float col_lse2[kMaxNZ];          // kModeDW: per-column lse * log2(e)
  float col_g[kMaxNZ];             // kModeDW: per-column g
  int32_t col_y[kMaxNZ];           // kModeDW: per-column target (INT32_MIN: column not valid)
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

constexpr int kBwdSharedBytes = static_cast<int>((sizeof(BwdShared) + 127) / 128 * 128);
constexpr int kBwdSmemLimit = 232448;  // per-block opt-in shared memory on sm_100

// Stage geometry of one compiled tiling: a stage holds one A unit (128 x 64) and the larger of
// the logit-phase B tile (NZ x 64) and the slice tile (64 x Hs).
template <int kNZ, int kHS>
struct BwdTile {
  static constexpr int stage_bytes = ((kAUnitBytes + (kNZ > kHS ? kNZ : kHS) * 128) + 1023) / 1024 * 1024;
  static constexpr int fit = (kBwdSmemLimit - kBwdSharedBytes) / stage_bytes;
  static constexpr int nstages = fit < kMaxStages ? fit : kMaxStages;
  static constexpr int smem = nstages * stage_bytes + kBwdSharedBytes;
  static_assert(nstages >= 2, "pipeline needs at least two stages");
  static_assert(kHS % 64 == 0 && kNZ % 64 == 0 && kHS + kNZ <= 512, "tile does not fit tensor memory");
};

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

// Everything one CTA of the cluster needs to know about its place in the work.
struct BwdCtx {
  uint32_t C, rank, cl, ncl, nslot;
  int64_t rows, total;
  int steps, nunits, KB, slice0;
  uint32_t ring_base;
};

// Bounded wait (single thread or per-thread).  On a timeout this CTA and its peers are told to stop.
template <bool kClusterAcq>
__device__ __forceinline__ bool bwd_wait(BwdShared& sh, const BwdArgs& a, uint32_t C, uint64_t* bar, uint32_t parity) {
  const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};
  const bool ok = mbar_wait<kClusterAcq>(bar, parity, wc);
  if (!ok) {
    const uint32_t la = smem_u32(const_cast<uint32_t*>(&sh.abort_flag));
    for (uint32_t q = 0; q < C; ++q) st_cluster_u32(mapa_shared(la, q), 1u);
  }
  return ok;
}

__device__ __forceinline__ void ring_advance(uint32_t& stage, uint32_t& phase, uint32_t nstages) {
  if (++stage == nstages) {
    stage = 0;
    phase ^= 1u;
  }
}

// ---------------- TMA producer (one thread) ----------------
struct TmaMaps {
  const CUtensorMap* stat;   // stationary operand, box {64, 128}
  const CUtensorMap* zb;     // streamed operand, box {64, NZ}  (logit phase B)
  const CUtensorMap* sl;     // streamed operand, box {64, 64}  (slice units)
  const CUtensorMap* dz;     // dZ scratch, box {64, 128}
};

template <int kNZ, int kHS>
__device__ __forceinline__ void bwd_tma_role(BwdShared& sh, const BwdArgs& a, const BwdCtx& x, const TmaMaps& m) {
  tma_prefetch_desc(m.stat);
  tma_prefetch_desc(m.zb);
  tma_prefetch_desc(m.sl);
  tma_prefetch_desc(m.dz);
  constexpr uint32_t nst = static_cast<uint32_t>(BwdTile<kNZ, kHS>::nstages);
  constexpr uint32_t sbytes = static_cast<uint32_t>(BwdTile<kNZ, kHS>::stage_bytes);
  constexpr uint32_t zbytes = kAUnitBytes + kNZ * 128;
  constexpr uint32_t obytes = kAUnitBytes + kHS * 128;
  constexpr int nsl = kHS / 64;
  constexpr int nkc = kNZ / 64;
  uint32_t stage = 0, phase = 0;

  StreamPos p, pz;  // p: step whose slice update is loaded; pz: step whose logit tile is loaded (p + C)
  p.zero();
  pz.zero();
  bool ok = true;
  const int64_t pro = static_cast<int64_t>(x.C) < x.total ? static_cast<int64_t>(x.C) : x.total;
  for (int64_t it = -pro; ok && it < x.total; ++it) {
    // the logit tile C steps ahead (the first C up front), then the slice update of step p
    if (pz.s < x.total) {
      if (pz.modc == x.rank) {
        const int ustat = (static_cast<int>(x.cl) + pz.u_idx * static_cast<int>(x.ncl)) * 128;
        const int ystr = pz.j * kNZ;
#pragma unroll 1
        for (int kb = 0; kb < x.KB; ++kb) {
          if (!bwd_wait<false>(sh, a, x.C, &sh.empty[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&sh.full[stage], zbytes);
          const uint32_t dst = x.ring_base + stage * sbytes;
          tma_load_2d(dst, m.stat, &sh.full[stage], kb * 64, ustat);
          tma_load_2d(dst + kAUnitBytes, m.zb, &sh.full[stage], kb * 64, ystr);
          ring_advance(stage, phase, nst);
        }
        if (!ok) break;
      }
      pz.next(x.steps, x.C, x.nslot);
    }
    if (it < 0) continue;
    // slice tiles of this CTA do not depend on the dZ tile: they are requested first, the dZ
    // chunks once the producer has published the tile
    const int dz_row = static_cast<int>((x.cl * x.nslot + p.slot) * 128);
    bool dz_ok = false;
#pragma unroll 1
    for (int kc = 0; kc < nkc; ++kc) {
      if (!bwd_wait<false>(sh, a, x.C, &sh.empty[stage], phase ^ 1u)) { ok = false; break; }
      mbar_arrive_expect_tx(&sh.full[stage], obytes);
      const uint32_t dst = x.ring_base + stage * sbytes;
      const int yrow = p.j * kNZ + kc * 64;
#pragma unroll
      for (int u = 0; u < nsl; ++u)
        tma_load_2d(dst + kAUnitBytes + u * kSlUnitBytes, m.sl, &sh.full[stage], x.slice0 + u * 64, yrow);
      if (!dz_ok) {
        if (!bwd_wait<true>(sh, a, x.C, &sh.dz_ready[p.slot], p.round & 1u)) { ok = false; break; }
        dz_ok = true;
      }
      tma_load_2d(dst, m.dz, &sh.full[stage], kc * 64, dz_row);
      ring_advance(stage, phase, nst);
    }
    if (!ok) break;
    p.next(x.steps, x.C, x.nslot);
  }
  // loads still in flight must land before the CTA may exit: the last fill of each stage
  for (uint32_t i = 0; i < nst; ++i) {
    const uint32_t ph = (i < stage) ? phase : (phase ^ 1u);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_test(&sh.full[i], ph))
      if (globaltimer_ns() - t0 > a.limit_ns) break;
  }
}

// ---------------- MMA issuer (one thread) ----------------
template <int kNZ, int kHS>
__device__ __forceinline__ void bwd_mma_role(BwdShared& sh, const BwdArgs& a, const BwdCtx& x, uint32_t tmem) {
  constexpr uint32_t nst = static_cast<uint32_t>(BwdTile<kNZ, kHS>::nstages);
  constexpr uint32_t idesc_z = idesc_bf16(128, kNZ, false, false);
  constexpr int n1 = kHS < 256 ? kHS : 256;  // slice update: one MMA of n1 columns, one of n2
  constexpr int n2 = kHS - n1;
  constexpr uint32_t idesc_o1 = idesc_bf16(128, n1, false, true);
  constexpr uint32_t idesc_o2 = idesc_bf16(128, n2 > 0 ? n2 : 64, false, true);
  constexpr uint32_t zcol = 512u - static_cast<uint32_t>(kNZ);
  constexpr int nkc = kNZ / 64;
  constexpr uint64_t sb_desc = static_cast<uint64_t>(BwdTile<kNZ, kHS>::stage_bytes >> 4);
  const uint64_t dk0 = sdesc_k_sw128(x.ring_base);                                // A operands
  const uint64_t dkb0 = sdesc_k_sw128(x.ring_base + kAUnitBytes);                 // logit-phase B
  const uint64_t dmb0 = sdesc_mn_sw128(x.ring_base + kAUnitBytes, kSlUnitBytes);  // slice B
  uint32_t stage = 0, phase = 0, zc = 0, oc = 0;

  StreamPos p, pz;
  p.zero();
  pz.zero();
  bool ok = true;
  const int64_t pro = static_cast<int64_t>(x.C) < x.total ? static_cast<int64_t>(x.C) : x.total;
  for (int64_t it = -pro; ok && it < x.total; ++it) {
    if (pz.s < x.total) {
      if (pz.modc == x.rank) {
        // logit tile z = A_stat[128 x H] * B_stream[NZ x H]^T into TMEM columns [512 - NZ, 512)
        if (!bwd_wait<false>(sh, a, x.C, &sh.z_empty, (zc & 1u) ^ 1u)) break;
        tc_fence_after();
#pragma unroll 1
        for (int kb = 0; kb < x.KB; ++kb) {
          if (!bwd_wait<false>(sh, a, x.C, &sh.full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = dk0 + stage * sb_desc;
          const uint64_t db = dkb0 + stage * sb_desc;
          umma_bf16(tmem + zcol, da, db, idesc_z, kb != 0 ? 1u : 0u);
          umma_bf16(tmem + zcol, da + 2, db + 2, idesc_z, 1u);
          umma_bf16(tmem + zcol, da + 4, db + 4, idesc_z, 1u);
          umma_bf16(tmem + zcol, da + 6, db + 6, idesc_z, 1u);
          umma_commit(&sh.empty[stage]);
          ring_advance(stage, phase, nst);
        }
        if (!ok) break;
        umma_commit(&sh.z_full);
        ++zc;
      }
      pz.next(x.steps, x.C, x.nslot);
    }
    if (it < 0) continue;
    // slice update of step p: O[:, 0:Hs] += dZ[128 x NZ] * S[NZ x Hs], K in chunks of 64
    if (p.j == 0) {
      if (!bwd_wait<false>(sh, a, x.C, &sh.o_empty, (oc & 1u) ^ 1u)) break;
      tc_fence_after();
    }
#pragma unroll 1
    for (int kc = 0; kc < nkc; ++kc) {
      if (!bwd_wait<false>(sh, a, x.C, &sh.full[stage], phase)) { ok = false; break; }
      tc_fence_after();
      // every chunk of the dZ tile has landed in shared memory (the full barrier completed): the
      // producer may refill its scratch slot.  Nothing this thread wrote needs ordering, so the
      // signal is relaxed (a release here stalls the issuing lane for ~0.4 us).
      if (kc == nkc - 1) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&sh.dz_free[p.slot]), p.modc));
      const uint64_t da = dk0 + stage * sb_desc;
      const uint64_t db = dmb0 + stage * sb_desc;
      const uint32_t acc0 = (p.j > 0 || kc > 0) ? 1u : 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // A: 16 K-columns = 32 bytes along the swizzled row; B: 16 K-rows = 2 KB of MN-major rows
        umma_bf16(tmem, da + 2 * k, db + (2048 >> 4) * k, idesc_o1, k == 0 ? acc0 : 1u);
        if constexpr (n2 > 0)
          umma_bf16(tmem + n1, da + 2 * k, db + (2048 >> 4) * k + ((4 * kSlUnitBytes) >> 4), idesc_o2,
                    k == 0 ? acc0 : 1u);
      }
      umma_commit(&sh.empty[stage]);
      ring_advance(stage, phase, nst);
    }
    if (!ok) break;
    if (p.j == x.steps - 1) {
      umma_commit(&sh.o_full);
      ++oc;
    }
    p.next(x.steps, x.C, x.nslot);
  }
  umma_commit(&sh.mma_done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(&sh.mma_done, 0))
    if (globaltimer_ns() - t0 > a.limit_ns) break;
}

// ---------------- epilogue: 4 warps, one accumulator lane (row) per thread ----------------
// All 128 threads take the same path; waits are made warp-uniform because tcgen05.ld is .aligned.
template <bool kClusterAcq>
__device__ __forceinline__ bool ep_wait(BwdShared& sh, const BwdArgs& a, uint32_t C, uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, bwd_wait<kClusterAcq>(sh, a, C, bar, parity)) != 0;
}

template <int kMode, int kNZ, int kHS>
__device__ __forceinline__ bool bwd_drain(BwdShared& sh, const BwdArgs& a, const BwdCtx& x, uint32_t tl, int row, int u,
                                          bool have_acc, uint32_t& oc) {
  if (have_acc) {
    if (!ep_wait<false>(sh, a, x.C, &sh.o_full, oc & 1u)) return false;
    tc_fence_after();
  }
  if (kMode == kModeDH) {
    const int64_t t = static_cast<int64_t>(u) * 128 + row;
    const bool v_ok = t < x.rows;
    uint16_t* dst = v_ok ? a.grad_hidden + static_cast<int64_t>(a.rowmap[t]) * a.H + x.slice0 : nullptr;
#pragma unroll 1
    for (int c = 0; c < kHS / 32; ++c) {
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
    float* dst = v_ok ? a.grad_w + vr * a.H + x.slice0 : nullptr;
#pragma unroll 1
    for (int c = 0; c < kHS / 32; ++c) {
      if (have_acc) {
        uint32_t v[32];
        tmem_ld32(tl + c * 32, v);
        tmem_ld_wait();
        if (v_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) d4[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      } else if (v_ok) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) d4[q] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  if (have_acc) {
    tc_fence_before();
    mbar_arrive(&sh.o_empty);
    ++oc;
  }
  return true;
}

template <int kMode, int kNZ, int kHS>
__device__ __forceinline__ void bwd_epilogue_role(BwdShared& sh, const BwdArgs& a, const BwdCtx& x, uint32_t tmem) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const int et = threadIdx.x - 64;  // 0..127
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  constexpr uint32_t zcol = 512u - static_cast<uint32_t>(kNZ);
  uint32_t zc = 0, oc = 0, epc = 0;
  float r_lse2 = 0.f, r_g = 0.f;
  int32_t r_y = -1;
  bool r_valid = false;

  if (kMode == kModeDW && x.steps == 0) {
    // no rows: every owned vocabulary tile gets a zero gradient
    for (int u = static_cast<int>(x.cl); u < x.nunits; u += static_cast<int>(x.ncl))
      bwd_drain<kMode, kNZ, kHS>(sh, a, x, tl, row, u, false, oc);
  }
  StreamPos p;
  p.zero();
  for (; p.s < x.total; p.next(x.steps, x.C, x.nslot)) {
    const int u = static_cast<int>(x.cl) + p.u_idx * static_cast<int>(x.ncl);
    if (kMode == kModeDH && p.j == 0) {
      const int64_t t = static_cast<int64_t>(u) * 128 + row;
      r_valid = t < x.rows;
      r_lse2 = r_valid ? a.lse[t] * kLog2e : 0.f;
      r_g = r_valid ? a.g[t] : 0.f;
      r_y = r_valid ? a.y[t] : -1;
    }
    if (p.modc == x.rank) {
      if (kMode == kModeDW) {
        // the previous step's column parameters are no longer read; stage this step's
        mbar_arrive(&sh.ep_bar);
        if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) break;
        for (int cc = et; cc < kNZ; cc += 128) {
          const int64_t t = static_cast<int64_t>(p.j) * kNZ + cc;
          const bool tv = t < x.rows;
          sh.col_lse2[cc] = tv ? a.lse[t] * kLog2e : 0.f;
          sh.col_g[cc] = tv ? a.g[t] : 0.f;
          sh.col_y[cc] = tv ? a.y[t] : INT32_MIN;
        }
        mbar_arrive(&sh.ep_bar);
        if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) break;
      }
      if (!ep_wait<false>(sh, a, x.C, &sh.z_full, zc & 1u)) break;
      tc_fence_after();
      if (p.round > 0) {
        if (!ep_wait<true>(sh, a, x.C, &sh.dz_free[p.slot], (p.round - 1) & 1u)) break;
      }
      uint16_t* dzrow = a.dz_scratch + (static_cast<int64_t>(x.cl * x.nslot + p.slot) * 128 + row) * kNZ;
      const int64_t vrow = static_cast<int64_t>(u) * 128 + row;  // kModeDW: this lane's vocabulary row
#pragma unroll 1
      for (int c = 0; c < kNZ / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tl + zcol + c * 32, v);
        tmem_ld_wait();
        float d[32];
        if (kMode == kModeDH) {
          const int vbase = p.j * kNZ + c * 32;
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
      mbar_arrive(&sh.ep_bar);
      if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) break;
      if (et == 0) {
        const uint32_t la = smem_u32(&sh.dz_ready[p.slot]);
        for (uint32_t q = 0; q < x.C; ++q) mbar_arrive_cluster(mapa_shared(la, q));
      }
    }
    if (p.j == x.steps - 1) {
      if (!bwd_drain<kMode, kNZ, kHS>(sh, a, x, tl, row, u, true, oc)) break;
    }
  }
}

template <int kMode, int kNZ, int kHS>
__global__ void __launch_bounds__(kBwdThreads, 1)
    k_bwd_cluster(const __grid_constant__ CUtensorMap tm_stat, const __grid_constant__ CUtensorMap tm_zb,
                  const __grid_constant__ CUtensorMap tm_sl, const __grid_constant__ CUtensorMap tm_dz, BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  BwdShared& sh = *reinterpret_cast<BwdShared*>(dsmem + BwdTile<kNZ, kHS>::nstages * BwdTile<kNZ, kHS>::stage_bytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  BwdCtx x;
  x.C = static_cast<uint32_t>(a.C);
  x.rank = cluster_ctarank();
  x.cl = cluster_id_x();
  x.ncl = ncluster_x();
  x.nslot = x.C * kSlotsPerCta;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    mbar_init(&sh.z_full, 1);
    mbar_init(&sh.z_empty, 128);
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.o_empty, 128);
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.ep_bar, 128);
    for (uint32_t i = 0; i < x.nslot; ++i) {
      mbar_init(&sh.dz_ready[i], 1);
      mbar_init(&sh.dz_free[i], x.C);
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

  x.ring_base = smem_u32(dsmem);
  // the 128B-swizzled tiles need 1024-byte aligned stages; refuse to run otherwise
  const bool misaligned = (x.ring_base & 1023u) != 0;
  if (misaligned && threadIdx.x == 0) raise_status(a.status, 4 /* BI_ERR_CUDA */);
  x.rows = misaligned ? 0 : *a.d_rows;
  const int mtiles = static_cast<int>((x.rows + 127) / 128);
  x.nunits = misaligned ? 0 : ((kMode == kModeDH) ? mtiles : a.nv128);
  x.steps = (kMode == kModeDH) ? a.nvz : static_cast<int>((x.rows + kNZ - 1) / kNZ);
  const int my_units = (static_cast<int>(x.cl) < x.nunits)
                           ? (x.nunits - static_cast<int>(x.cl) + static_cast<int>(x.ncl) - 1) / static_cast<int>(x.ncl)
                           : 0;
  x.total = static_cast<int64_t>(my_units) * x.steps;
  x.KB = a.H / 64;
  x.slice0 = static_cast<int>(x.rank) * a.Hs;

  if (warp == 0) {
    if (lane == 0) {
      const TmaMaps m{&tm_stat, &tm_zb, &tm_sl, &tm_dz};
      bwd_tma_role<kNZ, kHS>(sh, a, x, m);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) bwd_mma_role<kNZ, kHS>(sh, a, x, tmem);
    __syncwarp();
  } else {
    bwd_epilogue_role<kMode, kNZ, kHS>(sh, a, x, tmem);
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
