// kernels_lm.cuh -- the LM-head kernels: one cluster kernel template with three modes.
//
//   kModeFwd    token log-probabilities: z = h W^T tile by tile, a running reference maximum and
//               sum of exp per row, the target logit from its tile.  Logits exist only in TMEM.
//   kModeFwdDH  the same forward fused with dH.  With p = softmax(z_t), g_t = -c_i w_t and the
//               target column y = y_t left out of the sums,
//                   dL/dh_t = g_t sum_{v != y} p_v (W_y - W_v) = (g_t / s) (s' W_y - O'),
//               s' = sum_{v != y} e^{z_v - m}, s = s' + e^{z_y - m}, O' = sum_{v != y} e^{z_v - m} W_v
//               for a per-row reference m.  O' is accumulated on the tensor cores while the
//               vocabulary is swept (online rescaling whenever m moves).  Keeping the target out
//               of O' keeps dH accurate when p_y is close to 1 (no W_y - p_y W_y cancellation).
//   kModeDW     dW = dZ^T H with dZ_tv = g_t (1[v = y_t] - exp(z_tv - lse_t)) recomputed on chip.
//
// Sources: "Zero Mismatch, Simple Async RL", sections "Only one probability gap comes from old
// weights" (token logprob, unclipped IS weight) and "Alignment permits a simpler learning path"
// (group-mean advantage, token mean per response, mean over responses); "REINFORCE-Zero: kernel
// alignment ...", "Core insight" (a row's logprob must not depend on batch composition or on the
// order of floating-point operations chosen per call).
//
// Work split.  A cluster owns 128-row tiles ("units") of the stationary operand (hidden rows in
// the forward modes, vocabulary rows in kModeDW) and sweeps the streamed operand in steps of NZ
// rows.  The [128 x H] fp32 accumulator does not fit one SM's tensor memory, so H is split over
// the C CTAs of the cluster (Hs = H / C columns each).  The 128 x NZ logit tile of step s is
// computed by CTA s mod C with the full K = H; its epilogue turns the tile into a bf16 operand
// (P = e^{z - m} or dZ), publishes it through an L2 scratch slot, and every CTA TMA-loads it as
// the A operand of its own slice update O[:, Hs] += A[128 x NZ] S[NZ x Hs].
//
// Reference chain (forward modes).  The reference of step j of a unit is the running maximum of
// the logits of steps <= j, raised lazily: only when a tile's maximum exceeds the reference by
// more than kTau (so every P <= e^kTau).  The producer of step j receives m_{j-1} from the
// producer of step j-1 by a 128 x 4-byte st.async into its shared memory and passes m_j on.
// Each CTA keeps the sum of exp over its own tiles ("class" k = steps j == k mod C) against its
// latest reference; at the end of the sweep the C partials are combined in class order.
// Every decision is per row and every partition depends only on V and H, so a row's bits do not
// depend on the other rows, on T, or on where the row sits in the batch.
//
// Rescale group (kModeFwdDH only): four extra warps own the O rescale, so the producer
// epilogues never wait on steps of other CTAs and the chain hop is one DSMEM store.
//
// Issue rate: one lane issues every tcgen05.mma; a barrier wait costs it ~80 cycles, so each
// pipeline stage carries four MMAs of K = 16 x N >= 128 (>= 256 tensor cycles) per wait.
#pragma once

#include "sm100.cuh"

namespace bi {

constexpr int kAUnitBytes = 16384;  // [128 rows][64 bf16], 128B-swizzled
constexpr int kSlUnitBytes = 8192;  // [64 rows][64 bf16] MN-major slice unit
constexpr int kMaxStages = 4;
constexpr int kSlotsPerCta = 2;     // scratch slots per producer CTA
constexpr int kMaxCluster = 8;
constexpr int kMaxSlots = kMaxCluster * kSlotsPerCta;
constexpr int kMaxNZ = 256;
constexpr float kTau = 8.0f;        // lazy rescale threshold (natural-log units): P <= e^8
constexpr uint32_t kRsNone = 0xfffffffeu;  // rescale-group request: nothing to do (keep-alive)
constexpr uint32_t kRsStop = 0xffffffffu;  // rescale-group request: leave

enum LmMode : int { kModeFwd = 0, kModeFwdDH = 1, kModeDW = 2 };

template <int kMode>
struct LmThreads {  // TMA warp, MMA warp, 4 epilogue warps (+ 4 rescale warps in kModeFwdDH)
  static constexpr int value = (kMode == kModeFwdDH) ? 320 : 192;
};

// Column splits compiled in (NZ = logit-tile width, Hs = columns per CTA): the tiling of every
// H that has a split with Hs a multiple of 64, Hs <= 384 and C <= 8.
#define BI_LM_CONFIGS(X) X(256, 64) X(256, 128) X(256, 192) X(256, 256) X(192, 320) X(128, 384)

struct LmArgs {
  int32_t H, V;
  int32_t C;               // CTAs per cluster
  int32_t Hs;              // H / C
  int32_t NZ;              // streamed rows per step
  int64_t T;               // rows of the hidden-state tensor maps (upper bound)
  int32_t a_rows;          // rows of the stationary operand's logit-phase box: 0 for 128; fewer (a
                           // multiple of 8) only when one unit holds every row, which the rows
                           // past it then never see: the MMA's rows beyond read stale shared memory
                           // and give logits of rows past T, which nothing reads
  const int64_t* d_rows;   // number of valid rows on the device (nullptr: T)
  int32_t nvz;             // ceil(V / NZ)
  int32_t nv128;           // ceil(V / 128)
  const uint16_t* w_lm;    // [V, H] bf16 (kModeFwdDH reads W_y rows)
  // per (compact) row inputs
  const int32_t* y;        // targets
  const float* logmu;      // rollout log-probabilities (kModeFwdDH)
  const int32_t* respof;   // response of each row (kModeFwdDH)
  const double* coef;      // per-response c_i = A_i / (R* n_i) (kModeFwdDH)
  const int32_t* rowmap;   // compact row -> output row (nullptr: identity)
  // per (compact) row results
  float* lse_c;            // lse (kModeFwdDH writes, kModeDW reads)
  float* g_c;              // -c_i w_t (kModeFwdDH writes, kModeDW reads)
  float* tl_c;             // token loss, for the fixed-order reduction (kModeFwdDH)
  float* d3_c;             // D3 term, for the fixed-order reduction (kModeFwdDH)
  float* delta_c;          // log pi - log mu, for the KL estimators and the sequence gate (kModeFwdDH)
  uint8_t* clip_c;         // 1 where the PPO clip removed the token's gradient (kModeFwdDH)
  int32_t variant;         // loss variant: 0 unclipped, 1 PPO clip, 2 sequence gate (applied after)
  float eps_low, eps_high; // PPO clip range [1 - eps_low, 1 + eps_high]
  // outputs at output rows
  float* logprob;
  float* lse_out;          // nullable
  float* is_weight;        // nullable
  float* token_loss;       // nullable
  uint16_t* grad_hidden;   // [*, H] bf16 (kModeFwdDH)
  float* grad_w;           // [V, H] fp32 (kModeDW)
  // P store (kModeFwdDH, optional): every P tile stays in HBM for the dW kernel
  uint16_t* pbuf;          // [Tpad][p_ld] bf16, row = compact row, column = vocabulary id (nullptr: off)
  int64_t p_ld;            // nvz * NZ
  float* mhist;            // [nvz][Tpad] reference of each row at each step
  int64_t Tpad;            // ceil(T / 128) * 128
  float* sxr_c;            // [rows] s' / s = 1 - p_y (P store only)
  // scratch
  uint16_t* dz_scratch;    // [clusters * C * kSlotsPerCta * 128][NZ] bf16 (P or dZ tiles)
  float* alpha;            // [clusters * C * kSlotsPerCta][128] per-row O rescale factors (kModeFwdDH)
  float* fin;              // [clusters * C * 2][3][128] per-CTA (m, s', z_y) partials (forward modes)
  int32_t* status;
  uint64_t limit_ns;
  uint64_t force_timeout_ns;  // test hook: > 0 makes the epilogue wait on a barrier nobody signals
};

struct LmShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t z_full[2], z_empty[2];
  uint64_t o_full, o_empty, mma_done;
  uint64_t ep_bar;                 // rendezvous of the 128 epilogue threads (bounded, unlike bar.sync)
  uint64_t dz_ready[kMaxSlots];    // producer -> every CTA: the tile of this slot is published
  uint64_t dz_free[kMaxSlots];     // every CTA -> producer: the tile has landed in its shared memory
  uint64_t mref_full;              // previous producer -> this CTA: the reference arrived (tx bytes)
  uint64_t fin_full[2];            // every CTA -> every CTA: unit partials written (by unit parity)
  uint64_t o_drain;                // MMA: every O update issued so far completed
  uint64_t rs_req, rs_done;        // MMA <-> rescale group
  uint64_t never;                  // test hook: nothing arrives here
  uint32_t rflag[kMaxSlots];       // rescale needed at the step of this slot (written by its producer)
  uint32_t wvote[4];               // per-warp rescale votes of this CTA's epilogue
  uint32_t rs_slot;                // slot of the pending rescale request (or kRsNone / kRsStop)
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

// Arrays of one mode only, right after LmShared: the forward modes' reference received from the
// previous producer ([128] fp32), kModeDW's per-column parameters of the streamed rows of a step
// (lse * log2(e), g, target: [NZ] each).  Sized per mode so that the ring keeps every byte the
// other mode's arrays would take (at Hs = 320 that is the difference between 3 and 4 stages).
template <int kMode, int kNZ>
struct LmAux {
  static constexpr int bytes = (kMode == kModeDW) ? kNZ * 12 : 128 * 4;
};

constexpr int kLmSmemLimit = 232448;  // per-block opt-in shared memory on sm_100

// Stage geometry of one compiled tiling: a stage holds one A unit (128 x 64) and the larger of
// the logit-phase B tile (NZ x 64) and the slice tile (64 x Hs); LmShared and the mode's arrays
// follow the ring.
template <int kMode, int kNZ, int kHS>
struct LmTile {
  static constexpr int stage_bytes = ((kAUnitBytes + (kNZ > kHS ? kNZ : kHS) * 128) + 1023) / 1024 * 1024;
  static constexpr int shared_bytes =
      static_cast<int>(((sizeof(LmShared) + 15) / 16 * 16 + static_cast<size_t>(LmAux<kMode, kNZ>::bytes) + 127) / 128 *
                       128);
  static constexpr int fit = (kLmSmemLimit - shared_bytes) / stage_bytes;
  static constexpr int nstages = fit < kMaxStages ? fit : kMaxStages;
  static constexpr int smem = nstages * stage_bytes + shared_bytes;
  static_assert(nstages >= 2, "pipeline needs at least two stages");
  static_assert(kHS % 64 == 0 && kNZ % 64 == 0 && kHS + kNZ <= 512 && kNZ <= 256, "tile does not fit tensor memory");
};

// Tensor-memory columns of the logit tile: two buffers in kModeFwd (no accumulator there), one
// after the Hs accumulator columns otherwise.
template <int kMode, int kNZ>
struct ZBuf {
  static constexpr uint32_t count = (kMode == kModeFwd) ? 2u : 1u;
  __device__ static __forceinline__ uint32_t col(uint32_t b) {
    return (kMode == kModeFwd) ? b * 256u : 512u - static_cast<uint32_t>(kNZ);
  }
  __device__ static __forceinline__ uint32_t buf(uint32_t n) { return count == 2u ? (n & 1u) : 0u; }
  __device__ static __forceinline__ uint32_t parity(uint32_t n) { return count == 2u ? ((n >> 1) & 1u) : (n & 1u); }
};

// Position in a cluster's step stream, advanced without division.
struct StreamPos {
  int64_t s;        // stream index
  int u_idx;        // index of the unit among this cluster's units
  int j;            // step inside the unit
  uint32_t modc;    // s mod C  (the producer CTA of step s)
  uint32_t slot;    // s mod (C * kSlotsPerCta)  (scratch slot)
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
struct LmCtx {
  float* mref;                     // forward modes: [128] reference sent by the previous producer
  float* col_lse2;                 // kModeDW: [NZ] per-column lse * log2(e)
  float* col_g;                    // kModeDW: [NZ] per-column g
  int32_t* col_y;                  // kModeDW: [NZ] per-column target (INT32_MIN: column not valid)
  uint32_t C, rank, cl, ncl, nslot;
  int64_t rows, total;
  int steps, nunits, KB, slice0;
  uint32_t ring_base;
};

// Bounded wait.  On a timeout (or another role's abort) this CTA and its cluster peers stop.
template <bool kClusterAcq>
__device__ __forceinline__ bool lm_wait_for(LmShared& sh, const LmArgs& a, uint32_t C, uint64_t* bar, uint32_t parity,
                                            uint64_t limit_ns) {
  const WaitCtl wc{&sh.abort_flag, a.status, limit_ns};
  const bool ok = mbar_wait<kClusterAcq>(bar, parity, wc);
  if (!ok) {
    const uint32_t la = smem_u32(const_cast<uint32_t*>(&sh.abort_flag));
    for (uint32_t q = 0; q < C; ++q) st_cluster_u32(mapa_shared(la, q), 1u);
  }
  return ok;
}
template <bool kClusterAcq>
__device__ __forceinline__ bool lm_wait(LmShared& sh, const LmArgs& a, uint32_t C, uint64_t* bar, uint32_t parity) {
  return lm_wait_for<kClusterAcq>(sh, a, C, bar, parity, a.limit_ns);
}

// Warp-uniform outcome: tcgen05.ld/st that follow are .sync.aligned.
template <bool kClusterAcq>
__device__ __forceinline__ bool ep_wait(LmShared& sh, const LmArgs& a, uint32_t C, uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, lm_wait<kClusterAcq>(sh, a, C, bar, parity)) != 0;
}

__device__ __forceinline__ void ring_advance(uint32_t& stage, uint32_t& phase, uint32_t nstages) {
  if (++stage == nstages) {
    stage = 0;
    phase ^= 1u;
  }
}

// ---------------- TMA producer (one thread) ----------------
struct TmaMaps {
  const CUtensorMap* stat;  // stationary operand, box {64, 128}
  const CUtensorMap* zb;    // streamed operand, box {64, NZ}  (logit phase B)
  const CUtensorMap* sl;    // streamed operand seen as [cols / 64][rows][64], box {64, 64, Hs / 64}
  const CUtensorMap* dz;    // scratch tiles, box {64, 128}
};

template <int kMode, int kNZ, int kHS>
__device__ __forceinline__ void lm_tma_role(LmShared& sh, const LmArgs& a, const LmCtx& x, const TmaMaps& m) {
  tma_prefetch_desc(m.stat);
  tma_prefetch_desc(m.zb);
  if (kMode != kModeFwd) {
    tma_prefetch_desc(m.sl);
    tma_prefetch_desc(m.dz);
  }
  constexpr uint32_t nst = static_cast<uint32_t>(LmTile<kMode, kNZ, kHS>::nstages);
  constexpr uint32_t sbytes = static_cast<uint32_t>(LmTile<kMode, kNZ, kHS>::stage_bytes);
  const uint32_t zbytes = static_cast<uint32_t>((a.a_rows > 0 ? a.a_rows : 128) * 128 + kNZ * 128);
  constexpr uint32_t obytes = kAUnitBytes + kHS * 128;
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
          if (!lm_wait<false>(sh, a, x.C, &sh.empty[stage], phase ^ 1u)) { ok = false; break; }
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
    if (kMode != kModeFwd) {
      // slice tiles of this CTA do not depend on the published tile: they are requested first,
      // the tile's chunks once the producer has published it
      // the published tile: a scratch slot, or its place in the P store
      const bool stored = (kMode == kModeFwdDH) && a.pbuf != nullptr;
      const int dz_x0 = stored ? p.j * kNZ : 0;
      const int dz_row = stored ? (static_cast<int>(x.cl) + p.u_idx * static_cast<int>(x.ncl)) * 128
                                : static_cast<int>((x.cl * x.nslot + p.slot) * 128);
      bool dz_ok = false;
#pragma unroll 1
      for (int kc = 0; kc < nkc; ++kc) {
        if (!lm_wait<false>(sh, a, x.C, &sh.empty[stage], phase ^ 1u)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh.full[stage], obytes);
        const uint32_t dst = x.ring_base + stage * sbytes;
        const int yrow = p.j * kNZ + kc * 64;
        // the Hs / 64 blocks of this CTA's columns in one load (block-major view of the operand)
        tma_load_3d(dst + kAUnitBytes, m.sl, &sh.full[stage], 0, yrow, x.slice0 / 64);
        if (!dz_ok) {
          if (!lm_wait<true>(sh, a, x.C, &sh.dz_ready[p.slot], p.round & 1u)) { ok = false; break; }
          dz_ok = true;
        }
        tma_load_2d(dst, m.dz, &sh.full[stage], dz_x0 + kc * 64, dz_row);
        ring_advance(stage, phase, nst);
      }
      if (!ok) break;
    }
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
// One request to the rescale group, acknowledged before the issuer goes on.
__device__ __forceinline__ bool rs_handshake(LmShared& sh, const LmArgs& a, uint32_t C, uint32_t slot,
                                             uint32_t& rsc) {
  sh.rs_slot = slot;
  mbar_arrive(&sh.rs_req);  // release: the slot index is visible to the group's acquire
  if (!lm_wait<false>(sh, a, C, &sh.rs_done, rsc & 1u)) return false;
  ++rsc;
  return true;
}

template <int kMode, int kNZ, int kHS>
__device__ __forceinline__ void lm_mma_role(LmShared& sh, const LmArgs& a, const LmCtx& x, uint32_t tmem) {
  using ZB = ZBuf<kMode, kNZ>;
  constexpr uint32_t nst = static_cast<uint32_t>(LmTile<kMode, kNZ, kHS>::nstages);
  constexpr uint32_t idesc_z = idesc_bf16(128, kNZ, false, false);
  constexpr int n1 = kHS < 256 ? kHS : 256;  // slice update: one MMA of n1 columns, one of n2
  constexpr int n2 = kHS - n1;
  constexpr uint32_t idesc_o1 = idesc_bf16(128, n1, false, true);
  constexpr uint32_t idesc_o2 = idesc_bf16(128, n2 > 0 ? n2 : 64, false, true);
  constexpr int nkc = kNZ / 64;
  constexpr uint64_t sb_desc = static_cast<uint64_t>(LmTile<kMode, kNZ, kHS>::stage_bytes >> 4);
  const uint64_t dk0 = sdesc_k_sw128(x.ring_base);                                // A operands
  const uint64_t dkb0 = sdesc_k_sw128(x.ring_base + kAUnitBytes);                 // logit-phase B
  const uint64_t dmb0 = sdesc_mn_sw128(x.ring_base + kAUnitBytes, kSlUnitBytes);  // slice B
  uint32_t stage = 0, phase = 0, zc = 0, oc = 0, odc = 0, rsc = 0;

  StreamPos p, pz;
  p.zero();
  pz.zero();
  bool ok = true;
  const int64_t pro = static_cast<int64_t>(x.C) < x.total ? static_cast<int64_t>(x.C) : x.total;
  for (int64_t it = -pro; ok && it < x.total; ++it) {
    if (pz.s < x.total) {
      if (pz.modc == x.rank) {
        // logit tile z = A_stat[128 x H] * B_stream[NZ x H]^T
        const uint32_t b = ZB::buf(zc);
        const uint32_t zt = tmem + ZB::col(b);
        if (!lm_wait<false>(sh, a, x.C, &sh.z_empty[b], ZB::parity(zc) ^ 1u)) break;
        tc_fence_after();
#pragma unroll 1
        for (int kb = 0; kb < x.KB; ++kb) {
          if (!lm_wait<false>(sh, a, x.C, &sh.full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = dk0 + stage * sb_desc;
          const uint64_t db = dkb0 + stage * sb_desc;
          umma_bf16(zt, da, db, idesc_z, kb != 0 ? 1u : 0u);
          umma_bf16(zt, da + 2, db + 2, idesc_z, 1u);
          umma_bf16(zt, da + 4, db + 4, idesc_z, 1u);
          umma_bf16(zt, da + 6, db + 6, idesc_z, 1u);
          umma_commit(&sh.empty[stage]);
          ring_advance(stage, phase, nst);
        }
        if (!ok) break;
        umma_commit(&sh.z_full[b]);
        ++zc;
      }
      pz.next(x.steps, x.C, x.nslot);
    }
    if (it < 0) continue;
    if (kMode != kModeFwd) {
      // slice update of step p: O[:, 0:Hs] += A[128 x NZ] * S[NZ x Hs], K in chunks of 64
      if (p.j == 0) {
        if (!lm_wait<false>(sh, a, x.C, &sh.o_empty, (oc & 1u) ^ 1u)) break;
        tc_fence_after();
      } else if (kMode == kModeFwdDH) {
        // the producer of this step moved the reference of some row: O is rescaled first
        if (!lm_wait<true>(sh, a, x.C, &sh.dz_ready[p.slot], p.round & 1u)) break;
        if (sh.rflag[p.slot] != 0u) {
          umma_commit(&sh.o_drain);
          if (!lm_wait<false>(sh, a, x.C, &sh.o_drain, odc & 1u)) break;
          ++odc;
          tc_fence_before();
          if (!rs_handshake(sh, a, x.C, p.slot, rsc)) break;
          tc_fence_after();
        }
      }
#pragma unroll 1
      for (int kc = 0; kc < nkc; ++kc) {
        if (!lm_wait<false>(sh, a, x.C, &sh.full[stage], phase)) { ok = false; break; }
        tc_fence_after();
        // every chunk of the published tile has landed in shared memory (the full barrier
        // completed): the producer may refill its scratch slot.  Nothing this thread wrote needs
        // ordering, so the signal is relaxed (a release here stalls the issuing lane ~0.4 us).
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
        // keep-alive for the rescale group, whose waits are bounded: one request per unit
        if (kMode == kModeFwdDH && !rs_handshake(sh, a, x.C, kRsNone, rsc)) break;
      }
    }
    p.next(x.steps, x.C, x.nslot);
  }
  if (kMode == kModeFwdDH) rs_handshake(sh, a, x.C, kRsStop, rsc);
  umma_commit(&sh.mma_done);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(&sh.mma_done, 0))
    if (globaltimer_ns() - t0 > a.limit_ns) break;
}

// ---------------- rescale group (kModeFwdDH, 128 threads) ----------------
template <int kHS>
__device__ __forceinline__ void lm_rescale_role(LmShared& sh, const LmArgs& a, const LmCtx& x, uint32_t tmem) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  uint32_t rsc = 0;
  while (true) {
    if (!ep_wait<false>(sh, a, x.C, &sh.rs_req, rsc & 1u)) break;
    const uint32_t slot = sh.rs_slot;
    if (slot < static_cast<uint32_t>(kMaxSlots)) {
      tc_fence_after();
      const float alpha = __ldcg(a.alpha + static_cast<int64_t>(x.cl * x.nslot + slot) * 128 + row);
#pragma unroll 1
      for (int c = 0; c < kHS / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tl + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * alpha);
        tmem_st32(tl + c * 32, v);
      }
      tmem_st_wait();
      tc_fence_before();
    }
    mbar_arrive(&sh.rs_done);
    ++rsc;
    if (slot == kRsStop) break;
  }
}

// ---------------- epilogue helpers ----------------
// Store one 32-value chunk of bf16 to a 32-byte aligned address as two whole 32-byte sectors
// (sm_100 256-bit stores); the P store and the dZ scratch are laid out so that every chunk is.
__device__ __forceinline__ void store_bf16x32_sectors(uint16_t* dst, const float (&d)[32]) {
  uint32_t p[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) p[e] = pack_bf16x2(d[2 * e], d[2 * e + 1]);
  st_global_v8(dst, p);
  st_global_v8(dst + 16, p + 8);
}

// Store one 32-value chunk of bf16 to global memory (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float (&d)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_uint4(pack_bf16x2(d[8 * q + 0], d[8 * q + 1]), pack_bf16x2(d[8 * q + 2], d[8 * q + 3]),
                       pack_bf16x2(d[8 * q + 4], d[8 * q + 5]), pack_bf16x2(d[8 * q + 6], d[8 * q + 7]));
}

// Publish the tile of step p (already stored by every epilogue thread) to the cluster, with the
// step's rescale flag (OR of the four warp votes) written into every CTA first.
template <bool kWithFlag>
__device__ __forceinline__ bool publish_tile(LmShared& sh, const LmArgs& a, const LmCtx& x, const StreamPos& p,
                                             int et, uint32_t& epc) {
  __threadfence();
  fence_proxy_async_global();
  mbar_arrive(&sh.ep_bar);
  if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) return false;
  if (et == 0) {
    if (kWithFlag) {
      const uint32_t flag = sh.wvote[0] | sh.wvote[1] | sh.wvote[2] | sh.wvote[3];
      const uint32_t lf = smem_u32(&sh.rflag[p.slot]);
      for (uint32_t q = 0; q < x.C; ++q) st_cluster_u32(mapa_shared(lf, q), flag);
    }
    const uint32_t la = smem_u32(&sh.dz_ready[p.slot]);
    for (uint32_t q = 0; q < x.C; ++q) mbar_arrive_cluster(mapa_shared(la, q));
  }
  return true;
}

// ---------------- forward epilogue (kModeFwd, kModeFwdDH) ----------------
template <int kMode, int kNZ, int kHS>
__device__ __forceinline__ void lm_fwd_epilogue_role(LmShared& sh, const LmArgs& a, const LmCtx& x, uint32_t tmem) {
  using ZB = ZBuf<kMode, kNZ>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const int et = threadIdx.x - 64;  // 0..127
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  uint32_t zc = 0, oc = 0, epc = 0, mrc = 0, uc = 0;

  if (a.force_timeout_ns != 0) {
    if (!__all_sync(0xffffffffu, lm_wait_for<false>(sh, a, x.C, &sh.never, 0, a.force_timeout_ns))) return;
  }

  // per-row state of the current unit
  int64_t t = 0;
  bool valid = false;
  int32_t y = -1;
  float mp = -INFINITY, sp = 0.f, zyp = 0.f;  // this CTA's reference, sum of exp without the target, target logit

  StreamPos p;
  p.zero();
  for (; p.s < x.total; p.next(x.steps, x.C, x.nslot)) {
    if (p.j == 0) {
      const int u = static_cast<int>(x.cl) + p.u_idx * static_cast<int>(x.ncl);
      t = static_cast<int64_t>(u) * 128 + row;
      valid = t < x.rows;
      y = valid ? a.y[t] : -1;
      mp = -INFINITY;
      sp = 0.f;
      zyp = 0.f;
    }
    if (p.modc == x.rank) {
      // ---- producer of step p ----
      const uint32_t b = ZB::buf(zc);
      const uint32_t zt = tl + ZB::col(b);
      if (!ep_wait<false>(sh, a, x.C, &sh.z_full[b], ZB::parity(zc))) break;
      tc_fence_after();
      const int vbase0 = p.j * kNZ;
      // pass 1: the tile's row maximum over valid columns
      float M = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < kNZ / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(zt + c * 32, v);
        tmem_ld_wait();
        const int vb = vbase0 + c * 32;
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (vb + q < a.V) M = fmaxf(M, __uint_as_float(v[q]));
      }
      // the chain: the reference after the previous step, raised lazily
      float mprev = -INFINITY;
      if (p.j > 0) {
        if (!ep_wait<true>(sh, a, x.C, &sh.mref_full, mrc & 1u)) break;
        ++mrc;
        mprev = x.mref[row];
        if (et == 0) mbar_arrive_expect_tx(&sh.mref_full, 128 * 4);  // arm the next delivery
      }
      const float mnew = (M > mprev + kTau) ? M : mprev;
      if (p.j < x.steps - 1) {
        const uint32_t nxt = (p.modc + 1u == x.C) ? 0u : p.modc + 1u;
        st_async_u32(mapa_shared(smem_u32(&x.mref[row]), nxt), __float_as_uint(mnew),
                     mapa_shared(smem_u32(&sh.mref_full), nxt));
      }
      // this CTA's partial sum follows its own latest reference
      if (mnew != mp) {
        sp = (mp == -INFINITY) ? 0.f : sp * ex2_approx((mp - mnew) * kLog2e);
        mp = mnew;
      }
      const float mn2 = mnew * kLog2e;
      uint16_t* dzrow = nullptr;
      if (kMode == kModeFwdDH) {
        if (p.round > 0) {
          if (!ep_wait<true>(sh, a, x.C, &sh.dz_free[p.slot], (p.round - 1) & 1u)) break;
        }
        const int64_t urow = static_cast<int64_t>(static_cast<int>(x.cl) + p.u_idx * static_cast<int>(x.ncl)) * 128 + row;
        if (a.pbuf != nullptr) {
          dzrow = a.pbuf + urow * a.p_ld + p.j * kNZ;
          a.mhist[static_cast<int64_t>(p.j) * a.Tpad + urow] = mnew;
        } else {
          dzrow = a.dz_scratch + (static_cast<int64_t>(x.cl * x.nslot + p.slot) * 128 + row) * kNZ;
        }
      }
      // pass 2: P = e^{z - m} without the target column, the partial sum, the target logit
#pragma unroll 1
      for (int c = 0; c < kNZ / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(zt + c * 32, v);
        tmem_ld_wait();
        const int vb = vbase0 + c * 32;
        float d[32];
        float cs = 0.f;
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const float z = __uint_as_float(v[q]);
          const bool tgt = (vb + q == y);
          const bool in = (vb + q < a.V) && !tgt;
          const float pr = in ? ex2_approx(fmaf(z, kLog2e, -mn2)) : 0.f;
          cs += pr;
          d[q] = pr;
          if (tgt) zyp = z;
        }
        sp += cs;
        if (kMode == kModeFwdDH) store_bf16x32_sectors(dzrow + c * 32, d);
      }
      tc_fence_before();
      mbar_arrive(&sh.z_empty[b]);
      ++zc;
      if (kMode == kModeFwdDH) {
        // per-row rescale factor of O for this step, and whether any row of the tile needs it
        const float alpha = (mprev == mnew) ? 1.f : ex2_approx((mprev - mnew) * kLog2e);
        a.alpha[static_cast<int64_t>(x.cl * x.nslot + p.slot) * 128 + row] = alpha;
        const uint32_t need = __any_sync(0xffffffffu, p.j > 0 && alpha != 1.f) ? 1u : 0u;
        if (lane == 0) sh.wvote[quarter] = need;
        if (!publish_tile<true>(sh, a, x, p, et, epc)) break;
      }
    }
    if (p.j == x.steps - 1) {
      // ---- end of the sweep: combine the C class partials in class order ----
      const uint32_t par = uc & 1u;
      float* mine = a.fin + (static_cast<int64_t>(x.cl * x.C + x.rank) * 2 + par) * 384;
      mine[row] = mp;
      mine[128 + row] = sp;
      mine[256 + row] = zyp;
      __threadfence();
      mbar_arrive(&sh.ep_bar);
      if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) break;
      if (et == 0) {
        const uint32_t lf = smem_u32(&sh.fin_full[par]);
        for (uint32_t q = 0; q < x.C; ++q) mbar_arrive_cluster(mapa_shared(lf, q));
      }
      if (!ep_wait<true>(sh, a, x.C, &sh.fin_full[par], (uc >> 1) & 1u)) break;
      const float* base = a.fin + static_cast<int64_t>(x.cl * x.C) * 768 + par * 384;
      // class k (steps j == k mod C) sits on CTA (s0 + k) mod C, s0 = stream index of step 0
      const uint32_t jm = static_cast<uint32_t>(p.j) % x.C;
      const uint32_t k0 = (p.modc >= jm) ? p.modc - jm : p.modc + x.C - jm;
      float mstar = -INFINITY;
      for (uint32_t q = 0; q < x.C; ++q) mstar = fmaxf(mstar, __ldcg(base + q * 768 + row));
      float s_ex = 0.f;
      uint32_t q = k0;
      for (uint32_t k = 0; k < x.C; ++k) {
        const float mq = __ldcg(base + q * 768 + row);
        if (mq != -INFINITY) s_ex = fmaf(__ldcg(base + q * 768 + 128 + row), ex2_approx((mq - mstar) * kLog2e), s_ex);
        q = (q + 1u == x.C) ? 0u : q + 1u;
      }
      const bool ybad = valid && (y < 0 || y >= a.V);
      float lp = __int_as_float(0x7fc00000), lse = __int_as_float(0x7fc00000), s = 1.f;
      if (valid && !ybad) {
        const uint32_t qy0 = k0 + static_cast<uint32_t>(y / kNZ) % x.C;
        const uint32_t qy = (qy0 >= x.C) ? qy0 - x.C : qy0;
        const float zy = __ldcg(base + qy * 768 + 256 + row);
        s = s_ex + ex2_approx(fmaf(zy, kLog2e, -mstar * kLog2e));
        lse = mstar + logf(s);
        lp = zy - lse;
      }
      if (ybad && x.rank == 0) raise_status(a.status, 6 /* BI_ERR_BAD_TARGET */);
      const int64_t r = (a.rowmap != nullptr && valid) ? static_cast<int64_t>(a.rowmap[t]) : t;
      if (kMode == kModeFwdDH) {
        float g = 0.f;
        if (valid) {
          const float delta = lp - a.logmu[t];
          const float w = expf(delta);
          const float d3 = expm1f(delta) - delta;
          const double c = a.coef[a.respof[t]];
          float tlv = static_cast<float>(-c * static_cast<double>(w));
          uint8_t clipped = 0;
          g = tlv;
          if (a.variant == 1) {
            // -min(w A, clip(w) A) / (R* n) = -c min(w, 1 + eps_high) for A > 0 and
            // -c max(w, 1 - eps_low) for A < 0; the gradient flows only where w itself is the
            // selected term (c = A / (R* n) carries the sign of A)
            const float hi = 1.f + a.eps_high, lo = 1.f - a.eps_low;
            const bool pos = c > 0.0, neg = c < 0.0;
            const bool active = pos ? (w <= hi) : (neg && w >= lo);
            tlv = static_cast<float>(-c * static_cast<double>(pos ? fminf(w, hi) : fmaxf(w, lo)));
            g = active ? static_cast<float>(-c * static_cast<double>(w)) : 0.f;
            clipped = (pos || neg) && !active ? 1 : 0;
          }
          if (x.rank == 0) {
            a.logprob[r] = lp;
            if (a.is_weight) a.is_weight[r] = w;
            if (a.token_loss) a.token_loss[r] = tlv;
            a.lse_c[t] = lse;
            a.g_c[t] = g;
            a.tl_c[t] = tlv;
            a.d3_c[t] = d3;
            a.delta_c[t] = delta;
            a.clip_c[t] = clipped;
            if (a.sxr_c) a.sxr_c[t] = s_ex / s;
          }
        }
        // dH_t = (g / s) (s' W_y - O') on this CTA's columns; O', s' and s share the reference m*
        if (!ep_wait<false>(sh, a, x.C, &sh.o_full, oc & 1u)) break;
        tc_fence_after();
        const float gs = g / s;
        const uint16_t* wy = (valid && !ybad) ? a.w_lm + static_cast<int64_t>(y) * a.H + x.slice0 : nullptr;
        uint16_t* dst = valid ? a.grad_hidden + r * a.H + x.slice0 : nullptr;
        // row chunks are 64-byte multiples from the base: whole sectors when the base allows
        const bool sectors = (reinterpret_cast<uintptr_t>(a.grad_hidden) & 31u) == 0;
#pragma unroll 1
        for (int c = 0; c < kHS / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tl + c * 32, v);
          tmem_ld_wait();
          if (valid) {
            float d[32];
            if (wy != nullptr) {
              const uint4* w4 = reinterpret_cast<const uint4*>(wy + c * 32);
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const uint4 wv = w4[h];
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float w0 = __uint_as_float(ww[e] << 16);
                  const float w1 = __uint_as_float(ww[e] & 0xffff0000u);
                  d[8 * h + 2 * e] = gs * fmaf(s_ex, w0, -__uint_as_float(v[8 * h + 2 * e]));
                  d[8 * h + 2 * e + 1] = gs * fmaf(s_ex, w1, -__uint_as_float(v[8 * h + 2 * e + 1]));
                }
              }
            } else {
#pragma unroll
              for (int h = 0; h < 32; ++h) d[h] = __int_as_float(0x7fc00000);
            }
            if (sectors)
              store_bf16x32_sectors(dst + c * 32, d);
            else
              store_bf16x32(dst + c * 32, d);
          }
        }
        tc_fence_before();
        mbar_arrive(&sh.o_empty);
        ++oc;
      } else {
        if (valid && x.rank == 0) {
          a.logprob[r] = lp;
          if (a.lse_out) a.lse_out[r] = lse;
        }
      }
      ++uc;
    }
  }
}

// ---------------- dW epilogue (kModeDW) ----------------
template <int kNZ, int kHS>
__device__ __forceinline__ bool dw_drain(LmShared& sh, const LmArgs& a, const LmCtx& x, uint32_t tl, int row, int u,
                                         bool have_acc, uint32_t& oc) {
  if (have_acc) {
    if (!ep_wait<false>(sh, a, x.C, &sh.o_full, oc & 1u)) return false;
    tc_fence_after();
  }
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
  if (have_acc) {
    tc_fence_before();
    mbar_arrive(&sh.o_empty);
    ++oc;
  }
  return true;
}

template <int kNZ, int kHS>
__device__ __forceinline__ void lm_dw_epilogue_role(LmShared& sh, const LmArgs& a, const LmCtx& x, uint32_t tmem) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const int et = threadIdx.x - 64;  // 0..127
  const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  constexpr uint32_t zcol = 512u - static_cast<uint32_t>(kNZ);
  uint32_t zc = 0, oc = 0, epc = 0;
  (void)lane;

  if (x.steps == 0) {
    // no rows: every owned vocabulary tile gets a zero gradient
    for (int u = static_cast<int>(x.cl); u < x.nunits; u += static_cast<int>(x.ncl))
      dw_drain<kNZ, kHS>(sh, a, x, tl, row, u, false, oc);
  }
  StreamPos p;
  p.zero();
  for (; p.s < x.total; p.next(x.steps, x.C, x.nslot)) {
    const int u = static_cast<int>(x.cl) + p.u_idx * static_cast<int>(x.ncl);
    if (p.modc == x.rank) {
      // the previous step's column parameters are no longer read; stage this step's
      mbar_arrive(&sh.ep_bar);
      if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) break;
      for (int cc = et; cc < kNZ; cc += 128) {
        const int64_t tt = static_cast<int64_t>(p.j) * kNZ + cc;
        const bool tv = tt < x.rows;
        x.col_lse2[cc] = tv ? a.lse_c[tt] * kLog2e : 0.f;
        x.col_g[cc] = tv ? a.g_c[tt] : 0.f;
        x.col_y[cc] = tv ? a.y[tt] : INT32_MIN;
      }
      mbar_arrive(&sh.ep_bar);
      if (!ep_wait<false>(sh, a, x.C, &sh.ep_bar, (epc++) & 1u)) break;
      if (!ep_wait<false>(sh, a, x.C, &sh.z_full[0], zc & 1u)) break;
      tc_fence_after();
      if (p.round > 0) {
        if (!ep_wait<true>(sh, a, x.C, &sh.dz_free[p.slot], (p.round - 1) & 1u)) break;
      }
      uint16_t* dzrow = a.dz_scratch + (static_cast<int64_t>(x.cl * x.nslot + p.slot) * 128 + row) * kNZ;
      const int64_t vrow = static_cast<int64_t>(u) * 128 + row;  // this lane's vocabulary row
      const bool v_ok = vrow < a.V;
#pragma unroll 1
      for (int c = 0; c < kNZ / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tl + zcol + c * 32, v);
        tmem_ld_wait();
        float d[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int tc = c * 32 + q;
          const float pr = ex2_approx(fmaf(__uint_as_float(v[q]), kLog2e, -x.col_lse2[tc]));
          const int32_t yc = x.col_y[tc];
          const float oh = (static_cast<int64_t>(yc) == vrow) ? 1.f : 0.f;
          d[q] = (v_ok && yc != INT32_MIN) ? x.col_g[tc] * (oh - pr) : 0.f;
        }
        store_bf16x32_sectors(dzrow + c * 32, d);
      }
      tc_fence_before();
      mbar_arrive(&sh.z_empty[0]);
      ++zc;
      if (!publish_tile<false>(sh, a, x, p, et, epc)) break;
    }
    if (p.j == x.steps - 1) {
      if (!dw_drain<kNZ, kHS>(sh, a, x, tl, row, u, true, oc)) break;
    }
  }
}

// ---------------- the kernel ----------------
template <int kMode, int kNZ, int kHS>
__global__ void __launch_bounds__(LmThreads<kMode>::value, 1)
    k_lm_cluster(const __grid_constant__ CUtensorMap tm_stat, const __grid_constant__ CUtensorMap tm_zb,
                 const __grid_constant__ CUtensorMap tm_sl, const __grid_constant__ CUtensorMap tm_dz, LmArgs a) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  using Tile = LmTile<kMode, kNZ, kHS>;
  LmShared& sh = *reinterpret_cast<LmShared*>(dsmem + Tile::nstages * Tile::stage_bytes);
  uint8_t* aux = dsmem + Tile::nstages * Tile::stage_bytes + (sizeof(LmShared) + 15) / 16 * 16;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  LmCtx x;
  x.mref = reinterpret_cast<float*>(aux);                  // forward modes
  x.col_lse2 = reinterpret_cast<float*>(aux);              // kModeDW (the two never coexist)
  x.col_g = x.col_lse2 + kNZ;
  x.col_y = reinterpret_cast<int32_t*>(x.col_g + kNZ);
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.z_full[i], 1);
      mbar_init(&sh.z_empty[i], 128);
      mbar_init(&sh.fin_full[i], x.C);
    }
    mbar_init(&sh.o_full, 1);
    mbar_init(&sh.o_empty, 128);
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.ep_bar, 128);
    for (uint32_t i = 0; i < x.nslot; ++i) {
      mbar_init(&sh.dz_ready[i], 1);
      mbar_init(&sh.dz_free[i], x.C);
    }
    mbar_init(&sh.mref_full, 1);
    mbar_init(&sh.o_drain, 1);
    mbar_init(&sh.rs_req, 1);
    mbar_init(&sh.rs_done, 128);
    mbar_init(&sh.never, 1);
    mbar_arrive_expect_tx(&sh.mref_full, 128 * 4);  // armed for the first delivery
    sh.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // peers' barriers are initialised before any remote arrive or store
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  x.ring_base = smem_u32(dsmem);
  // the 128B-swizzled tiles need 1024-byte aligned stages; refuse to run otherwise
  const bool misaligned = (x.ring_base & 1023u) != 0;
  if (misaligned && threadIdx.x == 0) raise_status(a.status, 4 /* BI_ERR_CUDA */);
  x.rows = misaligned ? 0 : (a.d_rows ? *a.d_rows : a.T);
  const int mtiles = static_cast<int>((x.rows + 127) / 128);
  x.nunits = misaligned ? 0 : ((kMode == kModeDW) ? a.nv128 : mtiles);
  x.steps = (kMode == kModeDW) ? static_cast<int>((x.rows + kNZ - 1) / kNZ) : a.nvz;
  const int my_units = (static_cast<int>(x.cl) < x.nunits)
                           ? (x.nunits - static_cast<int>(x.cl) + static_cast<int>(x.ncl) - 1) / static_cast<int>(x.ncl)
                           : 0;
  x.total = static_cast<int64_t>(my_units) * x.steps;
  x.KB = a.H / 64;
  x.slice0 = static_cast<int>(x.rank) * a.Hs;

  if (warp == 0) {
    if (lane == 0) {
      const TmaMaps m{&tm_stat, &tm_zb, &tm_sl, &tm_dz};
      lm_tma_role<kMode, kNZ, kHS>(sh, a, x, m);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) lm_mma_role<kMode, kNZ, kHS>(sh, a, x, tmem);
    __syncwarp();
  } else if (warp < 6) {
    if constexpr (kMode == kModeDW)
      lm_dw_epilogue_role<kNZ, kHS>(sh, a, x, tmem);
    else
      lm_fwd_epilogue_role<kMode, kNZ, kHS>(sh, a, x, tmem);
  } else {
    if constexpr (kMode == kModeFwdDH) lm_rescale_role<kHS>(sh, a, x, tmem);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no peer touches this CTA's shared memory after this point
  if (sh.abort_flag != 0u) {
    // on the error path a peer's last DSMEM store may still be in flight towards this CTA
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 50000u) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bi
