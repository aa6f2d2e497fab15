// kernels_decode.cuh -- log pi for a few rows (decode-style scoring, T <= 128) on every SM, with
// the same bits as the cluster kernel (kernels_lm.cuh, kModeFwd), and nothing of size T x V in
// memory.
//
// "Zero Mismatch, Simple Async RL", section "Alignment permits a simpler learning path": rollout
// and learner logprobs bit-identical for the same weights and tokens, whether a row is scored
// alone or packed.  The cluster kernel gives a one-row call the same bits as a packed one, but it
// sweeps the whole vocabulary on one cluster.  Here the same arithmetic is spread over the GPU:
// k_lm_decode1 reads W once on every SM and leaves per-sub-tile row maxima, each step's reference
// and 32-column partial sums (about 1/18 of the rows' fp32 logits); k_lm_zscan combines them per
// row in the cluster kernel's order.  A call launches k_d1_zero (status word and maxima), then
// k_lm_decode1 (cooperative), then k_lm_zscan as a programmatic dependent of it.
#pragma once

#include "kernels_lm.cuh"

namespace bi {

// Programmatic dependent launch (sm_90+): a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream runs; it must wait for that
// kernel's completion (and its memory) before touching its results.  Without the launch attribute
// both instructions are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

constexpr int kDecodeRows = 128;  // rows one tile holds: the largest T this path serves
constexpr int kZtThreads = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

// ---------------------------------------------------------------------------------------------
// Single pass (k_lm_decode1): one cooperative launch, one CTA per SM, W read once.
//
// The vocabulary is cut into 128-column sub-tiles (an NZ-wide tile of the cluster kernel is NZ / 128
// of them; a logit column's value does not depend on the N of the instruction that computes it,
// only on its row of A, its row of B and the K order, which are the cluster kernel's).  Sub-tile
// s is handled by CTA s mod G in round s div G, which spreads the vocabulary evenly over the SMs.
// Per round a CTA computes its sub-tile's logits into one of four TMEM buffers, takes the row
// maxima over the valid columns and stores each as a tagged 64-bit word.  Two rounds later it
// forms the sub-tile's 32-column chunk sums: each row's reference chain is first advanced up to
// this tile, as the cluster kernel's producers pass it on, from the maxima of every sub-tile of the
// tiles up to this one, each read (and waited for, bounded, should its writer not have stored it
// yet) by every CTA for itself.  The CTA of a tile's first sub-tile writes the tile's references
// for the combine.  A round's sums need maxima of at most the next round, so by the schedule the
// entries are nearly always there; that every CTA is resident, on which the waits rely, is what
// the cooperative launch guarantees.
// ---------------------------------------------------------------------------------------------
// A sub-tile maximum travels between CTAs as one 64-bit word, the float's bits below a "written"
// tag: an aligned 8-byte access is single-copy atomic, so a reader that sees the tag sees the
// value, with no fence on either side (GPU-scope fences stall an SM whose TMA ring is in flight).
// The words are zeroed before the launch.
__device__ __forceinline__ void st_relaxed_gpu_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_gpu_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
constexpr uint64_t kD1Tag = uint64_t{1} << 32;
__device__ __forceinline__ float d1_value(uint64_t w) { return __uint_as_float(static_cast<uint32_t>(w)); }

// Where row `row`'s maximum of sub-tile `sub` lives: row-major for up to 32 rows (a warp walks up
// to 8 rows, its lanes over consecutive sub-tiles), sub-tile-major beyond (each row's owner
// thread walks the sub-tiles, and a warp's 32 rows of one sub-tile are one 256-byte line).
constexpr int kD1WarpRows = 32;    // up to this many rows: row-major maxima, 8 rows per epilogue warp
constexpr int kD1LaneEntries = 6;  // entries per lane per row loaded at once (a round's range is ~G)
__device__ __forceinline__ int64_t d1_slot(int64_t T, int nsub, int row, int sub) {
  return T <= kD1WarpRows ? static_cast<int64_t>(row) * nsub + sub : static_cast<int64_t>(sub) * T + row;
}

// The value of the entry at p, waiting (bounded) until its writer has stored it.  Returns false
// on a timeout or an abort.
__device__ __forceinline__ bool d1_entry(const uint64_t* p, float& v, volatile uint32_t* abort_flag,
                                         int32_t* status, uint64_t limit_ns) {
  uint64_t w = ld_relaxed_gpu_u64(p);
  if (w & kD1Tag) {
    v = d1_value(w);
    return true;
  }
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    w = ld_relaxed_gpu_u64(p);
    if (w & kD1Tag) {
      v = d1_value(w);
      return true;
    }
    if ((++spins & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        raise_status(status, 5 /* BI_ERR_TIMEOUT */);
        *abort_flag = 1u;
        return false;
      }
    }
  }
}

// Columns of a sub-tile (one MMA of that N): 128 where it divides the tile width NZ, else 64.  A
// narrower MMA costs the issuing thread about as much as a wide one, so sub-tiles are as wide as
// the balance over the SMs allows.
__host__ __device__ constexpr int d1_sub(int nz) { return nz % 128 == 0 ? 128 : 64; }
constexpr int kD1MaxStages = 24;
constexpr int kD1MaxBuf = 8;   // logit buffers in TMEM: 512 / sub-tile width
// Rounds between a sub-tile's maxima and its chunk sums (buffers - 2): a round's sums need every
// CTA's maxima of at most the next round.
__host__ __device__ constexpr int d1_lag(int sub) { return 512 / sub - 2; }
constexpr int kD1Smem = kLmSmemLimit;     // the ring takes what the resident rows leave

// Hidden rows, the A operand of every sub-tile, are either streamed with each stage (kAG = 0: a
// [128 x 64] box per stage) or, for T <= 8 kAG rows, loaded once and kept: the [128 x 64] A tile of
// K chunk kb is a window starting at kb kAG KB, whose first 8 kAG rows are the real ones (one or
// more 1 KB atoms of the 128-byte swizzle) and whose other rows are those of later chunks.  Those
// rows give logits of rows past T, which nothing reads; the windows overlap, so the rows cost
// (KB - 1) kAG KB + 16 KB instead of KB x 16 KB, and every stage of the ring carries W only.
__host__ __device__ constexpr int d1_a_bytes(int kag, int kb) { return kag == 0 ? 0 : ((kb - 1) * kag + 16) * 1024; }
// A stage: W rows [sub x 64] (and the hidden rows' [128 x 64] box when they are not resident).
__host__ __device__ constexpr int d1_stage_bytes(int kag, int sub) { return (kag == 0 ? kAUnitBytes : 0) + sub * 128; }

struct D1Shared {
  uint64_t full[kD1MaxStages], empty[kD1MaxStages];
  uint64_t z_full[kD1MaxBuf], z_empty[kD1MaxBuf];
  uint64_t a_full, mma_done, ep_bar;
  float mcs[kDecodeRows];  // each row's reference after tile jc - 1
  uint32_t tmem_base;
  volatile uint32_t abort_flag;
};

struct D1Args {
  int64_t T;          // real rows (<= 128)
  int32_t V, nvz, KB;
  int32_t nsub;       // sub-tiles: nvz * NZ / sub-tile width
  int32_t a_rows;     // rows of the streamed hidden-row box (kAG = 0): T rounded up to 8, <= 128
  int32_t smem;       // dynamic shared memory of the launch (<= kD1Smem)
  int32_t rounds;     // ceil(nsub / gridDim.x)
  uint64_t* smax;     // [T][nsub] (T <= 32) or [nsub][T] row maxima of each sub-tile over its valid
                      // columns, tagged (zero at launch): d1_slot
  float* mref;        // [nvz][T] reference of each row at each step
  float* csum;        // [T][nvz][NZ / 32] chunk sums
  float* zy;          // [T] target logits
  const int32_t* y;   // [T]
  int32_t* status;
  uint64_t limit_ns;
};

template <int kNZ, int kAG>
__global__ void __launch_bounds__(kZtThreads, 1)
    k_lm_decode1(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w, D1Args a) {
  // tm_h: hidden [T][H], box {64, kAG ? 8 kAG : 128}; tm_w: W [V][H], box {64, sub-tile width};
  // both 128-byte swizzled
  constexpr int kD1Sub = d1_sub(kNZ);
  constexpr int kD1Buf = 512 / kD1Sub;
  constexpr int kD1Lag = d1_lag(kD1Sub);
  constexpr int kSubPerTile = kNZ / kD1Sub;
  constexpr int kChunks = kNZ / 32;
  constexpr int kStageBytes = d1_stage_bytes(kAG, kD1Sub);
  extern __shared__ __align__(1024) uint8_t dsmem[];
  constexpr int kShBytes = static_cast<int>((sizeof(D1Shared) + 1023) / 1024 * 1024);
  D1Shared& sh = *reinterpret_cast<D1Shared*>(dsmem + a.smem - kShBytes);
  const int a_bytes = d1_a_bytes(kAG, a.KB);
  const int nst_i = (a.smem - kShBytes - a_bytes) / kStageBytes;
  const uint32_t nst = static_cast<uint32_t>(nst_i < kD1MaxStages ? nst_i : kD1MaxStages);
  // bytes a stage receives: W rows, and the real hidden rows (rounded up to 8) when they are
  // streamed; the MMA's rows past them read whatever the stage held and give logits of rows past
  // T, which nothing reads
  const uint32_t stage_tx = static_cast<uint32_t>((kAG == 0 ? a.a_rows * 128 : 0) + kD1Sub * 128);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x);
  const int b = static_cast<int>(blockIdx.x);
  // the combine kernel may be launched now; it waits for this grid's completion before reading
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kD1MaxStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    mbar_init(&sh.a_full, 1);
    for (int i = 0; i < kD1Buf; ++i) {
      mbar_init(&sh.z_full[i], 1);
      mbar_init(&sh.z_empty[i], 128);
    }
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.ep_bar, 128);
    sh.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  if (threadIdx.x < kDecodeRows) sh.mcs[threadIdx.x] = -INFINITY;
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t abase = smem_u32(dsmem);            // resident hidden rows (kAG > 0)
  const uint32_t ring = abase + static_cast<uint32_t>(a_bytes);
  const bool misaligned = (abase & 1023u) != 0 || nst < 2;
  if (misaligned && threadIdx.x == 0) raise_status(a.status, 4 /* BI_ERR_CUDA */);
  const int rounds = misaligned ? 0 : a.rounds;
  const WaitCtl wc{&sh.abort_flag, a.status, a.limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_h);
      tma_prefetch_desc(&tm_w);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      if (kAG > 0 && rounds > 0) {
        // the real rows of every K chunk, once: chunk kb's 8 kAG rows at kb kAG KB
        mbar_arrive_expect_tx(&sh.a_full, static_cast<uint32_t>(a.KB * kAG * 1024));
        for (int kb = 0; kb < a.KB; ++kb) tma_load_2d(abase + kb * kAG * 1024, &tm_h, &sh.a_full, kb * 64, 0);
      }
      for (int r = 0; ok && r < rounds; ++r) {
        const int sub = r * G + b;
        if (sub >= a.nsub) continue;
#pragma unroll 1
        for (int kb = 0; kb < a.KB; ++kb) {
          if (!mbar_wait<false>(&sh.empty[stage], phase ^ 1u, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&sh.full[stage], stage_tx);
          const uint32_t dst = ring + stage * kStageBytes;
          if (kAG == 0) {
            tma_load_2d(dst, &tm_h, &sh.full[stage], kb * 64, 0);
            tma_load_2d(dst + kAUnitBytes, &tm_w, &sh.full[stage], kb * 64, sub * kD1Sub);
          } else {
            tma_load_2d(dst, &tm_w, &sh.full[stage], kb * 64, sub * kD1Sub);
          }
          ring_advance(stage, phase, nst);
        }
      }
      if (kAG > 0 && rounds > 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_test(&sh.a_full, 0))
          if (globaltimer_ns() - t0 > a.limit_ns) break;
      }
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
      // the cluster kernel's instruction sequence per 64-column chunk of K, with N = sub-tile width
      constexpr uint32_t idesc = idesc_bf16(128, kD1Sub, false, false);
      constexpr uint64_t sb = static_cast<uint64_t>(kStageBytes >> 4);
      const uint64_t dk0 = sdesc_k_sw128(kAG == 0 ? ring : abase);
      const uint64_t dkb0 = sdesc_k_sw128(kAG == 0 ? ring + kAUnitBytes : ring);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      if (kAG > 0 && rounds > 0 && !mbar_wait<false>(&sh.a_full, 0u, wc)) ok = false;
      for (int r = 0; ok && r < rounds; ++r) {
        const int sub = r * G + b;
        if (sub >= a.nsub) continue;
        const uint32_t bb = static_cast<uint32_t>(r % kD1Buf);
        if (!mbar_wait<false>(&sh.z_empty[bb], ((r / kD1Buf) & 1u) ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t zt = tmem + bb * kD1Sub;
#pragma unroll 1
        for (int kb = 0; kb < a.KB; ++kb) {
          if (!mbar_wait<false>(&sh.full[stage], phase, wc)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = kAG == 0 ? dk0 + stage * sb : dk0 + static_cast<uint64_t>((kb * kAG * 1024) >> 4);
          const uint64_t db = dkb0 + stage * sb;
          umma_bf16(zt, da, db, idesc, kb != 0 ? 1u : 0u);
          umma_bf16(zt, da + 2, db + 2, idesc, 1u);
          umma_bf16(zt, da + 4, db + 4, idesc, 1u);
          umma_bf16(zt, da + 6, db + 6, idesc, 1u);
          umma_commit(&sh.empty[stage]);
          ring_advance(stage, phase, nst);
        }
        if (!ok) break;
        umma_commit(&sh.z_full[bb]);
      }
      umma_commit(&sh.mma_done);
      mbar_wait<false>(&sh.mma_done, 0u, wc);
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..127
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool warp_rows = static_cast<int64_t>(quarter * 32) < a.T;  // warp-uniform
    const bool real = row < a.T;
    const int32_t yt = real ? a.y[row] : -1;
    uint32_t epc = 0;
    int jc = 0;              // next tile of the rows' chains (the same for every row)
    bool ok = true;
    for (int r = 0; ok && r < rounds + kD1Lag; ++r) {
      if (r < rounds) {
        const int sub = r * G + b;
        if (sub < a.nsub) {
          const uint32_t bb = static_cast<uint32_t>(r % kD1Buf);
          if (!__all_sync(0xffffffffu, mbar_wait<false>(&sh.z_full[bb], (r / kD1Buf) & 1u, wc))) { ok = false; break; }
          tc_fence_after();
          if (warp_rows) {
            float M = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < kD1Sub / 32; ++c) {
              uint32_t v[32];
              tmem_ld32(tl + bb * kD1Sub + c * 32, v);
              tmem_ld_wait();
              const int vb = sub * kD1Sub + c * 32;
#pragma unroll
              for (int q = 0; q < 32; ++q)
                if (vb + q < a.V) M = fmaxf(M, __uint_as_float(v[q]));
            }
            if (real) st_relaxed_gpu_u64(a.smax + d1_slot(a.T, a.nsub, row, sub), kD1Tag | __float_as_uint(M));
          }
        }
      }
      const int qr = r - kD1Lag;
      if (qr < 0 || qr >= rounds) continue;
      const int sub = qr * G + b;
      if (sub >= a.nsub) continue;
      const int j = sub / kSubPerTile;
      const uint32_t bb = static_cast<uint32_t>(qr % kD1Buf);
      if (jc <= j) {
        // advance every row's chain over tiles jc .. j, as the cluster kernel's producers pass the
        // reference on.  The range's largest sub-tile maximum is checked first: only when it could
        // raise the reference are the tiles walked in order.  Up to 32 rows: a warp per group of
        // rows (coalesced loads, the ordered walk 32 tiles at a time over the lanes by shuffles).
        // More rows: each row's owner thread alone, its loads independent of one another.
        // (each entry is waited for until its writer has stored it: by the schedule it nearly
        // always has, the entries a round needs being at least two rounds old)
        const int lo = jc * kSubPerTile, hi = (j + 1) * kSubPerTile;
        bool good = true;
        if (a.T <= kD1WarpRows) {
          // up to 8 rows per warp (rows ew, ew + 4, ...): every lane loads all its entries of all
          // its rows before anything waits (one round trip), and only a lane that found one of
          // them not yet written loads its entries again, waiting for each
          const int ew = warp - 2;  // 0..3
          float mxr[8];
          uint64_t tags = kD1Tag;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            mxr[q] = -INFINITY;
            const int r = ew + 4 * q;
            if (r < static_cast<int>(a.T)) {
              const uint64_t* rr = a.smax + static_cast<int64_t>(r) * a.nsub;
#pragma unroll
              for (int k = 0; k < kD1LaneEntries; ++k) {
                const int i = lo + lane + 32 * k;
                if (i < hi) {
                  const uint64_t w = ld_relaxed_gpu_u64(rr + i);
                  tags &= w;
                  mxr[q] = fmaxf(mxr[q], d1_value(w));
                }
              }
              for (int i = lo + lane + 32 * kD1LaneEntries; i < hi; i += 32) {  // a wider range than a round's
                const uint64_t w = ld_relaxed_gpu_u64(rr + i);
                tags &= w;
                mxr[q] = fmaxf(mxr[q], d1_value(w));
              }
            }
          }
          if (!(tags & kD1Tag)) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              mxr[q] = -INFINITY;
              const int r = ew + 4 * q;
              if (r < static_cast<int>(a.T)) {
                const uint64_t* rr = a.smax + static_cast<int64_t>(r) * a.nsub;
                for (int i = lo + lane; i < hi && good; i += 32) {
                  float v;
                  good = d1_entry(rr + i, v, &sh.abort_flag, a.status, a.limit_ns);
                  mxr[q] = fmaxf(mxr[q], v);
                }
              }
            }
          }
          if (!__all_sync(0xffffffffu, good)) {
            good = false;
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int r = ew + 4 * q;
              if (r >= static_cast<int>(a.T)) break;  // warp-uniform
              const uint64_t* rr = a.smax + static_cast<int64_t>(r) * a.nsub;
              float m = sh.mcs[r];
              float mx = mxr[q];
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
              if (mx > m + kTau) {
                for (int base = jc; base <= j; base += 32) {
                  const bool has = base + lane <= j;
                  float Ml = -INFINITY;
                  if (has) {
#pragma unroll
                    for (int i = 0; i < kSubPerTile; ++i) Ml = fmaxf(Ml, d1_value(ld_relaxed_gpu_u64(rr + (base + lane) * kSubPerTile + i)));
                  }
                  // the tiles in order: the first whose maximum raises the reference sets it, and
                  // the search goes on past it with the new reference (the same decisions as one
                  // tile at a time, one ballot per raise)
                  int from = 0;
                  while (true) {
                    const uint32_t up = __ballot_sync(0xffffffffu, has && lane >= from && Ml > m + kTau);
                    if (up == 0u) break;
                    const int l = __ffs(static_cast<int>(up)) - 1;
                    m = __shfl_sync(0xffffffffu, Ml, l);
                    from = l + 1;
                  }
                }
              }
              if (lane == 0) sh.mcs[r] = m;
            }
          }
        } else if (real) {
          const uint64_t* rr = a.smax + row;  // entry of sub-tile i at rr + i T
          const int64_t Tr = a.T;
          float m = sh.mcs[row];
          float mx = -INFINITY;
          uint64_t tags = kD1Tag;
#pragma unroll 16
          for (int i = lo; i < hi; ++i) {
            const uint64_t w = ld_relaxed_gpu_u64(rr + i * Tr);
            tags &= w;
            mx = fmaxf(mx, d1_value(w));
          }
          if (!(tags & kD1Tag)) {
            // an entry was not there yet: the range again, waiting for each
            mx = -INFINITY;
            for (int i = lo; i < hi && good; ++i) {
              float v;
              good = d1_entry(rr + i * Tr, v, &sh.abort_flag, a.status, a.limit_ns);
              mx = fmaxf(mx, v);
            }
          }
          if (good && mx > m + kTau) {
            for (int t = jc; t <= j; ++t) {
              float M = -INFINITY;
#pragma unroll
              for (int i = 0; i < kSubPerTile; ++i)
                M = fmaxf(M, d1_value(ld_relaxed_gpu_u64(rr + (t * kSubPerTile + i) * Tr)));
              m = (M > m + kTau) ? M : m;
            }
          }
          sh.mcs[row] = m;
        }
        if (!good) sh.abort_flag = 1u;
        jc = j + 1;
        mbar_arrive(&sh.ep_bar);
        if (!__all_sync(0xffffffffu, mbar_wait<false>(&sh.ep_bar, (epc++) & 1u, wc))) { ok = false; break; }
      }
      const float mc = real ? sh.mcs[row] : 0.f;
      if (warp_rows) {
        if (real && sub % kSubPerTile == 0) a.mref[static_cast<int64_t>(j) * a.T + row] = mc;
        const float mn2 = (real ? mc : 0.f) * kLog2e;
        float* cs_out = a.csum + (static_cast<int64_t>(real ? row : 0) * a.nvz + j) * kChunks +
                        (sub % kSubPerTile) * (kD1Sub / 32);
#pragma unroll 1
        for (int c = 0; c < kD1Sub / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tl + bb * kD1Sub + c * 32, v);
          tmem_ld_wait();
          const int vb = sub * kD1Sub + c * 32;
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
      tc_fence_before();
      mbar_arrive(&sh.z_empty[bb]);
    }
    if (!ok && et == 0) sh.abort_flag = 1u;
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

// The status word and the tagged maxima zeroed in one launch: a maximum's reader waits for its
// writer's tag, so the words must start untagged.
__global__ void k_d1_zero(uint64_t* __restrict__ smax, int64_t n, int32_t* __restrict__ status) {
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i0 == 0) *status = 0;
  for (int64_t i = i0; i < n; i += static_cast<int64_t>(gridDim.x) * blockDim.x) smax[i] = 0;
}

constexpr int kZsThreads = 256;
constexpr int kZsBatch = 24;   // loads in flight per thread while staging (one batch at V = 151936)

// Dynamic shared memory of k_lm_zscan: one row's chunk sums and references.
__host__ __device__ constexpr size_t zscan_smem(int nvz, int nz) {
  return static_cast<size_t>(nvz) * (static_cast<size_t>(nz / 32) + 1) * 4;
}

// One block per row: the row's chunk sums and references are staged in shared memory by the whole
// block (coalesced), then C threads form the class partial sums (serial by definition) and one
// thread combines them.
template <int kNZ>
__global__ void __launch_bounds__(kZsThreads)
    k_lm_zscan(const float* __restrict__ csum, const float* __restrict__ mref, const float* __restrict__ zyb,
               const int32_t* __restrict__ y, int64_t T, int V, int nvz, int C, float* __restrict__ logprob,
               float* __restrict__ lse_out, int32_t* status) {
  constexpr int kChunks = kNZ / 32;
  extern __shared__ float zs[];
  float* cs = zs;                                            // [nvz][kChunks]
  float* mr = zs + static_cast<int64_t>(nvz) * kChunks;      // [nvz]
  __shared__ float cls[2 * 8];  // [8] class reference, [8] class sum
  const int64_t t = blockIdx.x;
  // launched as a programmatic dependent of k_lm_decode1: its sums are read only once it completed
  pdl_wait_primary();
  if (t >= T) return;
  const float* crow = csum + t * static_cast<int64_t>(nvz) * kChunks;
  // staged in batches of kZsBatch independent loads per thread, so that a batch costs one L2 round
  // trip rather than one per element
  const int ncs = nvz * kChunks;
#pragma unroll 1
  for (int base = 0; base < ncs + nvz; base += kZsThreads * kZsBatch) {
    float v[kZsBatch];
#pragma unroll
    for (int u = 0; u < kZsBatch; ++u) {
      const int i = base + u * kZsThreads + static_cast<int>(threadIdx.x);
      v[u] = i < ncs ? __ldcg(crow + i) : (i < ncs + nvz ? __ldcg(mref + static_cast<int64_t>(i - ncs) * T + t) : 0.f);
    }
#pragma unroll
    for (int u = 0; u < kZsBatch; ++u) {
      const int i = base + u * kZsThreads + static_cast<int>(threadIdx.x);
      if (i < ncs + nvz) zs[i] = v[u];  // cs, then mr right after it
    }
  }
  __syncthreads();
  // class k: its steps in order, rescaled at each change of reference
  if (static_cast<int>(threadIdx.x) < C) {
    const int k = threadIdx.x;
    float mp = -INFINITY, sp = 0.f;
#pragma unroll 2
    for (int j = k; j < nvz; j += C) {
      const float mnew = mr[j];
      if (mnew != mp) {
        sp = (mp == -INFINITY) ? 0.f : sp * ex2_approx((mp - mnew) * kLog2e);
        mp = mnew;
      }
#pragma unroll
      for (int c = 0; c < kChunks; ++c) sp += cs[j * kChunks + c];
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
