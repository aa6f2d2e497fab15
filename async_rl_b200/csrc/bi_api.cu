// bi_api.cu -- the C ABI declared in include/bi_isloss.h and include/bi_model.h: argument checks,
// workspace layout, tensor maps and the fixed launch sequences.  Nothing here allocates device
// memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "bi_isloss.h"
#include "bi_model.h"
#include "kernels_decode.cuh"
#include "kernels_dw.cuh"
#include "kernels_lm.cuh"
#include "kernels_model.cuh"
#include "kernels_small.cuh"

namespace {

using bi::Ctrl;
using bi::RedPart;

constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s for any single in-kernel wait
constexpr size_t kZscanSmemMax = 200 * 1024;      // one row's partial sums in the decode combine
constexpr int kMaxSms = 160;                      // upper bound used to size the dZ scratch
constexpr int kDzSlotsMax = 2 * kMaxSms;          // clusters * C * slots-per-CTA <= 2 * SMs

thread_local uint64_t g_force_timeout_ns = 0;

// ---------------------------------------------------------------------------------------------
// optional per-kernel timing (events around each launch; measurement tools only)
// ---------------------------------------------------------------------------------------------
enum KernelKind : int { kKPrep, kKRowmap, kKZeroRows, kKGather, kKLmFwd, kKLmFwdDH, kKLmDW, kKDwRows,
                        kKDwStream, kKSeqGate, kKRowParts, kKReduce, kKD3Partial, kKGemm, kKRmsNorm, kKLmZscan,
                        kKLmDecode1, kKD1Zero, kNumKinds };
const char* const kKindNames[kNumKinds] = {"k_prep", "k_rowmap", "k_zero_prompt_rows", "k_gather_rows",
                                           "k_lm_fwd", "k_lm_fwd_dh", "k_lm_dw", "k_dw_rows", "k_dw_stream",
                                           "k_seq_gate", "k_row_parts", "k_reduce_parts", "k_d3_partial",
                                           "k_gemm_pair", "k_rmsnorm", "k_lm_zscan", "k_lm_decode1",
                                           "k_d1_zero"};
static_assert(sizeof(bi::D3Out) == sizeof(bi_d3), "device-written diagnostics match the ABI struct");
struct Pending {
  int kind;
  cudaEvent_t a, b;
};
struct Profiler {
  bool on = false;
  bool failed = false;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
  double ms[kNumKinds] = {};
  int64_t n[kNumKinds] = {};
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) failed = true;
    return e;
  }
};
thread_local Profiler g_prof;

struct ProfScope {  // records an event pair around one launch when profiling is on
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  ProfScope(int k, cudaStream_t st) : kind(k), s(st) {
    if (g_prof.on) {
      a = g_prof.get();
      if (a) cudaEventRecord(a, s);
    }
  }
  ~ProfScope() {
    if (g_prof.on && a) {
      cudaEvent_t b = g_prof.get();
      if (b) {
        cudaEventRecord(b, s);
        g_prof.pending.push_back({kind, a, b});
      }
    }
  }
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t ctrl, lse_c, g_c, tl_c, d3_c, delta_c, clip_c, y_c, logmu_c, rowmap, respof, coef, cprefix, rej, red, hc,
      dz, alpha, fin;
  size_t sxr_c, mhist, hs, pbuf;  // the P store (loss layout with the store only)
  size_t zmref, zcsum, zy, zsmax;  // decode-style scoring (logprob layout, T <= 128)
  bool decode;
  size_t total;
  int nred;
  int64_t tpad, pcols;        // rows and columns the P store is sized for
};

constexpr size_t kFinBytes = static_cast<size_t>(kMaxSms) * 2 * 384 * sizeof(float);  // [CTAs][2][3][128]

// R == 0: the logprob-only layout (per-CTA partials only).  R > 0: the loss layout; with
// `store`, followed by the P store of the fused forward ([Tpad][V + 256] bf16, enough for any
// logit-tile width NZ <= 256), the per-step reference history ([ceil(V / 128)][Tpad] float) and
// the scaled hidden states of the dW GEMM ([Tpad][H] bf16).
// R == 0 with `decode` and 0 < T <= 128: followed by what the all-SM scoring path keeps: per-tile
// references ([ceil(V / 128)][T] fp32, enough for any tile width NZ >= 128), 32-column partial
// sums ([T][V / 32 + 8] fp32 at most), the target logits ([T] fp32) and the row maxima of
// 64-column sub-tiles ([T][V / 64 + 4] tagged 64-bit words at most).  Nothing of size T x V.
bool split_ok(int32_t H, int c);
int logit_cols(int Hs);

// Sub-tiles of the all-SM decode pass for the widest plan any valid split of H gives (the plan
// chosen on a device is one of them).
size_t decode_subtiles_max(int32_t H, int32_t V) {
  size_t n = 0;
  for (int c = 1; c <= bi::kMaxCluster; ++c) {
    if (!split_ok(H, c)) continue;
    const int nz = logit_cols(H / c);
    if (nz < 64) continue;
    const size_t ns = static_cast<size_t>((V + nz - 1) / nz) * static_cast<size_t>(nz / bi::d1_sub(nz));
    n = ns > n ? ns : n;
  }
  return n;
}

WsLayout ws_layout(int64_t T, int32_t H, int32_t V, int32_t R, bool store, bool decode = false) {
  WsLayout L{};
  const size_t t = static_cast<size_t>(T > 0 ? T : 1);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  const size_t nred = (t + bi::kRedBlock - 1) / bi::kRedBlock;
  // R == 0 also serves bi_d3_stats, whose block partials share the region
  L.fin = take(R > 0 || kFinBytes >= nred * sizeof(RedPart) ? kFinBytes : nred * sizeof(RedPart));
  if (R > 0) {
    // per-row arrays hold whole 128-row tiles (the dW kernel copies them in 64-row chunks)
    const size_t tp = (t + 127) / 128 * 128;
    L.ctrl = take(256);
    L.lse_c = take(tp * 4);
    L.g_c = take(tp * 4);
    L.tl_c = take(t * 4);
    L.d3_c = take(t * 4);
    L.delta_c = take(t * 4);
    L.clip_c = take(t);
    L.y_c = take(tp * 4);
    L.logmu_c = take(t * 4);
    L.rowmap = take(t * 4);
    L.respof = take(t * 4);
    L.coef = take(static_cast<size_t>(R) * 8);
    L.cprefix = take(static_cast<size_t>(R + 1) * 8);
    L.rej = take(static_cast<size_t>(R));
    L.nred = static_cast<int>(nred);
    L.red = take(static_cast<size_t>(L.nred) * sizeof(RedPart));
    L.hc = take(t * static_cast<size_t>(H) * 2);
    L.dz = take(static_cast<size_t>(kDzSlotsMax) * 128 * bi::kMaxNZ * 2);
    L.alpha = take(static_cast<size_t>(kDzSlotsMax) * 128 * 4);
    if (store) {
      L.tpad = static_cast<int64_t>((t + 127) / 128 * 128);
      L.pcols = (static_cast<int64_t>(V) + 127) / 128 * 128 + 256;
      L.sxr_c = take(tp * 4);
      L.hs = take(static_cast<size_t>(L.tpad) * static_cast<size_t>(H) * 2);
      L.mhist = take(static_cast<size_t>((V + 127) / 128) * static_cast<size_t>(L.tpad) * 4);
      L.pbuf = take(static_cast<size_t>(L.tpad) * static_cast<size_t>(L.pcols) * 2);
    }
  }
  if (R == 0 && decode && T > 0 && T <= bi::kDecodeRows) {
    L.decode = true;
    const size_t ntile = static_cast<size_t>((V + 127) / 128);
    L.zmref = take(t * ntile * 4);
    L.zcsum = take(t * (static_cast<size_t>(V + 31) / 32 + 8) * 4);
    L.zy = take(t * 4);
    L.zsmax = take(t * decode_subtiles_max(H, V) * 8);
  }
  L.total = o;
  return L;
}

// Column split of H over a cluster of C CTAs: Hs = H / C must be a multiple of 64 and at most
// 384 (its fp32 accumulator plus a logit tile of NZ >= 128 columns fill the 512 TMEM columns).
bool split_ok(int32_t H, int c) { return H % c == 0 && (H / c) % 64 == 0 && H / c <= 384; }
int logit_cols(int Hs) { return ((512 - Hs) < 256 ? (512 - Hs) : 256) / 64 * 64; }
// Any valid split exists (shape check that needs no device).
int cluster_split(int32_t H) {
  for (int c = 1; c <= bi::kMaxCluster; ++c)
    if (split_ok(H, c)) return c;
  return 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------------------------
// tensor maps (driver entry point fetched through the runtime; no libcuda link dependency)
// ---------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 row-major tensor [rows][cols], box {64 columns, box_rows rows}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same bf16 row-major [rows][cols] tensor seen as [cols / 64][rows][64]: one load brings
// `box_blocks` consecutive 64-column blocks of `box_rows` rows, each block a 128B-swizzled
// [box_rows][64] tile of its own (the MN-major operand layout), in a single TMA instruction.
bool make_map_blocks(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, int box_blocks) {
  EncodeTiledFn f = encode_fn();
  if (!f || cols % 64 != 0) return false;
  const cuuint64_t dims[3] = {64u, static_cast<cuuint64_t>(rows > 0 ? rows : 1), static_cast<cuuint64_t>(cols / 64)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, 128u};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_blocks)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------------------------
// per-device set-up (kernel attributes, SM count, cluster occupancy), done once per device
// ---------------------------------------------------------------------------------------------
struct DevInfo {
  bool ready = false;
  bool ok = false;
  int sms = 0;
  bool coop = false;                                // one k_lm_decode1 CTA fits on every SM, cooperatively
  int max_clusters[3][bi::kMaxCluster + 1] = {};  // [mode][C]
  int gemm_clusters = 0;                            // resident CTA pairs of the GEMM kernel
};
std::mutex g_dev_mu;
std::array<DevInfo, 64> g_dev;

template <int kMode>
int query_clusters(int C) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, 1, 1);
  cfg.blockDim = dim3(bi::LmThreads<kMode>::value, 1, 1);
  cfg.dynamicSmemBytes = bi::LmTile<kMode, 256, 256>::smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  // every compiled tiling needs one CTA per SM; the occupancy of one of them stands for all
  if (cudaOccupancyMaxActiveClusters(&n, bi::k_lm_cluster<kMode, 256, 256>, &cfg) != cudaSuccess) return 0;
  return n;
}

// Dynamic shared memory of a dW launch: at least half the SM's, so one CTA (and its 512 TMEM
// columns) per SM.
template <int kHS>
int dw_smem() {
  return bi::DwTile<kHS>::smem > bi::kLmSmemLimit / 2 + 1024 ? bi::DwTile<kHS>::smem : bi::kLmSmemLimit / 2 + 1024;
}
// Columns per dW item: the largest of 256, 192, 128, 64 that divides H.
int dw_split(int32_t H) {
  for (int hs = 256; hs >= 64; hs -= 64)
    if (H % hs == 0) return hs;
  return 0;
}

bool set_lm_attributes() {
  bool ok = true;
#define BI_SET_ATTR(NZ_, HS_)                                                                                  \
  ok = ok && cudaFuncSetAttribute(bi::k_lm_cluster<bi::kModeFwd, NZ_, HS_>,                                   \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,                                \
                                  bi::LmTile<bi::kModeFwd, NZ_, HS_>::smem) == cudaSuccess;                   \
  ok = ok && cudaFuncSetAttribute(bi::k_lm_cluster<bi::kModeFwdDH, NZ_, HS_>,                                 \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,                                \
                                  bi::LmTile<bi::kModeFwdDH, NZ_, HS_>::smem) == cudaSuccess;                 \
  ok = ok && cudaFuncSetAttribute(bi::k_lm_cluster<bi::kModeDW, NZ_, HS_>,                                    \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,                                \
                                  bi::LmTile<bi::kModeDW, NZ_, HS_>::smem) == cudaSuccess;
  BI_LM_CONFIGS(BI_SET_ATTR)
#undef BI_SET_ATTR
#define BI_SET_DW_ATTR(HS_)                                                                                     \
  ok = ok && cudaFuncSetAttribute(bi::k_dw_stream<HS_>, cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                  dw_smem<HS_>()) == cudaSuccess;
  BI_DW_CONFIGS(BI_SET_DW_ATTR)
#undef BI_SET_DW_ATTR
  ok = ok && cudaFuncSetAttribute(bi::k_gemm_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, bi::kGemmSmem) ==
                 cudaSuccess;
#define BI_SET_D1_ATTR(NZ_, AG_)                                                                            \
  ok = ok && cudaFuncSetAttribute(bi::k_lm_decode1<NZ_, AG_>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                  bi::kD1Smem) == cudaSuccess;
#define BI_SET_D1_ATTRS(NZ_) BI_SET_D1_ATTR(NZ_, 0) BI_SET_D1_ATTR(NZ_, 1) BI_SET_D1_ATTR(NZ_, 2) BI_SET_D1_ATTR(NZ_, 4)
  BI_SET_D1_ATTRS(256)
  BI_SET_D1_ATTRS(192)
  BI_SET_D1_ATTRS(128)
#undef BI_SET_D1_ATTRS
#undef BI_SET_D1_ATTR
  ok = ok && cudaFuncSetAttribute(bi::k_lm_zscan<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kZscanSmemMax)) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(bi::k_lm_zscan<192>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kZscanSmemMax)) == cudaSuccess;
  ok = ok && cudaFuncSetAttribute(bi::k_lm_zscan<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kZscanSmemMax)) == cudaSuccess;
  return ok;
}

int query_gemm_clusters() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(bi::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = bi::kGemmSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, bi::k_gemm_pair, &cfg) != cudaSuccess) return 0;
  return n;
}

const DevInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= static_cast<int>(g_dev.size())) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (d.ready) return d.ok ? &d : nullptr;
  d.ready = true;
  if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
  if (!set_lm_attributes()) return nullptr;
  for (int c = 1; c <= bi::kMaxCluster; ++c) {
    d.max_clusters[bi::kModeFwd][c] = query_clusters<bi::kModeFwd>(c);
    d.max_clusters[bi::kModeFwdDH][c] = query_clusters<bi::kModeFwdDH>(c);
    d.max_clusters[bi::kModeDW][c] = query_clusters<bi::kModeDW>(c);
  }
  d.gemm_clusters = query_gemm_clusters();
  int coop_attr = 0, per_sm = 0;
  d.coop = cudaDeviceGetAttribute(&coop_attr, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && coop_attr != 0 &&
           cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bi::k_lm_decode1<256, 0>, bi::kZtThreads,
                                                         bi::kD1Smem) == cudaSuccess &&
           per_sm >= 1;
  cudaGetLastError();
  d.ok = d.sms > 0 && d.sms <= kMaxSms;
  return d.ok ? &d : nullptr;
}

// Tiling for H: the split with the widest logit tile (NZ), then the most SMs in use.  It depends
// on H and the device only, so every call on a device (any T, any entry point) sees the same
// vocabulary tiles and the same C partial-sum classes: the bits of a row's logprob are a
// function of the row alone.
struct LmPlan {
  int C = 0, Hs = 0, NZ = 0;
};
LmPlan plan_lm(int32_t H, const DevInfo* di) {
  LmPlan best;
  int best_sms = -1;
  for (int c = 1; c <= bi::kMaxCluster; ++c) {
    if (!split_ok(H, c)) continue;
    const int hs = H / c, nz = logit_cols(hs);
    if (di->max_clusters[0][c] <= 0 || di->max_clusters[1][c] <= 0 || di->max_clusters[2][c] <= 0) continue;
    const int sms = di->max_clusters[1][c] * c;
    if (nz > best.NZ || (nz == best.NZ && sms > best_sms)) {
      best.C = c;
      best.Hs = hs;
      best.NZ = nz;
      best_sms = sms;
    }
  }
  return best;
}

template <int kMode, int kNZ, int kHS>
bi_status launch_lm(const CUtensorMap& tm_stat, const CUtensorMap& tm_zb, const CUtensorMap& tm_sl,
                    const CUtensorMap& tm_dz, const bi::LmArgs& a, int64_t units_upper, const DevInfo* di,
                    cudaStream_t s) {
  const int smem = bi::LmTile<kMode, kNZ, kHS>::smem;
  const int maxc = di->max_clusters[kMode][a.C];
  if (maxc <= 0) return BI_ERR_CUDA;
  int64_t ncl = units_upper < maxc ? units_upper : maxc;
  if (ncl < 1) ncl = 1;
  if (ncl * a.C * bi::kSlotsPerCta > kDzSlotsMax || ncl * a.C > kMaxSms) return BI_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ncl * a.C), 1, 1);
  cfg.blockDim = dim3(bi::LmThreads<kMode>::value, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfScope ps(kMode == bi::kModeFwd ? kKLmFwd : (kMode == bi::kModeFwdDH ? kKLmFwdDH : kKLmDW), s);
  return cudaLaunchKernelEx(&cfg, bi::k_lm_cluster<kMode, kNZ, kHS>, tm_stat, tm_zb, tm_sl, tm_dz, a) == cudaSuccess
             ? BI_OK
             : BI_ERR_CUDA;
}

unsigned blocks_for(int64_t n, int per) { return static_cast<unsigned>((n + per - 1) / per); }

template <int kHS>
bi_status launch_dw(const CUtensorMap& tm_p, const CUtensorMap& tm_h, const bi::DwArgs& a, const DevInfo* di,
                    cudaStream_t s) {
  const int grid = a.nitems < di->sms ? a.nitems : di->sms;
  ProfScope ps(kKDwStream, s);
  bi::k_dw_stream<kHS><<<grid > 0 ? grid : 1, bi::kDwThreads, dw_smem<kHS>(), s>>>(tm_p, tm_h, a);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

// The logprob-only forward (kModeFwd), shared by the two logprob entry points.
bi_status logprob_forward(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets, int64_t T, int32_t H,
                          int32_t V, float* logprob, float* lse, int32_t* dev_status, float* fin,
                          uint64_t force_timeout_ns, const DevInfo* di, cudaStream_t s) {
  const LmPlan pl = plan_lm(H, di);
  if (pl.C == 0) return BI_ERR_UNSUPPORTED_SHAPE;
  // fewer than 128 rows: one unit, whose hidden-row box holds the real rows only (rounded up to 8)
  const int a_rows = T < 128 ? static_cast<int>((T + 7) / 8 * 8) : 128;
  CUtensorMap tm_h, tm_wz, tm_w64;
  if (!make_map(&tm_h, hidden, T, H, a_rows) || !make_map(&tm_wz, w_lm, V, H, pl.NZ) ||
      !make_map(&tm_w64, w_lm, V, H, 64))
    return BI_ERR_CUDA;
  bi::LmArgs a{};
  a.a_rows = a_rows;
  a.H = H;
  a.V = V;
  a.C = pl.C;
  a.Hs = pl.Hs;
  a.NZ = pl.NZ;
  a.T = T;
  a.d_rows = nullptr;
  a.nvz = (V + pl.NZ - 1) / pl.NZ;
  a.nv128 = (V + 127) / 128;
  a.w_lm = w_lm;
  a.y = targets;
  a.logprob = logprob;
  a.lse_out = lse;
  a.fin = fin;
  a.status = dev_status;
  a.limit_ns = kWaitLimitNs;
  a.force_timeout_ns = force_timeout_ns;
  const int64_t units = (T + 127) / 128;
  bi_status st = BI_ERR_UNSUPPORTED_SHAPE;
  // the slice and scratch maps are not read in this mode; any valid map fills their places
#define BI_LAUNCH_FWD(NZ_, HS_)                                                                    \
  if (pl.NZ == NZ_ && pl.Hs == HS_)                                                              \
    st = launch_lm<bi::kModeFwd, NZ_, HS_>(tm_h, tm_wz, tm_w64, tm_w64, a, units, di, s);
  BI_LM_CONFIGS(BI_LAUNCH_FWD)
#undef BI_LAUNCH_FWD
  return st;
}

// Decode-style scoring (T <= 128 rows) on every SM (kernels_decode.cuh): one cooperative pass over
// W that leaves per-sub-tile row maxima, each step's reference and 32-column partial sums, then the
// per-row combine in the cluster kernel's order.  The same plan (C, NZ) as the cluster kernel, so
// the same bits.  Returns kDecodeUnsupported when the rows should go to the cluster kernel (no
// cooperative launch on this device, or a shape the combine does not hold in shared memory).
constexpr int kDecodeUnsupported = -1;

int logprob_decode(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets, int64_t T, int32_t H,
                   int32_t V, float* logprob, float* lse, int32_t* dev_status, uint8_t* ws, const WsLayout& L,
                   const DevInfo* di, cudaStream_t s) {
  const LmPlan pl = plan_lm(H, di);
  if (pl.C == 0 || pl.C > 8 || !di->coop || pl.NZ % 64 != 0) return kDecodeUnsupported;
  const int sub = bi::d1_sub(pl.NZ);
  const int nvz = (V + pl.NZ - 1) / pl.NZ;
  const size_t zsm = bi::zscan_smem(nvz, pl.NZ);
  if (zsm > kZscanSmemMax) return kDecodeUnsupported;
  // hidden rows kept resident in 1 KB atoms of 8 rows when few (the ring then carries W only).
  // The pass then also leaves room for the combine's block where four ring stages still fit, so
  // that the block is resident (waiting on the pass) before the pass ends: 228 KB of shared
  // memory per SM, 1 KB of it reserved per resident block, and up to 1 KB of the combine's own.
  constexpr size_t kSmPerSm = 233472, kPerBlock = 1024, kZsStatic = 1024;
  const int smem_lean = static_cast<int>((kSmPerSm - kPerBlock - (zsm + kZsStatic + kPerBlock)) / 1024 * 1024);
  auto fits = [&](int g, int smem) { return bi::d1_a_bytes(g, H / 64) + 4 * bi::d1_stage_bytes(g, sub) + 4096 <= smem; };
  int ag = T <= 8 ? 1 : (T <= 16 ? 2 : (T <= 32 ? 4 : 0));
  if (ag > 0 && !fits(ag, bi::kD1Smem)) ag = 0;
  const int d1_smem = (ag > 0 && smem_lean < bi::kD1Smem && fits(ag, smem_lean)) ? smem_lean : bi::kD1Smem;
  // streamed hidden rows: a box of T rows rounded up to 8 (whole 1 KB atoms of the swizzle), so
  // that no stage carries rows past T
  const int a_rows = ag > 0 ? 8 * ag : static_cast<int>(std::min<int64_t>(128, (T + 7) / 8 * 8));
  CUtensorMap tm_h, tm_w64;
  if (!make_map(&tm_h, hidden, T, H, a_rows) || !make_map(&tm_w64, w_lm, V, H, sub)) return BI_ERR_CUDA;
  const int nsub = nvz * (pl.NZ / sub);
  if (static_cast<size_t>(nsub) > decode_subtiles_max(H, V)) return kDecodeUnsupported;  // not held by L.zsmax
  const int G = nsub < di->sms ? nsub : di->sms;  // >= NZ / sub sub-tiles: every wait has a finite target
  bi::D1Args d{};
  d.T = T;
  d.V = V;
  d.nvz = nvz;
  d.KB = H / 64;
  d.nsub = nsub;
  d.a_rows = a_rows;
  d.smem = d1_smem;
  d.rounds = (nsub + G - 1) / G;
  d.smax = reinterpret_cast<uint64_t*>(ws + L.zsmax);
  d.mref = reinterpret_cast<float*>(ws + L.zmref);
  d.csum = reinterpret_cast<float*>(ws + L.zcsum);
  d.zy = reinterpret_cast<float*>(ws + L.zy);
  d.y = targets;
  d.status = dev_status;
  d.limit_ns = kWaitLimitNs;
  // the status word and the tagged maxima start at zero (a reader waits for its writer's tag)
  {
    ProfScope ps(kKD1Zero, s);
    const int64_t nz = T * static_cast<int64_t>(nsub);
    const unsigned zb = static_cast<unsigned>(std::min<int64_t>((nz + 255) / 256, 4 * di->sms));
    bi::k_d1_zero<<<zb, 256, 0, s>>>(d.smax, nz, dev_status);
    if (cudaGetLastError() != cudaSuccess) return BI_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G), 1, 1);
  cfg.blockDim = dim3(bi::kZtThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(d.smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaErrorInvalidValue;
  {
    ProfScope ps(kKLmDecode1, s);
#define BI_D1_LAUNCH(NZ_, AG_) \
  if (pl.NZ == NZ_ && ag == AG_) e = cudaLaunchKernelEx(&cfg, bi::k_lm_decode1<NZ_, AG_>, tm_h, tm_w64, d);
#define BI_D1_LAUNCHES(NZ_) BI_D1_LAUNCH(NZ_, 0) BI_D1_LAUNCH(NZ_, 1) BI_D1_LAUNCH(NZ_, 2) BI_D1_LAUNCH(NZ_, 4)
    BI_D1_LAUNCHES(256)
    BI_D1_LAUNCHES(192)
    BI_D1_LAUNCHES(128)
#undef BI_D1_LAUNCHES
#undef BI_D1_LAUNCH
  }
  if (e != cudaSuccess) return BI_ERR_CUDA;
  // the combine as a programmatic dependent of the pass: its launch overlaps the pass, and it waits
  // for the pass's completion before reading (a plain launch where the attribute is refused)
  ProfScope ps(kKLmZscan, s);
  cudaLaunchConfig_t zc = {};
  zc.gridDim = dim3(static_cast<unsigned>(T), 1, 1);
  zc.blockDim = dim3(bi::kZsThreads, 1, 1);
  zc.dynamicSmemBytes = zsm;
  zc.stream = s;
  cudaLaunchAttribute zattr[1];
  zattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  zattr[0].val.programmaticStreamSerializationAllowed = 1;
  zc.attrs = zattr;
  zc.numAttrs = 1;
  auto* zk = pl.NZ == 256 ? bi::k_lm_zscan<256> : (pl.NZ == 192 ? bi::k_lm_zscan<192> : bi::k_lm_zscan<128>);
  const int32_t Cz = pl.C;
  e = cudaLaunchKernelEx(&zc, zk, d.csum, d.mref, d.zy, targets, T, V, nvz, Cz, logprob, lse, dev_status);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    zc.numAttrs = 0;
    e = cudaLaunchKernelEx(&zc, zk, d.csum, d.mref, d.zy, targets, T, V, nvz, Cz, logprob, lse, dev_status);
  }
  return e == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // namespace

namespace {

// ---------------------------------------------------------------------------------------------
// Fixed scratch for bi_logprob_fwd_noalloc.  Some callers cannot allocate device memory at all:
// code that runs inside a host framework which owns every device allocation (a serving engine's
// fixed memory pool, a plugin given no allocator handle) has no way to hand this library a
// workspace.  For them, the forward's per-CTA partials live in this array instead.  It is a
// file-scope device array, so every GPU that loads the library holds it (480 KB) until the
// process exits.  Its size depends on the SM count only (one [2][3][128] block per CTA), so any
// T fits.  All calls share it: calls whose kernels overlap on the GPU (different streams,
// different host threads) race on it.
// ---------------------------------------------------------------------------------------------
constexpr size_t kNoAllocFloats = kFinBytes / sizeof(float);
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

// The array's name is only a host-side stand-in; the kernel needs its device address, looked up
// once per device with that device current (on the first call made on it).
float* noalloc_scratch_address() {
  static std::mutex mu;
  static std::array<float*, 64> addr{};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= static_cast<int>(addr.size())) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<float*>(p);
  }
  return addr[dev];
}

}  // namespace

extern "C" {

int32_t bi_version(void) { return 100; }

const char* bi_status_string(bi_status s) {
  switch (s) {
    case BI_OK: return "BI_OK";
    case BI_ERR_INVALID_ARG: return "BI_ERR_INVALID_ARG";
    case BI_ERR_UNSUPPORTED_SHAPE: return "BI_ERR_UNSUPPORTED_SHAPE";
    case BI_ERR_WORKSPACE: return "BI_ERR_WORKSPACE";
    case BI_ERR_CUDA: return "BI_ERR_CUDA";
    case BI_ERR_TIMEOUT: return "BI_ERR_TIMEOUT";
    case BI_ERR_BAD_TARGET: return "BI_ERR_BAD_TARGET";
    case BI_ERR_NONFINITE: return "BI_ERR_NONFINITE";
    case BI_ERR_BAD_OFFSETS: return "BI_ERR_BAD_OFFSETS";
  }
  return "BI_UNKNOWN";
}

void bi_debug_force_timeout_once(uint64_t limit_ns) { g_force_timeout_ns = limit_ns; }

void bi_profile_enable(int32_t on) { g_prof.on = on != 0; }

void bi_profile_reset(void) {
  for (int k = 0; k < kNumKinds; ++k) {
    g_prof.ms[k] = 0.0;
    g_prof.n[k] = 0;
  }
}

int32_t bi_profile_read(const char** names_out, double* ms_out, int64_t* launches_out, int32_t max_kernels) {
  for (const Pending& p : g_prof.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess)
      g_prof.failed = true;
    g_prof.ms[p.kind] += ms;
    g_prof.n[p.kind] += 1;
    g_prof.pool.push_back(p.a);
    g_prof.pool.push_back(p.b);
  }
  g_prof.pending.clear();
  if (g_prof.failed) return -1;
  int32_t m = 0;
  for (int k = 0; k < kNumKinds && m < max_kernels; ++k) {
    if (names_out) names_out[m] = kKindNames[k];
    if (ms_out) ms_out[m] = g_prof.ms[k];
    if (launches_out) launches_out[m] = g_prof.n[k];
    ++m;
  }
  return m;
}

size_t bi_workspace_bytes(int64_t T, int32_t H, int32_t V, int32_t R) {
  if (T < 0 || H <= 0 || V <= 0 || R < 0) return 0;
  return ws_layout(T, H, V, R, false, true).total;
}

size_t bi_workspace_bytes_min(int64_t T, int32_t H, int32_t V, int32_t R) {
  if (T < 0 || H <= 0 || V <= 0 || R < 0) return 0;
  return ws_layout(T, H, V, R, false).total;
}

size_t bi_workspace_bytes_pstore(int64_t T, int32_t H, int32_t V, int32_t R) {
  if (T < 0 || H <= 0 || V <= 0 || R < 1) return 0;
  return ws_layout(T, H, V, R, true).total;
}

bi_status bi_logprob_fwd(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets, int64_t T, int32_t H,
                         int32_t V, float* logprob, float* lse, int32_t* dev_status, void* ws, size_t ws_bytes,
                         void* stream) {
  const uint64_t force = g_force_timeout_ns;
  g_force_timeout_ns = 0;
  if (T < 0 || T >= (int64_t(1) << 31) || H <= 0 || V <= 0) return BI_ERR_INVALID_ARG;
  if (!dev_status || (T > 0 && (!hidden || !w_lm || !targets || !logprob))) return BI_ERR_INVALID_ARG;
  if (T > 0 && (!aligned16(hidden) || !aligned16(w_lm))) return BI_ERR_INVALID_ARG;
  if (H % 64 != 0 || cluster_split(H) == 0) return BI_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(T, H, V, 0, false);
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return BI_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DevInfo* di = device_info();
  if (!di) return BI_ERR_CUDA;
  // a few rows: the same bits from every SM when the workspace holds their logits (that path
  // zeroes the status word itself, in the launch that zeroes its tagged maxima)
  const WsLayout Ld = ws_layout(T, H, V, 0, false, true);
  if (T > 0 && Ld.decode && ws_bytes >= Ld.total && force == 0) {
    const int r = logprob_decode(hidden, w_lm, targets, T, H, V, logprob, lse, dev_status, static_cast<uint8_t*>(ws),
                                 Ld, di, s);
    if (r != kDecodeUnsupported) return static_cast<bi_status>(r);
  }
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return BI_ERR_CUDA;
  if (T == 0) return BI_OK;
  float* fin = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.fin);
  return logprob_forward(hidden, w_lm, targets, T, H, V, logprob, lse, dev_status, fin, force, di, s);
}

// Same computation as bi_logprob_fwd (same kernel, same tiles, same bits), with the per-CTA
// partials in the library's fixed scratch array instead of a caller workspace: no device
// allocation by anyone.
bi_status bi_logprob_fwd_noalloc(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets, int64_t T,
                                 int32_t H, int32_t V, float* logprob, float* lse, int32_t* dev_status,
                                 void* stream) {
  if (T < 0 || T >= (int64_t(1) << 31) || H <= 0 || V <= 0) return BI_ERR_INVALID_ARG;
  if (!dev_status || (T > 0 && (!hidden || !w_lm || !targets || !logprob))) return BI_ERR_INVALID_ARG;
  if (T > 0 && (!aligned16(hidden) || !aligned16(w_lm))) return BI_ERR_INVALID_ARG;
  if (H % 64 != 0 || cluster_split(H) == 0) return BI_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DevInfo* di = device_info();
  if (!di) return BI_ERR_CUDA;
  float* scratch = noalloc_scratch_address();
  if (!scratch) return BI_ERR_CUDA;
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return BI_ERR_CUDA;
  if (T == 0) return BI_OK;
  return logprob_forward(hidden, w_lm, targets, T, H, V, logprob, lse, dev_status, scratch, 0, di, s);
}

bi_status bi_is_loss_fwd_bwd(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets,
                             const float* rollout_logprob, const float* rewards, const int64_t* resp_offsets,
                             const int32_t* group_offsets, const int32_t* prompt_lens, int32_t R, int32_t G,
                             double resp_normalizer, const bi_loss_cfg* cfg, int64_t T, int32_t H, int32_t V,
                             float* loss, float* logprob,
                             float* is_weight, float* token_loss, bi_d3* d3, uint16_t* grad_hidden, float* grad_w,
                             int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || T >= (int64_t(1) << 31) || H <= 0 || V <= 0 || R < 1 || G < 1 || G > R) return BI_ERR_INVALID_ARG;
  if (!(resp_normalizer >= 0.0)) return BI_ERR_INVALID_ARG;
  const bi_loss_cfg lc = cfg ? *cfg : bi_loss_cfg{BI_LOSS_UNCLIPPED, 0.f, 0.f, 0.f, 0};
  if (lc.variant < BI_LOSS_UNCLIPPED || lc.variant > BI_LOSS_SEQ_GATE) return BI_ERR_INVALID_ARG;
  if ((lc.flags & ~BI_LOSS_STORE_P) != 0) return BI_ERR_INVALID_ARG;
  if (lc.variant == BI_LOSS_PPO_CLIP &&
      !(lc.eps_low >= 0.f && lc.eps_high >= 0.f && std::isfinite(lc.eps_low) && std::isfinite(lc.eps_high)))
    return BI_ERR_INVALID_ARG;
  if (lc.variant == BI_LOSS_SEQ_GATE && !(lc.gate >= 0.f)) return BI_ERR_INVALID_ARG;
  if (!dev_status || !w_lm || !rewards || !resp_offsets || !group_offsets || !loss || !grad_w)
    return BI_ERR_INVALID_ARG;
  if (T > 0 && (!hidden || !targets || !rollout_logprob || !logprob || !grad_hidden)) return BI_ERR_INVALID_ARG;
  if (!aligned16(w_lm) || !aligned16(grad_w) || (T > 0 && (!aligned16(hidden) || !aligned16(grad_hidden))))
    return BI_ERR_INVALID_ARG;
  if (H % 64 != 0 || cluster_split(H) == 0) return BI_ERR_UNSUPPORTED_SHAPE;
  // dW recomputes the logits tile by tile unless the caller opted in to the P store, which keeps
  // every exponentiated logit tile of the forward in the workspace for a GEMM-only dW
  const bool store = (lc.flags & BI_LOSS_STORE_P) != 0;
  if (store && dw_split(H) == 0) return BI_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(T, H, V, R, store);
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return BI_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DevInfo* di = device_info();
  if (!di) return BI_ERR_CUDA;
  const LmPlan pl = plan_lm(H, di);
  if (pl.C == 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return BI_ERR_CUDA;

  uint8_t* w8 = static_cast<uint8_t*>(ws);
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(w8 + L.ctrl);
  const int64_t* d_rows = &ctrl->n_scored;
  auto F = [&](size_t o) { return reinterpret_cast<float*>(w8 + o); };
  auto I = [&](size_t o) { return reinterpret_cast<int32_t*>(w8 + o); };
  const double rstar = resp_normalizer > 0.0 ? resp_normalizer : static_cast<double>(R);

  {
    ProfScope ps(kKPrep, s);
    bi::k_prep<<<1, 1024, 0, s>>>(rewards, resp_offsets, group_offsets, prompt_lens, R, G, rstar, T,
                                  reinterpret_cast<double*>(w8 + L.coef), reinterpret_cast<int64_t*>(w8 + L.cprefix),
                                  ctrl, dev_status);
  }
  if (T > 0) {
    ProfScope ps(kKRowmap, s);
    bi::k_rowmap<<<blocks_for(T, 256), 256, 0, s>>>(resp_offsets, prompt_lens, R, T,
                                                    reinterpret_cast<int64_t*>(w8 + L.cprefix), ctrl, targets,
                                                    rollout_logprob, I(L.rowmap), I(L.respof), I(L.y_c),
                                                    F(L.logmu_c), logprob, is_weight, token_loss);
  }
  const uint16_t* hc = hidden;
  if (T > 0 && prompt_lens) {
    {
      ProfScope ps(kKZeroRows, s);
      bi::k_zero_prompt_rows<<<blocks_for(T * 32, 256), 256, 0, s>>>(resp_offsets, prompt_lens, R, T, H, ctrl,
                                                                      grad_hidden);
    }
    uint16_t* hcw = reinterpret_cast<uint16_t*>(w8 + L.hc);
    ProfScope ps(kKGather, s);
    bi::k_gather_rows<<<blocks_for(T * 32, 256), 256, 0, s>>>(hidden, T, H, ctrl, I(L.rowmap), hcw);
    hc = hcw;
  }
  if (cudaGetLastError() != cudaSuccess) return BI_ERR_CUDA;

  CUtensorMap tm_h128, tm_hz, tm_hsl, tm_w128, tm_wz, tm_wsl, tm_dz, tm_p64, tm_hblk;
  const int64_t trows = T > 0 ? T : 1;
  const int nvz = (V + pl.NZ - 1) / pl.NZ;
  const int64_t p_ld = static_cast<int64_t>(nvz) * pl.NZ;  // <= L.pcols
  const void* hsrc = hc ? static_cast<const void*>(hc) : static_cast<const void*>(w8 + L.hc);
  // slice operands: the Hs / 64 column blocks of a CTA's slice, 64 rows, in one load
  if (!make_map(&tm_h128, hsrc, trows, H, 128) || !make_map(&tm_hz, hsrc, trows, H, pl.NZ) ||
      !make_map_blocks(&tm_hsl, hsrc, trows, H, 64, pl.Hs / 64) || !make_map(&tm_w128, w_lm, V, H, 128) ||
      !make_map(&tm_wz, w_lm, V, H, pl.NZ) || !make_map_blocks(&tm_wsl, w_lm, V, H, 64, pl.Hs / 64))
    return BI_ERR_CUDA;
  const int dw_hs = dw_split(H);
  if (store ? !(make_map(&tm_dz, w8 + L.pbuf, L.tpad, p_ld, 128) &&
                make_map_blocks(&tm_p64, w8 + L.pbuf, L.tpad, p_ld, 64, 4) &&
                make_map_blocks(&tm_hblk, w8 + L.hs, L.tpad, H, 64, dw_hs / 64))
            : !make_map(&tm_dz, w8 + L.dz, static_cast<int64_t>(kDzSlotsMax) * 128, pl.NZ, 128))
    return BI_ERR_CUDA;
  bi::LmArgs a{};
  a.H = H;
  a.V = V;
  a.C = pl.C;
  a.Hs = pl.Hs;
  a.NZ = pl.NZ;
  a.T = trows;
  a.d_rows = d_rows;
  a.nvz = (V + pl.NZ - 1) / pl.NZ;
  a.nv128 = (V + 127) / 128;
  a.w_lm = w_lm;
  a.y = I(L.y_c);
  a.logmu = F(L.logmu_c);
  a.respof = I(L.respof);
  a.coef = reinterpret_cast<const double*>(w8 + L.coef);
  a.rowmap = I(L.rowmap);
  a.lse_c = F(L.lse_c);
  a.g_c = F(L.g_c);
  a.tl_c = F(L.tl_c);
  a.d3_c = F(L.d3_c);
  a.delta_c = F(L.delta_c);
  a.clip_c = reinterpret_cast<uint8_t*>(w8 + L.clip_c);
  a.variant = lc.variant;
  a.eps_low = lc.eps_low;
  a.eps_high = lc.eps_high;
  a.logprob = logprob;
  a.is_weight = is_weight;
  a.token_loss = token_loss;
  a.grad_hidden = grad_hidden;
  a.grad_w = grad_w;
  a.dz_scratch = reinterpret_cast<uint16_t*>(w8 + L.dz);
  a.alpha = F(L.alpha);
  a.fin = F(L.fin);
  a.status = dev_status;
  a.limit_ns = kWaitLimitNs;
  bi::DwArgs da{};
  if (store) {
    a.pbuf = reinterpret_cast<uint16_t*>(w8 + L.pbuf);
    a.p_ld = p_ld;
    a.mhist = F(L.mhist);
    a.Tpad = L.tpad;
    a.sxr_c = F(L.sxr_c);
    da.H = H;
    da.V = V;
    da.Hs = dw_split(H);
    da.nsl = H / da.Hs;
    da.NZf = pl.NZ;
    da.nvz = nvz;
    da.Tpad = L.tpad;
    da.d_rows = d_rows;
    da.nv128 = a.nv128;
    da.nitems = ((a.nv128 + 1) / 2) * da.nsl;
    da.mhist = F(L.mhist);
    da.y_c = I(L.y_c);
    da.grad_w = grad_w;
    da.status = dev_status;
    da.limit_ns = kWaitLimitNs;
  }
  RedPart* parts = reinterpret_cast<RedPart*>(w8 + L.red);
  bi_status st = BI_ERR_UNSUPPORTED_SHAPE;
  // forward + dH over row tiles, the loss and D3 reductions, then dW over vocabulary tiles
#define BI_LAUNCH(NZ_, HS_)                                                                                  \
  if (pl.NZ == NZ_ && pl.Hs == HS_) {                                                                        \
    st = BI_OK;                                                                                            \
    if (T > 0) st = launch_lm<bi::kModeFwdDH, NZ_, HS_>(tm_h128, tm_wz, tm_wsl, tm_dz, a, (T + 127) / 128, di, s); \
    if (st == BI_OK) {                                                                                     \
      if (lc.variant == BI_LOSS_SEQ_GATE && T > 0) {                                                      \
        ProfScope ps(kKSeqGate, s);                                                                        \
        bi::k_seq_gate<<<R, 256, 0, s>>>(reinterpret_cast<const int64_t*>(w8 + L.cprefix), F(L.delta_c),  \
                                         I(L.rowmap), lc.gate, H, ctrl, F(L.g_c), F(L.tl_c), token_loss,  \
                                         grad_hidden, reinterpret_cast<uint8_t*>(w8 + L.rej));            \
      }                                                                                                    \
      {                                                                                                    \
        ProfScope ps(kKRowParts, s);                                                                       \
        bi::k_row_parts<<<L.nred, bi::kRedBlock, 0, s>>>(F(L.tl_c), F(L.d3_c), F(L.delta_c),             \
                                                         reinterpret_cast<const uint8_t*>(w8 + L.clip_c), \
                                                         ctrl, parts);                                     \
      }                                                                                                    \
      {                                                                                                    \
        ProfScope ps(kKReduce, s);                                                                         \
        const uint8_t* rej = (lc.variant == BI_LOSS_SEQ_GATE && T > 0)                                     \
                                 ? reinterpret_cast<const uint8_t*>(w8 + L.rej) : nullptr;                 \
        bi::k_reduce_parts<<<1, 1024, 0, s>>>(parts, L.nred, rej, R, loss, reinterpret_cast<bi::D3Out*>(d3), \
                                              dev_status);                                                 \
      }                                                                                                    \
      if (cudaGetLastError() != cudaSuccess) st = BI_ERR_CUDA;                                             \
    }                                                                                                      \
    if (st == BI_OK && !store) st = launch_lm<bi::kModeDW, NZ_, HS_>(tm_w128, tm_hz, tm_hsl, tm_dz, a, a.nv128, di, s); \
  }
  BI_LM_CONFIGS(BI_LAUNCH)
#undef BI_LAUNCH
  if (st == BI_OK && store) {
    {
      // scaled hidden states H' and the target entries of the P store, then the dW GEMM
      ProfScope ps(kKDwRows, s);
      bi::k_dw_rows<<<blocks_for(L.tpad * 32, 256), 256, 0, s>>>(
          static_cast<const uint16_t*>(hsrc), H, d_rows, L.tpad, F(L.lse_c), F(L.g_c), F(L.sxr_c), I(L.y_c),
          F(L.mhist), nvz, V, reinterpret_cast<uint16_t*>(w8 + L.hs), reinterpret_cast<uint16_t*>(w8 + L.pbuf),
          p_ld);
      if (cudaGetLastError() != cudaSuccess) return BI_ERR_CUDA;
    }
    st = BI_ERR_UNSUPPORTED_SHAPE;
#define BI_LAUNCH_DW(HS_) \
    if (da.Hs == HS_) st = launch_dw<HS_>(tm_p64, tm_hblk, da, di, s);
    BI_DW_CONFIGS(BI_LAUNCH_DW)
#undef BI_LAUNCH_DW
  }
  return st;
}

bi_status bi_d3_stats(const float* learner_logprob, const float* rollout_logprob, const uint8_t* mask, int64_t T,
                      bi_d3* out, int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || !out || !dev_status || (T > 0 && (!learner_logprob || !rollout_logprob))) return BI_ERR_INVALID_ARG;
  const size_t nred = static_cast<size_t>((T > 0 ? T : 1) + bi::kRedBlock - 1) / bi::kRedBlock;
  if (!ws || ws_bytes < nred * sizeof(RedPart) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return BI_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RedPart* parts = static_cast<RedPart*>(ws);
  // one partial per kD3BlockRows rows (the workspace holds one per kRedBlock rows, more than that)
  const size_t nblk = static_cast<size_t>((T > 0 ? T : 1) + bi::kD3BlockRows - 1) / bi::kD3BlockRows;
  {
    ProfScope ps(kKD3Partial, s);
    bi::k_d3_partial<<<static_cast<unsigned>(nblk), bi::kRedBlock, 0, s>>>(learner_logprob, rollout_logprob, mask, T,
                                                                           parts, dev_status);
  }
  ProfScope ps(kKReduce, s);
  bi::k_reduce_parts<<<1, 1024, 0, s>>>(parts, static_cast<int>(nblk), nullptr, 0, nullptr,
                                        reinterpret_cast<bi::D3Out*>(out), dev_status);
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_gemm_bf16(const uint16_t* x, const uint16_t* w, uint16_t* y, int64_t M, int32_t N, int32_t K,
                       int32_t* dev_status, void* stream) {
  if (!dev_status || !w || (M > 0 && (!x || !y))) return BI_ERR_INVALID_ARG;
  if (!aligned16(w) || (M > 0 && (!aligned16(x) || !aligned16(y)))) return BI_ERR_INVALID_ARG;
  // tile row coordinates (M rounded up to 256) must stay inside int32
  if (M < 0 || M > (int64_t{1} << 31) - 256) return BI_ERR_INVALID_ARG;
  if (N <= 0 || N % 8 != 0 || K <= 0 || K % 8 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return BI_ERR_CUDA;
  if (M == 0) return BI_OK;
  const DevInfo* di = device_info();
  if (!di || di->gemm_clusters <= 0) return BI_ERR_CUDA;
  CUtensorMap tm_x, tm_w;
  if (!make_map(&tm_x, x, M, K, 128) || !make_map(&tm_w, w, N, K, 128)) return BI_ERR_CUDA;
  bi::GemmArgs a{};
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.status = dev_status;
  a.limit_ns = kWaitLimitNs;
  const int64_t tiles = ((M + bi::kGemmTileM - 1) / bi::kGemmTileM) * ((N + bi::kGemmTileN - 1) / bi::kGemmTileN);
  const int64_t ncl = tiles < di->gemm_clusters ? tiles : di->gemm_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * ncl), 1, 1);
  cfg.blockDim = dim3(bi::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(bi::kGemmSmem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ProfScope ps(kKGemm, s);
  return cudaLaunchKernelEx(&cfg, bi::k_gemm_pair, tm_x, tm_w, a) == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

bi_status bi_rmsnorm(const uint16_t* x, const uint16_t* g, float eps, uint16_t* y, int64_t M, int32_t H,
                     int32_t* dev_status, void* stream) {
  if (!dev_status || !g || (M > 0 && (!x || !y))) return BI_ERR_INVALID_ARG;
  if (!aligned16(g) || (M > 0 && (!aligned16(x) || !aligned16(y)))) return BI_ERR_INVALID_ARG;
  if (M < 0 || !(eps >= 0.f) || !std::isfinite(eps)) return BI_ERR_INVALID_ARG;
  if (H <= 0 || H % 8 != 0) return BI_ERR_UNSUPPORTED_SHAPE;
  if (M > 0 && static_cast<const void*>(x) == static_cast<const void*>(y)) return BI_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s) != cudaSuccess) return BI_ERR_CUDA;
  if (M == 0) return BI_OK;
  const DevInfo* di = device_info();
  if (!di) return BI_ERR_CUDA;
  // a warp per row, 8 rows per block, rows strided over the grid.  The variant depends on H only:
  // rows of up to 3072 elements stay in registers (2 resident blocks per SM up to 2048, then 1),
  // longer rows take two passes (8 resident blocks per SM).
  const int64_t want = (M + bi::kNormThreads / 32 - 1) / (bi::kNormThreads / 32);
  const int kvec = (H + 255) / 256;
  const int64_t cap = static_cast<int64_t>(di->sms) * (kvec <= bi::kNormRegMaxVec ? bi::kNormRegBlocks(kvec) : 8);
  const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
  ProfScope ps(kKRmsNorm, s);
  switch (kvec) {
#define BI_NORM_CASE(V_)                                                                  \
  case V_:                                                                                \
    bi::k_rmsnorm_reg<V_><<<blocks, bi::kNormThreads, 0, s>>>(x, g, eps, y, M, H);        \
    break;
    BI_NORM_CASE(1) BI_NORM_CASE(2) BI_NORM_CASE(3) BI_NORM_CASE(4) BI_NORM_CASE(5) BI_NORM_CASE(6)
    BI_NORM_CASE(7) BI_NORM_CASE(8) BI_NORM_CASE(9) BI_NORM_CASE(10) BI_NORM_CASE(11) BI_NORM_CASE(12)
#undef BI_NORM_CASE
    default:
      bi::k_rmsnorm<<<blocks, bi::kNormThreads, 0, s>>>(x, g, eps, y, M, H);
  }
  return cudaGetLastError() == cudaSuccess ? BI_OK : BI_ERR_CUDA;
}

}  // extern "C"
