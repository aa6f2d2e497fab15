// kernels_small.cuh -- the light, memory-bound steps around the tensor-core kernels: offsets
// validation and per-response coefficients, the scored-row map, the gather of scored rows, the
// sequence gate of the comparison variant, and the fixed-order reductions of the loss, the D3
// statistics and the KL estimators.  No atomics take part in any sum: every reduction has a fixed
// tree shape that depends only on the number of rows.
//
// Definitions: "Zero Mismatch, Simple Async RL", sections "Only one probability gap comes from
// old weights" (w = pi / mu, D3 = mean of w - 1 - log w) and "Alignment permits a simpler
// learning path" (advantage = reward - group mean, tokens averaged within each response,
// no clipping, no gate; the clip and the gate exist here as the baselines the pages compare
// with).
#pragma once

#include "sm100.cuh"

namespace bi {

constexpr int kRedBlock = 256;

struct RedPart {
  double loss;
  double d3sum;
  double k1sum;        // sum of -delta
  double k2sum;        // sum of delta^2 / 2
  float d3max;
  int32_t pad;
  int64_t count;
  int64_t nonfinite;
  int64_t nclip;       // tokens whose gradient the clip removed
  int64_t nrej;        // responses the sequence gate rejected
};
__device__ __forceinline__ RedPart red_zero() { return RedPart{0.0, 0.0, 0.0, 0.0, -INFINITY, 0, 0, 0, 0, 0}; }

struct Ctrl {          // small device-side control block at the start of the workspace
  int64_t n_scored;    // number of scored (compact) rows
  int32_t valid;       // offsets passed validation
  int32_t pad;
};

// Largest i in [0, R) with off[i] <= r (off[R] > r is guaranteed by validation).
__device__ __forceinline__ int find_response(const int64_t* __restrict__ off, int R, int64_t r) {
  int lo = 0, hi = R - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One block.  Validates the offsets, then A_i = r_i - mean_group(r), n_i, c_i = A_i / (R* n_i)
// in float64, the exclusive prefix of n_i and the number of scored rows.
__global__ void k_prep(const float* __restrict__ rewards, const int64_t* __restrict__ off,
                       const int32_t* __restrict__ goff, const int32_t* __restrict__ plen, int R, int G,
                       double rstar, int64_t T, double* __restrict__ coef, int64_t* __restrict__ cprefix,
                       Ctrl* ctrl, int32_t* status) {
  __shared__ int bad;
  if (threadIdx.x == 0) {
    bad = 0;
    if (off[0] != 0 || off[R] != T || goff[0] != 0 || goff[G] != R) bad = 1;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < R; i += blockDim.x) {
    const int64_t len = off[i + 1] - off[i];
    const int64_t pl = plen ? plen[i] : 0;
    if (len < 0 || pl < 0 || pl > len) bad = 1;
  }
  for (int k = threadIdx.x; k < G; k += blockDim.x)
    if (goff[k + 1] < goff[k]) bad = 1;
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      raise_status(status, 8 /* BI_ERR_BAD_OFFSETS */);
      ctrl->n_scored = 0;
      ctrl->valid = 0;
    }
    return;
  }
  for (int k = threadIdx.x; k < G; k += blockDim.x) {
    const int a = goff[k], b = goff[k + 1];
    double sum = 0.0;
    for (int i = a; i < b; ++i) sum += static_cast<double>(rewards[i]);
    const double mean = (b > a) ? sum / static_cast<double>(b - a) : 0.0;
    for (int i = a; i < b; ++i) {
      const double A = static_cast<double>(rewards[i]) - mean;
      const int64_t n = (off[i + 1] - off[i]) - (plen ? plen[i] : 0);
      coef[i] = (n > 0) ? A / (rstar * static_cast<double>(n)) : 0.0;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t acc = 0;
    for (int i = 0; i < R; ++i) {
      cprefix[i] = acc;
      acc += (off[i + 1] - off[i]) - (plen ? plen[i] : 0);
    }
    cprefix[R] = acc;
    ctrl->n_scored = acc;
    ctrl->valid = 1;
  }
}

// One thread per packed row: compact index of scored rows, and zeros in the per-row outputs of
// prompt rows.
__global__ void k_rowmap(const int64_t* __restrict__ off, const int32_t* __restrict__ plen, int R, int64_t T,
                         const int64_t* __restrict__ cprefix, const Ctrl* ctrl, const int32_t* __restrict__ targets,
                         const float* __restrict__ logmu, int32_t* __restrict__ rowmap, int32_t* __restrict__ respof,
                         int32_t* __restrict__ y_c, float* __restrict__ logmu_c, float* __restrict__ logprob,
                         float* __restrict__ is_weight, float* __restrict__ token_loss) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= T || !ctrl->valid) return;
  const int i = find_response(off, R, r);
  const int64_t p = r - off[i];
  const int64_t pl = plen ? plen[i] : 0;
  if (p < pl) {
    logprob[r] = 0.f;
    if (is_weight) is_weight[r] = 0.f;
    if (token_loss) token_loss[r] = 0.f;
    return;
  }
  const int64_t k = cprefix[i] + (p - pl);
  rowmap[k] = static_cast<int32_t>(r);
  respof[k] = i;
  y_c[k] = targets[r];
  logmu_c[k] = logmu[r];
}

// One warp per packed row: zero the gradient row of prompt rows.
__global__ void k_zero_prompt_rows(const int64_t* __restrict__ off, const int32_t* __restrict__ plen, int R,
                                   int64_t T, int H, const Ctrl* ctrl, uint16_t* __restrict__ grad_hidden) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= T || !ctrl->valid) return;
  const int i = find_response(off, R, r);
  if (r - off[i] >= plen[i]) return;
  uint4* row = reinterpret_cast<uint4*>(grad_hidden + r * H);
  for (int q = lane; q < H / 8; q += 32) row[q] = make_uint4(0u, 0u, 0u, 0u);
}

// One warp per compact row: copy the scored hidden rows into the compact buffer and zero the rows
// that pad the last 128-row tile.
__global__ void k_gather_rows(const uint16_t* __restrict__ hidden, int64_t T, int H, const Ctrl* ctrl,
                              const int32_t* __restrict__ rowmap, uint16_t* __restrict__ hc) {
  const int64_t k = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t ns = ctrl->n_scored;
  const int64_t lim = ((ns + 127) / 128) * 128;
  if (k >= T || k >= lim) return;
  uint4* dst = reinterpret_cast<uint4*>(hc + k * H);
  if (k < ns) {
    const uint4* src = reinterpret_cast<const uint4*>(hidden + static_cast<int64_t>(rowmap[k]) * H);
    for (int q = lane; q < H / 8; q += 32) dst[q] = src[q];
  } else {
    for (int q = lane; q < H / 8; q += 32) dst[q] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Maximum that keeps a NaN operand (fmaxf would drop it): a NaN D3 term makes the max NaN, as it
// makes the mean NaN.
__device__ __forceinline__ float max_keep_nan(float a, float b) {
  return isnan(a) ? a : (isnan(b) ? b : fmaxf(a, b));
}

// Fixed-shape block reduction of a RedPart (warp butterflies, then warps in order).
__device__ __forceinline__ RedPart block_reduce(RedPart v) {
  for (int o = 16; o > 0; o >>= 1) {
    v.loss += __shfl_xor_sync(0xffffffffu, v.loss, o);
    v.d3sum += __shfl_xor_sync(0xffffffffu, v.d3sum, o);
    v.k1sum += __shfl_xor_sync(0xffffffffu, v.k1sum, o);
    v.k2sum += __shfl_xor_sync(0xffffffffu, v.k2sum, o);
    v.d3max = max_keep_nan(v.d3max, __shfl_xor_sync(0xffffffffu, v.d3max, o));
    v.count += __shfl_xor_sync(0xffffffffu, v.count, o);
    v.nonfinite += __shfl_xor_sync(0xffffffffu, v.nonfinite, o);
    v.nclip += __shfl_xor_sync(0xffffffffu, v.nclip, o);
    v.nrej += __shfl_xor_sync(0xffffffffu, v.nrej, o);
  }
  __shared__ RedPart wp[32];
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) wp[w] = v;
  __syncthreads();
  RedPart out = wp[0];
  if (threadIdx.x == 0) {
    for (int i = 1; i < nw; ++i) {
      out.loss += wp[i].loss;
      out.d3sum += wp[i].d3sum;
      out.k1sum += wp[i].k1sum;
      out.k2sum += wp[i].k2sum;
      out.d3max = max_keep_nan(out.d3max, wp[i].d3max);
      out.count += wp[i].count;
      out.nonfinite += wp[i].nonfinite;
      out.nclip += wp[i].nclip;
      out.nrej += wp[i].nrej;
    }
  }
  return out;
}

// Per-token diagnostic terms of one scored row: the D3 term (w - 1 - log w = expm1(delta) -
// delta) and the sampled KL estimators k1 = -delta, k2 = delta^2 / 2.
__device__ __forceinline__ void add_token(RedPart& v, float delta, float d3) {
  const double dd = static_cast<double>(delta);
  v.d3sum = static_cast<double>(d3);
  v.d3max = d3;
  v.k1sum = -dd;
  v.k2sum = 0.5 * dd * dd;
  v.count = 1;
  v.nonfinite = isfinite(d3) ? 0 : 1;
}

// One thread per compact row: the block partial of the token losses and diagnostic terms that
// the forward kernel left per row (loss = sum of token losses; D3, KL estimators, clip count).
__global__ void k_row_parts(const float* __restrict__ tl_c, const float* __restrict__ d3_c,
                            const float* __restrict__ delta_c, const uint8_t* __restrict__ clip_c,
                            const Ctrl* ctrl, RedPart* parts) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t ns = ctrl->n_scored;
  RedPart v = red_zero();
  if (k < ns) {
    add_token(v, delta_c[k], d3_c[k]);
    v.loss = static_cast<double>(tl_c[k]);
    v.nclip = clip_c[k];
  }
  const RedPart b = block_reduce(v);
  if (threadIdx.x == 0) parts[blockIdx.x] = b;
}

// bi_d3_stats: one block partial per kD3BlockRows rows.  A thread sums its rows in a fixed order
// (four consecutive rows per step, kD3Steps steps kRedBlock x 4 rows apart, so that every step of
// the block reads 4 KB of each input contiguously) before the block reduction, whose cost would
// otherwise outweigh the 9 bytes a row brings in.
constexpr int kD3Steps = 8;
constexpr int kD3BlockRows = kRedBlock * 4 * kD3Steps;

// One token into a thread's running sums (the counts are kept by the caller in 32 bits).
__device__ __forceinline__ void acc_token(RedPart& v, float delta, float d3) {
  const double dd = static_cast<double>(delta);
  v.d3sum += static_cast<double>(d3);
  v.d3max = max_keep_nan(v.d3max, d3);
  v.k1sum -= dd;
  v.k2sum += 0.5 * dd * dd;
}

__global__ void k_d3_partial(const float* __restrict__ lp, const float* __restrict__ mu,
                             const uint8_t* __restrict__ mask, int64_t T, RedPart* parts, int32_t* status) {
  // the status word starts at BI_OK here; only k_reduce_parts, launched after this kernel, raises it
  if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kD3BlockRows;
  // 16-byte loads where the arrays allow them (the API takes any float pointers)
  const bool vec = ((reinterpret_cast<uintptr_t>(lp) | reinterpret_cast<uintptr_t>(mu)) & 15u) == 0 &&
                   (mask == nullptr || (reinterpret_cast<uintptr_t>(mask) & 3u) == 0);
  RedPart v = red_zero();
  int32_t cnt = 0, nonfin = 0;  // at most kD3BlockRows / kRedBlock tokens per thread
#pragma unroll
  for (int k = 0; k < kD3Steps; ++k) {
    const int64_t t0 = base + (static_cast<int64_t>(k) * kRedBlock + threadIdx.x) * 4;
    float a[4], b[4];
    uint32_t m[4] = {1u, 1u, 1u, 1u};
    if (vec && t0 + 3 < T) {
      const float4 av = *reinterpret_cast<const float4*>(lp + t0);
      const float4 bv = *reinterpret_cast<const float4*>(mu + t0);
      a[0] = av.x; a[1] = av.y; a[2] = av.z; a[3] = av.w;
      b[0] = bv.x; b[1] = bv.y; b[2] = bv.z; b[3] = bv.w;
      if (mask != nullptr) {
        const uint32_t mw = *reinterpret_cast<const uint32_t*>(mask + t0);
#pragma unroll
        for (int e = 0; e < 4; ++e) m[e] = (mw >> (8 * e)) & 0xffu;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool in = t0 + e < T;
        a[e] = in ? lp[t0 + e] : 0.f;
        b[e] = in ? mu[t0 + e] : 0.f;
        m[e] = in ? (mask != nullptr ? mask[t0 + e] : 1u) : 0u;
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (m[e] != 0u) {
        const float delta = a[e] - b[e];
        const float d3 = expm1f(delta) - delta;
        acc_token(v, delta, d3);
        cnt += 1;
        nonfin += isfinite(d3) ? 0 : 1;
      }
    }
  }
  v.count = cnt;
  v.nonfinite = nonfin;
  const RedPart r = block_reduce(v);
  if (threadIdx.x == 0) parts[blockIdx.x] = r;
}

// One block per response (sequence-gate variant).  rho_i = mean of delta over the response's
// scored rows, summed in a fixed order in float64; a response with |rho_i| > gate (or a
// non-finite rho_i) is rejected: its rows get no loss and no gradient (token loss, g and the dH
// rows set to 0).  The decision is written to rej[i] (0 or 1) for every response, and the
// rejections are counted by k_reduce_parts in a fixed order.  Runs after the forward and before
// the reductions and dW.
__global__ void k_seq_gate(const int64_t* __restrict__ cprefix, const float* __restrict__ delta_c,
                           const int32_t* __restrict__ rowmap, float gate, int H, const Ctrl* ctrl,
                           float* __restrict__ g_c, float* __restrict__ tl_c, float* __restrict__ token_loss,
                           uint16_t* __restrict__ grad_hidden, uint8_t* __restrict__ rej) {
  const int i = blockIdx.x;
  if (!ctrl->valid) {
    if (threadIdx.x == 0) rej[i] = 0;
    return;
  }
  const int64_t k0 = cprefix[i], k1 = cprefix[i + 1];
  if (k1 <= k0) {
    if (threadIdx.x == 0) rej[i] = 0;
    return;
  }
  double part = 0.0;
  for (int64_t k = k0 + threadIdx.x; k < k1; k += blockDim.x) part += static_cast<double>(delta_c[k]);
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  __shared__ double wsum[32];
  __shared__ int reject;
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += wsum[w];
    const double rho = tot / static_cast<double>(k1 - k0);
    reject = !(fabs(rho) <= static_cast<double>(gate));
    rej[i] = reject ? 1 : 0;
  }
  __syncthreads();
  if (!reject) return;
  for (int64_t k = k0 + threadIdx.x; k < k1; k += blockDim.x) {
    g_c[k] = 0.f;
    tl_c[k] = 0.f;
    if (token_loss) token_loss[rowmap[k]] = 0.f;
  }
  const int q8 = H / 8;
  for (int64_t e = threadIdx.x; e < (k1 - k0) * q8; e += blockDim.x) {
    const int64_t k = k0 + e / q8;
    reinterpret_cast<uint4*>(grad_hidden + static_cast<int64_t>(rowmap[k]) * H)[e % q8] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// One block: sum the block partials in a fixed order; write the loss and the diagnostics.
struct D3Out {  // layout of bi_d3
  float mean;
  float max;
  int64_t count;
  int64_t n_nonfinite;
  float k1_mean;
  float k2_mean;
  int32_t n_clipped;
  int32_t n_rejected;
};

// `rej` (may be NULL): the sequence gate's per-response decisions, R of them.
__global__ void k_reduce_parts(const RedPart* __restrict__ parts, int nparts, const uint8_t* __restrict__ rej, int R,
                               float* loss, D3Out* d3, int32_t* status) {
  RedPart v = red_zero();
  if (rej != nullptr)
    for (int i = threadIdx.x; i < R; i += blockDim.x) v.nrej += rej[i];
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) {
    const RedPart p = parts[i];
    v.loss += p.loss;
    v.d3sum += p.d3sum;
    v.k1sum += p.k1sum;
    v.k2sum += p.k2sum;
    v.d3max = max_keep_nan(v.d3max, p.d3max);
    v.count += p.count;
    v.nonfinite += p.nonfinite;
    v.nclip += p.nclip;
  }
  const RedPart b = block_reduce(v);
  if (threadIdx.x == 0) {
    if (loss) *loss = static_cast<float>(b.loss);
    if (d3) {
      D3Out o;
      const bool any = b.count > 0;
      const double n = static_cast<double>(b.count);
      o.mean = any ? static_cast<float>(b.d3sum / n) : 0.f;
      o.max = any ? b.d3max : 0.f;
      o.count = b.count;
      o.n_nonfinite = b.nonfinite;
      o.k1_mean = any ? static_cast<float>(b.k1sum / n) : 0.f;
      o.k2_mean = any ? static_cast<float>(b.k2sum / n) : 0.f;
      o.n_clipped = static_cast<int32_t>(b.nclip);
      o.n_rejected = static_cast<int32_t>(b.nrej);
      *d3 = o;
    }
    if (b.nonfinite > 0 || (loss && !isfinite(b.loss))) raise_status(status, 7 /* BI_ERR_NONFINITE */);
  }
}

}  // namespace bi
