// sts.cuh -- sequential temperature scaling of the confidence head.
//
// freeaitool.com, "DeepSeek DSpark complete guide", section 4.1: the head's
// score c_k estimates the probability that draft token k is accepted given
// that every earlier one was; its raw scores are over-confident and are
// calibrated after training by one temperature per position, fitted from
// left to right (expected calibration error from 3-8 % to about 1 %).
// yage.ai, scheduler paragraph: the calibration runs on an offline set and
// aligns the estimated probabilities with the observed acceptance rates.
//
// Position j of calibration sequence n is observed when n_acc[n] >= j and
// accepted when n_acc[n] > j.  T_j minimises the Bernoulli likelihood of the
// observed labels under c = 1 / (1 + exp(-z / T_j)).  In theta = 1/T the
// likelihood is convex: its derivative g(theta) = sum (sigma(theta z) - y) z
// is non-decreasing with slope h = sum sigma (1 - sigma) z^2.  Every
// position runs the same search: g at both bounds of theta (a sign there
// settles the position on that bound), then from theta = 1 Newton steps
// kept inside a bracket of theta (its geometric midpoint when a step leaves
// it), until a step moves theta by at most kStsTol relative or after
// kStsIters steps.  Each step is one pass over the data for all positions:
//
//   sts_grad_kernel    lane l of a warp owns position l % K of row
//                      l / K (32 / K rows per warp step, so the K scores of
//                      a row are one coalesced read); fp64 sums of g and h
//                      per lane, block sums in a fixed order -> per-CTA
//                      partials; returns at once when no position is still
//                      searching
//   sts_update_kernel  warp j = position j: its lanes sum the per-CTA
//                      partials (lane l takes CTAs l, l + 32, ...; a fixed
//                      shuffle tree combines the lanes), then lane 0 takes
//                      the next step of the search
//
// The expected calibration error (observed pairs pooled, kStsBins bins of c)
// takes one more pass per temperature set, with per-thread bin sums in
// registers (static indices: each bin is a select), so every sum is taken in
// a fixed order and the result does not depend on scheduling.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kStsMaxK = 32;
constexpr int kStsThreads = 256;
constexpr int kStsWarps = kStsThreads / 32;
constexpr int kStsBins = 15;
constexpr int kStsIters = 40;
constexpr double kStsTol = 1e-13;
constexpr double kStsTMin = 0.05;
constexpr double kStsTMax = 20.0;
constexpr int kStsMaxGrid = 1184;  // eight CTAs per SM
constexpr int kStsUnroll = 4;      // row steps whose loads are issued together
constexpr int kStsBinVals = 2 * kStsBins + 1;  // per bin: sum c, sum y; then the pair count
constexpr int kStsPart = 4;                    // per CTA and position: g, h, count, non-zero

// Search state of one position, kept in the workspace between passes.
struct StsPos {
  double lo, hi;  // bracket of theta
  double theta;   // where the next pass evaluates the derivative
  int state;      // 0: lower bound evaluated next, 1: upper bound, 2: Newton, 3: settled
  int iters;      // Newton steps taken
};
// The workspace block of the search: the positions, then the number of
// positions still searching and the number of derivative passes made.
constexpr size_t kStsPosBytes = sizeof(StsPos) * kStsMaxK + 16;

__device__ __forceinline__ double sts_logistic(double x) { return 1.0 / (1.0 + exp(-x)); }

__global__ void sts_init_kernel(StsPos* __restrict__ pos, int* __restrict__ n_active, int K) {
  // n_active[0]: positions still searching; n_active[1]: passes made
  const int j = threadIdx.x;
  if (j < K) {
    StsPos p;
    p.lo = 1.0 / kStsTMax;
    p.hi = 1.0 / kStsTMin;
    p.theta = p.lo;
    p.state = 0;
    p.iters = 0;
    pos[j] = p;
  }
  if (j == 0) {
    n_active[0] = K;
    n_active[1] = 0;
  }
}

// Derivative and slope of every position's likelihood at its current theta
// (the first pass also counts the observed samples and notes any non-zero
// score): part [gridDim.x][K][kStsPart].
template <bool kFirst>
__global__ void __launch_bounds__(kStsThreads)
sts_grad_kernel(const float* __restrict__ z, const int32_t* __restrict__ n_acc, long long N, int K,
                const StsPos* __restrict__ pos, const int* __restrict__ n_active,
                double* __restrict__ part, unsigned* flags) {
  if (!kFirst && n_active[0] == 0) return;
  __shared__ double s_g[kStsWarps][32], s_h[kStsWarps][32];
  __shared__ int s_c[kStsWarps][32], s_nz[kStsWarps][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = 32 / K;                  // rows per warp step
  const int j = lane % K, rr = lane / K;  // this lane's position and row offset
  const bool live = rr < R;
  const double theta = pos[j].theta;
  double g = 0.0, h = 0.0;
  int c = 0, nz = 0;
  const long long step = (long long)gridDim.x * kStsWarps * R;
  // kStsUnroll row steps per iteration: every load is issued before any is
  // used (a lane past the data or past R reads nothing)
  for (long long n0 = ((long long)blockIdx.x * kStsWarps + warp) * R + rr; live && n0 < N;
       n0 += kStsUnroll * step) {
    int na[kStsUnroll];
    float zf[kStsUnroll];
#pragma unroll
    for (int u = 0; u < kStsUnroll; ++u) {
      const long long n = n0 + u * step;
      na[u] = -1;
      zf[u] = 0.0f;
      if (n < N) {
        na[u] = n_acc[n];
        zf[u] = z[n * K + j];
      }
    }
#pragma unroll
    for (int u = 0; u < kStsUnroll; ++u) {
      const long long n = n0 + u * step;
      if (n >= N) break;
      int a = na[u];
      if (a < 0 || a > K) {
        if (kFirst && j == 0) raise_flag(flags, DSPARK_FLAG_BAD_LENGTH);
        a = a < 0 ? 0 : K;
      }
      if (j > a) continue;
      const double zz = (double)zf[u];
      if (!isfinite(zz)) {
        if (kFirst) raise_flag(flags, DSPARK_FLAG_NONFINITE);
        continue;
      }
      const double y = a > j ? 1.0 : 0.0;
      const double sg = sts_logistic(theta * zz);
      g += (sg - y) * zz;
      h += sg * (1.0 - sg) * zz * zz;
      if (kFirst) {
        ++c;
        nz |= zz != 0.0;
      }
    }
  }
  s_g[warp][lane] = g;
  s_h[warp][lane] = h;
  s_c[warp][lane] = c;
  s_nz[warp][lane] = nz;
  __syncthreads();
  if (tid < K) {
    // position tid: lanes tid, tid + K, ... of every warp, in a fixed order
    double gs = 0.0, hs = 0.0;
    long long cs = 0;
    int any = 0;
    for (int w = 0; w < kStsWarps; ++w)
      for (int r = 0; r < R; ++r) {
        gs += s_g[w][r * K + tid];
        hs += s_h[w][r * K + tid];
        cs += s_c[w][r * K + tid];
        any |= s_nz[w][r * K + tid];
      }
    double* o = part + ((size_t)blockIdx.x * K + tid) * kStsPart;
    o[0] = gs;
    o[1] = hs;
    if (kFirst) {
      o[2] = (double)cs;
      o[3] = (double)any;
    }
  }
}

// Sum over the G per-CTA partials part[b * stride] by one warp, in a fixed
// order: lane l adds CTAs l, l + 32, ..., then a shuffle tree.
__device__ __forceinline__ double sts_warp_sum(const double* __restrict__ part, int G,
                                               size_t stride, int lane) {
  double v = 0.0;
  for (int b = lane; b < G; b += 32) v += part[(size_t)b * stride];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Warp j: position j's derivative and slope at the theta just evaluated,
// then (lane 0) the next step of its search.  Thread 0 stores how many
// positions still search and the number of passes made; after the last
// step the temperatures are written out.  Launch: one CTA of K warps.
__global__ void sts_update_kernel(const double* __restrict__ part, int G, int K,
                                  StsPos* __restrict__ pos, int* __restrict__ n_active,
                                  int step, int last_step, float* __restrict__ temps,
                                  int32_t* __restrict__ passes) {
  __shared__ int s_search[kStsMaxK];
  const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int before = n_active[0];  // positions searching when this step's pass ran
  StsPos p = pos[j];
  if (p.state < 3) {
    const size_t stride = (size_t)K * kStsPart;
    const double* pj = part + (size_t)j * kStsPart;
    const double g = sts_warp_sum(pj, G, stride, lane);
    const double h = sts_warp_sum(pj + 1, G, stride, lane);
    double cnt = 0.0, nz = 0.0;
    if (p.state == 0) {
      cnt = sts_warp_sum(pj + 2, G, stride, lane);
      nz = sts_warp_sum(pj + 3, G, stride, lane);
    }
    if (lane == 0) {
      if (p.state == 0) {  // the lower bound was evaluated (the first pass)
        if (cnt == 0.0 || nz == 0.0) {
          p.state = 3;  // nothing to fit: T = 1
          p.theta = 1.0;
        } else if (g >= 0.0) {
          p.state = 3;
        } else {
          p.state = 1;
          p.theta = p.hi;
        }
      } else if (p.state == 1) {  // the upper bound was evaluated
        if (g <= 0.0) {
          p.state = 3;
        } else {
          p.state = 2;
          p.theta = 1.0;
        }
      } else {  // a Newton point was evaluated
        if (g == 0.0) {
          p.state = 3;
        } else {
          if (g < 0.0)
            p.lo = p.theta;
          else
            p.hi = p.theta;
          const double newton = p.theta - g / h;
          if (h > 0.0 && fabs(newton - p.theta) <= kStsTol * p.theta) {
            p.theta = newton;
            p.state = 3;
          } else {
            p.theta = (h > 0.0 && newton > p.lo && newton < p.hi) ? newton : sqrt(p.lo * p.hi);
            if (++p.iters == kStsIters) p.state = 3;
          }
        }
      }
      pos[j] = p;
    }
  }
  if (lane == 0) {
    s_search[j] = p.state < 3;
    if (step == last_step) temps[j] = (float)(1.0 / p.theta);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int act = 0;
    for (int i = 0; i < K; ++i) act += s_search[i];
    if (before > 0) n_active[1] = step + 1;  // a pass ran at this step
    n_active[0] = act;
    if (step == last_step && passes != nullptr) *passes = n_active[1] + 2;  // + the two ECE passes
  }
}

// Calibration-error sums of one temperature set (unit = every T is 1, else
// the fitted thetas): part [gridDim.x][kStsBinVals].  Same lane mapping as
// the derivative pass; each lane keeps its bin sums in registers.
__global__ void __launch_bounds__(kStsThreads)
sts_ece_kernel(const float* __restrict__ z, const int32_t* __restrict__ n_acc, long long N, int K,
               const StsPos* __restrict__ pos, int unit, double* __restrict__ part,
               unsigned* flags) {
  (void)flags;
  __shared__ double s_red[kStsWarps][kStsBinVals];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = 32 / K;
  const int j = lane % K, rr = lane / K;
  const bool live = rr < R;
  const double theta = unit ? 1.0 : pos[j].theta;
  double sc[kStsBins], sy[kStsBins];
#pragma unroll
  for (int m = 0; m < kStsBins; ++m) sc[m] = sy[m] = 0.0;
  double total = 0.0;
  const long long step = (long long)gridDim.x * kStsWarps * R;
  for (long long n0 = ((long long)blockIdx.x * kStsWarps + warp) * R + rr; live && n0 < N;
       n0 += kStsUnroll * step) {
    int na[kStsUnroll];
    float zf[kStsUnroll];
#pragma unroll
    for (int u = 0; u < kStsUnroll; ++u) {
      const long long n = n0 + u * step;
      na[u] = -1;
      zf[u] = 0.0f;
      if (n < N) {
        na[u] = n_acc[n];
        zf[u] = z[n * K + j];
      }
    }
#pragma unroll
    for (int u = 0; u < kStsUnroll; ++u) {
      const long long n = n0 + u * step;
      if (n >= N) break;
      int a = na[u];
      a = a < 0 ? 0 : (a > K ? K : a);
      const double zz = (double)zf[u];
      if (j > a || !isfinite(zz)) continue;
      const double cf = sts_logistic(theta * zz);
      int bin = (int)(cf * kStsBins);
      if (bin > kStsBins - 1) bin = kStsBins - 1;
      const double y = a > j ? 1.0 : 0.0;
#pragma unroll
      for (int m = 0; m < kStsBins; ++m) {
        const bool in = bin == m;
        sc[m] += in ? cf : 0.0;
        sy[m] += in ? y : 0.0;
      }
      total += 1.0;
    }
  }
#pragma unroll
  for (int i = 0; i < kStsBinVals; ++i) {
    double v = i < kStsBins ? sc[i] : (i < 2 * kStsBins ? sy[i - kStsBins] : total);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (lane == 0) s_red[warp][i] = v;
  }
  __syncthreads();
  if (tid < kStsBinVals) {
    double v = 0.0;
    for (int w = 0; w < kStsWarps; ++w) v += s_red[w][tid];
    part[(size_t)blockIdx.x * kStsBinVals + tid] = v;
  }
}

// ECE = sum over bins |sum y - sum c| / pairs.  Warp i sums value i of the
// per-CTA sums (fixed order, as in the update); thread 0 combines.  Launch:
// one CTA of kStsBinVals warps.
__global__ void sts_ece_final_kernel(const double* __restrict__ part, int G, float* __restrict__ out) {
  __shared__ double s_v[kStsBinVals];
  const int i = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double v = sts_warp_sum(part + i, G, kStsBinVals, lane);
  if (lane == 0) s_v[i] = v;
  __syncthreads();
  if (threadIdx.x != 0) return;
  double e = 0.0;
  for (int m = 0; m < kStsBins; ++m) e += fabs(s_v[kStsBins + m] - s_v[m]);
  const double total = s_v[2 * kStsBins];
  *out = total > 0.0 ? (float)(e / total) : 0.0f;
}

inline int sts_grid(long long N) {
  long long g = (N + kStsThreads - 1) / kStsThreads;
  if (g > kStsMaxGrid) g = kStsMaxGrid;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace dspark
